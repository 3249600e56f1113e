#!/usr/bin/env python
"""Throughput of the SureLock decoding step on B200.

Default workload (--workload long8b): the LLaDA-8B shape (32 layers, d=4096,
32 heads x 128, SwiGLU 12288, vocab 126464), random-init bf16 weights, batch
4, 1024 random prompt ids + 1024 masked positions per sequence (N = 2048), 512
denoising steps in semi-autoregressive blocks of 64 positions, two tokens
unmasked per step, KL threshold eps = 0.05 with the confidence gate at the
0.5 quantile.  One bench step = one block of that decode (32 denoising steps:
the denoiser on the active rows with the sure test's statistics in the LM
head's epilogue, the lock decisions, unmasking and compaction); decodes run
back to back and the timed region starts at the first step of a decode, so
16 bench steps are exactly one decode.
--workload full8b: batch 1, 128 prompt + 256 masked (N = 384), 256 steps in
blocks of 32, one token per step, eps = 0.05; one bench step = one decode.

Reported (one JSON line from rank 0):
  value      denoising steps/s over all ranks, inputs resident in HBM
  e2e        the same through sl_sampler_generate with host prompts in and
             host tokens out (both copies inside the timed region)
  roofline   the dominant kernel (the tcgen05 GEMM): algorithmic bytes or
             FLOPs per launch / its CUDA-event launch time, against the
             measured peaks in MEASURED_PEAKS.json
  step_roofline  sum over the trajectory of max(F_t/peak_flops, B_t/peak_bw)
             divided by the measured decode time (the per-step roofline vs M_t)
  cpu_baseline   the CPU oracle on a bounded sample of the same step
Multi-GPU (torchrun): independent replicas, one decode per rank; the timed
region is bracketed by barriers and the max over ranks is taken.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload full8b|long8b] [--eps E] [--scripted] [--batch B]
                  [--gate-q Q] [--ablation none|no_kv_cache|gate_only] [--head-fusion on|off]
                  [--kv-reuse R]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import tempfile
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK, source="fallback")


# ------------------------------------------------------------- workload ---
def make_setup(name: str, eps, scripted: bool, batch=None, gate_q=None,
               ablation: str = "none", kv_reuse: int = 1) -> wl.SamplerSetup:
    """The workload's decode; `batch` (1..64 sequences per GPU) overrides its batch,
    `gate_q` its confidence gate, and `ablation` selects one of the pages'
    ablations (no_kv_cache, gate_only) instead of the method itself; `kv_reuse`
    R > 1 composes the method with K/V reuse for the active rows (all active
    rows recomputed every R steps)."""
    if name == "full8b":
        s = wl.cfg_full8b(eps=0.05 if eps is None else eps, scripted=scripted)
    elif name == "long8b":
        s = wl.cfg_long8b()
        if eps is not None:
            import dataclasses
            s = dataclasses.replace(s, eps=eps)
    else:
        raise SystemExit(f"unknown workload {name}")
    import dataclasses
    if batch is not None:
        if not 1 <= batch <= 64:
            raise SystemExit(f"--batch must be in [1, 64], got {batch}")
        s = dataclasses.replace(s, batch=batch)
    if gate_q is not None:
        if gate_q > 1.0:
            raise SystemExit(f"--gate-q must be <= 1 (< 0: gate off), got {gate_q}")
        s = dataclasses.replace(s, gate_q=gate_q)
    if ablation not in ("none", "no_kv_cache", "gate_only"):
        raise SystemExit(f"unknown ablation {ablation}")
    if ablation == "gate_only" and s.gate_q < 0:
        raise SystemExit("--ablation gate_only needs the confidence gate (--gate-q in [0, 1])")
    s = dataclasses.replace(s, no_kv_cache=ablation == "no_kv_cache",
                            gate_only=ablation == "gate_only")
    if kv_reuse < 1:
        raise SystemExit(f"--kv-reuse must be >= 1, got {kv_reuse}")
    if kv_reuse > 1 and (s.scripted or s.no_kv_cache):
        raise SystemExit("--kv-reuse composes with the sure test on the full cache only "
                         "(not with --scripted or --ablation no_kv_cache)")
    s = dataclasses.replace(s, kv_reuse=kv_reuse)
    s.validate()
    return s


def setup_from_args(args) -> wl.SamplerSetup:
    return make_setup(args.workload, args.eps, args.scripted, args.batch, args.gate_q,
                      args.ablation, getattr(args, "kv_reuse", 1))


DATA_DESC = "synthetic (random-init N(0,0.02) weights, uniform random prompt ids)"


def workload_config(args, setup: wl.SamplerSetup, world: int) -> dict:
    """The `config` object of the JSON line (the same for both arms)."""
    T = setup.steps
    return {"workload": f"{args.workload}: LLaDA-8B shape, batch {setup.batch}, "
                        f"{setup.prompt_len} prompt + {setup.gen_len} masked "
                        f"(N={setup.n_ctx}), {T} steps, blocks of {setup.block_len}, "
                        f"{setup.tokens_per_step} token(s)/step, eps={setup.eps}"
                        + (f", gate q={setup.gate_q}" if setup.gate_q >= 0 else "")
                        + (", scripted lock schedule" if setup.scripted else "")
                        + (", ablation: no KV cache (active rows' keys only)"
                           if setup.no_kv_cache else "")
                        + (", ablation: confidence gate only" if setup.gate_only else "")
                        + (", sure-test statistics in a separate pass after the LM head"
                           if getattr(args, "head_fusion", "on") == "off" else "")
                        + (f", K/V reuse for active rows (all recomputed every "
                           f"{setup.kv_reuse} steps)" if setup.kv_reuse > 1 else ""),
            "bench_step": (f"one full decode ({T} denoising steps)"
                           if bench_unit_steps(args, setup) == T else
                           f"one semi-autoregressive block ({setup.steps_per_block} denoising "
                           f"steps, 1/{setup.n_blocks} of a {T}-step decode); decodes run back "
                           f"to back and the timed region starts at a decode's first step"),
            "global_batch": world * setup.batch, "seq_len": setup.n_ctx,
            "parallelism": f"replicas{world}",
            "l2": "inputs larger than L2 (15 GB of weights streamed per step)"}


def gemm_traffic(alg_bytes_per_launch: float):
    """DRAM bytes per GEMM launch of this run: the committed ncu capture's ratio
    of measured DRAM bytes (read + write) to the library's algorithmic bytes
    over the same launches, applied to this run's algorithmic bytes per launch
    (the GEMM's traffic grows with the units it processes); None when the
    kernel source changed since the counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "gemm_tc_traffic.json")) as f:
            rec = json.load(f)
        for src, sha in rec["sources"].items():
            with open(os.path.join(ROOT, src), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != sha:
                    return None
        return float(rec["dram_bytes"]) / float(rec["algorithmic_bytes"]) * alg_bytes_per_launch
    except Exception:
        return None


def step_work(shape: wl.ModelShape, m_rows: int, batch: int, n_ctx: int):
    """Algorithmic FLOPs and HBM bytes of one denoising step on m_rows active
    rows (all sequences of the batch), attending to n_ctx keys per sequence."""
    d, f, V, L = shape.d_model, shape.d_ffn, shape.vocab, shape.n_layers
    lin = L * (4 * d * d + 3 * d * f) + V * d
    flops = 2.0 * m_rows * lin + 4.0 * L * m_rows * n_ctx * d
    byts = (2.0 * lin                          # weights, read once
            + batch * L * 2.0 * n_ctx * d * 2  # K/V of every position, read
            + L * 2.0 * m_rows * d * 2         # fresh K/V of the active rows, written
            + 4.0 * m_rows * V                 # posterior: this step's written, last step's read
            + 2.0 * m_rows * d)                # embedding gather
    return flops, byts


def stored_trajectory(workload: str):
    """The rows each step computes, as a GPU run of this exact workload
    recorded them (profiles/trajectory_*.json, copied from the bench line's
    "trajectory" = M_t, or its "computed_rows" under K/V reuse), or None.  It
    only weights the CPU oracle's timed sample by the work of each step; it is
    never an input or an expected value of a parity check."""
    import glob
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "trajectory_*.json"))):
        try:
            with open(path) as f:
                rec = json.load(f)
        except Exception:
            continue
        if rec.get("workload") == workload and rec.get("M_t"):
            rows = rec.get("computed_rows") or rec["M_t"]
            return np.asarray(rows, dtype=np.int64), os.path.basename(path)
    return None


def trajectory_from_lock_t(lock_t: np.ndarray, steps: int) -> np.ndarray:
    """Active rows at the start of every step: all rows minus those locked earlier."""
    lt = lock_t.reshape(-1)
    total = lt.size
    locked_at = np.bincount(lt[lt >= 0], minlength=steps)
    before = np.concatenate([[0], np.cumsum(locked_at)[:-1]])
    return total - before[:steps]


# --------------------------------------------------------------- clocks ---
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, path: str):
        self.gpu_id, self.path, self.proc = gpu_id, path, None

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", self.gpu_id], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for ln in open(self.path):
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 9:
                continue
            try:
                rows.append((float(p[1]), float(p[2]), float(p[3]), p[5], p[6], p[7], p[8]))
            except ValueError:
                continue
        if not rows:
            return None
        maxmhz = max(r[1] for r in rows)
        loaded = [r for r in rows if r[2] > 200.0] or rows
        reasons = set()
        for r in loaded:
            for name, v in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                "sw_power_cap"), r[3:]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": float(np.median([r[0] for r in loaded])), "sm_max_mhz": maxmhz,
                "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(r[2] for r in rows), "reasons": sorted(reasons)}


def gpu_id_for(dev) -> str:
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")
        return vis[dev.index or 0] if dev.index is not None and dev.index < len(vis) else vis[0]


# ---------------------------------------------------------- CPU oracle ---
def oracle_sample(setup: wl.SamplerSetup, traj: np.ndarray, layers: int = 2,
                  vocab_frac: int = 8, seed: int = 7):
    """Time the CPU oracle on a bounded sample of one denoising step at the
    densest point (every row active): `layers` transformer blocks on all
    B*N rows and the LM head + sure test on 1/vocab_frac of the vocabulary,
    with random weights of the real shape.  The step time is extrapolated to
    all layers and the full vocabulary, then to the trajectory in proportion to
    the algorithmic FLOPs of each step.  Returns (steps/s, description, threads)."""
    from oracle import model as om
    from oracle import surelock as osl
    shape = setup.shape
    d, f, V = shape.d_model, shape.d_ffn, shape.vocab
    B, N = setup.batch, setup.n_ctx
    rng = np.random.default_rng(seed)
    f32 = np.float32

    def w(*s):
        return rng.standard_normal(s, dtype=f32) * f32(0.02)

    Vs = V // vocab_frac
    h = rng.standard_normal((N, d), dtype=f32)
    pos = np.arange(N)
    one = np.ones(d, dtype=f32)
    lws = [{"wq": w(d, d), "wk": w(d, d), "wv": w(d, d), "wo": w(d, d), "w_gate": w(f, d),
            "w_up": w(f, d), "w_down": w(d, f), "attn_norm": one, "ffn_norm": one}
           for _ in range(layers)]
    head = w(Vs, d)
    ck = np.zeros((N, d), dtype=f32); cv = np.zeros((N, d), dtype=f32)
    t0 = time.perf_counter()
    for lw in lws:
        for _ in range(B):
            h = om.layer_forward(shape, lw, h, pos, ck, cv)
    t1 = time.perf_counter()
    z = om.rmsnorm(h, one, shape.rms_eps) @ head.T
    lp = osl.log_softmax(z)
    osl.kl_rows(lp, osl.log_softmax(z + f32(0.05)))
    osl.uncertainty(lp)
    osl.prediction(lp, 0)
    t2 = time.perf_counter()
    t_dense = (t1 - t0) * shape.n_layers / layers + (t2 - t1) * vocab_frac * B
    f_dense = step_work(shape, B * N, B, N)[0]
    t_traj = sum(t_dense * step_work(shape, int(m), B, N)[0] / f_dense for m in traj)
    threads = _blas_threads()
    desc = (f"oracle (NumPy float32) on {layers} of {shape.n_layers} layers x {B} sequence(s) "
            f"at M={B * N} rows + LM head/sure test on {Vs} of {V} vocab rows, extrapolated "
            f"to the full step ({t_dense:.2f} s) and to the {len(traj)}-step trajectory in "
            f"proportion to per-step FLOPs; measured {t2 - t0:.1f} s")
    return len(traj) / t_traj, desc, threads


def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ------------------------------------------------------------ GPU arm ---
class Ranks:
    """The replicas' process group (one rank per GPU under torchrun): a barrier
    around the timed region and the max over ranks of a time.  No data-path
    collective exists; nccl on the GPUs, gloo where there are none."""

    def __init__(self, world: int, backend: str = "nccl", device=None, timeout_s: int = 600):
        import torch
        self.world, self.dist = world, None
        self.device = device if device is not None else torch.device("cpu")
        if world > 1:
            import datetime
            import torch.distributed as dist
            kw = {"device_id": self.device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
            self.dist = dist

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, x: float) -> float:
        if self.dist is None:
            return x
        import torch
        t = torch.tensor([x], device=self.device, dtype=torch.float64)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.barrier()
            self.dist.destroy_process_group()
            self.dist = None


def bench_unit_steps(args, setup: wl.SamplerSetup) -> int:
    """Denoising steps per bench step: a whole decode (the default), so that
    any K timed steps weigh the decode's early, heavy steps (every row active)
    and its late, light ones as the decode itself does; or, for quick looks,
    one semi-autoregressive block (timed from a decode's first step, so a K
    that is not a multiple of the blocks per decode over-weights the first
    blocks)."""
    mode = getattr(args, "bench_step", "auto")
    if mode == "auto":
        mode = "decode"
    return setup.steps_per_block if mode == "block" else setup.steps


def aux_decodes(k: int, decode_ms: float, budget_ms: float = 20000.0) -> int:
    """Decodes of each instrumented / end-to-end pass: about `budget_ms` of
    decoding, at least one, at most the timed count."""
    return max(1, min(k, int(budget_ms // max(decode_ms, 1e-3))))


def carry_line(rec: dict, decodes: int, peaks: dict) -> dict:
    """The K/V reuse carry kernel over the instrumented decodes: its time per
    decode and its bandwidth (the reused rows' logits and lse read and written
    once) against the measured HBM copy peak."""
    ms, by = rec["ms"], rec["bytes"]
    gbs = by / (ms / 1e3) / 1e9 if ms > 0 else None
    return {"ms_per_decode": round(ms / max(1, decodes), 3),
            "launches_per_decode": rec["launches"] // max(1, decodes),
            "achieved_gbs": round(gbs, 1) if gbs else None,
            "frac_hbm": round(gbs / peaks["hbm_gbs"], 4) if gbs else None}


def replica_prompt_seed(rank: int) -> int:
    """Each replica decodes its own prompts."""
    return wl.SEED_PROMPTS + rank


def aggregate_rate(world: int, steps_per_rank: int, ms_max: float) -> float:
    """Denoising steps per second of the whole job: every rank's steps over the
    slowest rank's time."""
    return world * steps_per_rank / (ms_max / 1e3)


def run_ours(args, rank: int, world: int):
    import torch
    from token_locking_b200 import runtime as rt

    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    setup = setup_from_args(args)
    shape = setup.shape
    T = setup.steps
    ranks = Ranks(world, "nccl", dev)
    barrier, max_over_ranks = ranks.barrier, ranks.max

    weights = wl.torch_weights(shape, dev)
    torch.cuda.synchronize()
    model = rt.Model(shape, weights, "bf16")
    model.set_ablation(no_kv_cache=setup.no_kv_cache, gate_only=setup.gate_only)
    model.set_head_fusion(args.head_fusion == "on")
    s = rt.Sampler(model, setup.batch, setup.prompt_len, setup.gen_len, T, setup.block_len,
                   setup.tokens_per_step, setup.eps, setup.gate_q, setup.scripted)
    if setup.kv_reuse > 1:
        s.set_kv_reuse(setup.kv_reuse)
    prompts = wl.np_prompts(setup.batch, setup.prompt_len, shape.vocab, shape.mask_id,
                            seed=replica_prompt_seed(rank))
    d_prompts = torch.from_numpy(prompts).to(dev)
    t_tune = time.perf_counter()
    s.autotune()                 # GEMM tilings timed on this device (setup, untimed)
    t_tune = time.perf_counter() - t_tune

    def decode():
        s.start(d_prompts)
        for _ in range(T):
            s.step()

    # One bench step = `unit` denoising steps: a whole decode, or one
    # semi-autoregressive block of it (decodes then run back to back).
    unit = bench_unit_steps(args, setup)
    cursor = [0]                 # next denoising step of the running decode

    def run_unit():
        for _ in range(unit):
            if cursor[0] == 0:
                s.start(d_prompts)
            s.step()
            cursor[0] = (cursor[0] + 1) % T

    for _ in range(args.warmup):
        run_unit()
    while cursor[0] != 0:        # untimed: the timed region starts with a decode
        run_unit()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_id_for(dev), os.path.join(args.out_dir, f"clocks_rank{rank}.csv")) \
        if rank == 0 else None
    model.timing_read(reset=True)           # zero the library's kernel-launch counter
    barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
        time.sleep(0.4)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(args.steps):
        run_unit()
    ev1.record()
    torch.cuda.synchronize()
    ms_local = ev0.elapsed_time(ev1)
    while cursor[0] != 0:        # finish the running decode (untimed)
        run_unit()
    clk = clocks.stop() if clocks else None
    kernels_timed = model.timing_read(reset=True)["kernels"]
    barrier()
    ms = max_over_ranks(ms_local)
    # the instrumented and end-to-end passes run `aux` whole decodes (about 20 s
    # of decoding each): the timed region above is never shortened
    aux = aux_decodes(max(1, args.steps * unit // T), ms / args.steps * T / unit)

    # Per-kernel CUDA events around every GEMM / attention / lock launch.  An
    # event between two kernels also removes the programmatic-launch overlap at
    # that boundary, so this instrumented pass over the same K decodes is timed
    # separately from the headline number above.
    model.timing_read(reset=True)
    model.timing_enable(True)
    model.timing_read(reset=True)
    barrier()
    torch.cuda.synchronize()
    ei0, ei1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ei0.record()
    for _ in range(aux):
        decode()
    ei1.record()
    torch.cuda.synchronize()
    ms_instr = max_over_ranks(ei0.elapsed_time(ei1))
    model.timing_enable(False)
    tim = model.timing_read(reset=True)
    barrier()

    # trajectory of the last decode and per-step times of one more (untimed) decode
    st = s.state()
    traj = trajectory_from_lock_t(st["lock_t"].cpu().numpy(), T)
    s.start(d_prompts)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(T + 1)]
    evs[0].record()
    for t in range(T):
        s.step()
        evs[t + 1].record()
    torch.cuda.synchronize()
    step_ms = np.array([evs[t].elapsed_time(evs[t + 1]) for t in range(T)])
    traj2 = trajectory_from_lock_t(s.state()["lock_t"].cpu().numpy(), T)
    # the rows each step's forward runs on: M_t, or with K/V reuse the computed
    # rows between refreshes (read per step from one more untimed decode)
    rows_t, rows_t2 = traj, traj2
    if setup.kv_reuse > 1:
        s.start(d_prompts)
        got = []
        for t in range(T):
            m_act = sum(s.state()["active"].counts())
            s.step()
            got.append(m_act if t % setup.kv_reuse == 0 else sum(s.state()["computed"].counts()))
        rows_t = rows_t2 = np.array(got)

    # end to end: host prompts -> host tokens through the public call
    h_prompts = torch.from_numpy(prompts).pin_memory()
    h_out = torch.zeros((setup.batch, setup.n_ctx), dtype=torch.int32).pin_memory()
    s.generate_ptr(h_prompts.data_ptr(), h_out.data_ptr())
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(aux):
        s.generate_ptr(h_prompts.data_ptr(), h_out.data_ptr())
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    barrier()

    result = None
    if rank == 0:
        peaks = load_peaks()
        timed_steps = args.steps * unit
        value = aggregate_rate(world, timed_steps, ms)
        e2e_value = aggregate_rate(world, aux * T, e2e_ms)
        gen_tokens = world * timed_steps * setup.batch * setup.tokens_per_step
        # per-step roofline over the rows the timed steps compute (M_t, or the
        # computed rows under K/V reuse; the timed region starts at step 0 of a
        # decode), burst peaks
        pf = peaks["bf16_tflops"] * 1e12
        pb = peaks["hbm_gbs"] * 1e9
        roof_t = [max(fl / pf, by / pb) for fl, by in
                  (step_work(shape, int(m), setup.batch, setup.n_ctx) for m in rows_t)]
        roof = [roof_t[i % T] for i in range(timed_steps)]
        decode_ms = ms_local / timed_steps * T
        step_frac = (sum(roof) * 1e3) / ms_local
        flops_traj = sum(step_work(shape, int(m), setup.batch, setup.n_ctx)[0] for m in rows_t)
        flops_dense = T * step_work(shape, setup.batch * setup.n_ctx, setup.batch, setup.n_ctx)[0]
        # dominant kernel: the tensor-core GEMM
        g = tim["gemm"]
        t_f = g["flops"] / pf
        t_b = g["bytes"] / pb
        traffic = gemm_traffic(g["bytes"] / max(1, g["launches"]))
        # the GEMM is timed inside a long decode: a tensor-bound kernel runs at
        # the power-capped clock, so its peak is the sustained bf16 figure
        if t_b >= t_f:
            bound, ach, peak, unit = "hbm", g["bytes"] / (g["ms"] / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s"
            peak_kind = "HBM copy"
        else:
            bound, ach, peak, unit = ("tensor", g["flops"] / (g["ms"] / 1e3) / 1e12,
                                      peaks["bf16_tflops_sustained"], "TFLOP/s")
            peak_kind = "bf16 sustained (kernel timed inside the decode)"
        pfs = peaks["bf16_tflops_sustained"] * 1e12
        roof_s = [max(fl / pfs, by / pb) for fl, by in
                  (step_work(shape, int(rows_t[i % T]), setup.batch, setup.n_ctx)
                   for i in range(timed_steps))]
        step_frac_sustained = (sum(roof_s) * 1e3) / ms_local
        idx = list(range(0, T, 16)) + [T - 1]
        if setup.kv_reuse > 1:
            # every sampled step with its successor, so that steps between
            # refreshes are in the curve too
            idx = sorted({j for i in idx for j in (i, i + 1) if j < T})
        def roof_ms(m):
            fl, by = step_work(shape, int(m), setup.batch, setup.n_ctx)
            return max(fl / pf, by / pb) * 1e3

        curve = {"t": idx, "M_t": [int(traj2[i]) for i in idx],
                 "ms": [round(float(step_ms[i]), 3) for i in idx],
                 "roofline_frac": [round(roof_ms(rows_t2[i]) / float(step_ms[i]), 3) for i in idx]}
        if setup.kv_reuse > 1:
            curve["computed_rows"] = [int(rows_t2[i]) for i in idx]
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            v, desc, thr = oracle_sample(setup, rows_t)
            cpu = {"value": v, "unit": "denoise steps/s", "cores": thr, "kind": "oracle",
                   "sample": desc}
        result = {
            "metric": "LLaDA-8B-shape denoise steps/s & gen tok/s; % of per-step roofline vs M_t",
            "value": round(value, 3),
            "unit": "denoise steps/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms / args.steps, 3),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": DATA_DESC,
            "config": workload_config(args, setup, world),
            "gen_tok_s": round(gen_tokens / (ms / 1e3), 3),
            "e2e": {"value": round(e2e_value, 3), "unit": "denoise steps/s",
                    "gen_tok_s": round(world * aux * setup.batch * setup.gen_len
                                       / (e2e_ms / 1e3), 3),
                    "decodes": aux,
                    "h2d_bytes_per_step": int(prompts.nbytes),
                    "d2h_bytes_per_step": int(setup.batch * setup.n_ctx * 4)},
            "roofline": {"bound": bound, "achieved": round(ach, 2), "peak": peak, "unit": unit,
                         "frac": round(ach / peak, 4),
                         "traffic": round(traffic) if traffic else None,
                         "algorithmic_bytes_per_launch": round(g["bytes"] / max(1, g["launches"])),
                         "kernel": "gemm_tc_kernel (tcgen05)",
                         "launches": g["launches"], "kernel_ms": round(g["ms"], 3),
                         "peak_source": peaks["source"], "peak_kind": peak_kind,
                         "measured_in": f"instrumented pass of {aux} more decode(s) "
                                        f"({ms_instr / aux:.1f} ms/decode with events)"},
            "step_roofline": {"frac": round(step_frac, 4),
                              "frac_sustained": round(step_frac_sustained, 4),
                              "roofline_ms_per_decode": round(sum(roof_t) * 1e3, 3),
                              "measured_ms_per_decode": round(decode_ms, 3),
                              "timed_steps": timed_steps,
                              "peaks": "frac: burst (bf16_tflops, hbm_gbs); frac_sustained: "
                                       "bf16_tflops_sustained, hbm_gbs"},
            "algorithmic_flops_reduction": round(1.0 - flops_traj / flops_dense, 4),
            "kernel_time_ms": {k: round(tim[k]["ms"], 3) for k in ("gemm", "attn", "lock")},
            **({"reuse_carry": carry_line(tim["other"], aux, peaks)} if setup.kv_reuse > 1 else {}),
            "curve": curve,
            "trajectory": [int(m) for m in traj],
            **({"computed_rows": [int(m) for m in rows_t]} if setup.kv_reuse > 1 else {}),
            "cpu_baseline": cpu,
            "clocks": clk,
            "gpu_launches": int(kernels_timed),
            "autotune_s": round(t_tune, 2),
        }
    s.close()
    model.close()
    ranks.close()
    return result


# ------------------------------------------------------ reference arm ---
def run_reference(args, rank: int, world: int):
    """The CPU oracle on the machine's host cores, same metric and workload; each
    bench step is one bounded sample (see oracle_sample)."""
    if rank != 0:
        return None
    setup = setup_from_args(args)
    T = setup.steps
    cfg = workload_config(args, setup, world)
    # the trajectory the GPU arm recorded for this workload (the same M_t the
    # GPU arm's cpu_baseline uses), else a linear decay from N as a stand-in
    got = stored_trajectory(cfg["workload"])
    if got is not None and len(got[0]) == T:
        traj, traj_note = got[0], f"per-step rows from {got[1]}"
    else:
        traj = np.array([setup.batch * (setup.n_ctx - int(round(t * (setup.n_ctx - 1) / max(1, T))))
                         for t in range(T)])
        traj_note = "M_t trajectory: linear stand-in (no stored GPU trajectory)"
    for _ in range(args.warmup):
        oracle_sample(setup, traj, layers=1, vocab_frac=16)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v, desc, thr = oracle_sample(setup, traj, layers=1, vocab_frac=16)
        vals.append(v)
    wall = time.perf_counter() - t0
    value = float(np.mean(vals))
    desc = f"{desc}; {traj_note}"
    return {"impl": "reference", "metric":
            "LLaDA-8B-shape denoise steps/s & gen tok/s; % of per-step roofline vs M_t",
            "value": round(value, 6), "unit": "denoise steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(wall / args.steps * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": DATA_DESC, "config": cfg,
            "cpu_baseline": {"value": round(value, 6), "unit": "denoise steps/s", "cores": thr,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": round(value, 6), "unit": "denoise steps/s",
                    "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long8b",
                    help="long8b: LLaDA-8B shape, batch 4, N = 2048, 512 steps (the default); "
                         "full8b: batch 1, N = 384, 256 steps")
    ap.add_argument("--bench-step", default="auto", choices=["auto", "decode", "block"],
                    help="denoising steps per bench step: a whole decode (auto), or one "
                         "semi-autoregressive block (a quick look; biased towards the "
                         "first blocks unless K is a multiple of the blocks per decode)")
    ap.add_argument("--eps", type=float, default=None)
    ap.add_argument("--scripted", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences per GPU (default: the workload's own batch)")
    ap.add_argument("--gate-q", type=float, default=None,
                    help="confidence-gate quantile (default: the workload's; < 0 = off)")
    ap.add_argument("--ablation", default="none", choices=["none", "no_kv_cache", "gate_only"],
                    help="run one of the pages' ablations instead of the method")
    ap.add_argument("--head-fusion", default="on", choices=["on", "off"],
                    help="sure-test statistics in the LM head's epilogue (on) or in a "
                         "separate pass over the stored logits (off)")
    ap.add_argument("--kv-reuse", type=int, default=1,
                    help="compose the method with K/V reuse for the active rows: all active "
                         "rows are recomputed every R steps, between them only the masked and "
                         "just-unmasked ones (1 = off)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--out-dir", default=os.path.join(tempfile.gettempdir(), "surelock_bench"),
                    help="where the per-rank clock samples (CSV) are written")
    args = ap.parse_args()
    os.makedirs(args.out_dir, exist_ok=True)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        res = run_ours(args, rank, world)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
