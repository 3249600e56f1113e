"""Kernel-level benchmarks of the SureLock step on B200 (also the target of ncu
captures).

  python -m token_locking_b200.microbench layer [--m 2048,1024,...] [--iters K]
      One LLaDA-8B-shaped transformer block (d=4096, 32 heads x 128, SwiGLU
      12288) on M active rows of a sequence of N=2048 positions: random active
      subset (seed 2), cache filled N(0,1), hidden states N(0,1).  Runs the
      block through sl_layer_forward (gather of the active rows' inputs is the
      caller's; norms, fused QKV + RoPE + cache scatter, attention over all
      2048 keys, output projection + residual, SwiGLU FFN + residual).
  python -m token_locking_b200.microbench lock [--m 64,512,2048] [--iters K]
      The sure test on M rows of vocab 126464 bf16 logits, N(0,3) with a spike
      (row max + 8) on a random half of the rows, previous logits perturbed by
      N(0,0.05); KL test eps in {0.01, 0.05} with the 0.5-quantile confidence
      gate, then compaction.
  python -m token_locking_b200.microbench decode [--steps S] [--skip T] [--workload W]
      S denoising steps (after T untimed ones) of the LLaDA-8B-shaped decode:
      batch 1, N=384 (full8b, the default) or batch 4, N=2048 (long8b).
  python -m token_locking_b200.microbench gemm [--m 8,64,...]
      Sweep of the tensor-core GEMM tilings (tile width, 128/256-row tiles,
      K splits) on the LLaDA-8B projection shapes; one JSON line per tiling.

Each case prints one JSON line: the median time per call over --iters calls
(default 20; CUDA events, after 5 warm-up calls, L2 flushed before every call
by a 256 MB write), the roofline time of the case's algorithmic work and their
ratio.  The attn case times a warm back-to-back burst instead (mean per call).
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402
from token_locking_b200 import runtime as rt  # noqa: E402


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]) * 1e9, float(d["bf16_tflops"]) * 1e12, "measured"
    except Exception:
        return 6650e9, 1590e12, "fallback"


class _Flush:
    def __init__(self, dev):
        self.buf = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)

    def __call__(self):
        self.buf.fill_(1)


WARMUP = 5


def _time(fn, iters, flush, warmup=WARMUP):
    """Median CUDA-event time (ms) of one call over `iters` calls, each after an
    L2 flush, following `warmup` untimed calls."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(iters):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return float(np.median(times))


def layer_work(shape, M, N):
    d, f = shape.d_model, shape.d_ffn
    flops = 2.0 * M * (4 * d * d + 3 * d * f) + 4.0 * M * N * d
    byts = 2.0 * (4 * d * d + 3 * d * f) + 2.0 * 2 * N * d + 2.0 * 2 * M * d + 4.0 * 2 * M * d
    return flops, byts


def bench_layer(args, dev):
    shape = wl.ModelShape(n_layers=1, d_model=4096, n_heads=32, head_dim=128, d_ffn=12288,
                          vocab=126464, mask_id=126336, rope_theta=500000.0)
    N = wl.LAYER_MICRO_N
    w = wl.torch_weights(shape, dev)
    model = rt.Model(shape, w, "bf16")
    cache = rt.KVCache(model, 1, N)
    g = torch.Generator(device=dev).manual_seed(wl.SEED_MICRO)
    if not args.no_tune:
        model.autotune(cache, N)
    k, v = cache.view(0)
    k.normal_(generator=g)
    v.normal_(generator=g)
    pb, pf, src = _peaks()
    flush = _Flush(dev)
    out = []
    torch.cuda.synchronize()
    torch.cuda.profiler.start()          # ncu --profile-from-start off captures from here
    for M in args.m:
        act = rt.Active(1, N)
        act.load([wl.np_active_subset(N, M)])
        h0 = torch.randn((M, shape.d_model), device=dev, generator=g)
        h = h0.clone()

        def fn():
            h.copy_(h0)
            rt.layer_forward(model, cache, act, 0, h)

        ms = _time(fn, args.iters, flush)
        model.timing_enable(True)
        model.timing_read(reset=True)
        fn()
        torch.cuda.synchronize()
        tim = model.timing_read(reset=True)
        model.timing_enable(False)
        fl, by = layer_work(shape, M, N)
        roof = max(fl / pf, by / pb) * 1e3
        rec = {"case": "layer", "M": M, "N": N, "ms": round(ms, 4), "roofline_ms": round(roof, 4),
               "frac": round(roof / ms, 4), "bound": "tensor" if fl / pf > by / pb else "hbm",
               "gemm_ms": round(tim["gemm"]["ms"], 4), "attn_ms": round(tim["attn"]["ms"], 4),
               "gemm_GBps": round(tim["gemm"]["bytes"] / tim["gemm"]["ms"] / 1e6, 1),
               "gemm_TFLOPs": round(tim["gemm"]["flops"] / tim["gemm"]["ms"] / 1e9, 1),
               "attn_TFLOPs": round(tim["attn"]["flops"] / max(tim["attn"]["ms"], 1e-9) / 1e9, 1),
               "peaks": src}
        print(json.dumps(rec), flush=True)
        out.append(rec)
        act.close()
    torch.cuda.profiler.stop()
    model.close()
    return out


def bench_lock(args, dev):
    V = wl.LLADA8B.vocab
    pb, pf, src = _peaks()
    flush = _Flush(dev)
    torch.cuda.synchronize()
    torch.cuda.profiler.start()
    for M in args.m:
        z, zp, _ = wl.torch_lock_logits(M, V, dev)
        lse_prev = torch.logsumexp(zp.float(), 1).contiguous()
        act = rt.Active(1, M)
        R = M
        outs = dict(lse=torch.zeros(R, device=dev), kl=torch.zeros(R, device=dev),
                    unc=torch.zeros(R, device=dev), conf=torch.zeros(R, device=dev),
                    am=torch.zeros(R, device=dev, dtype=torch.int32),
                    lock=torch.zeros(R, device=dev, dtype=torch.uint8))
        masked = torch.zeros(R, device=dev, dtype=torch.uint8)
        locked = torch.zeros(R, device=dev, dtype=torch.uint8)
        lock_t = torch.zeros(R, device=dev, dtype=torch.int32)
        for eps in wl.LOCK_MICRO_EPS:
            def fn():
                rt.kl_lock(act, V, wl.LLADA8B.mask_id, z, zp, lse_prev, outs["lse"], masked,
                           outs["kl"], outs["unc"], outs["conf"], outs["am"], outs["lock"],
                           eps=eps, gate_q=wl.LOCK_MICRO_GATE_Q)

            act.reset()
            ms = _time(fn, args.iters, flush)
            n_lock = int(outs["lock"].sum())
            rt.compact_active(act, outs["lock"], locked, lock_t, 1)
            m_after = int(act.counts()[0])
            by = 4.0 * M * V + 16.0 * M
            roof = by / pb * 1e3
            print(json.dumps({"case": "lock", "M": M, "V": V, "eps": eps, "gate_q": 0.5,
                              "ms": round(ms, 4), "roofline_ms": round(roof, 4),
                              "frac": round(roof / ms, 4),
                              "GBps": round(by / ms / 1e6, 1), "locked": n_lock,
                              "M_after": m_after, "peaks": src}), flush=True)
        act.close()
    torch.cuda.profiler.stop()


def bench_decode(args, dev):
    setup = wl.cfg_long8b() if args.workload == "long8b" else wl.cfg_full8b(eps=0.05)
    shape = setup.shape
    w = wl.torch_weights(shape, dev)
    model = rt.Model(shape, w, "bf16")
    s = rt.Sampler(model, setup.batch, setup.prompt_len, setup.gen_len, setup.steps,
                   setup.block_len, setup.tokens_per_step, setup.eps, setup.gate_q)
    if args.kv_reuse > 1:
        s.set_kv_reuse(args.kv_reuse)
    max_rows = setup.batch * (setup.prompt_len + setup.gen_len)
    if args.tuning_in:
        for kind, M, bn, sp, var in json.load(open(args.tuning_in)):
            model.set_tuning(kind, M, bn, sp, var)
    elif not args.no_tune:
        s.autotune()
    if args.tuning_out:
        json.dump([[kind, M, *model.tuning(kind, M)] for kind in range(5)
                   for M in range(1, max_rows + 1)], open(args.tuning_out, "w"))
    prompts = torch.from_numpy(wl.np_prompts(setup.batch, setup.prompt_len, shape.vocab,
                                             shape.mask_id)).to(dev)
    s.start(prompts)
    if args.windows:
        # profiled windows of --steps steps starting at the given step indices;
        # the library's own count of algorithmic GEMM bytes over the same launches
        t, tot_b, tot_n = 0, 0.0, 0
        for w0 in (int(x) for x in args.windows.split(",")):
            while t < w0:
                s.step()
                t += 1
            torch.cuda.synchronize()
            model.timing_read(reset=True)
            model.timing_enable(True)
            torch.cuda.profiler.start()
            for _ in range(args.steps):
                s.step()
                t += 1
            torch.cuda.synchronize()
            torch.cuda.profiler.stop()
            tim = model.timing_read(reset=True)
            model.timing_enable(False)
            tot_b += tim["gemm"]["bytes"]
            tot_n += tim["gemm"]["launches"]
        print(json.dumps({"case": "decode_windows", "windows": args.windows, "steps": args.steps,
                          "gemm_launches": tot_n,
                          "gemm_algorithmic_bytes_per_launch": round(tot_b / max(1, tot_n))}))
        return
    for _ in range(args.skip):           # advance to later (smaller M) steps untimed
        s.step()
    torch.cuda.synchronize()
    torch.cuda.profiler.start()          # ncu --profile-from-start off captures from here
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    evs[0].record()
    for t in range(args.steps):
        s.step()
        evs[t + 1].record()
    torch.cuda.synchronize()
    torch.cuda.profiler.stop()
    ms = [evs[t].elapsed_time(evs[t + 1]) for t in range(args.steps)]
    print(json.dumps({"case": "decode", "steps": args.steps, "ms": [round(x, 3) for x in ms]}))


def bench_attn(args, dev):
    """sl_attention alone at the LLaDA-8B head layout (32 x 128), warm, for each
    layout (queries per CTA, key split) and the library's own choice: 128
    queries per CTA is the tensor-core kernel, 16/32/64 the mma.sync one.
    --batch B runs B sequences of M active rows each."""
    shape = wl.LLADA8B
    d = shape.d_model
    tiny = wl.ModelShape(n_layers=1, d_model=d, n_heads=shape.n_heads, head_dim=128, d_ffn=256,
                         vocab=256, mask_id=255, rope_theta=shape.rope_theta)
    model = rt.Model(tiny, wl.torch_weights(tiny, dev), "bf16")
    g = torch.Generator(device=dev).manual_seed(5)
    B = args.batch
    for n_ctx in args.n_ctx:
        cache = rt.KVCache(model, B, n_ctx)
        k, v = cache.view(0)
        k.copy_(torch.randn(k.shape, device=dev, generator=g).to(torch.bfloat16))
        v.copy_(torch.randn(v.shape, device=dev, generator=g).to(torch.bfloat16))
        for M in args.m:
            if M > n_ctx:
                continue
            act = rt.Active(B, n_ctx)
            act.load([np.sort(np.random.default_rng(M + b).choice(n_ctx, M, replace=False))
                      for b in range(B)])
            q = torch.randn((B * M, d), device=dev, generator=g).to(torch.bfloat16)
            o = torch.empty((B * M, d), device=dev, dtype=torch.bfloat16)
            for lay in args.attn_layouts:
                qpc, sp = lay[0], lay[1]
                kt = lay[2] if len(lay) > 2 else 0
                model.set_attention(qpc, sp, kt)

                def fn():
                    rt.attention(model, cache, act, 0, q, o)

                for _ in range(5):
                    fn()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(args.iters):
                    fn()
                e1.record()
                torch.cuda.synchronize()
                us = e0.elapsed_time(e1) * 1e3 / args.iters
                fl = 4.0 * B * M * n_ctx * d
                print(json.dumps({"case": "attn", "batch": B, "M": M, "n_ctx": n_ctx,
                                  "q_per_cta": qpc, "key_tile": kt,
                                  "splits": sp, "us": round(us, 2),
                                  "TFLOPs": round(fl / us / 1e6, 1)}), flush=True)
        cache.close()
    model.set_attention(0, 0)


def bench_gemm(args, dev):
    from token_locking_b200 import _abi as A
    d, f, V = 4096, 12288, 126464
    pb, pf, src = _peaks()
    g = torch.Generator(device=dev).manual_seed(3)

    def w(*s):
        return (torch.randn(s, device=dev, generator=g) * 0.02).to(torch.bfloat16)

    shapes = {"qkv": (3 * d, d), "o": (d, d), "gu": (2 * f, d), "down": (d, f)}
    if args.head:
        shapes["head"] = (V, d)
    if args.gemms:
        shapes = {k: shapes[k] if k != "head" else (V, d) for k in args.gemms.split(",")}
    # fixed tilings "bn:variant:splits,..." instead of the sweep
    fixed = [tuple(int(x) for x in t.split(":")) for t in args.tiles.split(",")] if args.tiles else None
    weights = {k: w(n, kk) for k, (n, kk) in shapes.items() if k != "gu"}
    wg, wu = w(f, d), w(f, d)
    flush = _Flush(dev)
    for M in args.m:
        for name, (N, K) in shapes.items():
            a = w(M, K)
            outb = torch.zeros((M, N), device=dev, dtype=torch.bfloat16)
            outf = torch.zeros((M, N), device=dev, dtype=torch.float32)
            outa = torch.zeros((M, f), device=dev, dtype=torch.bfloat16)
            sweep = fixed or [(bn, variant, sp)
                              for bn, variant in ((256, 0), (128, 0), (64, 0), (256, 1), (128, 1),
                                                  (64, 1), (256, 2), (128, 2))
                              for sp in (1, 2, 3, 4, 6, 8, 9, 12, 16, -1)]
            torch.cuda.profiler.start()          # ncu --profile-from-start off captures from here
            for bn, variant, sp in sweep:
                if bn < 128 and name == "qkv":
                    continue
                if (variant > 0 and M <= 128 and not fixed) or N % bn:
                    continue
                if sp != 1 and name == "head":
                    continue
                if variant == 3 and (M > 256 or bn != 128 or sp < 1 or name == "head"):
                    continue                     # swapped operands: few rows, 128 weight rows
                if True:
                    acc = sp != 1 or variant == 3  # fp32 partial sums (split K, swapped operands)
                    if name == "gu":
                        epi, b, b2, out = ((A.GEMM_ACCUM, wg, wu, outf) if acc else
                                           (A.GEMM_SWIGLU, wg, wu, outa))
                    elif name in ("o", "down"):
                        epi, b, b2, out = A.GEMM_RESID, weights[name], None, outf
                    else:
                        epi, b, b2, out = ((A.GEMM_ACCUM, weights[name], None, outf) if acc
                                           else (A.GEMM_STORE, weights[name], None, outb))

                    def fn():
                        rt.gemm_bf16(epi, a, b, out, b2=b2, bn=bn, splits=sp, variant=variant)

                    ms = _time(fn, args.iters, flush)
                    by = 2.0 * (N * K + M * K + M * N)
                    fl = 2.0 * M * N * K
                    print(json.dumps({"case": "gemm", "M": M, "gemm": name, "bn": bn,
                                      "variant": variant, "splits": sp,
                                      "us": round(ms * 1e3, 2),
                                      "GBps": round(by / ms / 1e6, 1),
                                      "TFLOPs": round(fl / ms / 1e9, 1)}), flush=True)
            torch.cuda.profiler.stop()
            if fixed:
                continue
            # the library's own choice
            if name == "gu":
                epi, b, b2, out = A.GEMM_SWIGLU, wg, wu, outa
            elif name in ("o", "down"):
                epi, b, b2, out = A.GEMM_RESID, weights[name], None, outf
            else:
                epi, b, b2, out = A.GEMM_STORE, weights[name], None, outb

            def fn():
                rt.gemm_bf16(epi, a, b, out, b2=b2, bn=0, splits=0)

            ms = _time(fn, args.iters, flush)
            print(json.dumps({"case": "gemm", "M": M, "gemm": name, "bn": 0, "variant": -1,
                              "splits": 0, "us": round(ms * 1e3, 2),
                              "GBps": round(2.0 * (N * K + M * K + M * N) / ms / 1e6, 1)}),
                  flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["layer", "lock", "decode", "gemm", "attn"])
    ap.add_argument("--head", action="store_true")
    ap.add_argument("--gemms", default=None, help="gemm case: comma list of qkv,o,gu,down,head")
    ap.add_argument("--tiles", default=None, help="gemm case: fixed bn:variant:splits list")
    ap.add_argument("--no-tune", action="store_true")
    ap.add_argument("--m", default=None)
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--steps", type=int, default=8)
    ap.add_argument("--skip", type=int, default=0, help="decode: denoising steps run before timing")
    ap.add_argument("--windows", default=None,
                    help="decode: profile --steps steps at each of these step indices")
    ap.add_argument("--n-ctx", default="384,2048", help="attn: key counts")
    ap.add_argument("--batch", type=int, default=1, help="attn: sequences")
    ap.add_argument("--workload", default="full8b", choices=["full8b", "long8b"],
                    help="decode: batch 1 x 384 positions, or batch 4 x 2048")
    ap.add_argument("--layouts", default="0:0,128:1:64,128:1:128,128:2:64,128:4:64,256:1,256:2,"
                    "16:1,32:1,64:1,16:2,16:4,64:4",
                    help="attn: queries-per-CTA:splits[:key tile] list (0:0 = the library's choice)")
    ap.add_argument("--tuning-out", default=None, help="decode: save the autotuned GEMM tilings")
    ap.add_argument("--kv-reuse", type=int, default=1,
                    help="decode: K/V reuse for the active rows, all recomputed every R steps")
    ap.add_argument("--tuning-in", default=None,
                    help="decode: load GEMM tilings instead of autotuning (e.g. under a profiler)")
    args = ap.parse_args()
    default = {"layer": wl.LAYER_MICRO_M, "lock": wl.LOCK_MICRO_M, "decode": (),
               "gemm": (8, 64, 128, 200, 256, 384, 1024), "attn": (8, 58, 198, 384)}[args.case]
    args.n_ctx = [int(x) for x in args.n_ctx.split(",")]
    args.attn_layouts = [tuple(int(v) for v in x.split(":")) for x in args.layouts.split(",")]
    args.m = [int(x) for x in args.m.split(",")] if args.m else list(default)
    dev = torch.device("cuda:0")
    {"layer": bench_layer, "lock": bench_lock, "decode": bench_decode,
     "gemm": bench_gemm, "attn": bench_attn}[args.case](args, dev)


if __name__ == "__main__":
    main()
