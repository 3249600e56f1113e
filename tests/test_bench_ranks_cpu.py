"""bench.py's host logic on the CPU: the replica plumbing on two gloo ranks (the
barrier, the max over ranks of a time, per-replica prompts, the whole-job rate,
the reference arm on rank 0 only), the workload flags, the clock summary, and
the per-step work behind the roofline fraction."""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    import workloads as wl
    ranks = bench.Ranks(world, "gloo", timeout_s=60)
    ranks.barrier()
    slowest = ranks.max(10.0 + 5.0 * rank)           # this rank's "time"
    prompts = wl.np_prompts(1, 16, 512, 511, seed=bench.replica_prompt_seed(rank))
    ref = bench.run_reference(None, rank, world) if rank != 0 else "skipped"
    ranks.close()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"max": slowest, "prompts": prompts.tolist(), "ref": ref}, f)


def test_two_gloo_ranks(tmp_path):
    mp.spawn(_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    r0 = json.load(open(tmp_path / "rank0.json"))
    r1 = json.load(open(tmp_path / "rank1.json"))
    assert r0["max"] == r1["max"] == 15.0              # both ranks see the slowest time
    assert r0["prompts"] != r1["prompts"]              # independent replicas
    assert r1["ref"] is None                           # the reference arm: rank 0 only


def test_aggregate_rate():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 3 decodes x 256 steps over the slowest rank's 1.5 s
    assert bench.aggregate_rate(2, 3 * 256, 1500.0) == 1024.0
    assert bench.aggregate_rate(1, 256, 1000.0) == 256.0


def test_batch_override():
    import types
    import pytest
    sys.path.insert(0, ROOT)
    import bench
    s = bench.make_setup("full8b", None, False, 8)
    assert (s.batch, s.n_ctx, s.steps) == (8, 384, 256)
    args = types.SimpleNamespace(workload="full8b")
    cfg = bench.workload_config(args, s, 2)
    assert cfg["global_batch"] == 16 and "batch 8" in cfg["workload"]
    assert bench.make_setup("long8b", None, False).batch == 4
    for bad in (0, 65):
        with pytest.raises(SystemExit):
            bench.make_setup("full8b", None, False, bad)


def test_ablation_and_gate_flags():
    import types
    import pytest
    sys.path.insert(0, ROOT)
    import bench
    s = bench.make_setup("full8b", None, False, None, None, "none")
    assert not s.no_kv_cache and not s.gate_only and s.gate_q < 0
    s = bench.make_setup("full8b", None, False, None, None, "no_kv_cache")
    assert s.no_kv_cache and not s.gate_only
    args = types.SimpleNamespace(workload="full8b")
    assert "no KV cache" in bench.workload_config(args, s, 1)["workload"]
    with pytest.raises(SystemExit):                  # gate-only needs the gate
        bench.make_setup("full8b", None, False, None, None, "gate_only")
    s = bench.make_setup("full8b", None, False, None, 0.5, "gate_only")
    assert s.gate_only and s.gate_q == 0.5
    cfg = bench.workload_config(args, s, 1)["workload"]
    assert "gate q=0.5" in cfg and "confidence gate only" in cfg
    for bad in (dict(gate_q=1.5), dict(ablation="nope")):
        kw = dict(gate_q=None, ablation="none")
        kw.update(bad)
        with pytest.raises(SystemExit):
            bench.make_setup("full8b", None, False, None, kw["gate_q"], kw["ablation"])
    # the command line reaches the same setup
    a = types.SimpleNamespace(workload="long8b", eps=None, scripted=False, batch=2, gate_q=None,
                              ablation="no_kv_cache")
    s = bench.setup_from_args(a)
    assert (s.batch, s.n_ctx, s.no_kv_cache, s.gate_q) == (2, 2048, True, 0.5)


def test_clock_sampler_summary(tmp_path):
    """The clocks object of the JSON line from nvidia-smi's CSV rows: median SM
    clock over the rows under load (power > 200 W), the max clock, and the
    throttle reasons seen active under load."""
    sys.path.insert(0, ROOT)
    import bench
    rows = [
        "0, 1980, 1965, 120.5, 0x0, Not Active, Not Active, Not Active, Not Active",   # idle
        "0, 1830, 1965, 980.1, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1820, 1965, 990.7, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1845, 1965, 960.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    path = tmp_path / "clocks.csv"
    path.write_text("\n".join(rows) + "\n")

    class Done:                       # stands in for the finished nvidia-smi process
        def terminate(self): pass
        def wait(self, timeout=None): return 0
        def kill(self): pass

    cs = bench.ClockSampler("GPU-x", str(path))
    cs.proc, cs.f = Done(), open(path)
    out = cs.stop()
    assert out["sm_mhz"] == 1830.0 and out["sm_max_mhz"] == 1965.0
    assert out["samples"] == 4 and out["samples_under_load"] == 3
    assert out["reasons"] == ["sw_power_cap"] and out["power_w_max"] == 990.7
    # a hardware slowdown under load is reported by name
    path.write_text("0, 1500, 1965, 700.0, 0x8, Active, Not Active, Not Active, Not Active\n")
    cs.f = open(path)
    assert bench.ClockSampler.stop(cs)["reasons"] == ["hw_slowdown"]
    # no nvidia-smi: no clocks object
    assert bench.ClockSampler("GPU-x", str(path)).stop() is None


def test_step_work_against_the_oracle_flop_model():
    """The bench's per-step roofline work: FLOPs equal the oracle's FLOP model
    (written separately), and the bytes at the LLaDA-8B shape match the stated
    figures (15.0 GB of weights; K/V, posterior and gather terms)."""
    sys.path.insert(0, ROOT)
    import bench
    import workloads as wl
    from oracle import surelock as osl
    shape = wl.LLADA8B
    for m, n in ((1, 384), (58, 384), (384, 384), (2048, 2048)):
        fl, _ = bench.step_work(shape, m, 1, n)
        assert fl == osl.flops_per_step(shape, m, n)
    _, b0 = bench.step_work(shape, 0, 1, 384)
    d, L, V = shape.d_model, shape.n_layers, shape.vocab
    weights = b0 - 1 * L * 2 * 384 * d * 2
    assert abs(weights / 1e9 - 15.0) < 0.05          # 2 (L (4d^2 + 3df) + Vd) bytes
    _, b1 = bench.step_work(shape, 1, 1, 384)
    assert b1 - b0 == L * 2 * d * 2 + 4 * V + 2 * d  # per active row: K/V write, posterior, gather
    _, b4 = bench.step_work(shape, 0, 4, 384)
    assert b4 - b0 == 3 * L * 2 * 384 * d * 2        # every sequence's cache is read


def test_trajectory_from_lock_steps():
    sys.path.insert(0, ROOT)
    import bench
    lock_t = np.array([-1, 0, 0, 2, -1, 1, 2, 2], dtype=np.int32)
    # all 8 rows active at step 0; 2 locked at step 0, 1 at step 1, 3 at step 2
    assert bench.trajectory_from_lock_t(lock_t, 4).tolist() == [8, 6, 5, 2]


def test_bench_step_unit():
    """A bench step is a whole decode for both workloads (unbiased for any K);
    --bench-step block takes one semi-autoregressive block (16 per long decode)."""
    import types
    sys.path.insert(0, ROOT)
    import bench
    long_ = bench.make_setup("long8b", None, False)
    short = bench.make_setup("full8b", None, False)
    a = types.SimpleNamespace(workload="long8b", bench_step="auto")
    assert bench.bench_unit_steps(a, long_) == 512
    assert "full decode" in bench.workload_config(a, long_, 1)["bench_step"]
    a = types.SimpleNamespace(workload="long8b", bench_step="block")
    assert bench.bench_unit_steps(a, long_) == 32 == long_.steps // 16
    assert "block" in bench.workload_config(a, long_, 1)["bench_step"]
    a = types.SimpleNamespace(workload="full8b", bench_step="auto")
    assert bench.bench_unit_steps(a, short) == 256
    assert "full decode" in bench.workload_config(a, short, 1)["bench_step"]
    a = types.SimpleNamespace(workload="long8b", bench_step="decode")
    assert bench.bench_unit_steps(a, long_) == 512
    # instrumented / end-to-end passes: about 20 s of decodes, at least one
    assert bench.aux_decodes(20, 19600.0) == 1
    assert bench.aux_decodes(20, 1250.0) == 16
    assert bench.aux_decodes(2, 100.0) == 2


def _bench_args(**kw):
    import types
    base = dict(gpus=1, steps=1, warmup=0, impl="reference", workload="long8b", bench_step="auto",
                eps=None, scripted=False, batch=None, gate_q=None, ablation="none",
                head_fusion="on", no_cpu_baseline=False)
    base.update(kw)
    return types.SimpleNamespace(**base)


def test_reference_arm_finds_the_stored_trajectory():
    """The reference arm weighs its oracle samples by the M_t trajectory a GPU
    run of the same workload recorded (profiles/trajectory_*.json): one per
    stored workload, as long as the decode, starting from every row active and
    never growing."""
    sys.path.insert(0, ROOT)
    import bench
    import numpy as np
    for kw in ({}, {"workload": "full8b", "eps": 0.05}, {"workload": "full8b", "eps": 0.0},
               {"workload": "full8b", "eps": 0.01}, {"workload": "full8b", "eps": 0.05,
                                                      "scripted": True}):
        a = _bench_args(**kw)
        setup = bench.setup_from_args(a)
        got = bench.stored_trajectory(bench.workload_config(a, setup, 1)["workload"])
        assert got is not None, kw
        traj, name = got
        assert len(traj) == setup.steps, (kw, name)
        assert traj[0] == setup.batch * setup.n_ctx
        assert np.all(np.diff(traj) <= 0) and traj[-1] >= 1
    # a workload no GPU run recorded has none
    a = _bench_args(workload="full8b", eps=0.2)
    setup = bench.setup_from_args(a)
    assert bench.stored_trajectory(bench.workload_config(a, setup, 1)["workload"]) is None


def test_head_fusion_arm_is_named_in_the_workload():
    sys.path.insert(0, ROOT)
    import bench
    on, off = _bench_args(), _bench_args(head_fusion="off")
    setup = bench.setup_from_args(on)
    w_on = bench.workload_config(on, setup, 1)["workload"]
    w_off = bench.workload_config(off, setup, 1)["workload"]
    assert w_on != w_off and "separate pass" in w_off and "separate pass" not in w_on


def test_kv_reuse_arm_is_named_and_checked():
    sys.path.insert(0, ROOT)
    import bench
    plain, reuse = _bench_args(), _bench_args(kv_reuse=4)
    s0, s4 = bench.setup_from_args(plain), bench.setup_from_args(reuse)
    assert s0.kv_reuse == 1 and s4.kv_reuse == 4
    w0 = bench.workload_config(plain, s0, 1)["workload"]
    w4 = bench.workload_config(reuse, s4, 1)["workload"]
    assert "K/V reuse" in w4 and "every 4 steps" in w4 and "K/V reuse" not in w0
    for bad in (dict(kv_reuse=0), dict(kv_reuse=2, scripted=True, workload="full8b"),
                dict(kv_reuse=2, ablation="no_kv_cache")):
        with pytest.raises(SystemExit):
            bench.setup_from_args(_bench_args(**bad))


def test_carry_line_arithmetic():
    sys.path.insert(0, ROOT)
    import bench
    got = bench.carry_line({"ms": 20.0, "bytes": 100e9 * 0.02, "launches": 768}, 2,
                           {"hbm_gbs": 6400.0})
    assert got == {"ms_per_decode": 10.0, "launches_per_decode": 384, "achieved_gbs": 100.0,
                   "frac_hbm": 0.0156}
    assert bench.carry_line({"ms": 0.0, "bytes": 0.0, "launches": 0}, 1,
                            {"hbm_gbs": 6400.0})["achieved_gbs"] is None


def test_reference_arm_weighs_reuse_workloads_by_their_computed_rows():
    """Under K/V reuse the reference arm's samples are weighted by the rows each
    step computed: all rows at step 0 (a refresh step), and fewer than the
    active rows in total (the two arrays come from two decodes of the run,
    which may lock a few rows at different steps, so they are not compared
    step by step)."""
    sys.path.insert(0, ROOT)
    import json as _json
    import bench
    import numpy as np
    for kw in ({"kv_reuse": 2}, {"kv_reuse": 4}, {"kv_reuse": 4, "eps": 0.01},
               {"kv_reuse": 4, "eps": 0.0}, {"kv_reuse": 4, "workload": "full8b", "eps": 0.05},
               {"kv_reuse": 4, "workload": "full8b", "eps": 0.0}):
        a = _bench_args(**kw)
        setup = bench.setup_from_args(a)
        got = bench.stored_trajectory(bench.workload_config(a, setup, 1)["workload"])
        assert got is not None, kw
        rows, name = got
        rec = _json.load(open(os.path.join(ROOT, "profiles", name)))
        m_t = np.asarray(rec["M_t"])
        assert len(rows) == len(m_t) == setup.steps, (kw, name)
        assert rows[0] == m_t[0] == setup.batch * setup.n_ctx
        assert np.all((rows >= 0) & (rows <= setup.batch * setup.n_ctx))
        assert rows.sum() < m_t.sum()
