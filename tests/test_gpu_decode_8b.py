"""Whole LLaDA-8B-shape decodes (32 layers, d_model 4096, 32 heads of 128,
d_ffn 12288, vocabulary 126464; random-init bf16 weights, seed 0, the bench's
prompts), teacher-forced against the oracle at the listed steps, in the launch
configuration the bench times (autotuned GEMM tilings, the default attention):

* batch 1, 128 prompt + 256 masked positions, 256 steps in blocks of 32, one
  token per step, for eps in {0, 0.01, 0.05} and the scripted schedule that
  takes M_t linearly down to 10% of N; checked at steps 0, 1, 2, 31, 32, 128,
  254 and 255 on every active row;
* batch 4, 1024 prompt + 1024 masked positions (N = 2048), 512 steps in blocks
  of 64, two tokens per step, eps 0.05 with the confidence gate at q = 0.5;
  checked on every active row at steps 255, 510 and 511, and at step 1 (every
  row active) on 32 sampled rows per sequence with per-block teacher forcing
  (each block attends over the GPU's cache after the step, which holds every
  active row's fresh K/V, so the oracle's work scales with the sample).

At each checked step: logits and log-probs within the bf16 tolerance of a
whole 32-block step (16 bf16 ulps of the largest logit, 0.5 for |z| in
[4, 8); see parity_util.deep_logit_tol), the fresh K/V the step wrote within
3e-2 relative (6e-2 for the eps = 0 arm's late steps, where every block input
carries the amplified difference), and the sure test, gate, unmasking and
compaction decided by the oracle on the GPU's own logits equal to the GPU's
outside the rounding bands.

Block by block: at steps 0 and 254 of the eps = 0 decode (every row active),
each of the 32 blocks is run on the oracle's own block input and must match
the oracle's block closely (parity_util.BLOCK_ULPS, BLOCK_RMS_FRAC) at every
depth and step; the chained difference is recorded alongside.

The observed errors are appended to the JSON-lines file named by
SL_PARITY_LOG when that variable is set.
"""
import json
import os
import time

import numpy as np
import pytest
import torch

import parity_8b as p8
import workloads as wl
from parity_util import BLOCK_RMS_FRAC, BLOCK_ULPS, bf16_ulp, deep_logit_tol
from oracle import model as om
from token_locking_b200 import runtime as rt

pytestmark = pytest.mark.gpu

CHECK4 = (0, 1, 2, 31, 32, 128, 254, 255)
CHECK5_FULL = (255, 510, 511)
CHECK5_SAMPLED = (1,)
SAMPLE5 = 32
KV_TOL = 3e-2


@pytest.fixture(scope="module")
def llada8b(cuda_dev):
    w = wl.torch_weights(wl.LLADA8B, cuda_dev)
    model = rt.Model(wl.LLADA8B, w, "bf16")
    w_or = p8.oracle_weights(w)
    yield model, w, w_or
    model.close()


def _log(rec):
    path = os.environ.get("SL_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")


def _rel(a, b):
    return float(np.abs(a - b).max() / max(1.0, float(np.abs(b).max())))


def _lp_err(z_gpu, z_or):
    """max |log p_gpu - log p_oracle| over the row's vocabulary (float64)."""
    def lsm(z):
        z = z.astype(np.float64)
        m = z.max(axis=-1, keepdims=True)
        return z - (m + np.log(np.exp(z - m).sum(axis=-1, keepdims=True)))
    return float(np.abs(lsm(z_gpu) - lsm(z_or)).max())


def _decode(llada8b, dev, setup, full_steps, sampled_steps, name, kv_tol=KV_TOL):
    model, _, w_or = llada8b
    shape = setup.shape
    B = setup.batch
    R = setup.kv_reuse
    s = rt.Sampler(model, B, setup.prompt_len, setup.gen_len, setup.steps, setup.block_len,
                   setup.tokens_per_step, setup.eps, setup.gate_q, setup.scripted)
    if R > 1:
        s.set_kv_reuse(R)
    s.autotune()
    prompts = wl.np_prompts(B, setup.prompt_len, shape.vocab, shape.mask_id,
                            seed=wl.SEED_PROMPTS)
    s.start(torch.from_numpy(prompts).to(dev))
    stats = {"mismatch": 0, "ambiguous": 0, "locks": 0, "unmask_amb": 0}
    worst = {"logits": 0.0, "kv": 0.0, "lp": 0.0}
    mask_prev = None          # K/V reuse: mask flags at the start of the previous step
    for t in range(setup.steps):
        if R > 1:
            mask_start = s.state()["masked"].cpu().numpy().astype(bool)
            if mask_prev is None:
                mask_prev = mask_start
        if t not in full_steps and t not in sampled_steps:
            s.step()
            if R > 1:
                mask_prev = mask_start
            continue
        full = t in full_steps
        snap = p8.snapshot(s, setup, want_cache=full)
        s.step()
        torch.cuda.synchronize()
        rt.device_check()
        g = p8.gpu_after(s, setup, t)
        t0 = time.time()
        refresh = R <= 1 or t % R == 0
        comp_gpu = None if refresh else s.state()["computed"].positions()
        j0 = 0
        for b in range(B):
            A_all = snap["act"][b]
            # the rows the step computes (all active rows unless K/V reuse
            # skips the unmasked ones between refreshes)
            A = A_all if refresh else A_all[snap["masked"][b, A_all] | mask_prev[b, A_all]]
            if not refresh:
                np.testing.assert_array_equal(comp_gpu[b], A)
                reused = np.setdiff1d(A_all, A)
                if full and len(reused):
                    kr, vr = p8.cache_rows(s, setup, b, reused)
                    np.testing.assert_array_equal(kr, snap["ck"][b][:, reused])
                    np.testing.assert_array_equal(vr, snap["cv"][b][:, reused])
                    np.testing.assert_array_equal(g["z"][b, reused], snap["z_prev"][b, reused])
            m = len(A)
            if m == 0:
                continue
            if full:
                z, ck, cv = p8.oracle_logits_full(shape, w_or, snap, b, A)
                zg = g["z"][b, A]
                kg, vg = p8.cache_rows(s, setup, b, A)
                kv = max(_rel(kg, ck[:, A]), _rel(vg, cv[:, A]))
                n_rows = m
            else:
                rng = np.random.default_rng(100 * t + b)
                idx = np.sort(rng.choice(m, min(SAMPLE5, m), replace=False))
                k_all, v_all = p8.cache_rows(s, setup, b, np.arange(setup.n_ctx))
                z, ks, vs = p8.oracle_logits_sampled(shape, w_or, snap["tokens"][b], A, idx,
                                                     k_all, v_all)
                zg = g["z"][b, A[idx]]
                kv = max(_rel(k_all[:, A[idx]], ks), _rel(v_all[:, A[idx]], vs))
                n_rows = len(idx)
            zerr = float(np.abs(zg - z).max())
            lperr = _lp_err(zg, z)
            worst["logits"] = max(worst["logits"], zerr)
            worst["kv"] = max(worst["kv"], kv)
            worst["lp"] = max(worst["lp"], lperr)
            _log({"test": name, "t": t, "b": b, "M": m, "rows_checked": n_rows,
                  "logits_max_abs_err": zerr, "logp_max_abs_err": lperr, "kv_max_rel_err": kv,
                  "z_max_abs": float(np.abs(z).max()), "oracle_s": round(time.time() - t0, 1)})
            tol = deep_logit_tol(float(np.abs(z).max()))
            assert zerr <= tol, f"{name} t={t} b={b}: logits err {zerr} > {tol}"
            assert kv <= kv_tol, f"{name} t={t} b={b}: fresh K/V rel err {kv}"
            assert lperr <= tol, f"{name} t={t} b={b}: log-prob err {lperr} > {tol}"
            p8.check_decisions(setup, t, b, A, snap, g, j0, stats,
                               A_all=None if refresh else A_all)
            j0 += m            # per-row outputs run over all sequences in order
        if R > 1:
            mask_prev = mask_start
    final = s.state()
    assert int(final["masked"].sum().item()) == 0, "positions left masked at the end"
    _log({"test": name, "summary": stats, "worst": worst})
    s.close()
    assert stats["mismatch"] == 0, stats
    return stats, worst


@pytest.mark.parametrize("arm", ["eps0", "eps0.01", "eps0.05", "scripted"])
def test_llada8b_b1_n384_teacher_forced(llada8b, cuda_dev, arm):
    setup = (wl.cfg_full8b(eps=0.05, scripted=True) if arm == "scripted"
             else wl.cfg_full8b(eps=float(arm[3:])))
    # with eps = 0 every row stays active, and a late step's K/V come from block
    # inputs that carry the amplified difference (up to 4 % of the residual's rms
    # in the last blocks at step 254)
    stats, _ = _decode(llada8b, cuda_dev, setup, CHECK4, (), f"cfg4-{arm}",
                       kv_tol=2 * KV_TOL if arm == "eps0" else KV_TOL)
    if arm == "eps0":
        assert stats["locks"] == 0
    else:
        assert stats["locks"] > 0


def test_llada8b_b1_n384_kv_reuse_teacher_forced(llada8b, cuda_dev):
    """The composition with K/V reuse (all active rows recomputed every 4 steps)
    at the batch-1 shape: steps 1, 2, 31, 254 and 255 fall between refreshes,
    where the computed list, the computed rows' logits, K/V and decisions, and
    the reused rows' unchanged cache entries and carried logits are checked."""
    import dataclasses
    setup = dataclasses.replace(wl.cfg_full8b(eps=0.05), kv_reuse=4)
    stats, _ = _decode(llada8b, cuda_dev, setup, CHECK4, (), "cfg4-reuse4")
    assert stats["locks"] > 0


def test_llada8b_b4_n2048_teacher_forced(llada8b, cuda_dev):
    setup = wl.cfg_long8b()
    stats, _ = _decode(llada8b, cuda_dev, setup, CHECK5_FULL, CHECK5_SAMPLED, "cfg5")
    assert stats["locks"] > 0


def test_llada8b_blocks_teacher_forced(llada8b, cuda_dev):
    """Every block of the 32 on the oracle's own block input (sl_layer_forward
    on all 384 rows of a fresh cache), at steps 0 and 254 of the batch-1 eps = 0
    decode: the block's output within BLOCK_ULPS bf16 ulps of the largest entry
    of its update and BLOCK_RMS_FRAC of the update's rms, at every depth and at
    both steps.  The chained difference (the GPU's blocks one after another)
    and the logits through the oracle's head are logged and held to the
    whole-step tolerance."""
    model, _, w_or = llada8b
    shape = wl.LLADA8B
    setup = wl.cfg_full8b(eps=0.0)
    s = rt.Sampler(model, 1, setup.prompt_len, setup.gen_len, setup.steps, setup.block_len,
                   setup.tokens_per_step, setup.eps, setup.gate_q, setup.scripted)
    s.autotune()
    prompts = wl.np_prompts(1, setup.prompt_len, shape.vocab, shape.mask_id,
                            seed=wl.SEED_PROMPTS)
    s.start(torch.from_numpy(prompts).to(cuda_dev))
    snaps = {}
    for t in range(255):
        if t in (0, 254):
            snaps[t] = s.state()["tokens"].cpu().numpy()[0].copy()
        s.step()
    torch.cuda.synchronize()
    s.close()
    N, d = setup.n_ctx, shape.d_model
    pos = np.arange(N, dtype=np.int32)
    for t, tok in snaps.items():
        hs = [np.asarray(w_or["tok_emb"][tok], dtype=np.float32)]
        ck = np.zeros((N, d), np.float32)
        cv = np.zeros((N, d), np.float32)
        for l in range(shape.n_layers):
            hs.append(om.layer_forward(shape, w_or["layers"][l], hs[-1], pos, ck, cv))
        cache = rt.KVCache(model, 1, N)
        act = rt.Active(1, N)
        act.load([pos])
        g = torch.from_numpy(hs[0]).to(cuda_dev)
        for l in range(shape.n_layers):
            x = torch.from_numpy(hs[l]).to(cuda_dev)
            rt.layer_forward(model, cache, act, l, x)
            rt.layer_forward(model, cache, act, l, g)
            torch.cuda.synchronize()
            rt.device_check()
            ref = hs[l + 1].astype(np.float64)
            upd = ref - hs[l]
            loc = np.abs(x.cpu().numpy() - ref)
            chn = np.abs(g.cpu().numpy() - ref)
            upd_rms = float(np.sqrt((upd ** 2).mean()))
            rec = {"test": "cfg4-blocks", "t": t, "layer": l,
                   "local_max": float(loc.max()), "local_rms": float(np.sqrt((loc ** 2).mean())),
                   "update_absmax": float(np.abs(upd).max()), "update_rms": upd_rms,
                   "chain_max": float(chn.max()), "chain_rms": float(np.sqrt((chn ** 2).mean())),
                   "residual_rms": float(np.sqrt((ref ** 2).mean()))}
            _log(rec)
            assert rec["local_max"] <= BLOCK_ULPS * bf16_ulp(rec["update_absmax"]), rec
            assert rec["local_rms"] <= BLOCK_RMS_FRAC * upd_rms, rec
        hf = om.rmsnorm(hs[-1], w_or["final_norm"], shape.rms_eps)
        z_ref = hf @ w_or["lm_head"].T
        hg = om.rmsnorm(g.cpu().numpy(), w_or["final_norm"], shape.rms_eps)
        zerr = float(np.abs(hg @ w_or["lm_head"].T - z_ref).max())
        _log({"test": "cfg4-blocks", "t": t, "logits_err_via_chain": zerr,
              "z_max_abs": float(np.abs(z_ref).max())})
        assert zerr <= deep_logit_tol(float(np.abs(z_ref).max())), (t, zerr)
        cache.close()
