"""Sure test, confidence gate, scripted schedule, compaction and unmasking on
the GPU against the oracle, on the same (bf16 or fp32) logits."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import surelock as osl
from token_locking_b200 import runtime as rt
from parity_util import BAND_D, BAND_U, compare_locks

pytestmark = pytest.mark.gpu


def _setup_logits(rows_total, V, dtype, seed, sigma_prev=0.05, spike=True):
    z, zp, _ = wl.np_lock_logits(rows_total, V, seed=seed, prev_sigma=sigma_prev,
                                 spike_frac=0.5 if spike else 0.0)
    if dtype == "bf16":
        z, zp = wl.round_bf16(z), wl.round_bf16(zp)
    return z.astype(np.float32), zp.astype(np.float32)


def _lse_of(z, lp):
    """logsumexp per row as z - log p at the row's largest (finite) logit."""
    i = np.argmax(z, axis=1)[:, None]
    return (np.take_along_axis(z, i, 1) - np.take_along_axis(lp, i, 1))[:, 0]


def _neg_inf_vocab_mask(z, zp, seed):
    """Logits with runs of -inf, as a vocabulary mask applied before the sure
    test leaves them: every row loses a contiguous range of ids plus scattered
    ids (same in both steps); the first rows lose the start of the vocabulary,
    so whole 8-wide groups at the front of a chunk are -inf; two rows gain a
    -inf in the previous step only (D must come out infinite there)."""
    rng = np.random.default_rng(seed)
    R, V = z.shape
    for r in range(R):
        a = 0 if r < 4 else int(rng.integers(0, V - 64))
        n = int(rng.integers(8, max(9, V // 4)))
        z[r, a:a + n] = -np.inf
        zp[r, a:a + n] = -np.inf
        cols = rng.choice(V, size=max(1, V // 50), replace=False)
        z[r, cols] = -np.inf
        zp[r, cols] = -np.inf
    for r in (R // 2, R - 1):
        col = int(np.argmax(np.where(np.isfinite(z[r]), z[r], -np.inf)))
        zp[r, col] = -np.inf
    return z, zp


def _run(dev, B, n_ctx, positions, V, dtype, eps, gate_q, has_prev, scripted_target, seed,
         masked_frac=0.3, sigma_prev=0.05, gate_only=False, neg_inf=False):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    R = B * n_ctx
    z, zp = _setup_logits(R, V, dtype, seed, sigma_prev)
    if neg_inf:
        z, zp = _neg_inf_vocab_mask(z, zp, seed + 7)
    rng = np.random.default_rng(seed + 100)
    masked = (rng.random(R) < masked_frac).astype(np.uint8)
    mask_id = V - 3
    # oracle inputs: log-probs of the exact stored values, lse_prev in fp64 -> fp32
    lp_cur_all = osl.log_softmax(z.astype(np.float64))
    lp_prev_all = osl.log_softmax(zp.astype(np.float64))
    lse_prev = _lse_of(zp.astype(np.float64), lp_prev_all).astype(np.float32)

    act = rt.Active(B, n_ctx)
    act.load(positions)
    cur = torch.from_numpy(z).to(dev, tdt)
    prv = torch.from_numpy(zp).to(dev, tdt)
    lse_p = torch.from_numpy(lse_prev).to(dev)
    lse_c = torch.zeros(R, device=dev)
    msk = torch.from_numpy(masked).to(dev)
    kl = torch.zeros(R, device=dev); unc = torch.zeros(R, device=dev)
    conf = torch.zeros(R, device=dev)
    amax = torch.zeros(R, device=dev, dtype=torch.int32)
    lock = torch.zeros(R, device=dev, dtype=torch.uint8)
    rt.kl_lock(act, V, mask_id, cur, prv, lse_p, lse_c, msk, kl, unc, conf, amax, lock,
               eps=eps, gate_q=gate_q, has_prev=has_prev, scripted_target=scripted_target,
               gate_only=gate_only)
    torch.cuda.synchronize()
    rt.device_check()
    out = dict(kl=kl.cpu().numpy(), unc=unc.cpu().numpy(), conf=conf.cpu().numpy(),
               argmax=amax.cpu().numpy(), lock=lock.cpu().numpy(), lse=lse_c.cpu().numpy())
    return act, out, dict(z=z, zp=zp, lp_cur=lp_cur_all, lp_prev=lp_prev_all, masked=masked,
                          mask_id=mask_id, lock_t=None), (msk, lock)


def _oracle_seq(pos_flat, ref, eps, gate_q, has_prev, scripted_target, gate_only=False):
    lp = ref["lp_cur"][pos_flat]
    lpp = ref["lp_prev"][pos_flat]
    D = osl.kl_rows(lp, lpp) if has_prev else np.full(len(pos_flat), np.inf)
    u = osl.uncertainty(lp)
    conf, pred = osl.prediction(lp, ref["mask_id"])
    masked = ref["masked"][pos_flat].astype(bool)
    hp = np.full(len(pos_flat), bool(has_prev))
    thr = osl.gate_threshold(u, gate_q) if gate_q >= 0 else np.inf
    if scripted_target >= 0:
        lock = osl.scripted_locks(D, masked, hp, pos_flat, len(pos_flat) - scripted_target)
    else:
        lock = osl.lock_decision(D, u, masked, hp, eps, gate_q, thr, gate_only)
    lse = _lse_of(ref["z"][pos_flat].astype(np.float64), lp)
    return dict(D=D, u=u, conf=conf, pred=pred, thr=thr, lock=lock, lse=lse)


CASES = [
    # B, n_ctx, counts, V, dtype, eps, gate_q, has_prev, scripted, sigma_prev
    (1, 64, [64], 512, "f32", 0.01, -1.0, True, -1, 0.2),
    (1, 300, [300], 4096, "bf16", 0.01, 0.5, True, -1, 0.2),
    (3, 100, [100, 7, 61], 1024, "bf16", 0.05, -1.0, True, -1, 0.2),
    (3, 100, [1, 0, 99], 1024, "bf16", 0.01, 0.5, True, -1, 0.2),
    (2, 50, [50, 33], 512, "f32", 0.01, 0.25, False, -1, 0.05),
    (2, 80, [80, 41], 2048, "bf16", 0.0, 0.5, True, -1, 0.05),
    (2, 80, [77, 41], 2048, "bf16", 0.0, -1.0, True, 30, 0.2),
    (1, 64, [64], 126464, "bf16", 0.01, 0.5, True, -1, 0.05),
    (1, 64, [64], 126464, "bf16", 0.05, 0.5, True, -1, 0.2),
    # the lock-test microbenchmark's larger row counts at the full vocabulary
    (1, 512, [512], 126464, "bf16", 0.01, 0.5, True, -1, 0.05),
    (1, 512, [512], 126464, "bf16", 0.05, 0.5, True, -1, 0.2),
    (1, 2048, [2048], 126464, "bf16", 0.01, 0.5, True, -1, 0.05),
    (1, 2048, [2048], 126464, "bf16", 0.05, 0.5, True, -1, 0.2),
]


NEG_INF_CASES = [
    (1, 64, [64], 1024, "f32", 0.05, 0.5, True, -1, 0.2),
    (2, 100, [100, 37], 4096, "bf16", 0.05, 0.5, True, -1, 0.2),
    (1, 64, [64], 126464, "bf16", 0.05, -1.0, True, -1, 0.2),
    (1, 64, [60], 2048, "bf16", 0.05, -1.0, False, -1, 0.2),
]


@pytest.mark.parametrize("case", CASES)
def test_kl_lock_matches_oracle(cuda_dev, case):
    _check_case(cuda_dev, case, neg_inf=False)


@pytest.mark.parametrize("case", NEG_INF_CASES)
def test_kl_lock_with_neg_inf_logits(cuda_dev, case):
    """Rows holding runs of -inf logits: no NaN anywhere, and the same D, u,
    conf, argmax, lse and lock flags as the oracle (0 log 0 = 0)."""
    _check_case(cuda_dev, case, neg_inf=True)


def _check_case(cuda_dev, case, neg_inf):
    B, n_ctx, counts, V, dtype, eps, gate_q, has_prev, scripted, sig = case
    rng = np.random.default_rng(sum(counts) + V)
    positions = [np.sort(rng.choice(n_ctx, c, replace=False)).astype(np.int32) for c in counts]
    act, out, ref, _ = _run(cuda_dev, B, n_ctx, positions, V, dtype, eps, gate_q, has_prev,
                            scripted, seed=V + B, sigma_prev=sig, neg_inf=neg_inf)
    M = sum(counts)
    for k in ("kl", "unc", "conf", "lse"):
        vals = out[k][:M] if k != "lse" else out[k]
        assert not np.any(np.isnan(vals)), f"NaN in {k}"
    j0 = 0
    n_mis = n_amb = 0
    for b in range(B):
        pf = positions[b] + b * n_ctx
        m = len(pf)
        o = _oracle_seq(pf, ref, eps, gate_q, has_prev, scripted)
        sl = slice(j0, j0 + m)
        np.testing.assert_array_equal(out["argmax"][sl], o["pred"])
        np.testing.assert_allclose(out["lse"][pf], o["lse"], rtol=2e-6, atol=2e-6)
        np.testing.assert_allclose(out["unc"][sl], o["u"], atol=2e-6)
        np.testing.assert_allclose(out["conf"][sl], o["conf"], rtol=2e-5, atol=1e-9)
        if has_prev:
            np.testing.assert_allclose(out["kl"][sl], o["D"], atol=2e-5, rtol=1e-4)
        else:
            assert np.all(np.isinf(out["kl"][sl]))
        if scripted >= 0:
            # exact: the schedule locks a fixed count by (D, position); ties in D
            # inside the band may swap, the count may not
            assert out["lock"][sl].sum() == o["lock"].sum()
            mis = np.sum(out["lock"][sl].astype(bool) != o["lock"])
            Ds = np.sort(o["D"][~ref["masked"][pf].astype(bool)])
            k = int(o["lock"].sum())
            if mis:
                assert k < len(Ds) and abs(Ds[k] - Ds[k - 1]) < BAND_D
        else:
            mi, am = compare_locks(out["lock"][sl], o["lock"], o["D"], o["u"], eps, o["thr"],
                                   gate_q >= 0)
            n_mis += mi
            n_amb += am
        j0 += m
    assert n_mis == 0, f"{n_mis} lock decisions differ outside the rounding band ({n_amb} ambiguous)"


def test_compaction_and_lock_bookkeeping(cuda_dev):
    B, n_ctx = 3, 200
    rng = np.random.default_rng(5)
    positions = [np.sort(rng.choice(n_ctx, c, replace=False)).astype(np.int32)
                 for c in (200, 17, 0)]
    act = rt.Active(B, n_ctx)
    act.load(positions)
    M = sum(len(p) for p in positions)
    lock_np = (rng.random(max(M, 1)) < 0.4).astype(np.uint8)[:M]
    lock = torch.from_numpy(np.concatenate([lock_np, np.zeros(B * n_ctx - M, np.uint8)])).to(cuda_dev)
    locked = torch.zeros(B * n_ctx, dtype=torch.uint8, device=cuda_dev)
    lock_t = torch.full((B * n_ctx,), -1, dtype=torch.int32, device=cuda_dev)
    rt.compact_active(act, lock, locked, lock_t, 7)
    torch.cuda.synchronize()
    new = act.positions()
    j0 = 0
    lk_all = locked.cpu().numpy()
    lt_all = lock_t.cpu().numpy()
    for b in range(B):
        m = len(positions[b])
        lk = lock_np[j0:j0 + m].astype(bool)
        want = osl.compact(positions[b], lk)
        np.testing.assert_array_equal(new[b], want)
        gone = positions[b][lk] + b * n_ctx
        assert np.all(lk_all[gone] == 1) and np.all(lt_all[gone] == 7)
        j0 += m
    assert lk_all.sum() == lock_np.sum()
    assert list(act.counts()) == [len(x) for x in new]


def test_compaction_of_every_row_and_of_none(cuda_dev):
    B, n_ctx = 2, 1500      # more rows than one block of threads
    act = rt.Active(B, n_ctx)
    act.reset()
    R = B * n_ctx
    locked = torch.zeros(R, dtype=torch.uint8, device=cuda_dev)
    lock_t = torch.full((R,), -1, dtype=torch.int32, device=cuda_dev)
    rt.compact_active(act, torch.zeros(R, dtype=torch.uint8, device=cuda_dev), locked, lock_t, 1)
    assert list(act.counts()) == [n_ctx, n_ctx]
    np.testing.assert_array_equal(act.positions()[1], np.arange(n_ctx))
    rt.compact_active(act, torch.ones(R, dtype=torch.uint8, device=cuda_dev), locked, lock_t, 2)
    assert list(act.counts()) == [0, 0]
    assert int(locked.sum()) == R and int((lock_t == 2).sum()) == R


@pytest.mark.parametrize("k", [1, 3, 40])
def test_unmask_topk_matches_oracle(cuda_dev, k):
    B, n_ctx = 2, 160
    rng = np.random.default_rng(k)
    positions = [np.sort(rng.choice(n_ctx, c, replace=False)).astype(np.int32) for c in (150, 90)]
    act = rt.Active(B, n_ctx)
    act.load(positions)
    M = sum(len(p) for p in positions)
    conf = np.round(rng.random(M), 2).astype(np.float32)      # many exact ties
    argmax = rng.integers(0, 500, M).astype(np.int32)
    masked = (rng.random(B * n_ctx) < 0.6).astype(np.uint8)
    tokens = rng.integers(0, 500, B * n_ctx).astype(np.int32)
    lo, hi = 40, 104
    pad = B * n_ctx - M
    t_conf = torch.from_numpy(np.concatenate([conf, np.zeros(pad, np.float32)])).to(cuda_dev)
    t_am = torch.from_numpy(np.concatenate([argmax, np.zeros(pad, np.int32)])).to(cuda_dev)
    t_tok = torch.from_numpy(tokens.copy()).to(cuda_dev)
    t_msk = torch.from_numpy(masked.copy()).to(cuda_dev)
    rt.unmask_topk(act, t_conf, t_am, lo, hi, k, t_tok, t_msk)
    torch.cuda.synchronize()
    want_tok, want_msk = tokens.copy(), masked.copy()
    j0 = 0
    for b in range(B):
        pos = positions[b]
        m = len(pos)
        sel = osl.unmask_select(pos, conf[j0:j0 + m].astype(np.float64),
                                masked[pos + b * n_ctx], lo, hi, k)
        want_tok[pos[sel] + b * n_ctx] = argmax[j0 + sel]
        want_msk[pos[sel] + b * n_ctx] = 0
        j0 += m
    np.testing.assert_array_equal(t_tok.cpu().numpy(), want_tok)
    np.testing.assert_array_equal(t_msk.cpu().numpy(), want_msk)


@pytest.mark.parametrize("eps,gate_q,has_prev", [(0.01, 0.5, True), (0.0, 0.25, True),
                                                 (-1.0, 0.9, True), (0.01, 0.5, False)])
def test_gate_only_matches_oracle(cuda_dev, eps, gate_q, has_prev):
    """The gate-only ablation: the gate alone decides, eps is ignored."""
    B, n_ctx, V = 3, 100, 1024
    rng = np.random.default_rng(77)
    positions = [np.sort(rng.choice(n_ctx, c, replace=False)).astype(np.int32) for c in (100, 9, 57)]
    act, out, ref, _ = _run(cuda_dev, B, n_ctx, positions, V, "bf16", eps, gate_q, has_prev, -1,
                            seed=31, sigma_prev=0.2, gate_only=True)
    j0 = n_mis = 0
    n_lock = 0
    for b in range(B):
        pf = positions[b] + b * n_ctx
        m = len(pf)
        o = _oracle_seq(pf, ref, eps, gate_q, has_prev, -1, gate_only=True)
        sl = slice(j0, j0 + m)
        mi, _ = compare_locks(out["lock"][sl], o["lock"], o["D"], o["u"], np.inf, o["thr"], True)
        n_mis += mi
        n_lock += int(out["lock"][sl].sum())
        j0 += m
    assert n_mis == 0
    assert (n_lock > 0) == has_prev


def test_gate_only_needs_the_gate(cuda_dev):
    positions = [np.arange(10, dtype=np.int32)]
    with pytest.raises(RuntimeError):
        _run(cuda_dev, 1, 10, positions, 512, "f32", 0.01, -1.0, True, -1, seed=3, gate_only=True)
