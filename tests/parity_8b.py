"""Helpers of the LLaDA-8B-shape parity tests: the device's bf16 weights seen by
the oracle as float32 arrays (converted one layer at a time, or kept on the
host when it has room), snapshots of a sampler's state, and the teacher-forced
comparison of one denoising step.

Teacher forcing: before a checked GPU step the oracle receives the GPU's state
(tokens, mask flags, active list, every layer's K/V cache, the previous step's
logits) and computes the same step in float32 on the same bf16 weights.  The
logits are compared within the bf16 tolerance; the decisions that floating
point takes (argmax, lock flags, unmasking) are taken by the oracle on the
GPU's own logits, so both sides decide in the same precision, and must agree
exactly outside the rounding bands; compaction must be the stable removal of
the locked rows.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import model as om
from oracle import surelock as osl
from parity_util import BAND_D, compare_locks, conf_ambiguous


def _host_gb() -> float:
    try:
        import psutil
        return psutil.virtual_memory().available / 1e9
    except Exception:
        return 0.0


class _Rows:
    """w["tok_emb"] for the oracle: rows gathered on the device, upcast on the host."""

    def __init__(self, t: torch.Tensor):
        self.t = t

    def __getitem__(self, idx):
        i = torch.from_numpy(np.asarray(idx, dtype=np.int64)).to(self.t.device)
        return self.t.index_select(0, i).float().cpu().numpy()


class _Layers:
    """w["layers"] for the oracle: each layer's bf16 weights as float32 arrays,
    converted on access and kept if `keep`."""

    def __init__(self, layers, keep: bool):
        self.dev = layers
        self.keep = keep
        self.memo = {}

    def __len__(self):
        return len(self.dev)

    def __getitem__(self, l):
        if l in self.memo:
            return self.memo[l]
        d = {k: v.float().cpu().numpy() for k, v in self.dev[l].items()}
        if self.keep:
            self.memo[l] = d
        return d

    def __iter__(self):
        for l in range(len(self)):
            yield self[l]


def oracle_weights(w_dev: dict) -> dict:
    """The device weights exactly as stored (bf16 values), as float32 for the
    oracle.  Layers stay on the device and are upcast when used unless the host
    has room to keep all of them."""
    n = len(w_dev["layers"])
    per_layer = sum(v.numel() for v in w_dev["layers"][0].values()) * 4 / 1e9
    keep = _host_gb() > per_layer * n + 24.0
    return {"tok_emb": _Rows(w_dev["tok_emb"]),
            "final_norm": w_dev["final_norm"].float().cpu().numpy(),
            "lm_head": w_dev["lm_head"].float().cpu().numpy(),
            "layers": _Layers(w_dev["layers"], keep)}


def snapshot(s, setup, want_cache=True) -> dict:
    """The sampler's state before its next step, on the host (float32)."""
    st = s.state()
    B, N = setup.batch, setup.n_ctx
    L = setup.shape.n_layers
    t = st["t"]
    prv = (t - 1) & 1 if t > 0 else 0
    out = {
        "t": t,
        "tokens": st["tokens"].cpu().numpy().copy(),
        "masked": st["masked"].cpu().numpy().astype(bool),
        "act": st["active"].positions(),
        "z_prev": st["logits"][prv].float().cpu().numpy().reshape(B, N, -1),
    }
    if want_cache:
        d = setup.shape.d_model
        ck = np.empty((B, L, N, d), dtype=np.float32)
        cv = np.empty((B, L, N, d), dtype=np.float32)
        for l in range(L):
            k, v = st["cache"].view(l)
            ck[:, l] = k.float().cpu().numpy().reshape(B, N, d)
            cv[:, l] = v.float().cpu().numpy().reshape(B, N, d)
        out["ck"], out["cv"] = ck, cv
    return out


def gpu_after(s, setup, t) -> dict:
    """The GPU's outputs of step t (read right after it)."""
    st = s.state()
    B, N = setup.batch, setup.n_ctx
    return {
        "z": st["logits"][t & 1].float().cpu().numpy().reshape(B, N, -1),
        "lse": st["lse"][t & 1].cpu().numpy().reshape(B, N),
        "kl": st["kl"].cpu().numpy(), "unc": st["unc"].cpu().numpy(),
        "conf": st["conf"].cpu().numpy(), "argmax": st["argmax"].cpu().numpy(),
        "lock": st["lock"].cpu().numpy().astype(bool),
        "act": st["active"].positions(),
        "tokens": st["tokens"].cpu().numpy(),
        "masked": st["masked"].cpu().numpy().astype(bool),
    }


def cache_rows(s, setup, b, rows) -> tuple:
    """The GPU cache's k, v [L, len(rows), d] of sequence b at `rows` (float32)."""
    st = s.state()
    N = setup.n_ctx
    idx = torch.from_numpy((b * N + np.asarray(rows)).astype(np.int64))
    ks, vs = [], []
    for l in range(setup.shape.n_layers):
        k, v = st["cache"].view(l)
        i = idx.to(k.device)
        ks.append(k.index_select(0, i).float().cpu().numpy())
        vs.append(v.index_select(0, i).float().cpu().numpy())
    return np.stack(ks), np.stack(vs)


def check_decisions(setup, t, b, A, snap, g, j0, stats, A_all=None):
    """Sure test, gate, unmasking and compaction of sequence b at step t, taken
    by the oracle on the GPU's logits; exact outside the rounding bands.  A are
    the rows the step computed; A_all the active rows when that is more (K/V
    reuse between refresh steps), which the compaction runs over."""
    shape = setup.shape
    m = len(A)
    sl_ = slice(j0, j0 + m)
    z = g["z"][b, A].astype(np.float64)
    lp = osl.log_softmax(z)
    lpp = osl.log_softmax(snap["z_prev"][b, A].astype(np.float64))
    hp = np.full(m, t > 0)
    rec = osl.lock_test(lp, lpp, hp, snap["masked"][b, A], A, shape, setup, t)
    np.testing.assert_array_equal(g["argmax"][sl_], rec["pred"])
    np.testing.assert_allclose(g["conf"][sl_], rec["conf"], rtol=2e-5)
    np.testing.assert_allclose(g["unc"][sl_], rec["u"], atol=2e-6)
    lse = z[:, 0] - lp[:, 0]
    np.testing.assert_allclose(g["lse"][b, A], lse, rtol=2e-6, atol=2e-6)
    if t > 0:
        np.testing.assert_allclose(g["kl"][sl_], rec["D"], atol=2e-5, rtol=1e-4)
    lock_g = g["lock"][sl_]
    if setup.scripted:
        assert lock_g.sum() == rec["lock"].sum(), f"t={t}: scripted lock count"
        diff = lock_g != rec["lock"]
        am = 0
        if rec["lock"].any():
            cut = rec["D"][rec["lock"]].max()
            am = int(np.sum(diff & (np.abs(rec["D"] - cut) < BAND_D)))
        mi = int(diff.sum()) - am
    else:
        mi, am = compare_locks(lock_g, rec["lock"], rec["D"], rec["u"], setup.eps, rec["thr"],
                               setup.gate_q >= 0)
    stats["mismatch"] += mi
    stats["ambiguous"] += am
    stats["locks"] += int(lock_g.sum())
    lo, hi = setup.block_bounds(t)
    conf = g["conf"][sl_].astype(np.float64)
    sel = osl.unmask_select(A, conf, snap["masked"][b, A], lo, hi, setup.tokens_per_step)
    want = snap["tokens"][b].copy()
    want[A[sel]] = g["argmax"][sl_][sel]
    if not np.array_equal(g["tokens"][b], want):
        cands = np.nonzero(snap["masked"][b, A] & (A >= lo) & (A < hi))[0]
        assert conf_ambiguous(conf, sel, cands), f"t={t} b={b}: unmasking differs"
        stats["unmask_amb"] += 1
    assert not np.any(lock_g & snap["masked"][b, A]), "a masked row locked"
    if A_all is None:
        np.testing.assert_array_equal(g["act"][b], osl.compact(A, lock_g))
    else:
        np.testing.assert_array_equal(g["act"][b], osl.compact(A_all, np.isin(A_all, A[lock_g])))
    assert np.array_equal(g["masked"][b], g["tokens"][b] == shape.mask_id)


def oracle_logits_full(shape, w_or, snap, b, A):
    """The oracle's step on every active row of sequence b from the snapshot
    (float32), and the cache rows it wrote.  Returns (z [M, V], ck, cv)."""
    ck = np.ascontiguousarray(snap["ck"][b])
    cv = np.ascontiguousarray(snap["cv"][b])
    z = om.forward_active(shape, w_or, snap["tokens"][b], A, ck, cv)
    return z, ck, cv


def oracle_logits_sampled(shape, w_or, tokens, A, rows_idx, ck_after, cv_after):
    """Per-layer teacher forcing for large steps: the oracle runs the sampled
    active rows (indices rows_idx into A) through every block, each block
    attending over the GPU's cache after the step (which holds every active
    row's fresh K/V of that block), so the work is proportional to the
    sample.  Returns (z [S, V], k, v [L, S, d]) with the sample's fresh K/V."""
    pos = A[rows_idx]
    h = w_or["tok_emb"][tokens[pos]]
    L = len(w_or["layers"])
    ks, vs = [], []
    for l in range(L):
        lw = w_or["layers"][l]
        ck = np.array(ck_after[l], dtype=np.float32)
        cv = np.array(cv_after[l], dtype=np.float32)
        h = om.layer_forward(shape, lw, h, pos, ck, cv)
        ks.append(ck[pos])
        vs.append(cv[pos])
    hf = om.rmsnorm(h, w_or["final_norm"], shape.rms_eps)
    return hf @ w_or["lm_head"].T, np.stack(ks), np.stack(vs)
