"""sl_kl_stats_noalloc: the sure-test statistics for callers that cannot
allocate device memory (their device memory belongs to another runtime's pool,
or a cudaMalloc and its implicit synchronisation is not allowed where they
run).  Its scratch is a static array inside the library, shared by every call.

The test calls it three times in a row through the C ABI, each on whatever the
previous call left in the shared scratch: bf16 logits with a previous
posterior, fp32 logits at the accepted maximum of 8192 rows without one
(has_prev = 0: D is +inf), and bf16 logits over the full 126464-token
vocabulary.  Each result is checked against the regular entry point
sl_kl_lock on the same inputs and, on sampled rows, against the oracle's
kl_rows / uncertainty / prediction on the exact stored logits, with the
tolerances of the other lock-test checks.  The file name keeps it last in
collection order."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import surelock as osl
from token_locking_b200 import runtime as rt

pytestmark = pytest.mark.gpu


def _inputs(dev, n_rows, V, dtype, seed):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    z, zp, _ = wl.np_lock_logits(n_rows, V, seed=seed, prev_sigma=0.2)
    cur = torch.from_numpy(z).to(dev, tdt)
    prv = torch.from_numpy(zp).to(dev, tdt)
    lse_prev = torch.logsumexp(prv.float(), dim=1).contiguous()
    return cur, prv, lse_prev


def _regular(dev, positions, n_ctx, V, mask_id, cur, prv, lse_prev, has_prev):
    act = rt.Active(1, n_ctx)
    act.load([positions])
    R = n_ctx
    out = {k: torch.zeros(R, device=dev) for k in ("kl", "unc", "conf", "lse")}
    out["argmax"] = torch.zeros(R, device=dev, dtype=torch.int32)
    lock = torch.zeros(R, device=dev, dtype=torch.uint8)
    masked = torch.zeros(R, device=dev, dtype=torch.uint8)
    rt.kl_lock(act, V, mask_id, cur, prv, lse_prev, out["lse"], masked, out["kl"], out["unc"],
               out["conf"], out["argmax"], lock, eps=0.01, has_prev=has_prev)
    return out


def _noalloc(dev, positions, V, mask_id, cur, prv, lse_prev, has_prev):
    rows = torch.from_numpy(positions.astype(np.int32)).to(dev)
    R = cur.shape[0]
    out = {k: torch.zeros(R, device=dev) for k in ("kl", "unc", "conf", "lse")}
    out["argmax"] = torch.zeros(R, device=dev, dtype=torch.int32)
    rt.kl_stats_noalloc(rows, V, mask_id, cur, prv if has_prev else None,
                        lse_prev if has_prev else None, out["lse"], out["kl"], out["unc"],
                        out["conf"], out["argmax"], has_prev=has_prev)
    return out


def _check_oracle(got, positions, cur, prv, mask_id, has_prev, n_sample, seed):
    """Sampled rows against the oracle on the exact stored logits (fp64)."""
    rng = np.random.default_rng(seed)
    js = np.sort(rng.choice(len(positions), min(n_sample, len(positions)), replace=False))
    pf = positions[js]
    idx = torch.from_numpy(pf.astype(np.int64)).to(cur.device)
    z = cur.index_select(0, idx).double().cpu().numpy()
    lp = osl.log_softmax(z)
    conf, pred = osl.prediction(lp, mask_id)
    u = osl.uncertainty(lp)
    lse = (z - lp)[:, 0]
    np.testing.assert_array_equal(got["argmax"][js], pred)
    np.testing.assert_allclose(got["unc"][js], u, atol=2e-6)
    np.testing.assert_allclose(got["conf"][js], conf, rtol=2e-5, atol=1e-9)
    np.testing.assert_allclose(got["lse"][pf], lse, rtol=2e-6, atol=2e-6)
    if has_prev:
        lpp = osl.log_softmax(prv.index_select(0, idx).double().cpu().numpy())
        np.testing.assert_allclose(got["kl"][js], osl.kl_rows(lp, lpp), atol=2e-5, rtol=1e-4)
    else:
        assert np.all(np.isposinf(got["kl"][js]))


def _check(a, b, positions):
    m = len(positions)
    for k in ("kl", "unc", "conf", "argmax", "lse"):
        a[k] = a[k].cpu().numpy()
        b[k] = b[k].cpu().numpy()
    np.testing.assert_array_equal(b["argmax"][:m], a["argmax"][:m])
    np.testing.assert_allclose(b["kl"][:m], a["kl"][:m], atol=2e-5, rtol=1e-4)
    np.testing.assert_allclose(b["unc"][:m], a["unc"][:m], atol=2e-6)
    np.testing.assert_allclose(b["conf"][:m], a["conf"][:m], rtol=2e-5)
    np.testing.assert_allclose(b["lse"][positions], a["lse"][positions], rtol=2e-6, atol=2e-6)


def test_noalloc_matches_regular_entry_point_and_oracle(cuda_dev):
    calls = [  # n_ctx, V, dtype, rows, has_prev, seed
        (300, 4096, "bf16", 211, 1, 11),
        (8192, 4096, "f32", 8192, 0, 12),
        (64, 126464, "bf16", 64, 1, 13),
    ]
    for n_ctx, V, dtype, m, has_prev, seed in calls:
        rng = np.random.default_rng(seed)
        positions = np.sort(rng.choice(n_ctx, m, replace=False)).astype(np.int32)
        cur, prv, lse_prev = _inputs(cuda_dev, n_ctx, V, dtype, seed)
        mask_id = V - 5
        ref = _regular(cuda_dev, positions, n_ctx, V, mask_id, cur, prv, lse_prev, has_prev)
        got = _noalloc(cuda_dev, positions, V, mask_id, cur, prv, lse_prev, has_prev)
        torch.cuda.synchronize()
        _check(ref, got, positions)
        _check_oracle(got, positions, cur, prv, mask_id, has_prev, 24, seed)


def test_noalloc_rejects_rows_beyond_its_scratch(cuda_dev):
    from token_locking_b200 import _abi as A
    rows = torch.zeros(8193, dtype=torch.int32, device=cuda_dev)
    buf = torch.zeros(8, device=cuda_dev)
    with pytest.raises(A.SureLockError) as e:
        rt.kl_stats_noalloc(rows, 512, 0, buf, buf, buf, buf, buf, buf, buf,
                            torch.zeros(8, dtype=torch.int32, device=cuda_dev))
    assert e.value.status == A.SL_ERR_INVALID and "8192" in str(e.value)
