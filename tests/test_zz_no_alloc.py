"""sl_kl_stats_noalloc: the sure-test statistics for callers that cannot
allocate device memory (their device memory belongs to another runtime's pool,
or a cudaMalloc and its implicit synchronisation is not allowed where they
run).  Its scratch is a static array inside the library, shared by every call.

The test calls it twice in a row through the C ABI (different row sets,
vocabularies and dtypes, so the second call runs on whatever the first one left
in the shared scratch) and checks each result against the regular entry point
sl_kl_lock on the same inputs, with the tolerances of the other lock-test
checks.  The file name keeps it last in collection order."""
import numpy as np
import pytest
import torch

import workloads as wl
from token_locking_b200 import runtime as rt

pytestmark = pytest.mark.gpu


def _inputs(dev, n_rows, V, dtype, seed):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    z, zp, _ = wl.np_lock_logits(n_rows, V, seed=seed, prev_sigma=0.2)
    cur = torch.from_numpy(z).to(dev, tdt)
    prv = torch.from_numpy(zp).to(dev, tdt)
    lse_prev = torch.logsumexp(prv.float(), dim=1).contiguous()
    return cur, prv, lse_prev


def _regular(dev, positions, n_ctx, V, mask_id, cur, prv, lse_prev):
    act = rt.Active(1, n_ctx)
    act.load([positions])
    R = n_ctx
    out = {k: torch.zeros(R, device=dev) for k in ("kl", "unc", "conf", "lse")}
    out["argmax"] = torch.zeros(R, device=dev, dtype=torch.int32)
    lock = torch.zeros(R, device=dev, dtype=torch.uint8)
    masked = torch.zeros(R, device=dev, dtype=torch.uint8)
    rt.kl_lock(act, V, mask_id, cur, prv, lse_prev, out["lse"], masked, out["kl"], out["unc"],
               out["conf"], out["argmax"], lock, eps=0.01)
    return out


def _noalloc(dev, positions, V, mask_id, cur, prv, lse_prev):
    rows = torch.from_numpy(positions.astype(np.int32)).to(dev)
    R = cur.shape[0]
    out = {k: torch.zeros(R, device=dev) for k in ("kl", "unc", "conf", "lse")}
    out["argmax"] = torch.zeros(R, device=dev, dtype=torch.int32)
    rt.kl_stats_noalloc(rows, V, mask_id, cur, prv, lse_prev, out["lse"], out["kl"], out["unc"],
                        out["conf"], out["argmax"])
    return out


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


def test_noalloc_matches_regular_entry_point_twice(cuda_dev):
    calls = [(300, 4096, "bf16", 211, 11), (64, 126464, "bf16", 64, 12)]
    for n_ctx, V, dtype, m, seed in calls:
        rng = np.random.default_rng(seed)
        positions = np.sort(rng.choice(n_ctx, m, replace=False)).astype(np.int32)
        cur, prv, lse_prev = _inputs(cuda_dev, n_ctx, V, dtype, seed)
        mask_id = V - 5
        ref = _regular(cuda_dev, positions, n_ctx, V, mask_id, cur, prv, lse_prev)
        got = _noalloc(cuda_dev, positions, V, mask_id, cur, prv, lse_prev)
        torch.cuda.synchronize()
        _check(ref, got, positions)


def test_noalloc_rejects_rows_beyond_its_scratch(cuda_dev):
    from token_locking_b200 import _abi as A
    rows = torch.zeros(8193, dtype=torch.int32, device=cuda_dev)
    buf = torch.zeros(8, device=cuda_dev)
    with pytest.raises(A.SureLockError) as e:
        rt.kl_stats_noalloc(rows, 512, 0, buf, buf, buf, buf, buf, buf, buf,
                            torch.zeros(8, dtype=torch.int32, device=cuda_dev))
    assert e.value.status == A.SL_ERR_INVALID and "8192" in str(e.value)
