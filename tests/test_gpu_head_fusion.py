"""The LM head fused with the sure test's statistics (sl_step_stats): the
epilogue of the LM-head GEMM stores the bf16 logits and takes per-tile
statistics of the stored values; a per-row merge writes lse, D, u, conf and
argmax.  Checked against

* sl_kl_lock, the separate pass, over the same stored logits: same argmax,
  and lse, D, u, conf within fp32 summation-order rounding;
* sl_step on the same state: the same logits up to the order in which split-K
  partial sums are added;
* the oracle's log_softmax / kl_rows / uncertainty / prediction on the stored
  logits (fp64): argmax exact, the rest within the lock-test tolerances;
* sl_lock_decide on the fused statistics: the same lock flags as sl_kl_lock;

for every LM-head tiling (tile width 64/128/192/256; 128-row, 256-row and
CTA-pair kernels), with and without a previous posterior, ragged batches, and
the full 126464-token vocabulary at the LLaDA-8B width.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import surelock as osl
from token_locking_b200 import runtime as rt
from parity_util import weights_to_device

pytestmark = pytest.mark.gpu

MINI = wl.ModelShape(n_layers=1, d_model=256, n_heads=2, head_dim=128, d_ffn=512,
                     vocab=3072, mask_id=3071, rope_theta=10000.0)
WIDE = wl.ModelShape(n_layers=1, d_model=4096, n_heads=32, head_dim=128, d_ffn=12288,
                     vocab=126464, mask_id=126336, rope_theta=500000.0)
G_HD = 4


def _state(model, shape, B, n_ctx, counts, dev, seed):
    rng = np.random.default_rng(seed)
    cache = rt.KVCache(model, B, n_ctx)
    act = rt.Active(B, n_ctx)
    act.load([np.sort(rng.choice(n_ctx, c, replace=False)).astype(np.int32) for c in counts])
    tokens = torch.from_numpy(rng.integers(0, shape.vocab - 1, (B, n_ctx)).astype(np.int32)).to(dev)
    return cache, act, tokens


def _run(model, shape, cache, act, tokens, dev, has_prev, eps=0.05, gate_q=0.5, seed=0):
    R = act.batch * act.n_ctx
    V = shape.vocab
    g = torch.Generator(device=dev).manual_seed(seed)
    prev = (torch.randn((R, V), device=dev, generator=g) * 2).to(torch.bfloat16)
    lse_prev = torch.logsumexp(prev.float(), dim=1).contiguous()
    masked = (torch.rand(R, device=dev, generator=g) < 0.3).to(torch.uint8)
    # fused
    z_f = torch.zeros((R, V), device=dev, dtype=torch.bfloat16)
    f = {k: torch.zeros(R, device=dev) for k in ("lse", "kl", "unc", "conf")}
    f["argmax"] = torch.zeros(R, device=dev, dtype=torch.int32)
    rt.step_stats(model, cache, act, tokens, z_f, prev if has_prev else None,
                  lse_prev if has_prev else None, f["lse"], f["kl"], f["unc"], f["conf"],
                  f["argmax"], has_prev=has_prev)
    lock_f = torch.zeros(R, device=dev, dtype=torch.uint8)
    rt.lock_decide(act, masked, f["kl"], f["unc"], lock_f, eps, gate_q, has_prev)
    # the separate statistics pass and decisions over the same stored logits
    u = {k: torch.zeros(R, device=dev) for k in ("lse", "kl", "unc", "conf")}
    u["argmax"] = torch.zeros(R, device=dev, dtype=torch.int32)
    lock_u = torch.zeros(R, device=dev, dtype=torch.uint8)
    rt.kl_lock(act, V, shape.mask_id, z_f, prev, lse_prev, u["lse"], masked, u["kl"], u["unc"],
               u["conf"], u["argmax"], lock_u, eps=eps, gate_q=gate_q, has_prev=has_prev)
    # and sl_step on the same state: the same logits (split-K GEMMs may add their
    # partial sums in another order, so within bf16 rounding rather than bitwise)
    z_u = torch.zeros_like(z_f)
    rt.step(model, cache, act, tokens, z_u)
    torch.cuda.synchronize()
    rt.device_check()
    return z_f, f, lock_f, z_u, u, lock_u, prev, masked


def _compare(shape, act, z_f, f, lock_f, z_u, u, lock_u, prev, has_prev, n_oracle_rows=12):
    rows = np.concatenate([p + b * act.n_ctx for b, p in enumerate(act.positions())])
    M = len(rows)
    zd = (z_f[rows].float() - z_u[rows].float()).abs().max().item()
    assert zd <= 5e-2, f"sl_step_stats and sl_step logits differ by {zd}"
    F = {k: v.cpu().numpy() for k, v in f.items()}
    U = {k: v.cpu().numpy() for k, v in u.items()}
    np.testing.assert_array_equal(F["argmax"][:M], U["argmax"][:M])
    np.testing.assert_allclose(F["lse"][rows], U["lse"][rows], rtol=2e-6, atol=2e-6)
    np.testing.assert_allclose(F["unc"][:M], U["unc"][:M], atol=2e-6)
    np.testing.assert_allclose(F["conf"][:M], U["conf"][:M], rtol=2e-5)
    if has_prev:
        np.testing.assert_allclose(F["kl"][:M], U["kl"][:M], atol=2e-5, rtol=1e-4)
    else:
        assert np.all(np.isposinf(F["kl"][:M]))
    # lock flags: the same except where D or u sits on a threshold within rounding
    diff = lock_f.cpu().numpy()[:M] != lock_u.cpu().numpy()[:M]
    assert diff.sum() <= max(1, M // 200), f"{diff.sum()} lock flags differ"
    # oracle on sampled rows of the stored logits
    rng = np.random.default_rng(M)
    js = np.sort(rng.choice(M, min(n_oracle_rows, M), replace=False))
    z = z_f[rows[js]].double().cpu().numpy()
    lp = osl.log_softmax(z)
    conf, pred = osl.prediction(lp, shape.mask_id)
    np.testing.assert_array_equal(F["argmax"][js], pred)
    np.testing.assert_allclose(F["unc"][js], osl.uncertainty(lp), atol=2e-6)
    np.testing.assert_allclose(F["conf"][js], conf, rtol=2e-5, atol=1e-9)
    np.testing.assert_allclose(F["lse"][rows[js]], (z - lp)[:, 0], rtol=2e-6, atol=2e-6)
    if has_prev:
        lpp = osl.log_softmax(prev[rows[js]].double().cpu().numpy())
        np.testing.assert_allclose(F["kl"][js], osl.kl_rows(lp, lpp), atol=2e-5, rtol=1e-4)


TILINGS = [(64, 0), (128, 0), (192, 0), (256, 0), (128, 1), (256, 1), (128, 2), (192, 2),
           (256, 2)]


@pytest.fixture(scope="module")
def mini(cuda_dev):
    w = weights_to_device(wl.np_weights(MINI, seed=0, std=0.05), "bf16", cuda_dev)
    model = rt.Model(MINI, w, "bf16")
    yield model
    model.close()


@pytest.mark.parametrize("bn,variant", TILINGS)
@pytest.mark.parametrize("has_prev", [True, False])
def test_fused_stats_every_head_tiling(mini, cuda_dev, bn, variant, has_prev):
    B, n_ctx, counts = 2, 300, [300, 141]
    M = sum(counts)
    mini.set_tuning(G_HD, M, bn, 1, variant)
    cache, act, tokens = _state(mini, MINI, B, n_ctx, counts, cuda_dev, seed=bn + variant)
    out = _run(mini, MINI, cache, act, tokens, cuda_dev, has_prev, seed=bn)
    _compare(MINI, act, *out[:7], has_prev=has_prev)
    cache.close()


@pytest.mark.parametrize("counts", [[1], [37], [128, 0, 5]])
def test_fused_stats_small_and_ragged(mini, cuda_dev, counts):
    B, n_ctx = len(counts), 160
    cache, act, tokens = _state(mini, MINI, B, n_ctx, counts, cuda_dev, seed=sum(counts))
    out = _run(mini, MINI, cache, act, tokens, cuda_dev, True, seed=3)
    _compare(MINI, act, *out[:7], has_prev=True)
    cache.close()


def test_fused_stats_full_vocabulary(cuda_dev):
    """The LLaDA-8B width and vocabulary (one block), 200 of 384 rows active."""
    w = wl.torch_weights(WIDE, cuda_dev, layers=1)
    model = rt.Model(WIDE, w, "bf16")
    cache, act, tokens = _state(model, WIDE, 1, 384, [200], cuda_dev, seed=9)
    out = _run(model, WIDE, cache, act, tokens, cuda_dev, True, eps=0.5, seed=4)
    _compare(WIDE, act, *out[:7], has_prev=True, n_oracle_rows=8)
    cache.close()
    model.close()
