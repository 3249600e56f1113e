"""One LLaDA-8B-shaped block (d_model 4096, 32 heads of 128, d_ffn 12288) on the
layer-microbenchmark inputs - block input N(0,1), cache N(0,1) over N = 2048
positions, a sorted random subset of M active rows - against the oracle on
sampled rows.  A row's block output depends only on its own input and the
whole cache, so the oracle first writes the fresh k, v of all M active rows
into a copy of the cache (two projections of every active row) and then runs
its block on 16 sampled rows; the GPU's fresh cache rows are checked on a
sample too, and every frozen cache row must be bitwise unchanged.  Both the
analytic tilings and the autotuned ones (which include the CTA-pair,
stream-K and 192-wide kernels) are covered."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import model as om
from token_locking_b200 import runtime as rt
from parity_util import to64, weights_for_oracle, weights_to_device

pytestmark = pytest.mark.gpu

N_CTX = 2048
SAMPLE = 16
# one block of the 8B shape; a small vocabulary (the block does not use it)
SHAPE8 = wl.ModelShape(n_layers=1, d_model=4096, n_heads=32, head_dim=128, d_ffn=12288,
                       vocab=256, mask_id=255, rope_theta=wl.LLADA8B.rope_theta)


@pytest.fixture(scope="module")
def block8(cuda_dev):
    w_np = wl.np_weights(SHAPE8, seed=0, std=0.02, gain_jitter=0.1)
    w_dev = weights_to_device(w_np, "bf16", cuda_dev)
    lw64 = weights_for_oracle(w_dev)["layers"][0]
    model = rt.Model(SHAPE8, w_dev, "bf16")
    cache = rt.KVCache(model, 1, N_CTX)
    rng = np.random.default_rng(2)
    d = SHAPE8.d_model
    ck = wl.round_bf16(rng.standard_normal((N_CTX, d)).astype(np.float32))
    cv = wl.round_bf16(rng.standard_normal((N_CTX, d)).astype(np.float32))
    yield model, cache, lw64, ck, cv
    model.close()


def _run(block8, cuda_dev, M):
    model, cache, lw64, ck, cv = block8
    d = SHAPE8.d_model
    k_dev, v_dev = cache.view(0)
    k_dev.copy_(torch.from_numpy(ck).to(cuda_dev, torch.bfloat16))
    v_dev.copy_(torch.from_numpy(cv).to(cuda_dev, torch.bfloat16))
    rng = np.random.default_rng(1000 + M)
    pos = np.sort(rng.choice(N_CTX, M, replace=False)).astype(np.int32)
    act = rt.Active(1, N_CTX)
    act.load([pos])
    h_np = rng.standard_normal((M, d)).astype(np.float32)
    h = torch.from_numpy(h_np).to(cuda_dev)
    rt.layer_forward(model, cache, act, 0, h)
    torch.cuda.synchronize()
    rt.device_check()

    # oracle: fresh k, v of every active row into a copy of the cache ...
    h64 = h_np.astype(np.float64)
    k_all, v_all = om.kv_of_block_input(SHAPE8, lw64, h64, pos)
    ck64, cv64 = ck.astype(np.float64), cv.astype(np.float64)
    ck64[pos], cv64[pos] = k_all, v_all
    # ... then the block on sampled rows (it rewrites their k, v identically)
    S = np.sort(rng.choice(M, min(SAMPLE, M), replace=False))
    ref = om.layer_forward(SHAPE8, lw64, h64[S], pos[S], ck64.copy(), cv64.copy())
    got = h.double().cpu().numpy()[S]
    err = np.abs(got - ref).max()
    print(f"M={M} tiling {[model.tuning(k, M) for k in range(4)]}: block output max err "
          f"{err:.4g} (|ref| max {np.abs(ref).max():.3g})")
    # bf16 activations and GEMM outputs around an fp32 residual of magnitude ~10:
    # observed 0.030-0.036 on B200; 0.1 leaves a 3x margin
    assert err <= 0.1, f"M={M}: block output max err {err}"

    k_got, v_got = to64(k_dev), to64(v_dev)
    frozen = np.ones(N_CTX, dtype=bool)
    frozen[pos] = False
    np.testing.assert_array_equal(k_got[frozen], ck[frozen])
    np.testing.assert_array_equal(v_got[frozen], cv[frozen])
    R = pos[np.sort(rng.choice(M, min(64, M), replace=False))]
    for got_c, ref_c in ((k_got, ck64), (v_got, cv64)):
        e = np.abs(got_c[R] - ref_c[R]).max()
        assert e <= 3e-2 * max(1.0, np.abs(ref_c[R]).max()), f"M={M}: fresh K/V max err {e}"


@pytest.mark.parametrize("M", [8, 64, 256, 512, 1024, 2048])
def test_block_8b_analytic_tilings(block8, cuda_dev, M):
    _run(block8, cuda_dev, M)


def test_qkv_tile_must_divide_segments(block8):
    """A fused Q|K|V tile takes its weight rows from one of Wq, Wk, Wv: a
    192-wide tile would straddle the 4096-row segments and is refused."""
    model = block8[0]
    with pytest.raises(RuntimeError):
        model.set_tuning(0, 64, 192, -1, 0)


_TUNED = {}


@pytest.mark.parametrize("M", [8, 200, 1024, 2048])
def test_block_8b_autotuned_tilings(block8, cuda_dev, M):
    model, cache = block8[0], block8[1]
    if not _TUNED:
        model.autotune(cache, N_CTX)
        _TUNED["done"] = True
    _run(block8, cuda_dev, M)
