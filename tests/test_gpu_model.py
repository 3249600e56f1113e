"""Denoiser on the active rows (sl_step / sl_layer_forward) against the oracle:
fp32 tiny model (1e-4) and bf16 models on the tensor-core path (5e-2), with
frozen cache rows for locked positions and ragged batches."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import model as om
from token_locking_b200 import runtime as rt
from parity_util import BLOCK_ULPS, LOGIT_TOL, bf16_ulp, to64, weights_for_oracle, weights_to_device

pytestmark = pytest.mark.gpu

MINI_BF16 = wl.ModelShape(n_layers=2, d_model=256, n_heads=2, head_dim=128, d_ffn=512,
                          vocab=1024, mask_id=1023, rope_theta=10000.0)


def _state(shape, B, n_ctx, counts, seed, dev, dtype):
    """Random tokens, an active subset per sequence and a cache whose non-active
    rows hold arbitrary frozen values."""
    rng = np.random.default_rng(seed)
    tokens = rng.integers(0, shape.vocab, (B, n_ctx)).astype(np.int32)
    positions = [np.sort(rng.choice(n_ctx, c, replace=False)).astype(np.int32) for c in counts]
    L, d = shape.n_layers, shape.d_model
    ck = (rng.standard_normal((L, B * n_ctx, d)) * 0.5).astype(np.float32)
    cv = (rng.standard_normal((L, B * n_ctx, d)) * 0.5).astype(np.float32)
    if dtype == "bf16":
        ck, cv = wl.round_bf16(ck), wl.round_bf16(cv)
    return tokens, positions, ck, cv


def _load_cache(cache, ck, cv, tdt):
    for l in range(ck.shape[0]):
        k, v = cache.view(l)
        k.copy_(torch.from_numpy(ck[l]).to(k.device, tdt))
        v.copy_(torch.from_numpy(cv[l]).to(v.device, tdt))


def _oracle_step(shape, w64, tokens, positions, ck, cv, n_ctx):
    """Oracle logits per sequence and the updated cache (float64)."""
    B = tokens.shape[0]
    L, d = shape.n_layers, shape.d_model
    zs = []
    ck2 = ck.astype(np.float64).reshape(L, B, n_ctx, d).copy()
    cv2 = cv.astype(np.float64).reshape(L, B, n_ctx, d).copy()
    for b in range(B):
        if len(positions[b]) == 0:
            zs.append(np.zeros((0, shape.vocab)))
            continue
        ckb = np.ascontiguousarray(ck2[:, b])
        cvb = np.ascontiguousarray(cv2[:, b])
        zs.append(om.forward_active(shape, w64, tokens[b], positions[b], ckb, cvb))
        ck2[:, b] = ckb
        cv2[:, b] = cvb
    return zs, ck2.reshape(L, B * n_ctx, d), cv2.reshape(L, B * n_ctx, d)


@pytest.mark.parametrize("shape,dtype,B,n_ctx,counts", [
    (wl.TINY, "f32", 1, 64, [64]),
    (wl.TINY, "f32", 1, 64, [23]),
    (wl.TINY, "f32", 3, 40, [40, 1, 17]),
    (MINI_BF16, "bf16", 1, 200, [200]),
    (MINI_BF16, "bf16", 2, 200, [131, 57]),
    (MINI_BF16, "bf16", 3, 96, [5, 0, 96]),
])
def test_step_matches_oracle(cuda_dev, shape, dtype, B, n_ctx, counts):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    w_np = wl.np_weights(shape, seed=0, std=0.02 if dtype == "f32" else 0.05, gain_jitter=0.1)
    w_dev = weights_to_device(w_np, dtype, cuda_dev)
    w64 = weights_for_oracle(w_dev)
    model = rt.Model(shape, w_dev, dtype)
    cache = rt.KVCache(model, B, n_ctx)
    act = rt.Active(B, n_ctx)
    tokens, positions, ck, cv = _state(shape, B, n_ctx, counts, seed=sum(counts), dev=cuda_dev,
                                       dtype=dtype)
    act.load(positions)
    _load_cache(cache, ck, cv, tdt)
    tok = torch.from_numpy(tokens).to(cuda_dev)
    logits = torch.full((B * n_ctx, shape.vocab), 123.0, device=cuda_dev, dtype=tdt)
    rt.step(model, cache, act, tok, logits)
    torch.cuda.synchronize()
    rt.device_check()
    zs, ck2, cv2 = _oracle_step(shape, w64, tokens, positions, ck, cv, n_ctx)
    lg = to64(logits)
    tol = LOGIT_TOL[dtype]
    written = np.zeros(B * n_ctx, dtype=bool)
    for b in range(B):
        rows = positions[b] + b * n_ctx
        written[rows] = True
        if len(rows):
            err = np.abs(lg[rows] - zs[b]).max()
            assert err <= tol, f"seq {b}: logits max err {err} > {tol}"
    assert np.all(lg[~written] == 123.0)                 # locked rows' logits untouched
    kv_tol = 1e-4 if dtype == "f32" else 3e-2
    for l in range(shape.n_layers):
        k, v = cache.view(l)
        k, v = to64(k), to64(v)
        # frozen rows bitwise unchanged; fresh rows equal the oracle's k, v
        np.testing.assert_array_equal(k[~written], ck[l][~written])
        np.testing.assert_array_equal(v[~written], cv[l][~written])
        assert np.abs(k[written] - ck2[l][written]).max() <= kv_tol * max(1.0, np.abs(ck2[l]).max())
        assert np.abs(v[written] - cv2[l][written]).max() <= kv_tol * max(1.0, np.abs(cv2[l]).max())
    model.close()


def test_layer_forward_bf16_matches_oracle(cuda_dev):
    """One block on given hidden states N(0,1) (the layer microbenchmark's input)."""
    shape = MINI_BF16
    B, n_ctx = 1, 300
    w_np = wl.np_weights(shape, seed=3, std=0.05)
    w_dev = weights_to_device(w_np, "bf16", cuda_dev)
    w64 = weights_for_oracle(w_dev)
    model = rt.Model(shape, w_dev, "bf16")
    cache = rt.KVCache(model, B, n_ctx)
    act = rt.Active(B, n_ctx)
    _, positions, ck, cv = _state(shape, B, n_ctx, [211], seed=4, dev=cuda_dev, dtype="bf16")
    act.load(positions)
    _load_cache(cache, ck, cv, torch.bfloat16)
    h_np = np.random.default_rng(5).standard_normal((211, shape.d_model)).astype(np.float32)
    h = torch.from_numpy(h_np).to(cuda_dev)
    rt.layer_forward(model, cache, act, 1, h)
    torch.cuda.synchronize()
    ckb = ck[1].astype(np.float64).copy()
    cvb = cv[1].astype(np.float64).copy()
    ref = om.layer_forward(shape, w64["layers"][1], h_np.astype(np.float64), positions[0], ckb, cvb)
    err = np.abs(h.double().cpu().numpy() - ref).max()
    # one block: within BLOCK_ULPS bf16 ulps of the largest entry of the block's
    # update (observed 0.0053 for an update of max 2.28: bound 0.0625)
    upd = np.abs(ref - h_np).max()
    assert err <= BLOCK_ULPS * bf16_ulp(upd), (err, upd)
    model.close()


def test_autotuned_step_matches_oracle(cuda_dev):
    """After autotuning, the tilings chosen per row count are valid and the step
    still agrees with the oracle (the tuning only changes the schedule)."""
    shape = MINI_BF16
    B, n_ctx = 2, 200
    w_np = wl.np_weights(shape, seed=0, std=0.05, gain_jitter=0.1)
    w_dev = weights_to_device(w_np, "bf16", cuda_dev)
    w64 = weights_for_oracle(w_dev)
    model = rt.Model(shape, w_dev, "bf16")
    cache = rt.KVCache(model, B, n_ctx)
    model.autotune(cache, B * n_ctx)
    for kind in range(5):
        for M in (1, 100, 257, 400):
            bn, sp, var = model.tuning(kind, M)
            assert bn in (64, 128, 192, 256) and (sp >= 1 or sp == -1) and var in (0, 1, 2, 3)
            # swapped operands only for projections in buckets of at most 256 rows
            assert var != 3 or (kind != 4 and M <= 256 and bn == 128 and sp >= 1)
    act = rt.Active(B, n_ctx)
    tokens, positions, ck, cv = _state(shape, B, n_ctx, [160, 130], seed=11, dev=cuda_dev,
                                       dtype="bf16")
    act.load(positions)
    _load_cache(cache, ck, cv, torch.bfloat16)
    tok = torch.from_numpy(tokens).to(cuda_dev)
    logits = torch.zeros((B * n_ctx, shape.vocab), device=cuda_dev, dtype=torch.bfloat16)
    rt.step(model, cache, act, tok, logits)
    torch.cuda.synchronize()
    rt.device_check()
    zs, _, _ = _oracle_step(shape, w64, tokens, positions, ck, cv, n_ctx)
    lg = to64(logits)
    for b in range(B):
        err = np.abs(lg[positions[b] + b * n_ctx] - zs[b]).max()
        assert err <= LOGIT_TOL["bf16"], err
    model.close()


@pytest.mark.parametrize("tiling", [(256, -1, 2), (128, -1, 0), (256, -1, 1), (128, 3, 2)])
def test_pinned_tilings_step_matches_oracle(cuda_dev, tiling):
    """Every projection GEMM pinned to one tiling (stream-K or split K, CTA
    pairs or single CTAs; the LM head keeps its own), through the workspace
    and finalize kernels of the split paths."""
    shape = MINI_BF16
    B, n_ctx = 2, 200
    w_np = wl.np_weights(shape, seed=1, std=0.05, gain_jitter=0.1)
    w_dev = weights_to_device(w_np, "bf16", cuda_dev)
    w64 = weights_for_oracle(w_dev)
    model = rt.Model(shape, w_dev, "bf16")
    cache = rt.KVCache(model, B, n_ctx)
    counts = [170, 123]
    M = sum(counts)
    bn, sp, var = tiling
    for kind in range(4):
        model.set_tuning(kind, M, bn, sp, var)
        assert model.tuning(kind, M) == (bn, sp, var)
    with pytest.raises(RuntimeError):
        model.set_tuning(4, M, 128, -1, 0)            # the LM head takes no K split
    act = rt.Active(B, n_ctx)
    tokens, positions, ck, cv = _state(shape, B, n_ctx, counts, seed=12, dev=cuda_dev, dtype="bf16")
    act.load(positions)
    _load_cache(cache, ck, cv, torch.bfloat16)
    tok = torch.from_numpy(tokens).to(cuda_dev)
    logits = torch.zeros((B * n_ctx, shape.vocab), device=cuda_dev, dtype=torch.bfloat16)
    rt.step(model, cache, act, tok, logits)
    torch.cuda.synchronize()
    rt.device_check()
    zs, ck2, cv2 = _oracle_step(shape, w64, tokens, positions, ck, cv, n_ctx)
    lg = to64(logits)
    for b in range(B):
        err = np.abs(lg[positions[b] + b * n_ctx] - zs[b]).max()
        assert err <= LOGIT_TOL["bf16"], err
    model.close()


@pytest.mark.parametrize("splits", [1, 3])
def test_swapped_operand_tilings_step_matches_oracle(cuda_dev, splits):
    """Every projection GEMM pinned to the swapped-operand kernel (the weight
    tile as the 128-row MMA operand, the 220 active rows as its N): Q|K|V and
    gate/up through the fp32 workspace and their finishing kernels, the output
    and down projections by reduce-add into the residual stream."""
    shape = MINI_BF16
    B, n_ctx = 2, 200
    w_np = wl.np_weights(shape, seed=2, std=0.05, gain_jitter=0.1)
    w_dev = weights_to_device(w_np, "bf16", cuda_dev)
    w64 = weights_for_oracle(w_dev)
    model = rt.Model(shape, w_dev, "bf16")
    cache = rt.KVCache(model, B, n_ctx)
    counts = [130, 90]
    M = sum(counts)
    for kind in range(4):
        model.set_tuning(kind, M, 128, splits, 3)
        assert model.tuning(kind, M) == (128, splits, 3)
    with pytest.raises(RuntimeError):
        model.set_tuning(4, M, 128, 1, 3)             # not for the LM head
    with pytest.raises(RuntimeError):
        model.set_tuning(0, 300, 128, 1, 3)           # a bucket above 256 rows
    act = rt.Active(B, n_ctx)
    tokens, positions, ck, cv = _state(shape, B, n_ctx, counts, seed=13, dev=cuda_dev, dtype="bf16")
    act.load(positions)
    _load_cache(cache, ck, cv, torch.bfloat16)
    tok = torch.from_numpy(tokens).to(cuda_dev)
    logits = torch.zeros((B * n_ctx, shape.vocab), device=cuda_dev, dtype=torch.bfloat16)
    rt.step(model, cache, act, tok, logits)
    torch.cuda.synchronize()
    rt.device_check()
    zs, ck2, cv2 = _oracle_step(shape, w64, tokens, positions, ck, cv, n_ctx)
    lg = to64(logits)
    for b in range(B):
        err = np.abs(lg[positions[b] + b * n_ctx] - zs[b]).max()
        assert err <= LOGIT_TOL["bf16"], err
    model.close()


MINI_768 = wl.ModelShape(n_layers=2, d_model=768, n_heads=6, head_dim=128, d_ffn=768,
                         vocab=1024, mask_id=1023, rope_theta=10000.0)


@pytest.mark.parametrize("splits,variant", [(1, 0), (-1, 2), (2, 1)])
def test_bn192_tilings_step_matches_oracle(cuda_dev, splits, variant):
    """192-column tiles for every projection (QKV, whose unsplit epilogue
    rotates whole heads, through its split path): the step agrees with the
    oracle and with the same step on the library's default tilings."""
    shape = MINI_768
    B, n_ctx = 1, 300
    # weight scale of the d_model = 256 models (logits of the same magnitude)
    w_np = wl.np_weights(shape, seed=2, std=0.05 * (256 / 768) ** 0.5, gain_jitter=0.1)
    w_dev = weights_to_device(w_np, "bf16", cuda_dev)
    w64 = weights_for_oracle(w_dev)
    counts = [260]
    M = sum(counts)
    tokens, positions, ck, cv = _state(shape, B, n_ctx, counts, seed=13, dev=cuda_dev, dtype="bf16")
    tok = torch.from_numpy(tokens).to(cuda_dev)

    def run(pin):
        model = rt.Model(shape, w_dev, "bf16")
        if pin:
            for kind in range(4):
                sp = 2 if (kind == 0 and splits == 1) else splits
                model.set_tuning(kind, M, 192, sp, variant)
            with pytest.raises(RuntimeError):
                model.set_tuning(0, M, 192, 1, 0)          # unsplit QKV needs whole heads
        cache = rt.KVCache(model, B, n_ctx)
        act = rt.Active(B, n_ctx)
        act.load(positions)
        _load_cache(cache, ck, cv, torch.bfloat16)
        logits = torch.zeros((B * n_ctx, shape.vocab), device=cuda_dev, dtype=torch.bfloat16)
        rt.step(model, cache, act, tok, logits)
        torch.cuda.synchronize()
        rt.device_check()
        model.close()
        return to64(logits)[positions[0]]

    pinned, default = run(True), run(False)
    zs, _, _ = _oracle_step(shape, w64, tokens, positions, ck, cv, n_ctx)
    assert np.abs(pinned - zs[0]).max() <= LOGIT_TOL["bf16"]
    assert np.abs(default - zs[0]).max() <= LOGIT_TOL["bf16"]
    assert np.abs(pinned - default).max() <= LOGIT_TOL["bf16"]
