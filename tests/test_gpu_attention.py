"""Attention of the active queries over every cached key (sl_attention, bf16
path) against the oracle's attention in fp64, for both kernels: the tensor-core
kernel (tcgen05 + TMEM, TMA-fed K/V; the library's default) with one or two
128-query tiles per CTA and its key range whole or split across CTAs (merged by
per-row tickets), and the mma.sync kernel in each warp layout (16, 32 or 64 queries per
CTA, the key tile shared by 4, 2 or 1 warps); ragged query counts (several
128-query tiles, partial last tiles), empty sequences and key counts off the
tile grids.  Every layout is pinned in turn (sl_model_set_attention) as well as
left to the library's cost model, and every call runs twice on the same
workspace so that a ticket left non-zero would show."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import model as om
from token_locking_b200 import runtime as rt
from parity_util import to64, weights_to_device

pytestmark = pytest.mark.gpu

SHAPE = wl.ModelShape(n_layers=1, d_model=512, n_heads=4, head_dim=128, d_ffn=512, vocab=1024,
                      mask_id=1023, rope_theta=10000.0)

CASES = [
    ([5], 384),             # a handful of queries over the bench's key count
    ([1], 64),              # one query, one key tile
    ([16, 3], 130),         # ragged key tail
    ([30, 17], 700),
    ([100, 64, 1], 384),    # query tiles of several sizes in one launch
    ([7], 4000),            # long key range (splits of many tiles)
    ([200], 2500),
    ([0, 40, 0], 260),      # empty sequences
    ([300], 700),           # three 128-query tiles, the last one partial
    ([129, 128, 1], 384),   # tile boundaries one row either side
    ([257, 384, 130], 640), # two-tile CTAs with a lone third tile, full pairs, one ragged
]


# (queries per CTA, cross-CTA key split[, key tile]); 0 = the library's cost
# model.  128 or 256 queries per CTA = the tensor-core kernel (one or two
# 128-query tiles sharing each K/V tile; the default): one tile with 64-key
# tiles runs two CTAs per SM, one tile with 128-key tiles and two tiles (64-key)
# one CTA per SM; 16/32/64 the mma.sync kernel.
LAYOUTS = [(0, 0), (128, 1, 64), (128, 2, 64), (128, 16, 64), (128, 1, 128), (128, 3, 128),
           (128, 16, 128), (256, 1), (256, 2), (256, 5),
           (16, 1), (32, 1), (64, 1), (16, 4), (32, 2), (64, 3)]


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("counts,n_ctx", CASES)
def test_attention_matches_oracle(cuda_dev, counts, n_ctx, layout):
    B = len(counts)
    H, dh, d = SHAPE.n_heads, SHAPE.head_dim, SHAPE.d_model
    w_dev = weights_to_device(wl.np_weights(SHAPE, seed=0, std=0.05), "bf16", cuda_dev)
    model = rt.Model(SHAPE, w_dev, "bf16")
    model.set_attention(*layout)
    cache = rt.KVCache(model, B, n_ctx)
    act = rt.Active(B, n_ctx)
    rng = np.random.default_rng(sum(counts) + n_ctx)
    positions = [np.sort(rng.choice(n_ctx, c, replace=False)).astype(np.int32) for c in counts]
    act.load(positions)
    k_np = wl.round_bf16(rng.standard_normal((B * n_ctx, d)).astype(np.float32))
    v_np = wl.round_bf16(rng.standard_normal((B * n_ctx, d)).astype(np.float32))
    k, v = cache.view(0)
    k.copy_(torch.from_numpy(k_np).to(cuda_dev, torch.bfloat16))
    v.copy_(torch.from_numpy(v_np).to(cuda_dev, torch.bfloat16))
    M = sum(counts)
    q_np = wl.round_bf16(rng.standard_normal((max(M, 1), d)).astype(np.float32))[:M]
    q = torch.from_numpy(q_np).to(cuda_dev, torch.bfloat16)
    o = torch.full((max(M, 1), d), 9.0, device=cuda_dev, dtype=torch.bfloat16)
    rt.attention(model, cache, act, 0, q, o)
    torch.cuda.synchronize()
    rt.device_check()
    got = to64(o)
    o2 = torch.full_like(o, -5.0)
    rt.attention(model, cache, act, 0, q, o2)
    torch.cuda.synchronize()
    rt.device_check()
    assert torch.equal(o[:M], o2[:M]), "a second call on the same workspace differs"
    off = 0
    for b, c in enumerate(counts):
        if c == 0:
            continue
        qb = q_np[off:off + c].astype(np.float64).reshape(c, H, dh)
        kb = k_np[b * n_ctx:(b + 1) * n_ctx].astype(np.float64).reshape(n_ctx, H, dh)
        vb = v_np[b * n_ctx:(b + 1) * n_ctx].astype(np.float64).reshape(n_ctx, H, dh)
        ref = om.attention(qb, kb, vb).reshape(c, d)
        # P is rounded to bf16 before P V, the output to bf16
        err = np.abs(got[off:off + c] - ref).max()
        assert err <= 2e-2 * max(1.0, np.abs(ref).max()), f"seq {b}: max err {err}"
        off += c
    model.close()


# ---------------------------------------------- ablation: no KV cache ---
# Queries see the keys of their own sequence's active rows only (key stamps).

NOKV_CASES = [
    ([5], 384, None),
    ([16, 3], 130, None),
    ([100, 64, 1], 384, None),
    ([200], 2500, None),
    ([0, 40, 0], 260, None),
    # every active row in the first key tile of a long range: whole key splits
    # and tiles see no visible key at all
    ([12], 4000, "head"),
    # active rows only at the end of the range
    ([9, 20], 3000, "tail"),
]
NOKV_LAYOUTS = [(0, 0), (128, 1, 64), (128, 4, 64), (128, 1, 128), (128, 4, 128), (256, 1),
                (256, 3), (16, 1), (32, 2), (64, 3), (16, 4)]


def _positions(rng, counts, n_ctx, where):
    out = []
    for c in counts:
        if where == "head":
            out.append(np.sort(rng.choice(64, c, replace=False)).astype(np.int32))
        elif where == "tail":
            out.append(np.sort(n_ctx - 1 - rng.choice(100, c, replace=False)).astype(np.int32))
        else:
            out.append(np.sort(rng.choice(n_ctx, c, replace=False)).astype(np.int32))
    return out


def _attention_case(cuda_dev, model, cache, act, positions, n_ctx, shape, dtype, rng):
    B = len(positions)
    H, dh, d = shape.n_heads, shape.head_dim, shape.d_model
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    rnd = wl.round_bf16 if dtype == "bf16" else (lambda x: x)
    act.load(positions)
    k_np = rnd(rng.standard_normal((B * n_ctx, d)).astype(np.float32))
    v_np = rnd(rng.standard_normal((B * n_ctx, d)).astype(np.float32))
    k, v = cache.view(0)
    k.copy_(torch.from_numpy(k_np).to(cuda_dev, tdt))
    v.copy_(torch.from_numpy(v_np).to(cuda_dev, tdt))
    M = sum(len(p) for p in positions)
    q_np = rnd(rng.standard_normal((max(M, 1), d)).astype(np.float32))[:M]
    q = torch.from_numpy(q_np).to(cuda_dev, tdt)
    o = torch.full((max(M, 1), d), 9.0, device=cuda_dev, dtype=tdt)
    rt.attention(model, cache, act, 0, q, o)
    torch.cuda.synchronize()
    rt.device_check()
    got = to64(o)
    off = 0
    worst = 0.0
    for b, pos in enumerate(positions):
        c = len(pos)
        if c == 0:
            continue
        qb = q_np[off:off + c].astype(np.float64).reshape(c, H, dh)
        kb = k_np[b * n_ctx:(b + 1) * n_ctx].astype(np.float64).reshape(n_ctx, H, dh)[pos]
        vb = v_np[b * n_ctx:(b + 1) * n_ctx].astype(np.float64).reshape(n_ctx, H, dh)[pos]
        ref = om.attention(qb, kb, vb).reshape(c, d)
        worst = max(worst, np.abs(got[off:off + c] - ref).max() / max(1.0, np.abs(ref).max()))
        off += c
    return worst


@pytest.mark.parametrize("layout", NOKV_LAYOUTS)
@pytest.mark.parametrize("counts,n_ctx,where", NOKV_CASES)
def test_attention_no_kv_cache_matches_oracle(cuda_dev, counts, n_ctx, where, layout):
    B = len(counts)
    w_dev = weights_to_device(wl.np_weights(SHAPE, seed=0, std=0.05), "bf16", cuda_dev)
    model = rt.Model(SHAPE, w_dev, "bf16")
    model.set_attention(*layout)
    model.set_ablation(no_kv_cache=True)
    cache = rt.KVCache(model, B, n_ctx)
    act = rt.Active(B, n_ctx)
    rng = np.random.default_rng(7 * sum(counts) + n_ctx)
    # two calls on one cache with different active sets: the second must not
    # see the first call's keys
    for _ in range(2):
        positions = _positions(rng, counts, n_ctx, where)
        err = _attention_case(cuda_dev, model, cache, act, positions, n_ctx, SHAPE, "bf16", rng)
        assert err <= 2e-2, f"max rel err {err}"
    model.close()


SHAPE_F32 = wl.ModelShape(n_layers=1, d_model=64, n_heads=4, head_dim=16, d_ffn=64, vocab=64,
                          mask_id=63, rope_theta=10000.0)


@pytest.mark.parametrize("counts,n_ctx,where", [([7, 0, 30], 100, None), ([5], 300, "tail"),
                                                ([3, 4], 200, "head")])
def test_attention_f32_no_kv_cache_matches_oracle(cuda_dev, counts, n_ctx, where):
    """fp32 path: 32-key chunks with no visible key, before and after the first."""
    B = len(counts)
    w_dev = weights_to_device(wl.np_weights(SHAPE_F32, seed=0, std=0.05), "f32", cuda_dev)
    model = rt.Model(SHAPE_F32, w_dev, "f32")
    model.set_ablation(no_kv_cache=True)
    cache = rt.KVCache(model, B, n_ctx)
    act = rt.Active(B, n_ctx)
    rng = np.random.default_rng(n_ctx)
    for _ in range(2):
        positions = _positions(rng, counts, n_ctx, where)
        err = _attention_case(cuda_dev, model, cache, act, positions, n_ctx, SHAPE_F32, "f32", rng)
        assert err <= 1e-5, f"max rel err {err}"
    model.close()
