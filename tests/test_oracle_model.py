"""Pins for the oracle denoiser (CPU only).

Each check ties the oracle to something other than itself: closed forms written
out from the definitions (tests/golden/closed_forms.json), scalar-loop brute
force (oracle.brute), or invariants of the operation."""
import json
import math
import os

import numpy as np
import pytest

import workloads as wl
from oracle import brute
from oracle import model as om

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")))

MICRO = wl.ModelShape(n_layers=2, d_model=16, n_heads=2, head_dim=8, d_ffn=24,
                      vocab=20, mask_id=19, rope_theta=10000.0)


def test_rmsnorm_closed_form():
    c = GOLD["rmsnorm_3_4"]
    y = om.rmsnorm(np.array([c["x"]]), np.ones(2), c["eps"])
    np.testing.assert_allclose(y[0], c["y"], rtol=1e-15)


def test_rmsnorm_gain_and_brute():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 7))
    g = 1 + 0.3 * rng.standard_normal(7)
    np.testing.assert_allclose(om.rmsnorm(x, g, 1e-5), brute.rmsnorm(x.tolist(), g.tolist(), 1e-5),
                               rtol=1e-13)
    # gains scale channels: rmsnorm(x, g) = rmsnorm(x, 1) * g
    np.testing.assert_allclose(om.rmsnorm(x, g, 1e-5), om.rmsnorm(x, np.ones(7), 1e-5) * g, rtol=1e-14)


def test_silu_closed_form():
    assert om.silu(np.array(GOLD["silu_1"]["x"])) == pytest.approx(GOLD["silu_1"]["y"], rel=1e-15)
    assert om.silu(np.array(0.0)) == 0.0
    assert om.silu(np.array(40.0)) == pytest.approx(40.0, rel=1e-15)


def test_rope_closed_form():
    c = GOLD["rope_dh4_pos1"]
    x = np.array(c["x"]).reshape(1, 1, 4)
    y = om.rope(x, np.array([c["pos"]]), c["theta"])
    np.testing.assert_allclose(y[0, 0], c["y"], rtol=1e-14)


def test_rope_invariants():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 3, 16))
    k = rng.standard_normal((1, 3, 16))
    # position 0 is the identity
    np.testing.assert_array_equal(om.rope(q, np.array([0]), 1e4), q)
    # the rotation keeps each pair's norm, hence the vector norm
    np.testing.assert_allclose(np.linalg.norm(om.rope(q, np.array([37]), 1e4), axis=-1),
                               np.linalg.norm(q, axis=-1), rtol=1e-13)
    # scores depend on the relative position only
    def score(p1, p2):
        return np.sum(om.rope(q, np.array([p1]), 1e4) * om.rope(k, np.array([p2]), 1e4), axis=-1)
    np.testing.assert_allclose(score(5, 2), score(105, 102), rtol=1e-10, atol=1e-12)
    # matches the scalar loop
    y = om.rope(q, np.array([11]), 1e4)
    for h in range(3):
        np.testing.assert_allclose(y[0, h], brute.rope_vec(q[0, h].tolist(), 11, 1e4), rtol=1e-13)


def test_attention_brute_and_special_cases():
    rng = np.random.default_rng(7)
    M, N, H, dh = 3, 5, 2, 4
    q = rng.standard_normal((M, H, dh))
    k = rng.standard_normal((N, H, dh))
    v = rng.standard_normal((N, H, dh))
    o = om.attention(q, k, v)
    for m in range(M):
        for h in range(H):
            ref = brute.attention_head(q[m, h].tolist(), k[:, h].tolist(), v[:, h].tolist())
            np.testing.assert_allclose(o[m, h], ref, rtol=1e-13)
    # identical keys: uniform weights, output = mean of the values
    ke = np.repeat(k[:1], N, axis=0)
    np.testing.assert_allclose(om.attention(q, ke, v), np.broadcast_to(v.mean(0), (M, H, dh)),
                               rtol=1e-13)
    # one key aligned with a huge query dominates: output = its value
    qb = np.zeros((1, 1, dh)); qb[0, 0, 0] = 1e3
    kb = np.zeros((N, 1, dh)); kb[3, 0, 0] = 1.0
    np.testing.assert_allclose(om.attention(qb, kb, v[:, :1]), v[3:4, :1], rtol=1e-12)


def _micro_weights(seed=0):
    return om.cast_weights(wl.np_weights(MICRO, seed=seed, std=0.3, gain_jitter=0.2), np.float64)


def test_forward_active_matches_loops_with_frozen_rows():
    """Whole denoiser on an active subset over a cache holding frozen rows."""
    w = _micro_weights()
    N, L, d = 6, MICRO.n_layers, MICRO.d_model
    rng = np.random.default_rng(8)
    tokens = rng.integers(0, MICRO.vocab, N).astype(np.int32)
    ck = rng.standard_normal((L, N, d))
    cv = rng.standard_normal((L, N, d))
    pos = np.array([0, 2, 3, 5], dtype=np.int32)
    bk, bv = ck.tolist(), cv.tolist()
    z = om.forward_active(MICRO, w, tokens, pos, ck, cv)
    wl_ = {k: (v.tolist() if hasattr(v, "tolist") else v) for k, v in w.items() if k != "layers"}
    wl_["layers"] = [{k: v.tolist() for k, v in lw.items()} for lw in w["layers"]]
    zb = brute.forward_active(MICRO, wl_, tokens.tolist(), pos.tolist(), bk, bv)
    np.testing.assert_allclose(z, zb, rtol=1e-11, atol=1e-12)
    # frozen rows (1 and 4) are untouched, fresh rows agree with the loops
    np.testing.assert_allclose(ck, np.array(bk), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(cv, np.array(bv), rtol=1e-11, atol=1e-12)


def test_forward_active_all_rows_equals_full_forward_bitwise():
    """With every row active and the cache fully overwritten, the gathered,
    cached computation is the unmodified denoiser, bit for bit."""
    w = _micro_weights(1)
    N = 7
    rng = np.random.default_rng(9)
    tokens = rng.integers(0, MICRO.vocab, N).astype(np.int32)
    ck = np.zeros((MICRO.n_layers, N, MICRO.d_model))
    cv = np.zeros_like(ck)
    z = om.forward_active(MICRO, w, tokens, np.arange(N, dtype=np.int32), ck, cv)
    np.testing.assert_array_equal(z, om.forward_full(MICRO, w, tokens))


def test_kv_of_block_input_reproduces_cache():
    w = _micro_weights(2)
    N = 5
    tokens = np.arange(N, dtype=np.int32)
    ck = np.zeros((MICRO.n_layers, N, MICRO.d_model)); cv = np.zeros_like(ck)
    pos = np.arange(N, dtype=np.int32)
    blk = []
    om.forward_active(MICRO, w, tokens, pos, ck, cv, blk)
    for l in range(MICRO.n_layers):
        k, v = om.kv_of_block_input(MICRO, w["layers"][l], blk[l], pos)
        np.testing.assert_array_equal(k, ck[l])
        np.testing.assert_array_equal(v, cv[l])


# ------------------------------------------- ablation: no KV cache ---

def _micro_case(seed, N):
    rng = np.random.default_rng(seed)
    tokens = rng.integers(0, MICRO.vocab, N).astype(np.int32)
    ck = rng.standard_normal((MICRO.n_layers, N, MICRO.d_model))
    cv = rng.standard_normal((MICRO.n_layers, N, MICRO.d_model))
    return tokens, ck, cv


def test_no_kv_cache_matches_loops():
    """Queries attend to the active rows only: vectorised vs scalar loops."""
    w = _micro_weights()
    tokens, ck, cv = _micro_case(10, 6)
    pos = np.array([0, 2, 3, 5], dtype=np.int32)
    bk, bv = ck.tolist(), cv.tolist()
    z = om.forward_active(MICRO, w, tokens, pos, ck, cv, no_kv_cache=True)
    wl_ = {k: (v.tolist() if hasattr(v, "tolist") else v) for k, v in w.items() if k != "layers"}
    wl_["layers"] = [{k: v.tolist() for k, v in lw.items()} for lw in w["layers"]]
    zb = brute.forward_active(MICRO, wl_, tokens.tolist(), pos.tolist(), bk, bv, no_kv_cache=True)
    np.testing.assert_allclose(z, zb, rtol=1e-11, atol=1e-12)
    # and it is a different computation from the method's (locked keys matter there)
    z_full = om.forward_active(MICRO, w, tokens, pos, *_micro_case(10, 6)[1:])
    assert np.abs(z - z_full).max() > 1e-3


def test_no_kv_cache_contiguous_run_is_the_full_denoiser_on_it():
    """A contiguous active run [p0, p0 + M) attending only to itself is the
    unmodified denoiser on that sub-sequence: rotary scores depend on relative
    positions only, so the absolute offset p0 drops out (up to rounding)."""
    w = _micro_weights(3)
    N, p0, M = 11, 4, 5
    tokens, ck, cv = _micro_case(11, N)
    pos = np.arange(p0, p0 + M, dtype=np.int32)
    z = om.forward_active(MICRO, w, tokens, pos, ck, cv, no_kv_cache=True)
    np.testing.assert_allclose(z, om.forward_full(MICRO, w, tokens[p0:p0 + M]), rtol=1e-10, atol=1e-10)


def test_no_kv_cache_ignores_locked_rows_cache():
    w = _micro_weights(4)
    N = 8
    tokens, ck, cv = _micro_case(12, N)
    pos = np.array([1, 2, 6], dtype=np.int32)
    locked = np.setdiff1d(np.arange(N), pos)
    ck2, cv2 = ck.copy(), cv.copy()
    ck2[:, locked] += 5.0
    cv2[:, locked] -= 3.0
    za = om.forward_active(MICRO, w, tokens, pos, ck.copy(), cv.copy(), no_kv_cache=True)
    zb = om.forward_active(MICRO, w, tokens, pos, ck2.copy(), cv2.copy(), no_kv_cache=True)
    np.testing.assert_array_equal(za, zb)
    # the method reads those rows, so the same change moves its logits
    zc = om.forward_active(MICRO, w, tokens, pos, ck.copy(), cv.copy())
    zd = om.forward_active(MICRO, w, tokens, pos, ck2.copy(), cv2.copy())
    assert np.abs(zc - zd).max() > 1e-3


def test_no_kv_cache_with_every_row_active_is_the_method_bitwise():
    w = _micro_weights(5)
    N = 7
    tokens, ck, cv = _micro_case(13, N)
    pos = np.arange(N, dtype=np.int32)
    np.testing.assert_array_equal(
        om.forward_active(MICRO, w, tokens, pos, ck.copy(), cv.copy(), no_kv_cache=True),
        om.forward_active(MICRO, w, tokens, pos, ck.copy(), cv.copy()))
