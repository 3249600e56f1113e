"""The seeded input generators shared by the oracle and the CUDA path hold the
recipe the parity tests and benchmarks rely on: prompt ids never equal [MASK],
active subsets are sorted and unique, lock-test logits carry the stated spike
and perturbation, the bf16 rounding is round-to-nearest-even, and every draw is
reproducible from its seed."""
import numpy as np
import pytest
import torch

import workloads as wl


def test_prompts_avoid_mask_and_cover_the_vocabulary():
    V = 64
    for mask_id in (0, 17, V - 1):
        p = wl.np_prompts(8, 4000, V, mask_id, seed=3)
        assert p.dtype == np.int32 and p.shape == (8, 4000)
        assert p.min() >= 0 and p.max() < V
        assert not np.any(p == mask_id)
        counts = np.bincount(p.ravel(), minlength=V)
        others = np.delete(counts, mask_id)
        # uniform over the V - 1 other ids: every id drawn, none far off the mean
        assert others.min() > 0
        assert np.abs(others - others.mean()).max() < 6 * np.sqrt(others.mean())
    np.testing.assert_array_equal(wl.np_prompts(2, 9, 50, 49), wl.np_prompts(2, 9, 50, 49))


def test_initial_tokens_layout():
    pr = wl.np_prompts(3, 5, 40, 39)
    tok, msk = wl.initial_tokens(pr, 7, 39)
    assert tok.shape == (3, 12) and msk.shape == (3, 12)
    np.testing.assert_array_equal(tok[:, :5], pr)
    assert np.all(tok[:, 5:] == 39)
    assert np.all(msk[:, :5] == 0) and np.all(msk[:, 5:] == 1)


@pytest.mark.parametrize("m", [1, 8, 64, 2048])
def test_active_subset_sorted_unique_in_range(m):
    a = wl.np_active_subset(2048, m)
    assert a.dtype == np.int32 and a.shape == (m,)
    assert np.all(np.diff(a) > 0)
    assert a.min() >= 0 and a.max() < 2048


def test_lock_logits_recipe():
    m, V = 400, 4096
    z, zp, spiked = wl.np_lock_logits(m, V, seed=5)
    assert z.dtype == np.float32 and z.shape == (m, V)
    assert 0.4 < spiked.mean() < 0.6
    top2 = np.sort(z, axis=1)[:, -2:]
    gap = top2[:, 1] - top2[:, 0]
    # spiked rows: the spiked entry sits 8 above the rest of the row
    np.testing.assert_allclose(gap[spiked], 8.0, atol=1e-4)
    # unspiked rows: a plain N(0, 3) row; the gap between its two largest of
    # 4096 draws is about exponential with mean 3 / sqrt(2 ln 4096) ~ 0.74, so
    # none comes near the spike
    assert np.median(gap[~spiked]) < 1.0
    assert gap[~spiked].max() < 7.0
    body = z[~spiked]
    assert abs(body.std() - 3.0) < 0.05 and abs(body.mean()) < 0.05
    d = zp - z
    assert abs(d.std() - 0.05) < 0.002 and abs(d.mean()) < 0.002
    z2, zp2, s2 = wl.np_lock_logits(m, V, seed=5)
    np.testing.assert_array_equal(z, z2)
    np.testing.assert_array_equal(zp, zp2)
    # the literal variant adds 8 to one entry of the row instead
    zl, _, sl = wl.np_lock_logits(m, V, seed=5, literal_spike=True)
    np.testing.assert_array_equal(sl, spiked)
    diff = zl - z
    assert np.all(diff[~spiked] == 0)


def test_bf16_rounding_is_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 20000),
        np.array([0.0, -0.0, 1.0, -1.0, np.inf, -np.inf, 3.0e38, -3.0e38, 1e-40, -1e-40],
                 dtype=np.float32),
        # exact ties between two bf16 values: 1 + 2^-8 (to even: 1.0), 1 + 3 * 2^-8 (up)
        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)], dtype=np.float32),
    ]).astype(np.float32)       # both sides round the same float32 values
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(wl.to_bf16_bits(x), want)
    np.testing.assert_array_equal(wl.round_bf16(x),
                                  torch.from_numpy(x).to(torch.bfloat16).float().numpy())
    assert np.isnan(wl.round_bf16(np.array([np.nan], dtype=np.float32)))[0]


def test_weights_reproducible_and_scaled():
    shape = wl.ModelShape(n_layers=2, d_model=64, n_heads=4, head_dim=16, d_ffn=128, vocab=96,
                          mask_id=95, rope_theta=1e4)
    a = wl.np_weights(shape, seed=0)
    b = wl.np_weights(shape, seed=0)
    c = wl.np_weights(shape, seed=1)
    np.testing.assert_array_equal(a["layers"][1]["w_down"], b["layers"][1]["w_down"])
    assert not np.array_equal(a["lm_head"], c["lm_head"])
    allw = np.concatenate([a["tok_emb"].ravel(), a["lm_head"].ravel()] +
                          [v.ravel() for lw in a["layers"] for k, v in lw.items()
                           if not k.endswith("norm")])
    assert abs(allw.std() - 0.02) < 0.0005
    assert all(np.all(lw["attn_norm"] == 1) for lw in a["layers"])
    j = wl.np_weights(shape, seed=0, gain_jitter=0.1)
    # gains are drawn after every matrix: the matrices are unchanged
    np.testing.assert_array_equal(j["lm_head"], a["lm_head"])
    g = np.concatenate([lw["ffn_norm"] for lw in j["layers"]])
    assert abs(g.mean() - 1.0) < 0.05 and 0.05 < g.std() < 0.15


def test_torch_weights_recipe():
    """The device-side generator of the benchmark's weights, run on the CPU:
    bf16 [out, in] matrices N(0, std), unit gains, reproducible from the seed,
    and `layers` truncating the same draw sequence."""
    shape = wl.ModelShape(n_layers=3, d_model=128, n_heads=1, head_dim=128, d_ffn=256, vocab=512,
                          mask_id=511, rope_theta=1e4)
    cpu = torch.device("cpu")
    a = wl.torch_weights(shape, cpu)
    b = wl.torch_weights(shape, cpu)
    assert a["tok_emb"].dtype == torch.bfloat16 and tuple(a["tok_emb"].shape) == (512, 128)
    assert tuple(a["layers"][0]["w_gate"].shape) == (256, 128)
    assert tuple(a["layers"][0]["w_down"].shape) == (128, 256)
    assert tuple(a["lm_head"].shape) == (512, 128) and len(a["layers"]) == 3
    assert torch.equal(a["layers"][2]["wv"], b["layers"][2]["wv"])
    assert torch.all(a["final_norm"] == 1) and torch.all(a["layers"][1]["ffn_norm"] == 1)
    allw = torch.cat([a["tok_emb"].float().ravel()] +
                     [v.float().ravel() for lw in a["layers"] for k, v in lw.items()
                      if not k.endswith("norm")])
    assert abs(allw.std().item() - 0.02) < 0.001 and abs(allw.mean().item()) < 0.001
    # fewer layers: the same first draws
    c = wl.torch_weights(shape, cpu, layers=1)
    assert len(c["layers"]) == 1 and torch.equal(c["layers"][0]["wq"], a["layers"][0]["wq"])
    assert not torch.equal(wl.torch_weights(shape, cpu, seed=7)["lm_head"], a["lm_head"])
