"""One whole sl_step of a two-layer model at the LLaDA-8B width (d_model 4096,
32 heads of 128, d_ffn 12288) with the full 126464-token vocabulary, against
the oracle on sampled rows, over a cache that already holds rows at the
positions that are not active (their K/V must be read and left untouched).

Every layer's keys depend on every active row, so the oracle runs layer 1 on
all M active rows, writes layer 2's fresh k, v of all M rows into its copy of
the cache (two projections per row), and finishes layer 2, the final norm and
the LM head on 16 sampled rows.  The oracle computes in fp32 on the device's
bf16 weights (an 8B-width layer in fp64 would take minutes on the host)."""
import json
import os

import numpy as np
import pytest
import torch

import workloads as wl
from parity_util import wide_logit_tol
from oracle import model as om
from token_locking_b200 import runtime as rt

pytestmark = pytest.mark.gpu

SHAPE = wl.ModelShape(n_layers=2, d_model=4096, n_heads=32, head_dim=128, d_ffn=12288,
                      vocab=126464, mask_id=126336, rope_theta=wl.LLADA8B.rope_theta)
N_CTX = 384
SAMPLE = 16


def oracle_sampled(w, tokens_np, pos, ck0, cv0, S):
    """Logits of the sampled active rows S and both layers' caches after the
    step: layer 1 on all active rows, layer 2's fresh k, v of all active rows,
    then layer 2, the final norm and the LM head on the sampled rows."""
    lw0, lw1 = w["layers"]
    h = w["tok_emb"][tokens_np[pos]].astype(np.float32)
    ck = [c.copy() for c in ck0]
    cv = [c.copy() for c in cv0]
    h1 = om.layer_forward(SHAPE, lw0, h, pos, ck[0], cv[0])
    k2, v2 = om.kv_of_block_input(SHAPE, lw1, h1, pos)
    ck[1][pos], cv[1][pos] = k2, v2
    h2 = om.layer_forward(SHAPE, lw1, h1[S], pos[S], ck[1].copy(), cv[1].copy())
    hf = om.rmsnorm(h2, w["final_norm"], SHAPE.rms_eps)
    return hf @ w["lm_head"].T, ck, cv


@pytest.fixture(scope="module")
def step8(cuda_dev):
    w_dev = wl.torch_weights(SHAPE, cuda_dev)
    torch.cuda.synchronize()

    def host(t):
        return t.float().cpu().numpy()

    w = {k: host(v) for k, v in w_dev.items() if k != "layers"}
    w["layers"] = [{k: host(v) for k, v in lw.items()} for lw in w_dev["layers"]]
    model = rt.Model(SHAPE, w_dev, "bf16")
    yield model, w
    model.close()


@pytest.mark.parametrize("M", [384, 200, 37])
def test_step_8b_width_full_vocab(step8, cuda_dev, M):
    model, w = step8
    cache = rt.KVCache(model, 1, N_CTX)
    act = rt.Active(1, N_CTX)
    rng = np.random.default_rng(M)
    d = SHAPE.d_model
    ck0 = [wl.round_bf16(rng.standard_normal((N_CTX, d)).astype(np.float32)) for _ in range(2)]
    cv0 = [wl.round_bf16(rng.standard_normal((N_CTX, d)).astype(np.float32)) for _ in range(2)]
    for l in range(2):
        k, v = cache.view(l)
        k.copy_(torch.from_numpy(ck0[l]).to(cuda_dev, torch.bfloat16))
        v.copy_(torch.from_numpy(cv0[l]).to(cuda_dev, torch.bfloat16))
    pos = np.sort(rng.choice(N_CTX, M, replace=False)).astype(np.int32)
    act.load([pos])
    tokens_np = wl.np_prompts(1, N_CTX, SHAPE.vocab, SHAPE.mask_id, seed=M)[0]
    tokens = torch.from_numpy(tokens_np).to(cuda_dev)
    logits = torch.zeros((N_CTX, SHAPE.vocab), device=cuda_dev, dtype=torch.bfloat16)
    rt.step(model, cache, act, tokens, logits)
    torch.cuda.synchronize()
    rt.device_check()

    S = np.sort(rng.choice(M, min(SAMPLE, M), replace=False))
    z_ref, ck, cv = oracle_sampled(w, tokens_np, pos, ck0, cv0, S)
    z_gpu = logits.float().cpu().numpy()[pos[S]]
    err = np.abs(z_gpu - z_ref).max()
    print(f"M={M}: logits max err {err:.4g} (|z| max {np.abs(z_ref).max():.3g})")
    path = os.environ.get("SL_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"test": "width8b-2layers", "M": M, "logits_max_abs_err": float(err),
                                "z_max_abs": float(np.abs(z_ref).max())}) + "\n")
    # bf16 activations, GEMM outputs and logits around fp32 residuals over two
    # 8B-width layers and the full vocabulary (parity_util.wide_logit_tol)
    tol = wide_logit_tol(float(np.abs(z_ref).max()))
    assert err <= tol, f"M={M}: logits max err {err} > {tol}"
    frozen = np.ones(N_CTX, dtype=bool)
    frozen[pos] = False
    for l in range(2):
        k, v = cache.view(l)
        kg, vg = k.float().cpu().numpy(), v.float().cpu().numpy()
        np.testing.assert_array_equal(kg[frozen], ck0[l][frozen])
        np.testing.assert_array_equal(vg[frozen], cv0[l][frozen])
        e = max(np.abs(kg[pos] - ck[l][pos]).max(), np.abs(vg[pos] - cv[l][pos]).max())
        assert e <= 3e-2 * max(1.0, np.abs(ck[l][pos]).max()), f"M={M} layer {l}: fresh K/V err {e}"
