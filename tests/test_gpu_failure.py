"""Failure detection on the GPU without a GPU fault.

* A bounded wait that runs out: with the GEMM's wait limit shortened to 20 ms
  and one operand copy left out (the library's test hook), the MMA warp's wait
  gives up; the kernel records SL_ERR_TIMEOUT in the device error word, drains
  its copies, frees its TMEM and returns.  The next launch must then be exact.
* Token ids outside [0, vocab): host prompts are refused before anything is
  enqueued (SL_ERR_INVALID); a bad id already on the device is embedded as
  zeros and reported by sl_device_check as SL_ERR_STATE, never used as an
  address; the next step with valid ids is unaffected.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from token_locking_b200 import _abi as A
from token_locking_b200 import runtime as rt
from parity_util import weights_to_device

pytestmark = pytest.mark.gpu

MINI_BF16 = wl.ModelShape(n_layers=2, d_model=256, n_heads=2, head_dim=128, d_ffn=512,
                          vocab=1024, mask_id=1023, rope_theta=10000.0)


def _gemm_ref(a, b):
    return (a.double() @ b.double().T).float()


def test_gemm_wait_runs_out_and_context_stays_usable(cuda_dev):
    g = torch.Generator(device=cuda_dev)
    g.manual_seed(3)
    M, N, K = 256, 512, 1024
    a = torch.randn(M, K, device=cuda_dev, generator=g).to(torch.bfloat16)
    b = torch.randn(N, K, device=cuda_dev, generator=g).to(torch.bfloat16)
    out = torch.zeros(M, N, device=cuda_dev, dtype=torch.bfloat16)
    rt.device_check(clear=True)
    try:
        rt.debug_set_wait_limit(20_000_000)          # 20 ms
        rt.debug_inject_lost_load()
        rt.gemm_bf16(A.GEMM_STORE, a, b, out, bn=128, splits=1, variant=0)
        torch.cuda.synchronize()
        with pytest.raises(A.SureLockError) as e:
            rt.device_check(clear=True)
        assert e.value.status == A.SL_ERR_TIMEOUT
        rt.device_check(clear=True)                   # cleared: nothing recorded since
    finally:
        rt.debug_set_wait_limit(0)
    # the hook was one-shot and the context survived: the same GEMM is exact now
    out.zero_()
    rt.gemm_bf16(A.GEMM_STORE, a, b, out, bn=128, splits=1, variant=0)
    torch.cuda.synchronize()
    rt.device_check(clear=True)
    ref = _gemm_ref(a, b)
    err = (out.float() - ref).abs().max().item()
    assert err <= 4e-3 * ref.abs().max().item()


def test_wait_limit_outside_range_is_refused(cuda_dev):
    for ns in (10, 3_000_000_000):
        with pytest.raises(A.SureLockError) as e:
            rt.debug_set_wait_limit(ns)
        assert e.value.status == A.SL_ERR_INVALID
    rt.debug_set_wait_limit(0)


def _mini_model(dev):
    w_np = wl.np_weights(MINI_BF16, seed=0, std=0.05)
    w_dev = weights_to_device(w_np, "bf16", dev)
    return rt.Model(MINI_BF16, w_dev, "bf16"), w_dev


def test_out_of_range_host_prompt_is_refused(cuda_dev):
    model, _ = _mini_model(cuda_dev)
    s = rt.Sampler(model, 2, 16, 32, 8, 32, 4, 0.01)
    prompts = wl.np_prompts(2, 16, MINI_BF16.vocab, MINI_BF16.mask_id)
    for bad in (MINI_BF16.vocab, -1):
        p = prompts.copy()
        p[1, 5] = bad
        with pytest.raises(A.SureLockError) as e:
            s.generate(p)
        assert e.value.status == A.SL_ERR_INVALID and "prompt id" in str(e.value)
    rt.device_check(clear=True)                      # nothing was enqueued
    out = s.generate(prompts)                        # valid prompts still decode
    assert np.array_equal(out[:, :16], prompts)
    assert np.all((out >= 0) & (out < MINI_BF16.vocab))
    s.close()
    model.close()


def test_out_of_range_device_token_is_reported_not_read(cuda_dev):
    model, _ = _mini_model(cuda_dev)
    B, n_ctx, V = 1, 64, MINI_BF16.vocab
    cache = rt.KVCache(model, B, n_ctx)
    act = rt.Active(B, n_ctx)
    act.reset()
    rng = np.random.default_rng(4)
    tokens = rng.integers(0, V - 1, (B, n_ctx)).astype(np.int32)
    good = torch.from_numpy(tokens).to(cuda_dev)
    logits_ref = torch.zeros(B * n_ctx, V, device=cuda_dev, dtype=torch.bfloat16)
    rt.step(model, cache, act, good, logits_ref)
    torch.cuda.synchronize()
    rt.device_check(clear=True)
    for bad_id in (V, 1 << 30, -7):
        bad = tokens.copy()
        bad[0, 9] = bad_id
        logits = torch.zeros_like(logits_ref)
        rt.step(model, cache, act, torch.from_numpy(bad).to(cuda_dev), logits)
        torch.cuda.synchronize()
        with pytest.raises(A.SureLockError) as e:
            rt.device_check(clear=True)
        assert e.value.status == A.SL_ERR_STATE and "token id" in str(e.value)
        assert torch.isfinite(logits.float()).all()
    # the error word was cleared and a valid step reproduces the first one (all
    # rows are active, so every cache row is rewritten before it is read; split-K
    # sums may add in another order, hence a bf16-rounding tolerance)
    logits = torch.zeros_like(logits_ref)
    rt.step(model, cache, act, good, logits)
    torch.cuda.synchronize()
    rt.device_check(clear=True)
    assert (logits.float() - logits_ref.float()).abs().max().item() <= 2e-2
    act.close()
    cache.close()
    model.close()
