"""Seeded synthetic workloads shared by the CUDA path's tests/bench and the oracle.

This module holds shapes, sampler settings and seeded random-number draws only.
It contains none of the method's arithmetic (no normalisation, attention,
softmax, KL, gate, compaction or sampling): both the oracle and the CUDA path
receive the arrays produced here as inputs.

The workloads follow the five settings used to evaluate SureLock
("Stopping Computation for Converged Tokens in Masked Diffusion-LM Decoding"):
a tiny fp32 model for exhaustive checks, one LLaDA-8B-shaped layer, the lock
test on LLaDA-sized vocabularies, and the full LLaDA-8B shape at batch 1
(N=384) and batch 4 (N=2048).  The pages evaluate on WikiText-103, MT-Bench
and HumanEval with trained LLaDA-8B weights; none of that is available here,
so random-init weights N(0, 0.02) and uniform random prompt ids stand in.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np

SEED_WEIGHTS = 0
SEED_PROMPTS = 1
SEED_MICRO = 2


@dataclasses.dataclass(frozen=True)
class ModelShape:
    n_layers: int
    d_model: int
    n_heads: int
    head_dim: int
    d_ffn: int
    vocab: int
    mask_id: int
    rope_theta: float
    rms_eps: float = 1e-5

    def linear_params_per_layer(self) -> int:
        d, f = self.d_model, self.d_ffn
        return 4 * d * d + 3 * d * f

    def linear_params(self) -> int:
        """Parameters touched by the per-row GEMMs of one step (layers + LM head)."""
        return self.n_layers * self.linear_params_per_layer() + self.vocab * self.d_model


# Tiny fp32 MDLM: 2 layers, d=64, 4 heads of 16, SwiGLU 256, vocab 512.
TINY = ModelShape(n_layers=2, d_model=64, n_heads=4, head_dim=16, d_ffn=256,
                  vocab=512, mask_id=511, rope_theta=10000.0)

# LLaDA-8B shape: 32 layers, d=4096, 32 heads of 128, SwiGLU 12288, vocab 126464.
# The [MASK] id 126336 is LLaDA's convention; the pages do not state it.
LLADA8B = ModelShape(n_layers=32, d_model=4096, n_heads=32, head_dim=128,
                     d_ffn=12288, vocab=126464, mask_id=126336,
                     rope_theta=500000.0)


@dataclasses.dataclass(frozen=True)
class SamplerSetup:
    """One semi-autoregressive SureLock decode: prompt + masked region."""
    shape: ModelShape
    dtype: str            # "f32" or "bf16"
    batch: int
    prompt_len: int
    gen_len: int
    steps: int
    block_len: int
    tokens_per_step: int
    eps: float
    gate_q: float = -1.0  # < 0: confidence gate off
    scripted: bool = False
    # ablations: the confidence gate as the only lock criterion; queries that
    # see the active rows' keys only (locked rows' cached K/V unused)
    gate_only: bool = False
    no_kv_cache: bool = False
    # K/V reuse for active rows, refresh interval R (1 = off): between refresh
    # steps the active rows that are neither masked nor just unmasked are not
    # recomputed; their cached K/V and last posterior stand in for them
    kv_reuse: int = 1

    @property
    def n_ctx(self) -> int:
        return self.prompt_len + self.gen_len

    @property
    def n_blocks(self) -> int:
        return self.gen_len // self.block_len

    @property
    def steps_per_block(self) -> int:
        return self.steps // self.n_blocks

    def validate(self) -> None:
        assert self.gen_len % self.block_len == 0
        assert self.steps % self.n_blocks == 0
        assert self.steps_per_block * self.tokens_per_step == self.block_len

    def block_bounds(self, t: int):
        """[lo, hi) of the block being decoded at step t (absolute positions)."""
        b = t // self.steps_per_block
        lo = self.prompt_len + b * self.block_len
        return lo, lo + self.block_len

    def scripted_target(self, t: int) -> int:
        """Scripted lock schedule: target active count after step t,
        round-half-up of N - 0.9 N (t+1)/(T-1), so M_t decays linearly to 10% of N."""
        n = self.n_ctx
        x = n - 0.9 * n * (t + 1) / (self.steps - 1)
        return int(math.floor(x + 0.5))


CFG_TINY = SamplerSetup(TINY, "f32", batch=1, prompt_len=16, gen_len=48, steps=16,
                        block_len=48, tokens_per_step=3, eps=0.01)


def cfg_full8b(eps: float = 0.05, scripted: bool = False) -> SamplerSetup:
    return SamplerSetup(LLADA8B, "bf16", batch=1, prompt_len=128, gen_len=256,
                        steps=256, block_len=32, tokens_per_step=1, eps=eps,
                        scripted=scripted)


def cfg_long8b() -> SamplerSetup:
    return SamplerSetup(LLADA8B, "bf16", batch=4, prompt_len=1024, gen_len=1024,
                        steps=512, block_len=64, tokens_per_step=2, eps=0.05,
                        gate_q=0.5)


LAYER_MICRO_M = (2048, 1024, 512, 256, 64, 8)
LAYER_MICRO_N = 2048
LOCK_MICRO_M = (64, 512, 2048)
LOCK_MICRO_EPS = (0.01, 0.05)
LOCK_MICRO_GATE_Q = 0.5


# ----------------------------------------------------------------------------
# numpy generators (host, used by CPU tests and small GPU cases)
# ----------------------------------------------------------------------------

def np_weights(shape: ModelShape, seed: int = SEED_WEIGHTS, std: float = 0.02,
               gain_jitter: float = 0.0, dtype=np.float32) -> dict:
    """Random-init weights, row-major [out, in].  Draw order: tok_emb, then per
    layer wq, wk, wv, wo, w_gate, w_up, w_down, then lm_head, then (if
    gain_jitter > 0) the norm gains 1 + gain_jitter * N(0, 1)."""
    rng = np.random.default_rng(seed)
    d, f, V, L = shape.d_model, shape.d_ffn, shape.vocab, shape.n_layers

    def nrm(*s):
        return (rng.standard_normal(s, dtype=np.float32) * std).astype(dtype)

    w = {"tok_emb": nrm(V, d), "layers": []}
    for _ in range(L):
        w["layers"].append({"wq": nrm(d, d), "wk": nrm(d, d), "wv": nrm(d, d),
                            "wo": nrm(d, d), "w_gate": nrm(f, d), "w_up": nrm(f, d),
                            "w_down": nrm(d, f)})
    w["lm_head"] = nrm(V, d)
    for lw in w["layers"]:
        for g in ("attn_norm", "ffn_norm"):
            if gain_jitter > 0:
                lw[g] = (1.0 + gain_jitter * rng.standard_normal(d)).astype(dtype)
            else:
                lw[g] = np.ones(d, dtype=dtype)
    if gain_jitter > 0:
        w["final_norm"] = (1.0 + gain_jitter * rng.standard_normal(d)).astype(dtype)
    else:
        w["final_norm"] = np.ones(d, dtype=dtype)
    return w


def np_prompts(batch: int, prompt_len: int, vocab: int, mask_id: int,
               seed: int = SEED_PROMPTS) -> np.ndarray:
    """Uniform prompt ids in [0, vocab) without mask_id, shape [batch, prompt_len]."""
    rng = np.random.default_rng(seed)
    r = rng.integers(0, vocab - 1, size=(batch, prompt_len), dtype=np.int64)
    return np.where(r >= mask_id, r + 1, r).astype(np.int32)


def initial_tokens(prompts: np.ndarray, gen_len: int, mask_id: int):
    """x_0 = prompt followed by gen_len [MASK] ids; returns (tokens, masked)."""
    b, p = prompts.shape
    tok = np.full((b, p + gen_len), mask_id, dtype=np.int32)
    tok[:, :p] = prompts
    masked = np.zeros((b, p + gen_len), dtype=np.uint8)
    masked[:, p:] = 1
    return tok, masked


def np_active_subset(n_ctx: int, m: int, seed: int = SEED_MICRO) -> np.ndarray:
    """Sorted random m-subset of [0, n_ctx) (the layer microbench's active rows)."""
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(n_ctx, size=m, replace=False)).astype(np.int32)


def np_lock_logits(m: int, vocab: int, seed: int = SEED_MICRO, sigma: float = 3.0,
                   spike_frac: float = 0.5, spike: float = 8.0,
                   prev_sigma: float = 0.05, literal_spike: bool = False):
    """Lock-test logits (float32, before any rounding): z ~ N(0, sigma) with a
    spiked entry on a random spike_frac of rows, and z_prev = z + N(0, prev_sigma).

    The spiked entry is set to (row max + spike); literal_spike=True instead adds
    spike to a random entry.  Returns (z, z_prev, spiked_rows)."""
    rng = np.random.default_rng(seed)
    z = (rng.standard_normal((m, vocab), dtype=np.float32) * sigma)
    spiked = rng.random(m) < spike_frac
    where = rng.integers(0, vocab, size=m)
    rows = np.nonzero(spiked)[0]
    if literal_spike:
        z[rows, where[rows]] += spike
    else:
        z[rows, where[rows]] = z[rows].max(axis=1) + spike
    z_prev = z + rng.standard_normal((m, vocab), dtype=np.float32) * prev_sigma
    return z, z_prev, spiked


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round-to-nearest-even), returned as uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    nan = np.isnan(x)
    out = rounded.astype(np.uint16)
    out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest bfloat16 value, kept as float32."""
    return bf16_bits_to_f32(to_bf16_bits(x))


# ----------------------------------------------------------------------------
# torch generators (device, for the LLaDA-8B-shaped workloads)
# ----------------------------------------------------------------------------

def torch_weights(shape: ModelShape, device, seed: int = SEED_WEIGHTS,
                  std: float = 0.02, layers: Optional[int] = None):
    """bf16 random-init weights generated on `device` with torch's generator.
    Same draw order as np_weights (values differ: another generator)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    d, f, V = shape.d_model, shape.d_ffn, shape.vocab
    L = shape.n_layers if layers is None else layers

    def nrm(*s):
        t = torch.empty(s, device=device, dtype=torch.bfloat16)
        t.normal_(0.0, std, generator=g)
        return t

    w = {"tok_emb": nrm(V, d), "layers": []}
    for _ in range(L):
        w["layers"].append({"wq": nrm(d, d), "wk": nrm(d, d), "wv": nrm(d, d),
                            "wo": nrm(d, d), "w_gate": nrm(f, d), "w_up": nrm(f, d),
                            "w_down": nrm(d, f),
                            "attn_norm": torch.ones(d, device=device, dtype=torch.bfloat16),
                            "ffn_norm": torch.ones(d, device=device, dtype=torch.bfloat16)})
    w["lm_head"] = nrm(V, d)
    w["final_norm"] = torch.ones(d, device=device, dtype=torch.bfloat16)
    return w


def torch_lock_logits(m: int, vocab: int, device, seed: int = SEED_MICRO,
                      sigma: float = 3.0, spike_frac: float = 0.5, spike: float = 8.0,
                      prev_sigma: float = 0.05):
    """Device version of np_lock_logits returning bf16 (z, z_prev) and the spiked mask."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    z = torch.randn((m, vocab), device=device, generator=g) * sigma
    spiked = torch.rand(m, device=device, generator=g) < spike_frac
    where = torch.randint(0, vocab, (m,), device=device, generator=g)
    rows = torch.nonzero(spiked).flatten()
    z[rows, where[rows]] = z[rows].max(dim=1).values + spike
    z_prev = z + torch.randn((m, vocab), device=device, generator=g) * prev_sigma
    return z.to(torch.bfloat16), z_prev.to(torch.bfloat16), spiked
