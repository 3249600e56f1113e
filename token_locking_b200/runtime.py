"""Python binding of libsurelock.so: argument marshalling only.

PyTorch supplies device memory and streams; every step of the decoding path
(gather, projections, attention, LM head, sure test, gate, compaction,
unmasking) runs in the library's CUDA kernels.  Device buffers owned by the
library are exposed to Python as zero-copy torch views through the CUDA array
interface.
"""
from __future__ import annotations

import ctypes as C
from typing import Optional, Sequence

import numpy as np
import torch

from . import _abi as A

_TORCH_DT = {A.SL_F32: torch.float32, A.SL_BF16: torch.bfloat16}


def _dtype_code(dtype) -> int:
    if dtype in ("bf16", torch.bfloat16, A.SL_BF16):
        return A.SL_BF16
    if dtype in ("f32", "fp32", torch.float32, A.SL_F32):
        return A.SL_F32
    raise ValueError(f"unsupported dtype {dtype!r}")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return t.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        s = torch.cuda.current_stream()
    return s.cuda_stream


class _DevView:
    """Zero-copy view of library-owned device memory (CUDA array interface)."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (ptr, False), "version": 3, "strides": None}


def device_view(ptr: int, shape, dtype: torch.dtype) -> torch.Tensor:
    ts = {torch.float32: "<f4", torch.int32: "<i4", torch.uint8: "|u1", torch.bfloat16: "<i2",
          torch.int16: "<i2"}[dtype]
    t = torch.as_tensor(_DevView(ptr, shape, ts), device="cuda")
    return t.view(torch.bfloat16) if dtype == torch.bfloat16 else t


class Model:
    """sl_model over torch weight tensors (kept alive by this object).

    weights: dict with tok_emb [V,d], final_norm [d], lm_head [V,d] and
    layers: list of dicts (attn_norm, wq, wk, wv, wo, ffn_norm, w_gate, w_up,
    w_down), all contiguous CUDA tensors of the model dtype."""

    def __init__(self, shape, weights: dict, dtype="bf16"):
        self.shape = shape
        self.dtype = _dtype_code(dtype)
        self.torch_dtype = _TORCH_DT[self.dtype]
        self._w = weights
        cfg = A.Config(shape.n_layers, shape.d_model, shape.n_heads, shape.head_dim, shape.d_ffn,
                       shape.vocab, shape.mask_id, shape.rms_eps, shape.rope_theta, self.dtype)
        names = ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down")
        arr = (A.LayerWeights * shape.n_layers)()
        for l, lw in enumerate(weights["layers"]):
            for n in names:
                t = lw[n]
                if t.dtype != self.torch_dtype:
                    raise ValueError(f"layer {l} {n}: dtype {t.dtype}, expected {self.torch_dtype}")
                setattr(arr[l], n, _ptr(t))
        self._layers_arr = arr
        w = A.Weights(_ptr(weights["tok_emb"]), _ptr(weights["final_norm"]),
                      _ptr(weights["lm_head"]), C.cast(arr, C.POINTER(A.LayerWeights)))
        h = C.c_void_p()
        A.check(A.lib().sl_model_create(C.byref(cfg), C.byref(w), C.byref(h)), "sl_model_create")
        self.handle = h

    def close(self):
        if getattr(self, "handle", None):
            A.lib().sl_model_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def autotune(self, cache: "KVCache", max_rows: int, stream=None):
        """Time the GEMM tilings on this device and keep the fastest per row count."""
        A.check(A.lib().sl_model_autotune(self.handle, cache.handle, max_rows, _stream(stream)),
                "sl_model_autotune")

    def tuning(self, kind: int, M: int):
        """(bn, splits, variant) of GEMM `kind` at M rows."""
        bn, sp, var = C.c_int(), C.c_int(), C.c_int()
        A.check(A.lib().sl_model_tuning(self.handle, kind, M, C.byref(bn), C.byref(sp),
                                        C.byref(var)), "sl_model_tuning")
        return bn.value, sp.value, var.value

    def set_attention(self, queries_per_cta: int = 0, splits: int = 0, key_tile: int = 0):
        """Pin the attention layout (0 = the library's cost model)."""
        A.check(A.lib().sl_model_set_attention(self.handle, queries_per_cta, splits),
                "sl_model_set_attention")
        A.check(A.lib().sl_model_set_attention_keys(self.handle, key_tile),
                "sl_model_set_attention_keys")

    def set_ablation(self, no_kv_cache: bool = False, gate_only: bool = False):
        """Ablations of the method: attention without the locked rows' cached
        K/V; the confidence gate as the only lock criterion of the samplers."""
        flags = (A.ABLATE_NO_KV_CACHE if no_kv_cache else 0) | (A.ABLATE_GATE_ONLY if gate_only else 0)
        A.check(A.lib().sl_model_set_ablation(self.handle, flags), "sl_model_set_ablation")

    def set_head_fusion(self, enable: bool = True):
        """Samplers take the sure test's statistics from the LM head's epilogue
        (True, the default) or from a separate pass over the logits."""
        A.check(A.lib().sl_model_set_head_fusion(self.handle, 1 if enable else 0),
                "sl_model_set_head_fusion")

    def set_tuning(self, kind: int, M: int, bn: int, splits: int, variant: int):
        """Pin GEMM `kind`'s tiling for the row-count bucket of M (splits -1: stream-K)."""
        A.check(A.lib().sl_model_set_tuning(self.handle, kind, M, bn, splits, variant),
                "sl_model_set_tuning")

    def timing_enable(self, on: bool = True):
        A.check(A.lib().sl_timing_enable(self.handle, 1 if on else 0), "sl_timing_enable")

    def timing_read(self, reset: bool = True) -> dict:
        t = A.Timing()
        A.check(A.lib().sl_timing_read(self.handle, C.byref(t), 1 if reset else 0), "sl_timing_read")
        names = ["gemm", "attn", "lock", "other"]
        out = {n: {"ms": t.ms[i], "bytes": t.bytes[i], "flops": t.flops[i],
                   "launches": int(t.launches[i])} for i, n in enumerate(names)}
        out["kernels"] = int(t.kernels)
        return out


class KVCache:
    def __init__(self, model: Model, batch: int, n_ctx: int):
        self.model, self.batch, self.n_ctx = model, batch, n_ctx
        h = C.c_void_p()
        A.check(A.lib().sl_kv_cache_create(model.handle, batch, n_ctx, C.byref(h)),
                "sl_kv_cache_create")
        self.handle = h
        self.owned = True

    @classmethod
    def wrap(cls, handle, model: Model, batch: int, n_ctx: int):
        self = cls.__new__(cls)
        self.model, self.batch, self.n_ctx, self.handle, self.owned = model, batch, n_ctx, handle, False
        return self

    def reset(self, stream=None):
        A.check(A.lib().sl_kv_cache_reset(self.handle, _stream(stream)), "sl_kv_cache_reset")

    def view(self, layer: int):
        """(k, v) of one layer as torch views [batch*n_ctx, d_model]."""
        k, v = C.c_void_p(), C.c_void_p()
        A.check(A.lib().sl_kv_cache_view(self.handle, layer, C.byref(k), C.byref(v)),
                "sl_kv_cache_view")
        shape = (self.batch * self.n_ctx, self.model.shape.d_model)
        return (device_view(k.value, shape, self.model.torch_dtype),
                device_view(v.value, shape, self.model.torch_dtype))

    def close(self):
        if getattr(self, "handle", None) and self.owned:
            A.lib().sl_kv_cache_destroy(self.handle)
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Active:
    """The active set A_t: flat ascending positions b*n_ctx+i plus offsets."""

    def __init__(self, batch: int, n_ctx: int):
        self.batch, self.n_ctx = batch, n_ctx
        h = C.c_void_p()
        A.check(A.lib().sl_active_create(batch, n_ctx, C.byref(h)), "sl_active_create")
        self.handle = h
        self.owned = True

    @classmethod
    def wrap(cls, handle, batch: int, n_ctx: int):
        self = cls.__new__(cls)
        self.batch, self.n_ctx, self.handle, self.owned = batch, n_ctx, handle, False
        return self

    def reset(self, stream=None):
        A.check(A.lib().sl_active_reset(self.handle, _stream(stream)), "sl_active_reset")

    def load(self, positions: Sequence[np.ndarray], stream=None):
        counts = np.array([len(p) for p in positions], dtype=np.int32)
        flat = (np.concatenate([np.asarray(p, dtype=np.int32) for p in positions])
                if counts.sum() else np.zeros(1, dtype=np.int32))
        A.check(A.lib().sl_active_load(self.handle, counts.ctypes.data_as(C.POINTER(C.c_int32)),
                                       flat.ctypes.data_as(C.POINTER(C.c_int32)), _stream(stream)),
                "sl_active_load")

    def counts(self) -> np.ndarray:
        out = np.zeros(self.batch, dtype=np.int32)
        A.check(A.lib().sl_active_counts(self.handle, out.ctypes.data_as(C.POINTER(C.c_int32))),
                "sl_active_counts")
        return out

    def view(self):
        """(rows [M], seq_off [batch+1]) as int32 torch views (current M)."""
        r, o = C.c_void_p(), C.c_void_p()
        A.check(A.lib().sl_active_view(self.handle, C.byref(r), C.byref(o)), "sl_active_view")
        m = int(self.counts().sum())
        rows = device_view(r.value, (self.batch * self.n_ctx,), torch.int32)[:m]
        return rows, device_view(o.value, (self.batch + 1,), torch.int32)

    def positions(self):
        """Per-sequence ascending local positions (host copy)."""
        rows, off = self.view()
        rows = rows.cpu().numpy()
        off = off.cpu().numpy()
        return [rows[off[b]:off[b + 1]] - b * self.n_ctx for b in range(self.batch)]

    def close(self):
        if getattr(self, "handle", None) and self.owned:
            A.lib().sl_active_destroy(self.handle)
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def step(model: Model, cache: KVCache, active: Active, tokens: torch.Tensor,
         logits: torch.Tensor, stream=None):
    A.check(A.lib().sl_step(model.handle, cache.handle, active.handle, _ptr(tokens), _ptr(logits),
                            _stream(stream)), "sl_step")


def layer_forward(model: Model, cache: KVCache, active: Active, layer: int, h: torch.Tensor,
                  stream=None):
    """One block on the active rows; h [M, d] fp32 is updated in place."""
    if h.dtype != torch.float32:
        raise ValueError("hidden states must be fp32")
    A.check(A.lib().sl_layer_forward(model.handle, cache.handle, active.handle, layer, _ptr(h),
                                     _stream(stream)), "sl_layer_forward")


def attention(model: Model, cache: KVCache, active: Active, layer: int, q: torch.Tensor,
              o: torch.Tensor, stream=None):
    A.check(A.lib().sl_attention(model.handle, cache.handle, active.handle, layer, _ptr(q),
                                 _ptr(o), _stream(stream)), "sl_attention")


def gemm_bf16(epi: int, a: torch.Tensor, b: torch.Tensor, out: torch.Tensor, b2=None, ldo=None,
              row_map=None, bn: int = 0, splits: int = 0, variant: int = 0, stream=None):
    """out (op)= a @ b.T on the tensor cores (see sl_gemm_bf16)."""
    M, K = a.shape
    N = b.shape[0] * (2 if b2 is not None else 1)
    ldo = out.shape[-1] if ldo is None else ldo
    A.check(A.lib().sl_gemm_bf16(epi, _ptr(a), M, K, _ptr(b), _ptr(b2), N, _ptr(out), ldo,
                                 _ptr(row_map), bn, splits, variant, _stream(stream)),
            "sl_gemm_bf16")


def device_check(clear: bool = True):
    A.check(A.lib().sl_device_check(1 if clear else 0), "sl_device_check")


def debug_set_wait_limit(ns: int):
    """Barrier-wait limit of later GEMM launches in ns (0 = the default 2 s)."""
    A.check(A.lib().sl_debug_set_wait_limit(int(ns)), "sl_debug_set_wait_limit")


def debug_inject_lost_load():
    """The next 1-SM GEMM launch leaves out its first stage's copies (test hook)."""
    A.check(A.lib().sl_debug_inject_lost_load(), "sl_debug_inject_lost_load")


def kl_lock(active: Active, vocab: int, mask_id: int, logits_cur: torch.Tensor,
            logits_prev: Optional[torch.Tensor], lse_prev: Optional[torch.Tensor],
            lse_cur: torch.Tensor, masked: torch.Tensor, kl: torch.Tensor, unc: torch.Tensor,
            conf: torch.Tensor, argmax: torch.Tensor, lock: torch.Tensor, eps: float,
            gate_q: float = -1.0, has_prev: bool = True, scripted_target: int = -1,
            gate_only: bool = False, stream=None):
    p = A.LockParams(eps, gate_q, 1 if has_prev else 0, scripted_target, 1 if gate_only else 0)
    A.check(A.lib().sl_kl_lock(active.handle, vocab, mask_id, _dtype_code(logits_cur.dtype),
                               _ptr(logits_cur), _ptr(logits_prev), _ptr(lse_prev), _ptr(lse_cur),
                               _ptr(masked), C.byref(p), _ptr(kl), _ptr(unc), _ptr(conf),
                               _ptr(argmax), _ptr(lock), _stream(stream)), "sl_kl_lock")


def step_stats(model: Model, cache: KVCache, active: Active, tokens: torch.Tensor,
               logits: torch.Tensor, logits_prev: Optional[torch.Tensor],
               lse_prev: Optional[torch.Tensor], lse_cur: torch.Tensor, kl: torch.Tensor,
               unc: torch.Tensor, conf: torch.Tensor, argmax: torch.Tensor,
               has_prev: bool = True, stream=None):
    """sl_step with the sure test's statistics taken in the LM head's epilogue."""
    A.check(A.lib().sl_step_stats(model.handle, cache.handle, active.handle, _ptr(tokens),
                                  _ptr(logits), _ptr(logits_prev), _ptr(lse_prev),
                                  1 if has_prev else 0, _ptr(lse_cur), _ptr(kl), _ptr(unc),
                                  _ptr(conf), _ptr(argmax), _stream(stream)), "sl_step_stats")


def lock_decide(active: Active, masked: torch.Tensor, kl: torch.Tensor, unc: torch.Tensor,
                lock: torch.Tensor, eps: float, gate_q: float = -1.0, has_prev: bool = True,
                scripted_target: int = -1, gate_only: bool = False, stream=None):
    """The lock flags from precomputed statistics (sl_lock_decide)."""
    p = A.LockParams(eps, gate_q, 1 if has_prev else 0, scripted_target, 1 if gate_only else 0)
    A.check(A.lib().sl_lock_decide(active.handle, _ptr(masked), C.byref(p), _ptr(kl), _ptr(unc),
                                   _ptr(lock), _stream(stream)), "sl_lock_decide")


def kl_stats_noalloc(rows: torch.Tensor, vocab: int, mask_id: int, logits_cur: torch.Tensor,
                     logits_prev: Optional[torch.Tensor], lse_prev: Optional[torch.Tensor],
                     lse_cur: torch.Tensor, kl: torch.Tensor, unc: torch.Tensor,
                     conf: torch.Tensor, argmax: torch.Tensor, has_prev: bool = True,
                     stream=None):
    """Sure-test statistics without any device allocation by the library
    (sl_kl_stats_noalloc): for hosts that own all device memory themselves."""
    if rows.dtype != torch.int32:
        raise ValueError("rows must be int32")
    A.check(A.lib().sl_kl_stats_noalloc(_ptr(rows), rows.numel(), vocab, mask_id,
                                        _dtype_code(logits_cur.dtype), _ptr(logits_cur),
                                        _ptr(logits_prev), _ptr(lse_prev), _ptr(lse_cur),
                                        1 if has_prev else 0, _ptr(kl), _ptr(unc), _ptr(conf),
                                        _ptr(argmax), _stream(stream)), "sl_kl_stats_noalloc")


def unmask_topk(active: Active, conf: torch.Tensor, argmax: torch.Tensor, block_lo: int,
                block_hi: int, k: int, tokens: torch.Tensor, masked: torch.Tensor, stream=None):
    A.check(A.lib().sl_unmask_topk(active.handle, _ptr(conf), _ptr(argmax), block_lo, block_hi, k,
                                   _ptr(tokens), _ptr(masked), _stream(stream)), "sl_unmask_topk")


def compact_active(active: Active, lock: torch.Tensor, locked: torch.Tensor, lock_t: torch.Tensor,
                   step_idx: int, stream=None):
    A.check(A.lib().sl_compact_active(active.handle, _ptr(lock), _ptr(locked), _ptr(lock_t),
                                      step_idx, _stream(stream)), "sl_compact_active")


class Sampler:
    """Library-driven SureLock decode (sl_sampler_*)."""

    def __init__(self, model: Model, batch: int, prompt_len: int, gen_len: int, steps: int,
                 block_len: int, tokens_per_step: int, eps: float, gate_q: float = -1.0,
                 scripted: bool = False):
        self.model = model
        self.batch = batch
        self.n_ctx = prompt_len + gen_len
        self.prompt_len = prompt_len
        self.params = A.SamplerParams(prompt_len, gen_len, steps, block_len, tokens_per_step,
                                      eps, gate_q, 1 if scripted else 0)
        h = C.c_void_p()
        A.check(A.lib().sl_sampler_create(model.handle, batch, C.byref(self.params), C.byref(h)),
                "sl_sampler_create")
        self.handle = h

    def start(self, prompts: torch.Tensor, stream=None):
        A.check(A.lib().sl_sampler_start(self.handle, _ptr(prompts), _stream(stream)),
                "sl_sampler_start")

    def set_kv_reuse(self, period: int):
        """K/V reuse for the active rows with refresh interval `period` (1 = off);
        between decodes only."""
        A.check(A.lib().sl_sampler_set_kv_reuse(self.handle, int(period)),
                "sl_sampler_set_kv_reuse")

    def step(self, stream=None):
        A.check(A.lib().sl_sampler_step(self.handle, _stream(stream)), "sl_sampler_step")

    def generate(self, prompts_host: np.ndarray, out_host: Optional[np.ndarray] = None,
                 stream=None) -> np.ndarray:
        """Whole decode from host prompts [batch, prompt_len] to host tokens."""
        pr = np.ascontiguousarray(prompts_host, dtype=np.int32)
        if out_host is None:
            out_host = np.zeros((self.batch, self.n_ctx), dtype=np.int32)
        A.check(A.lib().sl_sampler_generate(self.handle, pr.ctypes.data, out_host.ctypes.data,
                                            _stream(stream)), "sl_sampler_generate")
        return out_host

    def generate_ptr(self, h_prompts_ptr: int, h_out_ptr: int, stream=None):
        A.check(A.lib().sl_sampler_generate(self.handle, h_prompts_ptr, h_out_ptr,
                                            _stream(stream)), "sl_sampler_generate")

    def autotune(self, stream=None):
        """Autotune the model's GEMM tilings for this sampler's batch and length."""
        st = A.SamplerState()
        A.check(A.lib().sl_sampler_get_state(self.handle, C.byref(st)), "sl_sampler_get_state")
        cache = KVCache.wrap(st.cache, self.model, st.batch, st.n_ctx)
        self.model.autotune(cache, st.batch * st.n_ctx, stream)

    def state(self) -> dict:
        st = A.SamplerState()
        A.check(A.lib().sl_sampler_get_state(self.handle, C.byref(st)), "sl_sampler_get_state")
        B, N, V = st.batch, st.n_ctx, self.model.shape.vocab
        dt = self.model.torch_dtype
        R = B * N
        return {
            "t": st.t,
            "tokens": device_view(st.tokens, (B, N), torch.int32),
            "masked": device_view(st.masked, (B, N), torch.uint8),
            "locked": device_view(st.locked, (B, N), torch.uint8),
            "lock_t": device_view(st.lock_t, (B, N), torch.int32),
            "logits": [device_view(st.logits[i], (R, V), dt) for i in range(2)],
            "lse": [device_view(st.lse[i], (R,), torch.float32) for i in range(2)],
            "kl": device_view(st.kl, (R,), torch.float32),
            "unc": device_view(st.unc, (R,), torch.float32),
            "conf": device_view(st.conf, (R,), torch.float32),
            "argmax": device_view(st.argmax, (R,), torch.int32),
            "lock": device_view(st.lock, (R,), torch.uint8),
            "cache": KVCache.wrap(st.cache, self.model, B, N),
            "active": Active.wrap(st.active, B, N),
            "computed": Active.wrap(st.computed, B, N) if st.computed else None,
        }

    def close(self):
        if getattr(self, "handle", None):
            A.lib().sl_sampler_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
