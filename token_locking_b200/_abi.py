"""ctypes declarations of libsurelock.so (include/surelock.h).

Argument marshalling only: every step of the decoding path runs in the CUDA
library.  Loading fails loudly when the library is missing; there is no CPU
fallback.
"""
from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsurelock.so")

SL_OK, SL_ERR_INVALID, SL_ERR_CUDA, SL_ERR_OOM, SL_ERR_UNSUPPORTED, SL_ERR_TIMEOUT, SL_ERR_STATE = range(7)
SL_F32, SL_BF16 = 0, 1
SL_MAX_BATCH = 64
K_GEMM, K_ATTN, K_LOCK, K_OTHER, K_COUNT = range(5)
GEMM_STORE, GEMM_RESID, GEMM_SWIGLU, GEMM_ACCUM = range(4)
ABLATE_NO_KV_CACHE, ABLATE_GATE_ONLY = 1, 2
STATUS_NAMES = ["SL_OK", "SL_ERR_INVALID", "SL_ERR_CUDA", "SL_ERR_OOM", "SL_ERR_UNSUPPORTED",
                "SL_ERR_TIMEOUT", "SL_ERR_STATE"]


class Config(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("d_model", C.c_int), ("n_heads", C.c_int),
                ("head_dim", C.c_int), ("d_ffn", C.c_int), ("vocab", C.c_int),
                ("mask_id", C.c_int), ("rms_eps", C.c_float), ("rope_theta", C.c_float),
                ("dtype", C.c_int)]


class LayerWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm",
                                          "w_gate", "w_up", "w_down")]


class Weights(C.Structure):
    _fields_ = [("tok_emb", C.c_void_p), ("final_norm", C.c_void_p), ("lm_head", C.c_void_p),
                ("layers", C.POINTER(LayerWeights))]


class LockParams(C.Structure):
    _fields_ = [("eps", C.c_float), ("gate_q", C.c_float), ("has_prev", C.c_int),
                ("scripted_target", C.c_int), ("gate_only", C.c_int)]


class SamplerParams(C.Structure):
    _fields_ = [("prompt_len", C.c_int), ("gen_len", C.c_int), ("steps", C.c_int),
                ("block_len", C.c_int), ("tokens_per_step", C.c_int), ("eps", C.c_float),
                ("gate_q", C.c_float), ("scripted", C.c_int)]


class SamplerState(C.Structure):
    _fields_ = [("tokens", C.c_void_p), ("masked", C.c_void_p), ("locked", C.c_void_p),
                ("lock_t", C.c_void_p), ("logits", C.c_void_p * 2), ("lse", C.c_void_p * 2),
                ("kl", C.c_void_p), ("unc", C.c_void_p), ("conf", C.c_void_p),
                ("argmax", C.c_void_p), ("lock", C.c_void_p), ("cache", C.c_void_p),
                ("active", C.c_void_p), ("t", C.c_int), ("batch", C.c_int), ("n_ctx", C.c_int),
                ("computed", C.c_void_p)]


class Timing(C.Structure):
    _fields_ = [("ms", C.c_double * K_COUNT), ("bytes", C.c_double * K_COUNT),
                ("flops", C.c_double * K_COUNT), ("launches", C.c_longlong * K_COUNT),
                ("kernels", C.c_longlong)]


_P = C.c_void_p
_I = C.c_int
# name -> (restype, argtypes); the full exported surface of include/surelock.h
SIGNATURES = {
    "sl_last_error": (C.c_char_p, []),
    "sl_version": (C.c_char_p, []),
    "sl_model_create": (_I, [C.POINTER(Config), C.POINTER(Weights), C.POINTER(_P)]),
    "sl_model_destroy": (None, [_P]),
    "sl_kv_cache_create": (_I, [_P, _I, _I, C.POINTER(_P)]),
    "sl_kv_cache_reset": (_I, [_P, _P]),
    "sl_kv_cache_view": (_I, [_P, _I, C.POINTER(_P), C.POINTER(_P)]),
    "sl_kv_cache_destroy": (None, [_P]),
    "sl_active_create": (_I, [_I, _I, C.POINTER(_P)]),
    "sl_active_reset": (_I, [_P, _P]),
    "sl_active_load": (_I, [_P, C.POINTER(C.c_int32), C.POINTER(C.c_int32), _P]),
    "sl_active_counts": (_I, [_P, C.POINTER(C.c_int32)]),
    "sl_active_view": (_I, [_P, C.POINTER(_P), C.POINTER(_P)]),
    "sl_active_destroy": (None, [_P]),
    "sl_step": (_I, [_P, _P, _P, _P, _P, _P]),
    "sl_kl_lock": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, C.POINTER(LockParams),
                        _P, _P, _P, _P, _P, _P]),
    "sl_step_stats": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P]),
    "sl_lock_decide": (_I, [_P, _P, C.POINTER(LockParams), _P, _P, _P, _P]),
    "sl_model_set_head_fusion": (_I, [_P, _I]),
    "sl_kl_stats_noalloc": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P]),
    "sl_unmask_topk": (_I, [_P, _P, _P, _I, _I, _I, _P, _P, _P]),
    "sl_compact_active": (_I, [_P, _P, _P, _P, _I, _P]),
    "sl_model_set_ablation": (_I, [_P, _I]),
    "sl_sampler_create": (_I, [_P, _I, C.POINTER(SamplerParams), C.POINTER(_P)]),
    "sl_sampler_start": (_I, [_P, _P, _P]),
    "sl_sampler_set_kv_reuse": (_I, [_P, _I]),
    "sl_sampler_step": (_I, [_P, _P]),
    "sl_sampler_generate": (_I, [_P, _P, _P, _P]),
    "sl_sampler_get_state": (_I, [_P, C.POINTER(SamplerState)]),
    "sl_sampler_destroy": (None, [_P]),
    "sl_layer_forward": (_I, [_P, _P, _P, _I, _P, _P]),
    "sl_attention": (_I, [_P, _P, _P, _I, _P, _P, _P]),
    "sl_gemm_bf16": (_I, [_I, _P, _I, _I, _P, _P, _I, _P, _I, _P, _I, _I, _I, _P]),
    "sl_model_autotune": (_I, [_P, _P, _I, _P]),
    "sl_model_tuning": (_I, [_P, _I, _I, C.POINTER(_I), C.POINTER(_I), C.POINTER(_I)]),
    "sl_model_set_tuning": (_I, [_P, _I, _I, _I, _I, _I]),
    "sl_model_set_attention": (_I, [_P, _I, _I]),
    "sl_model_set_attention_keys": (_I, [_P, _I]),
    "sl_timing_enable": (_I, [_P, _I]),
    "sl_timing_read": (_I, [_P, C.POINTER(Timing), _I]),
    "sl_device_check": (_I, [_I]),
    "sl_debug_set_wait_limit": (_I, [C.c_ulonglong]),
    "sl_debug_inject_lost_load": (_I, []),
}

_lib = None


def lib():
    """The loaded library with argtypes set.  Raises if it was never built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m token_locking_b200.build` "
                "(the SureLock path has no CPU fallback)")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


class SureLockError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib().sl_last_error().decode(errors="replace")
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else str(status)
        super().__init__(f"{where}: {name}: {msg}")
        self.status = status


def check(status: int, where: str) -> None:
    if status != SL_OK:
        raise SureLockError(status, where)
