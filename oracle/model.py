"""Oracle denoiser: a bidirectional masked-diffusion transformer evaluated on the
active rows only.  Test infrastructure (see the package docstring).

What the pages fix:
  * Locked positions skip their query projection and FFN sublayers; their
    attention keys and values stay cached so active positions still attend to
    them (Abstract; Paper-Notes, "Key design: permanent locking").
  * Attention uses K^all[L_t] <- C.k[L_t]: the cached keys of locked rows stand
    in for fresh ones (Paper-Notes, "permanent locking", core idea).
  * A locked token's block input is frozen and its K/V are cached for every
    layer (gist.science/it, section 2 "Azione di Blocco").
  * Per-step cost O(M N d) for attention and O(M d^2) for the FFN
    (gist.science/nl section 2 "Complexiteitsvermindering"; gist.science/it
    section 2 "Complessita Computazionale").

Readings where the pages are silent (the plainest reading consistent with them):
  * RMSNorm with eps = rms_eps (1e-5) and per-channel gains; no biases anywhere;
    untied LM head; SwiGLU FFN  W_down( silu(W_gate b) * (W_up b) ).
  * Rotary embedding in rotate-half form on pairs (i, i + head_dim/2) with
    frequency theta^(-2i/head_dim), applied to q and k at the absolute position.
  * Scaled dot-product attention 1/sqrt(head_dim), bidirectional, softmax over
    all N keys of the sequence.
  * K/V projections are skipped for locked rows too: with a frozen block input
    they would reproduce the cached values exactly.
  * Weights are row-major [out, in]; y = x @ W.T.

Ablation (Paper-Notes, ablation table, row "no KV cache": locked tokens can no
longer be attended, so their information is lost):
  * `no_kv_cache=True` restricts every query's keys to the active rows of its
    sequence (their fresh k, v); the cached rows of locked positions are not
    read at all.  Positions, and so the rotary angles, stay absolute.
"""
from __future__ import annotations

import numpy as np


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """y = x / sqrt(mean(x^2) + eps) * g over the last axis.
    Reading (the pages are silent on the model): RMSNorm with per-channel gains."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def silu(x: np.ndarray) -> np.ndarray:
    """x * sigmoid(x), the gate of the SwiGLU FFN (reading: the pages are silent
    on the FFN; LLaDA-style SwiGLU)."""
    return x / (1.0 + np.exp(-x))


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding.  x: [M, H, dh], pos: [M] absolute positions.
    Reading (the pages are silent on positions): rotate-half RoPE at the
    absolute position, so active and cached keys keep their places.

    For i < dh/2, the pair (x_i, x_{i+dh/2}) is rotated by angle pos * theta^(-2i/dh):
      out_i        = x_i cos - x_{i+dh/2} sin
      out_{i+dh/2} = x_{i+dh/2} cos + x_i sin
    """
    dh = x.shape[-1]
    half = dh // 2
    dt = x.dtype
    inv = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / dh)
    ang = pos.astype(np.float64)[:, None] * inv[None, :]          # [M, half]
    cos = np.cos(ang).astype(dt)[:, None, :]
    sin = np.sin(ang).astype(dt)[:, None, :]
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def softmax(s: np.ndarray, axis: int = -1) -> np.ndarray:
    """exp(s - max) / sum exp(s - max) along `axis` (the attention weights)."""
    m = np.max(s, axis=axis, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def attention(q: np.ndarray, k_all: np.ndarray, v_all: np.ndarray) -> np.ndarray:
    """Bidirectional attention of M queries over all N keys of one sequence.

    q: [M, H, dh]; k_all, v_all: [N, H, dh] (cached rows for locked positions,
    fresh rows for active ones).  Returns [M, H, dh].
    Abstract: the keys and values of a locked position stay cached and the
    active positions keep attending to them; Paper-Notes, "permanent locking":
    K^all[L_t] <- C.k[L_t]."""
    dh = q.shape[-1]
    qh = np.transpose(q, (1, 0, 2))               # [H, M, dh]
    kh = np.transpose(k_all, (1, 2, 0))           # [H, dh, N]
    vh = np.transpose(v_all, (1, 0, 2))           # [H, N, dh]
    s = np.matmul(qh, kh) / np.sqrt(np.asarray(dh, dtype=q.dtype))
    p = softmax(s, axis=-1)
    o = np.matmul(p, vh)                          # [H, M, dh]
    return np.transpose(o, (1, 0, 2))


def layer_forward(shape, lw: dict, h: np.ndarray, pos: np.ndarray,
                  ck: np.ndarray, cv: np.ndarray, no_kv_cache: bool = False) -> np.ndarray:
    """One transformer block on the active rows of one sequence.

    h: [M, d] block input of the active rows at positions `pos` (ascending).
    ck, cv: [N, d] this layer's cache for the sequence; rows `pos` are
    overwritten with the fresh k, v (the scatter into C), all other rows are
    read as they are (frozen K/V of locked positions).  With no_kv_cache the
    queries attend to the rows `pos` only.  Returns the block output [M, d].
    Abstract: locked positions skip the query projection and feed-forward
    sublayers; gist.science/it section 2, "Azione di Blocco": their block input
    is frozen and their K/V are cached for every layer."""
    H, dh = shape.n_heads, shape.head_dim
    M = h.shape[0]
    a = rmsnorm(h, lw["attn_norm"], shape.rms_eps)
    q = (a @ lw["wq"].T).reshape(M, H, dh)
    k = (a @ lw["wk"].T).reshape(M, H, dh)
    v = (a @ lw["wv"].T).reshape(M, H, dh)
    q = rope(q, pos, shape.rope_theta)
    k = rope(k, pos, shape.rope_theta)
    ck[pos] = k.reshape(M, H * dh)
    cv[pos] = v.reshape(M, H * dh)
    keys = pos if no_kv_cache else np.arange(ck.shape[0])
    n = keys.shape[0]
    o = attention(q, ck[keys].reshape(n, H, dh), cv[keys].reshape(n, H, dh)).reshape(M, H * dh)
    h = h + o @ lw["wo"].T
    b = rmsnorm(h, lw["ffn_norm"], shape.rms_eps)
    h = h + (silu(b @ lw["w_gate"].T) * (b @ lw["w_up"].T)) @ lw["w_down"].T
    return h


def forward_active(shape, w: dict, tokens: np.ndarray, pos: np.ndarray,
                   ck: np.ndarray, cv: np.ndarray, block_inputs: list = None,
                   no_kv_cache: bool = False) -> np.ndarray:
    """Logits z [M, V] of the active rows `pos` of one sequence.

    tokens: [N] current ids x_t; ck, cv: [L, N, d] the sequence's cache,
    updated in place at rows `pos`.  If block_inputs is a list, the input h of
    every block is appended to it (used to check that K/V of locked rows are
    reproducible from their frozen block inputs).  no_kv_cache: the ablation
    in which the active rows attend to one another only.
    gist.science/nl section 2, "Complexiteitsvermindering": the step costs
    O(M N d) for attention and O(M d^2) for the projections and FFN."""
    h = w["tok_emb"][tokens[pos]]
    for l, lw in enumerate(w["layers"]):
        if block_inputs is not None:
            block_inputs.append(h.copy())
        h = layer_forward(shape, lw, h, pos, ck[l], cv[l], no_kv_cache)
    hf = rmsnorm(h, w["final_norm"], shape.rms_eps)
    return hf @ w["lm_head"].T


def kv_of_block_input(shape, lw: dict, h: np.ndarray, pos: np.ndarray):
    """k (after RoPE) and v [M, d] that a block would produce from input h
    (gist.science/it section 2, "Azione di Blocco": a locked row's cached K/V
    are those of its frozen block input)."""
    H, dh = shape.n_heads, shape.head_dim
    M = h.shape[0]
    a = rmsnorm(h, lw["attn_norm"], shape.rms_eps)
    k = rope((a @ lw["wk"].T).reshape(M, H, dh), pos, shape.rope_theta)
    v = a @ lw["wv"].T
    return k.reshape(M, H * dh), v


def forward_full(shape, w: dict, tokens: np.ndarray) -> np.ndarray:
    """Logits [N, V] of the unmodified denoiser on every position of one
    sequence: the comparison run of the Abstract, the sampler with locking
    switched off.  Written without any gather, cache or scatter, so it is an
    independent restatement of the same block."""
    H, dh = shape.n_heads, shape.head_dim
    N = tokens.shape[0]
    pos = np.arange(N)
    h = w["tok_emb"][tokens]
    for lw in w["layers"]:
        a = rmsnorm(h, lw["attn_norm"], shape.rms_eps)
        q = rope((a @ lw["wq"].T).reshape(N, H, dh), pos, shape.rope_theta)
        k = rope((a @ lw["wk"].T).reshape(N, H, dh), pos, shape.rope_theta)
        v = (a @ lw["wv"].T).reshape(N, H, dh)
        o = attention(q, k, v).reshape(N, H * dh)
        h = h + o @ lw["wo"].T
        b = rmsnorm(h, lw["ffn_norm"], shape.rms_eps)
        h = h + (silu(b @ lw["w_gate"].T) * (b @ lw["w_up"].T)) @ lw["w_down"].T
    hf = rmsnorm(h, w["final_norm"], shape.rms_eps)
    return hf @ w["lm_head"].T


def cast_weights(w: dict, dtype) -> dict:
    """Copy of a weight dict with every array cast to dtype."""
    out = {k: np.asarray(v, dtype=dtype) for k, v in w.items() if k != "layers"}
    out["layers"] = [{k: np.asarray(v, dtype=dtype) for k, v in lw.items()}
                     for lw in w["layers"]]
    return out
