"""Scalar-loop restatements for tiny shapes -- TEST INFRASTRUCTURE ONLY.

Each function re-derives one piece of the oracle from its textbook definition
with explicit Python loops over math.* scalars (no NumPy reductions, no matrix
products), so a slip in the vectorised oracle (a dropped term, a transposed
operand, a wrong sign or index) shows up as a mismatch.  Only for shapes small
enough that the loops finish in well under a second.
"""
from __future__ import annotations

import math


def rmsnorm(x, g, eps):
    """x: list of rows (lists of floats)."""
    out = []
    for row in x:
        ms = sum(v * v for v in row) / len(row)
        r = 1.0 / math.sqrt(ms + eps)
        out.append([row[i] * r * g[i] for i in range(len(row))])
    return out


def matvec_rows(x, w):
    """y[m][o] = sum_i x[m][i] * w[o][i]  (w row-major [out, in])."""
    return [[sum(row[i] * wo[i] for i in range(len(row))) for wo in w] for row in x]


def rope_vec(vec, p, theta):
    """Rotate-half RoPE on one head vector at position p."""
    dh = len(vec)
    half = dh // 2
    out = [0.0] * dh
    for i in range(half):
        a = p * theta ** (-2.0 * i / dh)
        c, s = math.cos(a), math.sin(a)
        out[i] = vec[i] * c - vec[i + half] * s
        out[i + half] = vec[i + half] * c + vec[i] * s
    return out


def attention_head(q, keys, vals):
    """softmax(q . k_n / sqrt(dh)) weighted sum of vals, one query, one head."""
    dh = len(q)
    sc = [sum(q[i] * k[i] for i in range(dh)) / math.sqrt(dh) for k in keys]
    mx = max(sc)
    e = [math.exp(s - mx) for s in sc]
    tot = sum(e)
    return [sum(e[n] * vals[n][i] for n in range(len(vals))) / tot for i in range(dh)]


def silu(x):
    """x * sigmoid(x) on one scalar."""
    return x / (1.0 + math.exp(-x))


def forward_active(shape, w, tokens, pos, ck, cv, no_kv_cache=False):
    """Loop restatement of the denoiser on active rows `pos` of one sequence.
    ck, cv: lists [L][N][d] updated in place at rows `pos`.  With no_kv_cache a
    query sees the keys of the rows `pos` only.  Returns logits."""
    H, dh, d = shape.n_heads, shape.head_dim, shape.d_model
    N = len(ck[0])
    seen = list(pos) if no_kv_cache else list(range(N))
    h = [list(map(float, w["tok_emb"][tokens[p]])) for p in pos]
    for l, lw in enumerate(w["layers"]):
        a = rmsnorm(h, lw["attn_norm"], shape.rms_eps)
        q = matvec_rows(a, lw["wq"])
        k = matvec_rows(a, lw["wk"])
        v = matvec_rows(a, lw["wv"])
        for m, p in enumerate(pos):
            for hh in range(H):
                sl = slice(hh * dh, (hh + 1) * dh)
                q[m][sl] = rope_vec(q[m][sl], p, shape.rope_theta)
                k[m][sl] = rope_vec(k[m][sl], p, shape.rope_theta)
            ck[l][p] = list(k[m])
            cv[l][p] = list(v[m])
        o = []
        for m in range(len(pos)):
            row = []
            for hh in range(H):
                sl = slice(hh * dh, (hh + 1) * dh)
                row += attention_head(q[m][sl], [ck[l][n][sl] for n in seen],
                                      [cv[l][n][sl] for n in seen])
            o.append(row)
        ow = matvec_rows(o, lw["wo"])
        h = [[h[m][i] + ow[m][i] for i in range(d)] for m in range(len(pos))]
        b = rmsnorm(h, lw["ffn_norm"], shape.rms_eps)
        g = matvec_rows(b, lw["w_gate"])
        u = matvec_rows(b, lw["w_up"])
        act = [[silu(g[m][j]) * u[m][j] for j in range(len(g[m]))] for m in range(len(pos))]
        dn = matvec_rows(act, lw["w_down"])
        h = [[h[m][i] + dn[m][i] for i in range(d)] for m in range(len(pos))]
    hf = rmsnorm(h, w["final_norm"], shape.rms_eps)
    return matvec_rows(hf, w["lm_head"])


def log_softmax_row(z):
    """z - log(sum exp z) for one row, shifted by its max."""
    mx = max(z)
    lse = mx + math.log(sum(math.exp(v - mx) for v in z))
    return [v - lse for v in z]


def kl(p_log, q_log):
    """sum_v p(v) (log p(v) - log q(v)) for one row of log-probabilities."""
    return sum(math.exp(a) * (a - b) for a, b in zip(p_log, q_log))


def lower_quantile(values, q):
    """Smallest value v such that at least floor(q (n-1)) + 1 values are <= v
    (the lower order statistic, defined by counting instead of sorting)."""
    n = len(values)
    need = int(math.floor(q * (n - 1))) + 1
    best = None
    for v in values:
        if sum(1 for x in values if x <= v) >= need and (best is None or v < best):
            best = v
    return best


def topk_positions(cands, k):
    """cands: list of (pos, conf).  The k positions with the highest conf, ties
    to the lower position, found by pairwise dominance counting."""
    chosen = []
    for p, c in cands:
        better = sum(1 for p2, c2 in cands if (c2 > c) or (c2 == c and p2 < p))
        if better < k:
            chosen.append(p)
    return sorted(chosen)
