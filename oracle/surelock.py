"""Oracle for SureLock's lock test, active-set bookkeeping and sampler.
Test infrastructure (see the package docstring).

Sources (the pages on "Stopping Computation for Converged Tokens in Masked
Diffusion-LM Decoding"):
  * Two disjoint sets per step: the active set A_t, which is computed, and the
    locked set L_t, which is skipped but whose K/V stay cached; the active set
    only shrinks (Paper-Notes, "Method: overall framework" and "permanent
    locking", design motivation; "Key findings": M_t decreases monotonically).
  * Lock criterion D_t^(i) = KL(p_t^(i) || p_{t-1}^(i)) <= eps (Paper-Notes,
    "lock criterion: step-to-step KL"; gist.science/it section 2 "Criterio di
    Blocco"), tested at unmasked positions (Abstract: "when the posterior at an
    unmasked position has stabilized across steps").
  * Optional confidence gate u_t^(i) = 1 - max_v p_t^(i)(v) <= q_m(u_t)
    (Paper-Notes, "optional confidence gate"), q_m a percentile of u among the
    active tokens (gist.science/it section 2, "Filtro di Confidenza").
  * After the lock step t*, the posterior stays frozen: p_hat_t = p_{t*}
    (Paper-Notes, "permanent locking", core idea).
  * The comparison run is the same sampler with locking switched off (Abstract).

Readings where the pages are silent (the plainest reading consistent with them):
  R4  "unmasked" means not [MASK] in the step's input x_t; prompt positions count.
  R5  no previous posterior at t = 0, so nothing locks at t = 0.
  R6  eps <= 0 disables locking (the pages' test D <= eps would fire at D = 0).
  R7  D is clamped at 0 (rounding can make it slightly negative).
  R8  q_m is the lower order statistic: sorted(u over A_t)[floor(q (|A_t|-1))],
      over all active rows of the sequence, masked or not; comparison <=.
  R9  ties: argmax takes the lowest vocab id, unmasking takes the lowest
      position, compaction keeps ascending position order.
  R11 semi-autoregressive blocks over the generated region; each step unmasks
      the k highest-confidence masked positions of the current block, where
      confidence and prediction are taken over v != [MASK].
  R22 composition with K/V reuse for the active rows (refresh interval R): all
      of A_t computed when t mod R = 0, else the active rows masked now or at
      the start of the previous step; the others keep their cached K/V and last
      posterior and are not tested (step()); the gate quantile of R8 is then
      taken over the computed rows.
  Scripted mode: instead of the KL test, lock the eligible (unmasked, with a
  previous posterior) active rows in ascending (D, position) order until the
  active count reaches a target.

Ablations (Paper-Notes, ablation table):
  * gate only ("confidence gate only"): the gate is the sole lock criterion,
    lock_j = not masked_j and has_prev_j and u_j <= thr.  Only the KL
    inequality is dropped; eligibility stays as in the full test, so nothing
    locks at t = 0 and a row is first tested the step after it is unmasked.
    eps plays no part; the gate must be on (gate_q >= 0).
  * no KV cache (the table's note: locked tokens drop out of attention): the denoiser's queries
    see the keys of the active rows only (model.forward_active, no_kv_cache).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np

from . import model as om


def log_softmax(z: np.ndarray) -> np.ndarray:
    """log p = z - logsumexp(z) over the last axis: the per-position posterior
    p_t that the lock criterion compares (Paper-Notes, "lock criterion")."""
    m = np.max(z, axis=-1, keepdims=True)
    return z - (m + np.log(np.sum(np.exp(z - m), axis=-1, keepdims=True)))


def kl_rows(lp_cur: np.ndarray, lp_prev: np.ndarray) -> np.ndarray:
    """D = max(0, sum_v p_cur(v) (log p_cur(v) - log p_prev(v))) per row: the
    step-to-step KL of the lock criterion (Paper-Notes, "lock criterion";
    gist.science/it section 2, "Criterio di Blocco"), clamped at 0 (reading R7).
    A term with p_cur(v) = 0 (a -inf logit) is 0, the usual 0 log 0 = 0 of the
    KL's definition; p_cur(v) > 0 with p_prev(v) = 0 makes D infinite."""
    p = np.exp(lp_cur)
    with np.errstate(invalid="ignore"):
        terms = np.where(p > 0, p * (lp_cur - lp_prev), 0.0)
    return np.maximum(0.0, np.sum(terms, axis=-1))


def uncertainty(lp_cur: np.ndarray) -> np.ndarray:
    """u = 1 - max_v p(v) per row (all vocab entries, [MASK] included): the
    gate's uncertainty (Paper-Notes, "optional confidence gate")."""
    return 1.0 - np.exp(np.max(lp_cur, axis=-1))


def prediction(lp_cur: np.ndarray, mask_id: int):
    """(conf, pred): the largest probability over v != mask_id and its lowest
    index; this is what the sampler unmasks with (readings R9, R11: the pages
    name the sampler but not its details)."""
    lp = np.array(lp_cur, copy=True)
    lp[..., mask_id] = -np.inf
    pred = np.argmax(lp, axis=-1)           # first occurrence = lowest id
    conf = np.exp(np.take_along_axis(lp, pred[..., None], axis=-1)[..., 0])
    return conf, pred.astype(np.int32)


def gate_threshold(u_active: np.ndarray, q: float) -> float:
    """q-quantile of u over the active rows, lower order statistic: q_m(u_t) of
    the gate (Paper-Notes, "optional confidence gate"; gist.science/it section
    2, "Filtro di Confidenza"; reading R8 for the order statistic)."""
    m = u_active.shape[0]
    if m == 0:
        return np.inf
    r = int(np.floor(q * (m - 1)))
    return np.sort(u_active, kind="stable")[r]


def lock_decision(D, u, masked, has_prev, eps: float, gate_q: float, thr,
                  gate_only: bool = False):
    """lock_j = eps>0 and not masked_j and has_prev_j and D_j<=eps and
    (gate off or u_j <= thr).  gate_only: lock_j = not masked_j and has_prev_j
    and u_j <= thr, whatever eps and D.
    Paper-Notes, "lock criterion" and "optional confidence gate"; Abstract:
    only unmasked positions are tested; readings R4-R6; gate only: the
    Paper-Notes ablation table."""
    if gate_only:
        if gate_q < 0:
            raise ValueError("the gate-only criterion needs the confidence gate (gate_q >= 0)")
        return (~masked.astype(bool)) & has_prev.astype(bool) & (u <= thr)
    if eps <= 0:
        return np.zeros(D.shape, dtype=bool)
    ok = (~masked.astype(bool)) & has_prev.astype(bool) & (D <= eps)
    if gate_q >= 0:
        ok &= (u <= thr)
    return ok


def scripted_locks(D, masked, has_prev, pos, n_lock: int):
    """Lock the n_lock eligible rows with the smallest (D, position): the
    scripted schedule of the benchmark (a fixed M_t decay, not from the pages)."""
    elig = (~masked.astype(bool)) & has_prev.astype(bool)
    idx = np.nonzero(elig)[0]
    order = idx[np.lexsort((pos[idx], D[idx]))]
    lock = np.zeros(D.shape, dtype=bool)
    lock[order[:max(0, n_lock)]] = True
    return lock


def compact(act: np.ndarray, lock: np.ndarray) -> np.ndarray:
    """Stable removal of the locked rows from the active list: the active set
    only shrinks (Paper-Notes, "permanent locking"; reading R9 for the order)."""
    return act[~lock]


def unmask_select(pos: np.ndarray, conf: np.ndarray, masked_rows: np.ndarray,
                  lo: int, hi: int, k: int) -> np.ndarray:
    """Indices (into the active rows) of the k masked rows in [lo, hi) with the
    highest confidence, ties to the lower position (reading R11: the
    semi-autoregressive sampler the pages compare against)."""
    cand = np.nonzero(masked_rows.astype(bool) & (pos >= lo) & (pos < hi))[0]
    order = cand[np.lexsort((pos[cand], -conf[cand]))]
    return order[:k]


@dataclasses.dataclass
class State:
    """Sampler state for a batch of sequences."""
    tokens: np.ndarray        # [B, N] int32
    masked: np.ndarray        # [B, N] bool
    act: List[np.ndarray]     # per sequence: ascending active positions
    locked: np.ndarray        # [B, N] bool
    lock_t: np.ndarray        # [B, N] int32, -1 if never locked
    has_prev: np.ndarray      # [B, N] bool
    ck: np.ndarray            # [B, L, N, d]
    cv: np.ndarray            # [B, L, N, d]
    lp_prev: np.ndarray       # [B, N, V]  last posterior (frozen p_hat for locked rows)
    # mask flags at the start of the previous step (K/V reuse: a row unmasked
    # during that step is computed once more before it can be reused)
    masked_before: Optional[np.ndarray] = None

    def copy(self) -> "State":
        return State(self.tokens.copy(), self.masked.copy(), [a.copy() for a in self.act],
                     self.locked.copy(), self.lock_t.copy(), self.has_prev.copy(),
                     self.ck.copy(), self.cv.copy(), self.lp_prev.copy(),
                     None if self.masked_before is None else self.masked_before.copy())


def init_state(shape, tokens: np.ndarray, masked: np.ndarray, dtype=np.float64) -> State:
    """A_0 = every position, nothing locked, no previous posterior (reading R5),
    an all-zero cache."""
    B, N = tokens.shape
    L, d, V = shape.n_layers, shape.d_model, shape.vocab
    return State(tokens=tokens.astype(np.int32).copy(), masked=masked.astype(bool).copy(),
                 act=[np.arange(N, dtype=np.int32) for _ in range(B)],
                 locked=np.zeros((B, N), dtype=bool),
                 lock_t=np.full((B, N), -1, dtype=np.int32),
                 has_prev=np.zeros((B, N), dtype=bool),
                 ck=np.zeros((B, L, N, d), dtype=dtype), cv=np.zeros((B, L, N, d), dtype=dtype),
                 lp_prev=np.zeros((B, N, V), dtype=dtype),
                 masked_before=masked.astype(bool).copy())


def lock_test(lp: np.ndarray, lp_prev: np.ndarray, has_prev: np.ndarray,
              masked: np.ndarray, pos: np.ndarray, shape, setup, t: int,
              n_active_target: Optional[int] = None):
    """The sure test of one sequence's active rows.  Returns a dict with D, u,
    conf, pred, thr and the lock flags (the pieces above, in the order of
    Paper-Notes, "lock criterion" and "optional confidence gate")."""
    D = np.full(lp.shape[0], np.inf, dtype=lp.dtype)
    hp = has_prev.astype(bool)
    if np.any(hp):
        D[hp] = kl_rows(lp[hp], lp_prev[hp])
    u = uncertainty(lp)
    conf, pred = prediction(lp, shape.mask_id)
    thr = gate_threshold(u, setup.gate_q) if setup.gate_q >= 0 else np.inf
    if setup.scripted:
        target = setup.scripted_target(t) if n_active_target is None else n_active_target
        lock = scripted_locks(D, masked, hp, pos, lp.shape[0] - target)
    else:
        lock = lock_decision(D, u, masked, hp, setup.eps, setup.gate_q, thr,
                             setup.gate_only)
    return {"D": D, "u": u, "conf": conf, "pred": pred, "thr": thr, "lock": lock}


def step(shape, w: dict, st: State, setup, t: int, record_block_inputs: bool = False):
    """One SureLock denoising step t on every sequence, updating `st` in place.

    Order: forward on A_t (fresh K/V scattered into C) -> log-softmax -> sure
    test on the mask flags at the start of the step -> unmask the top-k of the
    current block -> record p_t for the active rows (frozen for those that lock)
    -> remove the locked rows from A_t.  Returns one record per sequence.
    Paper-Notes, "Method: overall framework" (compute A_t, serve L_t from the
    cache) and "permanent locking" (a locked row's posterior is frozen).

    With setup.kv_reuse = R > 1 (the pages' composition with cross-step reuse:
    Paper-Notes, "permanent locking", design motivation, sets SureLock's
    permanent removal against dLLM-Cache's per-step choice of what to compute;
    "loss / training strategy" and gist.science/it section 4, "Ortogonalita",
    call the two orthogonal and stackable; the scheme itself is this
    restatement's reading) the forward
    runs on all of A_t only when t mod R = 0.  Between those refresh steps it
    runs on the active rows that are masked or were masked at the start of the
    previous step; the other active rows keep their cached K/V and their last
    posterior, are not tested, and stay active."""
    out = []
    lo, hi = setup.block_bounds(t)
    R = getattr(setup, "kv_reuse", 1)
    if R > 1 and (setup.scripted or setup.no_kv_cache):
        # the scripted lock count is defined over the whole active set, and the
        # no-cache ablation has no stale K/V to reuse
        raise ValueError("K/V reuse composes with the sure test on the full cache only")
    refresh = R <= 1 or t % R == 0
    if st.masked_before is None:
        st.masked_before = st.masked.copy()
    masked_start = st.masked.copy()
    for b in range(st.tokens.shape[0]):
        A = st.act[b]
        # the rows computed this step: all of A_t, or, between refresh steps of
        # the K/V reuse, its masked rows and the rows unmasked during the
        # previous step (reading: composition with K/V reuse for active rows)
        C = A if refresh else A[st.masked[b, A] | st.masked_before[b, A]]
        blk = [] if record_block_inputs else None
        z = om.forward_active(shape, w, st.tokens[b], C, st.ck[b], st.cv[b], blk,
                              setup.no_kv_cache)
        lp = log_softmax(z)
        masked_rows = st.masked[b, C].copy()
        rec = lock_test(lp, st.lp_prev[b, C], st.has_prev[b, C], masked_rows, C,
                        shape, setup, t)
        sel = unmask_select(C, rec["conf"], masked_rows, lo, hi, setup.tokens_per_step)
        st.tokens[b, C[sel]] = rec["pred"][sel]
        st.masked[b, C[sel]] = False
        st.lp_prev[b, C] = lp
        st.has_prev[b, C] = True
        lk = rec["lock"]
        st.locked[b, C[lk]] = True
        st.lock_t[b, C[lk]] = t
        st.act[b] = compact(A, np.isin(A, C[lk]))
        rec.update({"z": z, "lp": lp, "pos": C, "active": A, "unmasked": C[sel],
                    "block_inputs": blk})
        out.append(rec)
    st.masked_before = masked_start
    return out


def surelock_sampler(shape, w: dict, tokens: np.ndarray, masked: np.ndarray, setup,
                     dtype=np.float64, keep_records: bool = False):
    """Full SureLock decode.  Returns (final tokens, final log-probs [B, N, V],
    active counts per step [T+1, B], per-step records if keep_records).
    Paper-Notes, "Method: overall framework"; "key findings": M_t only falls."""
    st = init_state(shape, tokens, masked, dtype)
    counts = [[len(a) for a in st.act]]
    recs = []
    for t in range(setup.steps):
        r = step(shape, w, st, setup, t)
        counts.append([len(a) for a in st.act])
        if keep_records:
            recs.append(r)
    return st.tokens, st.lp_prev, np.array(counts), (recs if keep_records else None), st


def plain_sampler(shape, w: dict, tokens: np.ndarray, masked: np.ndarray, setup):
    """The sampler with locking switched off: every step runs the full denoiser on all
    N positions (no active set, no cache).  Returns (final tokens, final
    log-probs [B, N, V])."""
    tok = tokens.astype(np.int32).copy()
    msk = masked.astype(bool).copy()
    B, N = tok.shape
    lp = None
    pos = np.arange(N, dtype=np.int32)
    lps = [None] * B
    for t in range(setup.steps):
        lo, hi = setup.block_bounds(t)
        for b in range(B):
            lp = log_softmax(om.forward_full(shape, w, tok[b]))
            conf, pred = prediction(lp, shape.mask_id)
            sel = unmask_select(pos, conf, msk[b], lo, hi, setup.tokens_per_step)
            tok[b, sel] = pred[sel]
            msk[b, sel] = False
            lps[b] = lp
    return tok, np.stack(lps)


def flops_per_step(shape, m_rows: int, n_ctx_rows: int) -> float:
    """Algorithmic FLOPs of one step on m_rows active rows attending to
    n_ctx_rows keys: 2 M (L (4 d^2 + 3 d f) + V d) + 4 L M N d (gist.science/nl
    section 2, "Complexiteitsvermindering": O(M d^2) for the projections and FFN,
    O(M N d) for attention)."""
    d, f, V, L = shape.d_model, shape.d_ffn, shape.vocab, shape.n_layers
    return 2.0 * m_rows * (L * (4 * d * d + 3 * d * f) + V * d) + 4.0 * L * m_rows * n_ctx_rows * d
