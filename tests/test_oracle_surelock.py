"""Pins for the oracle's lock test, bookkeeping and sampler (CPU only)."""
import json
import math
import os

import numpy as np
import pytest

import workloads as wl
from oracle import brute
from oracle import model as om
from oracle import surelock as sl

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")))


# ---------------------------------------------------------------- lock test --

def test_log_softmax_normalised_and_shift_invariant():
    rng = np.random.default_rng(0)
    z = rng.standard_normal((4, 50)) * 3
    lp = sl.log_softmax(z)
    np.testing.assert_allclose(np.exp(lp).sum(-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(sl.log_softmax(z + 123.0), lp, atol=1e-12)
    for r in range(4):
        np.testing.assert_allclose(lp[r], brute.log_softmax_row(z[r].tolist()), atol=1e-13)


def test_kl_bernoulli_closed_form():
    c = GOLD["bernoulli_kl"]
    d = sl.kl_rows(np.log(np.array([c["p"]])), np.log(np.array([c["q"]])))
    assert d[0] == pytest.approx(c["kl"], rel=1e-14)
    # the opposite direction differs: the test is KL(p_t || p_{t-1}), not symmetric
    d_rev = sl.kl_rows(np.log(np.array([c["q"]])), np.log(np.array([c["p"]])))
    assert abs(d_rev[0] - c["kl"]) > 1e-3


def test_kl_with_zero_probability_entries():
    """Entries with a -inf logit have probability 0 and add no term to the KL
    (0 log 0 = 0 in its definition), so a two-outcome pair padded with -inf
    logits keeps the Bernoulli closed form; an outcome the previous posterior
    gave probability 0 while the current one does not makes D infinite."""
    c = GOLD["bernoulli_kl"]
    ninf = -np.inf
    lp = np.array([[np.log(c["p"][0]), ninf, np.log(c["p"][1]), ninf]])
    lq = np.array([[np.log(c["q"][0]), ninf, np.log(c["q"][1]), ninf]])
    d = sl.kl_rows(lp, lq)
    assert d[0] == pytest.approx(c["kl"], rel=1e-14)
    # current posterior puts 0 where the previous one did not: still finite
    lq2 = np.array([[np.log(0.3), np.log(0.1), np.log(0.6), ninf]])
    want = c["p"][0] * math.log(c["p"][0] / 0.3) + c["p"][1] * math.log(c["p"][1] / 0.6)
    assert sl.kl_rows(lp, lq2)[0] == pytest.approx(want, rel=1e-13)
    # current puts mass where the previous had none: infinite divergence
    assert sl.kl_rows(lq2, lp)[0] == np.inf
    # log_softmax of logits with -inf entries: those stay -inf, the rest normalise
    z = np.array([[1.0, ninf, 2.0, ninf]])
    lpz = sl.log_softmax(z)
    assert np.isneginf(lpz[0, 1]) and np.isneginf(lpz[0, 3])
    assert np.exp(lpz[0, [0, 2]]).sum() == pytest.approx(1.0, rel=1e-15)


def test_kl_zero_nonneg_shift_and_brute():
    rng = np.random.default_rng(1)
    z = rng.standard_normal((6, 40)) * 2
    lp = sl.log_softmax(z)
    assert np.all(sl.kl_rows(lp, lp) == 0.0)                   # identical posteriors
    lq = sl.log_softmax(z + rng.standard_normal(z.shape))
    d = sl.kl_rows(lp, lq)
    assert np.all(d > 0)                                        # Gibbs' inequality
    np.testing.assert_allclose(sl.kl_rows(lp, sl.log_softmax(z + 5.0)), 0.0, atol=1e-13)
    for r in range(6):
        assert d[r] == pytest.approx(brute.kl(lp[r].tolist(), lq[r].tolist()), rel=1e-12)


def test_kl_small_perturbation_limit():
    """KL(p || softmax(z + s eta)) -> s^2/2 Var_p(eta) as s -> 0."""
    rng = np.random.default_rng(2)
    z = rng.standard_normal((3, 64))
    eta = rng.standard_normal((3, 64))
    s = 1e-4
    lp = sl.log_softmax(z)
    p = np.exp(lp)
    var = (p * eta ** 2).sum(-1) - ((p * eta).sum(-1)) ** 2
    np.testing.assert_allclose(sl.kl_rows(lp, sl.log_softmax(z + s * eta)), 0.5 * s * s * var,
                               rtol=1e-3)


def test_uncertainty_and_prediction():
    V, mask = 10, 9
    z = np.zeros((3, V))
    z[0, 4] = 50.0                       # peaked: u -> 0
    z[2, mask] = 5.0; z[2, 1] = 2.0; z[2, 3] = 2.0   # [MASK] largest, tie between 1 and 3
    lp = sl.log_softmax(z)
    u = sl.uncertainty(lp)
    assert u[0] < 1e-15
    assert u[1] == pytest.approx(1 - 1 / V, rel=1e-15)         # uniform row
    conf, pred = sl.prediction(lp, mask)
    assert pred[0] == 4 and pred[1] == 0 and pred[2] == 1       # lowest id among ties, mask skipped
    assert conf[2] == pytest.approx(math.exp(2) / (math.exp(5) + 2 * math.exp(2) + 7), rel=1e-14)
    # u counts [MASK]; conf does not
    assert u[2] == pytest.approx(1 - math.exp(5) / (math.exp(5) + 2 * math.exp(2) + 7), rel=1e-14)


@pytest.mark.parametrize("m", [1, 2, 5, 8, 33])
@pytest.mark.parametrize("q", [0.0, 0.25, 0.5, 0.9, 1.0])
def test_gate_threshold_lower_order_statistic(m, q):
    rng = np.random.default_rng(m)
    u = rng.random(m)
    u[:m // 3] = u[0]                                        # ties
    thr = sl.gate_threshold(u, q)
    assert thr == np.quantile(u, q, method="lower")
    assert thr == brute.lower_quantile(u.tolist(), q)


def test_lock_decision_truth_table():
    D = np.array([0.001, 0.001, 0.001, 0.02, 0.001, 0.001])
    u = np.array([0.1, 0.1, 0.1, 0.1, 0.9, 0.1])
    masked = np.array([0, 1, 0, 0, 0, 0], dtype=bool)
    hp = np.array([1, 1, 0, 1, 1, 1], dtype=bool)
    assert sl.lock_decision(D, u, masked, hp, 0.01, -1, np.inf).tolist() == \
        [True, False, False, False, True, True]
    assert sl.lock_decision(D, u, masked, hp, 0.01, 0.5, 0.5).tolist() == \
        [True, False, False, False, False, True]
    assert not sl.lock_decision(D * 0, u, masked, hp, 0.0, -1, np.inf).any()   # eps = 0: never
    # D exactly at eps locks (<=), u exactly at thr passes (<=)
    assert sl.lock_decision(np.array([0.01]), np.array([0.3]), np.array([False]), np.array([True]),
                            0.01, 0.5, 0.3).tolist() == [True]


def test_gate_only_truth_table():
    """Gate-only ablation: the gate alone decides among unmasked rows with a
    previous posterior; D and eps play no part."""
    D = np.array([0.001, 5.0, 0.001, 0.02, 0.001, 7.0])
    u = np.array([0.1, 0.1, 0.1, 0.1, 0.9, 0.5])
    masked = np.array([0, 0, 1, 0, 0, 0], dtype=bool)
    hp = np.array([1, 1, 1, 0, 1, 1], dtype=bool)
    for eps in (0.0, 0.01, -1.0):
        assert sl.lock_decision(D, u, masked, hp, eps, 0.5, 0.5, gate_only=True).tolist() == \
            [True, True, False, False, False, True]
    with pytest.raises(ValueError):
        sl.lock_decision(D, u, masked, hp, 0.01, -1, np.inf, gate_only=True)


def test_gate_only_is_the_full_test_with_an_unbounded_eps():
    """gate_only == the KL test with eps = +inf (D <= inf always holds), the
    identity by which the library runs the ablation."""
    rng = np.random.default_rng(21)
    for trial in range(30):
        n = int(rng.integers(1, 40))
        D = rng.exponential(0.05, n) * (rng.random(n) < 0.9) + (rng.random(n) < 0.1) * 1e30
        u = np.round(rng.random(n), 2)
        masked = rng.random(n) < 0.3
        hp = rng.random(n) < 0.8
        q = float(rng.random())
        thr = sl.gate_threshold(u, q)
        np.testing.assert_array_equal(
            sl.lock_decision(D, u, masked, hp, 0.0, q, thr, gate_only=True),
            sl.lock_decision(D, u, masked, hp, np.inf, q, thr))


def test_scripted_locks_brute():
    rng = np.random.default_rng(3)
    n = 12
    D = np.round(rng.random(n), 1)                          # many ties in D
    masked = rng.random(n) < 0.3
    hp = rng.random(n) < 0.8
    pos = np.sort(rng.choice(100, n, replace=False))
    for k in range(0, n + 2):
        lock = sl.scripted_locks(D, masked, hp, pos, k)
        elig = [(D[i], pos[i], i) for i in range(n) if (not masked[i]) and hp[i]]
        want = {i for _, _, i in sorted(elig)[:k]}
        assert set(np.nonzero(lock)[0].tolist()) == want


def test_compact_stable():
    act = np.array([1, 4, 5, 9, 12, 20])
    lock = np.array([0, 1, 0, 0, 1, 0], dtype=bool)
    assert sl.compact(act, lock).tolist() == [a for a, l in zip(act, lock) if not l]


def test_unmask_select_brute():
    rng = np.random.default_rng(4)
    for trial in range(20):
        n = int(rng.integers(1, 15))
        pos = np.sort(rng.choice(40, n, replace=False))
        conf = np.round(rng.random(n), 1)
        masked = rng.random(n) < 0.7
        lo, hi, k = 5, 30, int(rng.integers(1, 5))
        sel = sl.unmask_select(pos, conf, masked, lo, hi, k)
        cands = [(int(pos[i]), conf[i]) for i in range(n) if masked[i] and lo <= pos[i] < hi]
        assert sorted(pos[sel].tolist()) == brute.topk_positions(cands, k)


# ------------------------------------------------------------------ sampler --

def _tiny(seed_w=0, gain_jitter=0.0):
    cfg = wl.CFG_TINY
    cfg.validate()
    w = om.cast_weights(wl.np_weights(cfg.shape, seed=seed_w, gain_jitter=gain_jitter), np.float64)
    pr = wl.np_prompts(cfg.batch, cfg.prompt_len, cfg.shape.vocab, cfg.shape.mask_id)
    tok, msk = wl.initial_tokens(pr, cfg.gen_len, cfg.shape.mask_id)
    return cfg, w, tok, msk


def test_eps_zero_equals_plain_sampler_bitwise():
    """eps = 0 never locks, so SureLock is exactly the sampler without locking."""
    import dataclasses
    cfg, w, tok, msk = _tiny()
    cfg0 = dataclasses.replace(cfg, eps=0.0)
    t1, lp1, counts, _, _ = sl.surelock_sampler(cfg.shape, w, tok, msk, cfg0)
    t2, lp2 = sl.plain_sampler(cfg.shape, w, tok, msk, cfg0)
    assert np.all(counts == cfg.n_ctx)
    np.testing.assert_array_equal(t1, t2)
    np.testing.assert_array_equal(lp1, lp2)
    assert not np.any(t1 == cfg.shape.mask_id)


def test_sampler_invariants_tiny():
    cfg, w, tok, msk = _tiny()
    st = sl.init_state(cfg.shape, tok, msk)
    prev_act = st.act[0].copy()
    frozen = {}
    n_locked_total = 0
    for t in range(cfg.steps):
        masked_before = st.masked[0].copy()
        locked_before = st.locked[0].copy()
        rec = sl.step(cfg.shape, w, st, cfg, t, record_block_inputs=True)[0]
        A = rec["pos"]
        lk = rec["lock"]
        # masked positions never lock; nothing locks without a previous posterior
        assert not np.any(masked_before[A[lk]])
        if t == 0:
            assert not lk.any()
        # locks never revert, the active set only shrinks and stays sorted
        assert np.all(st.locked[0] >= locked_before)
        assert len(st.act[0]) <= len(prev_act)
        assert np.all(np.diff(st.act[0]) > 0)
        assert set(st.act[0].tolist()) <= set(prev_act.tolist())
        assert set(st.act[0].tolist()) == set(np.nonzero(~st.locked[0])[0].tolist())
        # K/V of locked rows: reproducible from their frozen block inputs
        # (recomputed from all of the step's block inputs: same matrix shapes,
        # same rounding, so equality is bitwise)
        kv = [om.kv_of_block_input(cfg.shape, w["layers"][l], rec["block_inputs"][l], A)
              for l in range(cfg.shape.n_layers)]
        for j in np.nonzero(lk)[0]:
            p = A[j]
            for l in range(cfg.shape.n_layers):
                np.testing.assert_array_equal(kv[l][0][j], st.ck[0, l, p])
                np.testing.assert_array_equal(kv[l][1][j], st.cv[0, l, p])
            frozen[p] = (st.ck[0, :, p].copy(), st.cv[0, :, p].copy(), st.lp_prev[0, p].copy(),
                         st.tokens[0, p])
        n_locked_total += int(lk.sum())
        # frozen cache rows and posterior of earlier locks are bitwise unchanged
        for p, (k, v, lp, tk) in frozen.items():
            np.testing.assert_array_equal(st.ck[0, :, p], k)
            np.testing.assert_array_equal(st.cv[0, :, p], v)
            np.testing.assert_array_equal(st.lp_prev[0, p], lp)
            assert st.tokens[0, p] == tk
        prev_act = st.act[0].copy()
    assert n_locked_total > 10          # the tiny workload does exercise locking
    assert not np.any(st.tokens == cfg.shape.mask_id)


def test_sampler_huge_eps_locks_every_eligible_row_at_step_one():
    import dataclasses
    cfg, w, tok, msk = _tiny()
    cfg_big = dataclasses.replace(cfg, eps=1e9)
    st = sl.init_state(cfg.shape, tok, msk)
    sl.step(cfg.shape, w, st, cfg_big, 0)
    unmasked_after_0 = ~st.masked[0]
    rec = sl.step(cfg.shape, w, st, cfg_big, 1)[0]
    # every row that was unmasked at the start of step 1 locks; masked rows stay
    assert set(rec["pos"][rec["lock"]].tolist()) == set(np.nonzero(unmasked_after_0)[0].tolist())


def test_gate_only_locks_rows_at_or_below_threshold():
    import dataclasses
    cfg, w, tok, msk = _tiny()
    cfg_g = dataclasses.replace(cfg, eps=1e9, gate_q=0.5)
    st = sl.init_state(cfg.shape, tok, msk)
    sl.step(cfg.shape, w, st, cfg_g, 0)
    rec = sl.step(cfg.shape, w, st, cfg_g, 1)[0]
    assert np.all(rec["u"][rec["lock"]] <= rec["thr"])
    assert rec["thr"] == np.quantile(rec["u"], 0.5, method="lower")
    assert 0 < rec["lock"].sum() < len(rec["pos"])


def test_scripted_schedule_follows_target():
    import dataclasses
    cfg, w, tok, msk = _tiny()
    cfg_s = dataclasses.replace(cfg, scripted=True, eps=0.0)
    st = sl.init_state(cfg.shape, tok, msk)
    for t in range(cfg.steps):
        m_before = len(st.act[0])
        n_elig = int(np.sum(~st.masked[0, st.act[0]] & st.has_prev[0, st.act[0]]))
        sl.step(cfg.shape, w, st, cfg_s, t)
        want = max(cfg_s.scripted_target(t), m_before - n_elig, 0)
        assert len(st.act[0]) == min(m_before, want)


def test_scripted_target_formula():
    cfg = wl.cfg_full8b(scripted=True)
    assert cfg.scripted_target(0) == 383            # 384 - 1.355 -> 382.6 -> 383
    assert cfg.scripted_target(cfg.steps - 2) == 38   # 384 - 345.6 = 38.4 at t+1 = T-1
    tg = [cfg.scripted_target(t) for t in range(cfg.steps - 1)]
    assert all(a >= b for a, b in zip(tg, tg[1:]))
    # the target never asks to lock masked rows: masked count after step t is 256-(t+1)
    assert all(tg[t] >= 256 - (t + 1) for t in range(cfg.steps - 1))


def test_flops_model():
    s = wl.LLADA8B
    # per-row linear FLOPs 2 (L (4 d^2 + 3 d f) + V d) = 2 * 7.497e9
    assert sl.flops_per_step(s, 1, 0) == pytest.approx(2 * 7.497e9, rel=1e-3)
    assert sl.flops_per_step(s, 10, 100) - sl.flops_per_step(s, 10, 0) == 4 * 32 * 10 * 100 * 4096


# ---------------------------------------------------------------- ablations --

def test_gate_only_sampler_equals_unbounded_eps_with_gate():
    import dataclasses
    cfg, w, tok, msk = _tiny()
    a = sl.surelock_sampler(cfg.shape, w, tok, msk, dataclasses.replace(cfg, gate_q=0.3, gate_only=True))
    b = sl.surelock_sampler(cfg.shape, w, tok, msk, dataclasses.replace(cfg, gate_q=0.3, eps=1e30))
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    np.testing.assert_array_equal(a[2], b[2])
    assert a[2][-1, 0] < cfg.n_ctx            # the gate alone does lock rows


def test_no_kv_cache_sampler_without_locks_is_the_plain_sampler():
    import dataclasses
    cfg, w, tok, msk = _tiny()
    c0 = dataclasses.replace(cfg, eps=0.0, no_kv_cache=True)
    t1, lp1, counts, _, _ = sl.surelock_sampler(cfg.shape, w, tok, msk, c0)
    t2, lp2 = sl.plain_sampler(cfg.shape, w, tok, msk, c0)
    assert np.all(counts == cfg.n_ctx)
    np.testing.assert_array_equal(t1, t2)
    np.testing.assert_array_equal(lp1, lp2)


def test_no_kv_cache_sampler_departs_only_after_the_first_lock():
    """The ablation changes nothing until some row is locked; from the step
    after the first lock the active rows' posteriors differ."""
    import dataclasses
    cfg, w, tok, msk = _tiny()
    st_a = sl.init_state(cfg.shape, tok, msk)
    st_b = sl.init_state(cfg.shape, tok, msk)
    cfg_b = dataclasses.replace(cfg, no_kv_cache=True)
    first_lock = None
    for t in range(cfg.steps):
        ra = sl.step(cfg.shape, w, st_a, cfg, t)[0]
        rb = sl.step(cfg.shape, w, st_b, cfg_b, t)[0]
        if first_lock is None:
            np.testing.assert_array_equal(ra["lp"], rb["lp"])
            np.testing.assert_array_equal(ra["lock"], rb["lock"])
            if ra["lock"].any():
                first_lock = t
        elif t == first_lock + 1:
            assert np.abs(ra["lp"] - rb["lp"]).max() > 1e-6
            break
        assert np.all(np.diff(st_b.act[0]) > 0)
    assert first_lock is not None


# ---- composition with K/V reuse for the active rows (refresh interval R) ----

def _reuse_state_trace(cfg, w, tok, msk):
    """Run the decode step by step; per step the active set and mask flags at
    its start, the record, and snapshots of the cache and posteriors."""
    st = sl.init_state(cfg.shape, tok, msk)
    out = []
    for t in range(cfg.steps):
        snap = (st.act[0].copy(), st.masked[0].copy(), st.locked[0].copy(),
                st.ck.copy(), st.cv.copy(), st.lp_prev.copy())
        rec = sl.step(cfg.shape, w, st, cfg, t, record_block_inputs=True)[0]
        out.append((snap, rec))
    return st, out


@pytest.mark.parametrize("R", [2, 3])
def test_kv_reuse_computed_rows_and_frozen_rows(R):
    """Between refresh steps (t mod R != 0) only the active rows that are masked,
    or were masked at the start of the previous step, are computed; every other
    active row keeps its cached K/V and its last posterior bitwise, and only
    computed rows can lock.  Refresh steps compute all of A_t."""
    import dataclasses
    cfg, w, tok, msk = _tiny()
    c = dataclasses.replace(cfg, kv_reuse=R)
    st, trace = _reuse_state_trace(c, w, tok, msk)
    prev_mask = msk[0].astype(bool)
    n_reused = n_locks = 0
    for t, ((A, mask0, locked0, ck0, cv0, lp0), rec) in enumerate(trace):
        C = rec["pos"]
        np.testing.assert_array_equal(rec["active"], A)
        if t % R == 0:
            np.testing.assert_array_equal(C, A)
        else:
            np.testing.assert_array_equal(C, A[mask0[A] | prev_mask[A]])
            assert set(np.nonzero(mask0)[0].tolist()) <= set(C.tolist())
        reused = np.setdiff1d(A, C)
        n_reused += len(reused)
        nxt = trace[t + 1][0] if t + 1 < len(trace) else (st.act[0], st.masked[0], st.locked[0],
                                                             st.ck, st.cv, st.lp_prev)
        for p in reused:
            np.testing.assert_array_equal(nxt[3][0, :, p], ck0[0, :, p])
            np.testing.assert_array_equal(nxt[4][0, :, p], cv0[0, :, p])
            np.testing.assert_array_equal(nxt[5][0, p], lp0[0, p])
        # the computed rows' cache entries are those of this step's block inputs
        for l in range(c.shape.n_layers):
            k, v = om.kv_of_block_input(c.shape, w["layers"][l], rec["block_inputs"][l], C)
            np.testing.assert_array_equal(k, nxt[3][0, l, C])
            np.testing.assert_array_equal(v, nxt[4][0, l, C])
        # locks: among computed rows only, never on a row masked at the step's start
        new_locks = np.nonzero(nxt[2] & ~locked0)[0]
        np.testing.assert_array_equal(new_locks, C[rec["lock"]])
        assert not np.any(mask0[new_locks])
        np.testing.assert_array_equal(nxt[0], np.setdiff1d(A, new_locks))
        n_locks += len(new_locks)
        prev_mask = mask0
    assert n_reused > 20 and n_locks > 10       # both mechanisms are exercised
    assert not np.any(st.tokens == c.shape.mask_id)


@pytest.mark.parametrize("R", [2, 3, 7])
def test_kv_reuse_is_exact_for_a_single_block(R):
    """With one block a row's K/V depend on its own token and position only, and
    an unmasked token never changes, so a row recomputed once after its
    unmasking has exact K/V from then on.  Reuse (like locking) then changes no
    decision: the decode's tokens are those of the sampler without locking.
    A computed set that missed the rows unmasked in the previous step would
    leave their mask-token K/V in the cache and change the tokens."""
    import dataclasses
    shape1 = dataclasses.replace(wl.TINY, n_layers=1)
    c = dataclasses.replace(wl.CFG_TINY, shape=shape1, kv_reuse=R, eps=0.05)
    w = om.cast_weights(wl.np_weights(shape1, seed=0, std=0.2), np.float64)
    pr = wl.np_prompts(c.batch, c.prompt_len, shape1.vocab, shape1.mask_id)
    tok, msk = wl.initial_tokens(pr, c.gen_len, shape1.mask_id)
    t_reuse = sl.surelock_sampler(shape1, w, tok, msk, c)[0]
    t_plain = sl.plain_sampler(shape1, w, tok, msk, c)[0]
    np.testing.assert_array_equal(t_reuse, t_plain)


def test_kv_reuse_is_an_approximation_with_two_blocks():
    """With two blocks the second block's K/V of a reused row depend on the
    other rows, so the first step between refreshes already departs from the
    recomputing sampler on the rows it does compute; R = 1 is SureLock."""
    import dataclasses
    cfg, w, tok, msk = _tiny()
    st1 = sl.init_state(cfg.shape, tok, msk)
    st2 = sl.init_state(cfg.shape, tok, msk)
    st3 = sl.init_state(cfg.shape, tok, msk)
    c2 = dataclasses.replace(cfg, kv_reuse=2)
    c1 = dataclasses.replace(cfg, kv_reuse=1)
    for t in range(2):
        r1 = sl.step(cfg.shape, w, st1, cfg, t)[0]
        r2 = sl.step(cfg.shape, w, st2, c2, t)[0]
        r3 = sl.step(cfg.shape, w, st3, c1, t)[0]
        np.testing.assert_array_equal(r1["lp"], r3["lp"])
    C = r2["pos"]
    assert len(C) < len(r1["pos"])
    j = np.searchsorted(r1["pos"], C)
    assert np.abs(r1["lp"][j] - r2["lp"]).max() > 1e-6


def test_kv_reuse_rejects_the_scripted_schedule_and_the_no_cache_ablation():
    import dataclasses
    cfg, w, tok, msk = _tiny()
    for kw in ({"scripted": True}, {"no_kv_cache": True}):
        c = dataclasses.replace(cfg, kv_reuse=2, **kw)
        st = sl.init_state(cfg.shape, tok, msk)
        with pytest.raises(ValueError):
            sl.step(cfg.shape, w, st, c, 0)


def test_semi_ar_blocks_fill_in_order():
    """The semi-autoregressive schedule: each step unmasks exactly k positions,
    all inside the current block; a block has no masked position left after its
    steps, and no later block is touched before it is current (two blocks of 24
    positions, 8 steps each, 3 per step)."""
    import dataclasses
    cfg, w, tok, msk = _tiny()
    c = dataclasses.replace(cfg, block_len=24, steps=16, tokens_per_step=3)
    c.validate()
    st = sl.init_state(c.shape, tok, msk)
    for t in range(c.steps):
        lo, hi = c.block_bounds(t)
        before = st.masked[0].copy()
        sl.step(c.shape, w, st, c, t)
        newly = np.nonzero(before & ~st.masked[0])[0]
        assert len(newly) == c.tokens_per_step
        assert np.all((newly >= lo) & (newly < hi))
        if (t + 1) % c.steps_per_block == 0:
            assert not st.masked[0, lo:hi].any()
        assert st.masked[0, hi:].all()
    assert not st.masked.any()


def test_sequences_of_a_batch_are_independent():
    """Two sequences stepped together give, bitwise, what each gives alone: the
    gate quantile, the unmasking and the compaction are per sequence."""
    import dataclasses
    cfg, w, _, _ = _tiny()
    c2 = dataclasses.replace(cfg, batch=2, gate_q=0.5, eps=0.05)
    pr = wl.np_prompts(2, c2.prompt_len, c2.shape.vocab, c2.shape.mask_id, seed=11)
    tok, msk = wl.initial_tokens(pr, c2.gen_len, c2.shape.mask_id)
    both = sl.surelock_sampler(c2.shape, w, tok, msk, c2)
    c1 = dataclasses.replace(c2, batch=1)
    for b in range(2):
        one = sl.surelock_sampler(c1.shape, w, tok[b:b + 1], msk[b:b + 1], c1)
        np.testing.assert_array_equal(both[0][b], one[0][0])
        np.testing.assert_array_equal(both[1][b], one[1][0])
        np.testing.assert_array_equal(both[2][:, b], one[2][:, 0])
