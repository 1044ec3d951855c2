"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each test checks the oracle against a closed form, a special case that reduces
to a library routine, a brute-force enumeration, an invariant, or a worked
example of the DSpark pages -- never against a retyped copy of its own loops.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy import special, stats

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(a):
    return synth.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def _f(a):
    return synth.bf16_bits_to_f32(a).astype(np.float64)


def _tiny_draft_inputs(nb, gamma, V, r, w_std, seed):
    rng = np.random.default_rng(seed)
    W1 = _bf16(rng.normal(0, w_std, (V, r)))
    W2 = _bf16(rng.normal(0, w_std, (r, V)))
    U = _bf16(rng.normal(0, 1.0, (nb, gamma, V)))
    anchor = rng.integers(0, V, nb).astype(np.int32)
    return U, anchor, W1, W2


# ---------------------------------------------------------------------------
# Markov head (gdymind.com "DSpark", section 4): B = W1 W2 "in principle a full
# V x V matrix" -- the low-rank path must equal drafting with the materialised
# full transition matrix.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("V,r,gamma,nb", [(64, 8, 6, 3), (300, 16, 5, 4), (1000, 256, 3, 2)])
def test_draft_equals_full_transition_matrix(oracle_mod, V, r, gamma, nb):
    U, anchor, W1, W2 = _tiny_draft_inputs(nb, gamma, V, r, 0.6, seed=V)
    Bfull = _f(W1) @ _f(W2)                      # [V, V] in fp64
    x, logit, gap = oracle_mod.draft(U, anchor, W1, W2)
    Uf = _f(U)
    for i in range(nb):
        prev = anchor[i]
        for k in range(gamma):
            l = Uf[i, k] + Bfull[prev]
            xk = int(np.argmax(l))
            assert x[i, k] == xk
            assert logit[i, k] == pytest.approx(l[xk], abs=1e-10)
            srt = np.sort(l)
            assert gap[i, k] == pytest.approx(srt[-1] - srt[-2], abs=1e-10)
            prev = xk
    # the bias must actually move the choice somewhere in these cases
    plain = np.argmax(Uf, axis=2)
    assert (plain != x).any()


def test_draft_zero_factor_is_parallel_argmax(oracle_mod):
    V, r, gamma, nb = 500, 32, 7, 5
    U, anchor, W1, W2 = _tiny_draft_inputs(nb, gamma, V, r, 0.5, seed=11)
    for zero in ("W1", "W2"):
        a = np.zeros_like(W1) if zero == "W1" else W1
        b = np.zeros_like(W2) if zero == "W2" else W2
        x, logit, _ = oracle_mod.draft(U, anchor, a, b)
        np.testing.assert_array_equal(x, np.argmax(_f(U), axis=2))
        np.testing.assert_array_equal(logit, np.max(_f(U), axis=2))


def test_draft_ties_take_smallest_index(oracle_mod):
    V, r, gamma = 64, 8, 4
    U = np.zeros((1, gamma, V), dtype=np.uint16)
    U[0, :, [5, 9, 40]] = _bf16([3.0])[0]
    x, logit, gap = oracle_mod.draft(U, np.array([2], np.int32), np.zeros((V, r), np.uint16),
                                     np.zeros((r, V), np.uint16))
    assert (x == 5).all() and (logit == 3.0).all() and (gap == 0.0).all()


def test_draft_rejects_bad_anchor(oracle_mod):
    U, anchor, W1, W2 = _tiny_draft_inputs(1, 2, 64, 8, 0.1, seed=1)
    with pytest.raises(ValueError):
        oracle_mod.draft(U, np.array([64], np.int32), W1, W2)


@pytest.mark.parametrize("mode", [0, 1])
def test_draft_forced_on_its_own_tokens_is_the_free_running_draft(oracle_mod, mode):
    # teacher forcing with x_{k-1} = the tokens the free-running draft picked must give
    # back that draft exactly (greedy and Gumbel-max, whose noise is keyed by position)
    V, r, gamma, nb = 400, 16, 7, 5
    U, anchor, W1, W2 = _tiny_draft_inputs(nb, gamma, V, r, 0.4, seed=21)
    x, l, g = oracle_mod.draft(U, anchor, W1, W2, mode=mode, tau=0.8, seed=5)
    prev = np.concatenate([anchor[:, None], x[:, :-1]], axis=1)
    xf, lf, gf = oracle_mod.draft(U, anchor, W1, W2, mode=mode, tau=0.8, seed=5, forced_prev=prev)
    np.testing.assert_array_equal(xf, x)
    np.testing.assert_array_equal(lf, l)
    np.testing.assert_array_equal(gf, g)


def test_draft_forced_position_is_a_one_step_draft_from_that_token(oracle_mod):
    # greedy: position k forced to x_{k-1} = t equals a one-position draft whose anchor
    # is t and whose base logits are U[:, k-1] (catches an off-by-one in the forcing)
    V, r, gamma, nb = 300, 16, 6, 4
    U, anchor, W1, W2 = _tiny_draft_inputs(nb, gamma, V, r, 0.5, seed=22)
    prev = np.random.default_rng(3).integers(0, V, (nb, gamma)).astype(np.int32)
    xf, lf, gf = oracle_mod.draft(U, anchor, W1, W2, forced_prev=prev)
    for k in range(gamma):
        x1, l1, g1 = oracle_mod.draft(U[:, k:k + 1].copy(), prev[:, k].copy(), W1, W2)
        np.testing.assert_array_equal(xf[:, k], x1[:, 0])
        np.testing.assert_array_equal(lf[:, k], l1[:, 0])
        np.testing.assert_array_equal(gf[:, k], g1[:, 0])


def test_draft_forced_rejects_out_of_range_tokens(oracle_mod):
    U, anchor, W1, W2 = _tiny_draft_inputs(2, 3, 64, 8, 0.1, seed=1)
    prev = np.zeros((2, 3), np.int32)
    prev[1, 2] = 64
    with pytest.raises(ValueError):
        oracle_mod.draft(U, anchor, W1, W2, forced_prev=prev)


# ---------------------------------------------------------------------------
# Gumbel-max: frequencies must follow softmax(l / tau)
# ---------------------------------------------------------------------------
def test_gumbel_max_frequencies_follow_softmax(oracle_mod):
    V, r, gamma, nb, tau = 8, 4, 50, 2000, 0.7
    l = np.array([0.0, 0.5, -1.0, 1.25, 0.25, -0.5, 1.0, 0.75], dtype=np.float32)
    U = np.broadcast_to(_bf16(l), (nb, gamma, V)).copy()
    W1 = np.zeros((V, r), np.uint16)
    W2 = np.zeros((r, V), np.uint16)
    x, logit, _ = oracle_mod.draft(U, np.zeros(nb, np.int32), W1, W2, mode=1, tau=tau, seed=1234)
    counts = np.bincount(x.ravel(), minlength=V)
    p = special.softmax(_f(_bf16(l)) / tau)
    chi2, pval = stats.chisquare(counts, p * counts.sum())
    assert pval > 1e-4, (counts, p * counts.sum(), pval)
    # the reported logit is the unperturbed one at the chosen token
    np.testing.assert_array_equal(logit, _f(_bf16(l))[x])


def test_gumbel_small_temperature_is_greedy(oracle_mod):
    V, r, gamma, nb = 200, 8, 6, 6
    U, anchor, W1, W2 = _tiny_draft_inputs(nb, gamma, V, r, 0.3, seed=5)
    xg, _, gapg = oracle_mod.draft(U, anchor, W1, W2, mode=0)
    xs, _, _ = oracle_mod.draft(U, anchor, W1, W2, mode=1, tau=1e-6, seed=99)
    # noise is at most about 17 in size, so with tau = 1e-6 only gaps below 4e-5 can flip
    ok = gapg > 1e-4
    assert ok.mean() > 0.9
    np.testing.assert_array_equal(xg[ok], xs[ok])


def test_noise_key_uses_request_position_and_vocab(oracle_mod):
    g = {(b, k, v): oracle_mod.gumbel(7, b, k, v) for b in range(3) for k in (1, 2) for v in range(9)}
    assert len(set(g.values())) == len(g)


# ---------------------------------------------------------------------------
# Philox4x32-10 (SC'11): each round is a bijection.  The inverse below undoes a
# round with the published multipliers and Weyl constants; a wrong constant or
# word wiring in the oracle breaks the round trip.  (Agreement with other
# Philox implementations is not pinned: no known-answer vectors are at hand.)
# ---------------------------------------------------------------------------
_M0, _M1 = 0xD2511F53, 0xCD9E8D57
_W0, _W1 = 0x9E3779B9, 0xBB67AE85
_MASK = 0xFFFFFFFF


def _philox_inverse(y, key):
    keys = [((key[0] + i * _W0) & _MASK, (key[1] + i * _W1) & _MASK) for i in range(10)]
    inv0, inv1 = pow(_M0, -1, 1 << 32), pow(_M1, -1, 1 << 32)
    y0, y1, y2, y3 = (int(t) for t in y)
    for k0, k1 in reversed(keys):
        x2 = (y1 * inv1) & _MASK
        x0 = (y3 * inv0) & _MASK
        x1 = y0 ^ ((_M1 * x2) >> 32) ^ k0
        x3 = y2 ^ ((_M0 * x0) >> 32) ^ k1
        y0, y1, y2, y3 = x0, x1, x2, x3
    return [y0, y1, y2, y3]


def test_philox_rounds_invert(oracle_mod):
    rng = np.random.default_rng(3)
    for _ in range(200):
        ctr = rng.integers(0, 2**32, 4, dtype=np.uint64).astype(np.uint32)
        key = rng.integers(0, 2**32, 2, dtype=np.uint64).astype(np.uint32)
        out = oracle_mod.philox4x32_10(ctr, key)
        assert _philox_inverse(out, [int(k) for k in key]) == [int(c) for c in ctr]


def test_philox_output_is_uniform(oracle_mod):
    words = np.concatenate([oracle_mod.philox4x32_10([i, 0, 5, 0], [1, 2]) for i in range(4096)])
    hist = np.bincount((words >> 28).astype(np.int64), minlength=16)
    assert stats.chisquare(hist).pvalue > 1e-4


def test_uniform_from_word_stays_inside_open_interval(oracle_mod):
    assert oracle_mod.uniform_from_word(0) == 2.0**-24
    assert oracle_mod.uniform_from_word(0xFFFFFFFF) == 1.0 - 2.0**-24
    assert oracle_mod.uniform_from_word(1 << 31) == 0.5 + 2.0**-24


# ---------------------------------------------------------------------------
# Confidence head + Sequential Temperature Scaling + survival product
# (gdymind.com "DSpark", section 5)
# ---------------------------------------------------------------------------
def _conf_inputs(B, gamma, d, r, V, seed):
    rng = np.random.default_rng(seed)
    h = _bf16(rng.normal(0, 1, (B, gamma, d)))
    W1 = _bf16(rng.normal(0, 0.5, (V, r)))
    w = _bf16(rng.normal(0, 1 / math.sqrt(d + r), d + r))
    anchor = rng.integers(0, V, B).astype(np.int32)
    x = rng.integers(0, V, (B, gamma)).astype(np.int32)
    T = rng.uniform(1, 3, gamma).astype(np.float32)
    return h, anchor, x, W1, w, T


def test_confidence_one_hot_weights_select_inputs(oracle_mod):
    B, gamma, d, r, V = 3, 5, 24, 8, 50
    h, anchor, x, W1, w, T = _conf_inputs(B, gamma, d, r, V, 1)
    ones = np.ones(gamma, np.float32)
    hf, Ef = _f(h), _f(W1)
    prev = np.concatenate([anchor[:, None], x[:, :-1]], axis=1)   # x_{k-1}, x_0 = anchor
    for i in (0, 7, d - 1):
        e = np.zeros(d + r, np.uint16); e[i] = _bf16([1.0])[0]
        out = oracle_mod.confidence(h, anchor, x, W1, e, 0.25, ones)
        np.testing.assert_allclose(out["z"], hf[:, :, i] + 0.25, rtol=0, atol=1e-12)
        np.testing.assert_allclose(out["c"], special.expit(hf[:, :, i] + 0.25), rtol=1e-12)
    for j in (0, 3, r - 1):
        e = np.zeros(d + r, np.uint16); e[d + j] = _bf16([1.0])[0]
        out = oracle_mod.confidence(h, anchor, x, W1, e, -0.5, ones)
        np.testing.assert_allclose(out["z"], Ef[prev, j] - 0.5, rtol=0, atol=1e-12)


def test_confidence_zero_weights_give_bias_only(oracle_mod):
    B, gamma, d, r, V = 2, 6, 16, 8, 30
    h, anchor, x, W1, w, T = _conf_inputs(B, gamma, d, r, V, 2)
    out = oracle_mod.confidence(h, anchor, x, W1, np.zeros(d + r, np.uint16), 1.0, T)
    np.testing.assert_allclose(out["c"], np.broadcast_to(special.expit(1.0 / T.astype(np.float64)),
                                                         (B, gamma)), rtol=1e-13)


def test_sts_temperature_scales_the_logit(oracle_mod):
    B, gamma, d, r, V = 4, 7, 32, 16, 80
    h, anchor, x, W1, w, T = _conf_inputs(B, gamma, d, r, V, 3)
    c1 = oracle_mod.confidence(h, anchor, x, W1, w, 1.0, np.ones(gamma, np.float32))["c"]
    cT = oracle_mod.confidence(h, anchor, x, W1, w, 1.0, T)["c"]
    # T = 1 is the plain sigmoid of the logit; any T divides that same logit
    np.testing.assert_allclose(special.logit(cT) * T, special.logit(c1), rtol=1e-9, atol=1e-9)
    big = oracle_mod.confidence(h, anchor, x, W1, w, 1.0, np.full(gamma, 1e30, np.float32))["c"]
    np.testing.assert_allclose(big, 0.5, atol=1e-12)


def test_survival_is_cumulative_product_and_never_increases(oracle_mod):
    B, gamma, d, r, V = 6, 12, 40, 16, 100
    h, anchor, x, W1, w, T = _conf_inputs(B, gamma, d, r, V, 4)
    out = oracle_mod.confidence(h, anchor, x, W1, w, 2.0, T)
    c, P64, P32 = out["c"], out["P64"], out["P32"]
    np.testing.assert_allclose(P64[:, 0], c[:, 0], rtol=1e-15)
    np.testing.assert_allclose(P64[:, 1:] / P64[:, :-1], c[:, 1:], rtol=1e-12)
    assert (np.diff(P64, axis=1) <= 0).all() and (P64 > 0).all() and (P64 <= 1).all()
    assert (np.diff(P32.astype(np.float64), axis=1) <= 0).all()
    np.testing.assert_allclose(P32, P64, rtol=1e-5)
    # the fp32 product takes one rounding per step, with each factor rounded to fp32 first
    np.testing.assert_array_equal(P32[:, 0], c[:, 0].astype(np.float32))


def test_confidence_rejects_bad_temperature(oracle_mod):
    h, anchor, x, W1, w, T = _conf_inputs(1, 2, 8, 4, 10, 5)
    with pytest.raises(ValueError):
        oracle_mod.confidence(h, anchor, x, W1, w, 0.0, np.array([1.0, 0.0], np.float32))


# ---------------------------------------------------------------------------
# Hardware-aware prefix scheduler (wispaper.ai "The Hardware-Aware Prefix
# Scheduler"; gdymind.com "DSpark", section 6)
# ---------------------------------------------------------------------------
def _objective(P, L, Tstep):
    """Expected tokens per second of a verify-length choice, exact numerator."""
    B = P.shape[0]
    num = B << 46
    for b in range(B):
        for k in range(L[b]):
            num += math.floor(float(P[b, k]) * 2.0**46)
    return math.ldexp(float(num) / float(Tstep[B + sum(L)]), -46)


def _tables(B, gamma, rng):
    n = B * (gamma + 1) + 1
    yield np.full(n, 1000.0)                                          # flat
    yield 1000.0 + 90.0 * np.arange(n)                                # linear
    yield 500.0 + 300.0 * np.maximum(0, np.arange(n) - B - 2)         # knee
    yield rng.uniform(100.0, 2000.0, n)                               # arbitrary
    yield np.sort(rng.uniform(100.0, 2000.0, n))                      # increasing staircase


@pytest.mark.parametrize("B,gamma", [(1, 1), (1, 4), (2, 3), (3, 2), (3, 4), (2, 4)])
def test_schedule_matches_brute_force_enumeration(oracle_mod, B, gamma):
    rng = np.random.default_rng(100 * B + gamma)
    for trial in range(6):
        P = synth.monotone_scores(B, gamma, seed=trial * 31 + B, tie_frac=0.3 if trial % 2 else 0.0,
                                  zero_frac=0.3 if trial == 4 else 0.0)
        for Tstep in _tables(B, gamma, rng):
            L, N, F, _ = oracle_mod.schedule(P, Tstep)
            best, best_n = -1.0, None
            for Ls in itertools.product(range(gamma + 1), repeat=B):
                f = _objective(P, Ls, Tstep)
                if f > best:
                    best, best_n = f, sum(Ls)
                elif f == best:
                    best_n = min(best_n, sum(Ls))
            assert F == best
            assert _objective(P, L, Tstep) == best
            assert N == int(L.sum()) == best_n


@pytest.mark.parametrize("B,gamma", [(32768, 2), (1024, 64)])
def test_schedule_largest_sizes_closed_form(oracle_mod, B, gamma):
    # every score 1 and a flat curve: verify everything, F = (B + B gamma) / T exactly.
    # The fixed-point numerator (B + B gamma) 2^46 must not overflow at these sizes.
    T = 15000.0
    L, N, F, _ = oracle_mod.schedule(np.ones((B, gamma), np.float32), np.full(B * (gamma + 1) + 1, T))
    assert (L == gamma).all() and N == B * gamma
    assert F == (B + B * gamma) / T
    # halve every score: F = (B + B gamma / 2) / T, still everything verified
    L, N, F, _ = oracle_mod.schedule(np.full((B, gamma), 0.5, np.float32),
                                     np.full(B * (gamma + 1) + 1, T))
    assert N == B * gamma and F == (B + B * gamma / 2) / T


def test_schedule_flat_curve_verifies_everything(oracle_mod):
    B, gamma = 4, 8
    P = synth.monotone_scores(B, gamma, seed=9)
    L, N, F, _ = oracle_mod.schedule(P, np.full(B * (gamma + 1) + 1, 20000.0))
    assert (L == gamma).all() and N == B * gamma


def test_schedule_steep_curve_verifies_nothing(oracle_mod):
    B, gamma = 4, 8
    P = synth.monotone_scores(B, gamma, seed=9)
    n = np.arange(B * (gamma + 1) + 1, dtype=np.float64)
    L, N, F, _ = oracle_mod.schedule(P, 1000.0 * 4.0 ** n)
    assert (L == 0).all() and N == 0 and F == B / (1000.0 * 4.0 ** B)
    assert F * 1e6 == pytest.approx(B / 256.0 * 1e3)   # tokens per second at a 256 ms step


def test_schedule_lengths_are_prefixes_of_the_global_order(oracle_mod):
    B, gamma = 16, 6
    P = synth.monotone_scores(B, gamma, seed=4, tie_frac=0.4)
    Tstep = 1000.0 + 40.0 * np.arange(B * (gamma + 1) + 1)
    L, N, F, F_all = oracle_mod.schedule(P, Tstep)
    assert 0 < N < B * gamma and F == F_all.max() and int(np.argmax(F_all)) == N
    # every kept score is >= every dropped one
    kept = np.concatenate([P[b, :L[b]] for b in range(B)])
    dropped = np.concatenate([P[b, L[b]:] for b in range(B)])
    assert kept.min() >= dropped.max()


def test_schedule_worked_examples_of_the_pages(oracle_mod):
    with open(os.path.join(GOLDEN, "scheduler_worked_examples.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        P = np.array(case["P"], dtype=np.float32)
        L, N, F, F_all = oracle_mod.schedule(P, np.array(case["tstep_us"]))
        assert L.tolist() == case["expected_L"], case["name"]
        np.testing.assert_allclose(F_all[:len(case["F_by_N"])], case["F_by_N"], rtol=2e-4)


def test_schedule_negative_zero_scores_count_as_zero(oracle_mod):
    # -0.0 equals +0.0 as a number: the same lengths, N* and objective as with +0.0,
    # and exact zeros keep their (b asc, k asc) order behind every positive score
    B, gamma = 24, 6
    rng = np.random.default_rng(8)
    P = synth.monotone_scores(B, gamma, seed=2, tie_frac=0.2, zero_frac=0.6, neg_zero=True)
    assert np.signbit(P).any()
    Pp = np.where(P == 0.0, np.float32(0.0), P).astype(np.float32)
    for Tstep in _tables(B, gamma, rng):
        a = oracle_mod.schedule(P, Tstep)
        b = oracle_mod.schedule(Pp, Tstep)
        np.testing.assert_array_equal(a[0], b[0])
        assert a[1] == b[1] and a[2] == b[2]
        np.testing.assert_array_equal(a[3], b[3])


def test_schedule_rejects_scores_outside_unit_interval(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.schedule(np.array([[1.5, 0.5]], np.float32), np.ones(4))


# ---------------------------------------------------------------------------
# Strict prefix-match verification (seventnews.com article: the first rejected
# token and everything after it are dropped)
# ---------------------------------------------------------------------------
def test_verify_special_cases(oracle_mod):
    gamma = 5
    x = np.array([[1, 2, 3, 4, 5]] * 5, np.int32)
    t = np.array([[1, 2, 3, 4, 5, 6],      # all agree
                  [9, 2, 3, 4, 5, 6],      # first disagrees
                  [1, 2, 9, 4, 5, 6],      # third disagrees
                  [1, 2, 3, 4, 9, 6],      # fifth disagrees, beyond L
                  [1, 2, 3, 4, 5, 6]], np.int32)
    L = np.array([5, 3, 4, 3, 0], np.int32)
    acc, bonus = oracle_mod.verify(x, L, t)
    assert acc.tolist() == [5, 0, 2, 3, 0]
    assert bonus.tolist() == [6, 9, 9, 4, 1]


def test_verify_random_against_mask_formulation(oracle_mod):
    x, L, t = synth.verify_inputs(300, 9, 50, seed=2, agree=0.8)
    acc, bonus = oracle_mod.verify(x, L, t)
    k = np.arange(9)[None, :]
    bad = (x != t[:, :9]) & (k < L[:, None])
    expect = np.where(bad.any(axis=1), bad.argmax(axis=1), L)
    np.testing.assert_array_equal(acc, expect)
    np.testing.assert_array_equal(bonus, t[np.arange(300), expect])


def test_verify_rejects_length_beyond_gamma(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.verify(np.zeros((1, 3), np.int32), np.array([4], np.int32),
                          np.zeros((1, 4), np.int32))


# ---------------------------------------------------------------------------
# Sequential Temperature Scaling, fitting (gdymind.com "DSpark", section 5,
# "Sequential Temperature Scaling"): per position, left to right, a 1-D grid
# search for the temperature minimising the ECE of the cumulative product, with
# the temperatures of earlier positions frozen.
# ---------------------------------------------------------------------------
def test_ece_hand_computed_values(oracle_mod):
    # one sample per bin: the ECE is the mean |y - P|
    P = np.array([0.1, 0.2, 0.85, 0.9])
    acc = np.array([0, 1, 1, 1], np.int32)           # labels at k = 1: acc >= 1
    assert oracle_mod.ece(P, acc, 1) == pytest.approx((0.1 + 0.8 + 0.15 + 0.1) / 4, abs=1e-15)
    # two samples in one bin (0.30 and 0.32 both fall in [4/15, 5/15)): the gap is
    # taken between the bin's sums, not sample by sample
    P = np.array([0.30, 0.32])
    assert oracle_mod.ece(P, np.array([1, 0], np.int32), 1) == pytest.approx(abs(1 - 0.62) / 2,
                                                                           abs=1e-15)
    # P = 1 lands in the last bin; labels use acc >= k
    P = np.array([1.0, 1.0, 0.0])
    acc = np.array([3, 2, 0], np.int32)
    assert oracle_mod.ece(P, acc, 3) == pytest.approx(1.0 / 3, abs=1e-15)
    assert oracle_mod.ece(P, acc, 2) == pytest.approx(0.0, abs=1e-15)
    # one bin: ECE is |mean label - mean score|
    rng = np.random.default_rng(0)
    P = rng.random(1000)
    acc = rng.integers(0, 3, 1000).astype(np.int32)
    assert oracle_mod.ece(P, acc, 1, n_bins=1) == pytest.approx(abs((acc >= 1).mean() - P.mean()),
                                                                abs=1e-13)


def _two_group_calibration():
    """Two groups of 50 blocks, exactly calibrated at T = (2, 3) on the grid.

    Position 1: sigmoid(z / 2) is 0.3 in group A and 0.7 in group B, and 15 and 35
    blocks of them accept.  Position 2: sigmoid(z / 3) is 0.8 for every block,
    so the cumulative products are 0.24 and 0.56, and 12 and 28 blocks accept
    both drafts.  Every other temperature moves the scores off the label rates.
    """
    za = 2.0 * math.log(0.3 / 0.7)
    zb = 2.0 * math.log(0.7 / 0.3)
    z2 = 3.0 * math.log(4.0)
    z = np.zeros((100, 2), np.float32)
    z[:50, 0], z[50:, 0], z[:, 1] = za, zb, z2
    acc = np.zeros(100, np.int32)
    acc[:12] = 2; acc[12:15] = 1                       # group A: 15 accept #1, 12 accept #2
    acc[50:78] = 2; acc[78:85] = 1                     # group B: 35 accept #1, 28 accept #2
    return z, acc


def test_sts_fit_exact_calibration_is_found(oracle_mod):
    z, acc = _two_group_calibration()
    T, e = oracle_mod.sts_fit(z, acc, t_min=0.5, t_step=0.01, n_t=451)
    # z is stored in fp32, so the zero of the ECE sits within 1e-6 of (2, 3)
    np.testing.assert_allclose(T, [2.0, 3.0], atol=1e-9)
    assert (e < 1e-6).all()
    # with position 1 frozen at its raw scores (T = 1: 0.155 and 0.845) instead of
    # its fitted ones, the product at T_2 = 3 would be 0.124 and 0.676 against
    # label rates 0.24 and 0.56, so the zero at (2, 3) pins the frozen prefix too


def test_sts_fit_scales_with_the_logits(oracle_mod):
    # sigmoid((2 z) / (2 T)) = sigmoid(z / T) bit for bit, and the doubled grid
    # 1.0 + 0.02 i is exactly twice 0.5 + 0.01 i: the fit must double exactly
    z, acc = synth.calibration_set(3000, 6, seed=3)
    T, e = oracle_mod.sts_fit(z, acc, t_min=0.5, t_step=0.01, n_t=451)
    T2, e2 = oracle_mod.sts_fit(2 * z, acc, t_min=1.0, t_step=0.02, n_t=451)
    np.testing.assert_array_equal(T2, 2 * T)
    np.testing.assert_array_equal(e2, e)


def test_sts_fit_each_choice_is_the_grid_minimum(oracle_mod):
    # with T_1..T_{k-1} frozen, no grid temperature at k beats T_k; each candidate's
    # ECE is the oracle's ECE of the explicitly formed product.  Run once frozen at
    # the fit's own choices and once at other temperatures (T_fixed).
    z, acc = synth.calibration_set(800, 4, seed=4)
    grid = 0.5 + 0.01 * np.arange(451)
    T_own, _ = oracle_mod.sts_fit(z, acc)
    for fixed in (None, T_own[::-1].copy() + 0.3):
        T, e, G = oracle_mod.sts_fit(z, acc, T_fixed=fixed, return_grid=True)
        frozen = T if fixed is None else fixed
        P = np.ones(800)
        for k in range(4):
            eces = [oracle_mod.ece(P * special.expit(z[:, k].astype(np.float64) / t), acc, k + 1)
                    for t in grid]
            i = int(np.argmin(eces))
            assert T[k] == grid[i] and e[k] == pytest.approx(eces[i], abs=1e-15)
            np.testing.assert_allclose(G[k], eces, rtol=0, atol=1e-15)
            P = P * special.expit(z[:, k].astype(np.float64) / frozen[k])
        if fixed is not None:
            assert not np.array_equal(T[1:], T_own[1:])     # the frozen prefix matters


def test_sts_fit_recovers_the_true_temperature(oracle_mod):
    # labels drawn from an exactly logistic survival chain with known T*: the
    # fitted temperatures converge to T* as the calibration set grows
    rng = np.random.default_rng(7)
    N, Tstar = 60000, np.array([1.5, 2.4, 3.3])
    z = rng.normal(2.5, 2.5, (N, 3)).astype(np.float32)
    ok = rng.random((N, 3)) < special.expit(z.astype(np.float64) / Tstar)
    acc = np.where(ok.all(axis=1), 3, np.argmin(ok, axis=1)).astype(np.int32)
    T, e = oracle_mod.sts_fit(z, acc)
    np.testing.assert_allclose(T, Tstar, atol=0.2)
    assert (e < 0.01).all()


def test_sts_fit_rejects_bad_arguments(oracle_mod):
    z, acc = _two_group_calibration()
    with pytest.raises(ValueError):
        oracle_mod.sts_fit(z, acc, t_min=0.0)
    with pytest.raises(ValueError):
        oracle_mod.sts_fit(z, acc, n_bins=0)


# ---------------------------------------------------------------------------
# RNN head (gdymind.com "DSpark", section 4, second instantiation of the sequential
# block: a recurrent state over the block's prefix).  No equations on the pages: the
# Elman reading s_k = tanh(W1[x_{k-1}] + s_{k-1} Whh), bias = bf16(s_k) W2 is pinned
# only by its special cases (parity unpinned against the pages).
# ---------------------------------------------------------------------------
def _rnn_inputs(nb, gamma, V, r, seed, whh_std):
    U, anchor, W1, W2 = _tiny_draft_inputs(nb, gamma, V, r, 0.5, seed=seed)
    rng = np.random.default_rng(seed + 1)
    Whh = _bf16(rng.normal(0, whh_std, (r, r)))
    return U, anchor, W1, W2, Whh


@pytest.mark.parametrize("mode", [0, 1])
def test_rnn_without_recurrence_is_a_markov_head_on_tanh_table(oracle_mod, mode):
    # Whh = 0: s_k = tanh(W1[x_{k-1}]), so the RNN head drafts exactly like the Markov
    # head whose table is bf16(fp32(tanh(W1)))
    V, r, gamma, nb = 300, 16, 6, 4
    U, anchor, W1, W2, _ = _rnn_inputs(nb, gamma, V, r, 5, 0.0)
    Z = np.zeros((r, r), np.uint16)
    W1t = synth.f32_to_bf16_bits(np.tanh(_f(W1)).astype(np.float32))
    x_r, l_r, g_r = oracle_mod.draft_rnn(U, anchor, W1, W2, Z, mode=mode, tau=0.8, seed=3)
    x_m, l_m, g_m = oracle_mod.draft(U, anchor, W1t, W2, mode=mode, tau=0.8, seed=3)
    np.testing.assert_array_equal(x_r, x_m)
    np.testing.assert_array_equal(l_r, l_m)
    np.testing.assert_array_equal(g_r, g_m)


def test_rnn_state_carries_the_prefix_beyond_the_last_token(oracle_mod):
    # two requests with different anchors are forced to the same x_1 by a large base
    # logit; at position 2 the Markov head (Whh = 0) then sees identical inputs, the RNN
    # head does not: its state still holds the anchor
    V, r, gamma = 64, 8, 2
    U, _, W1, W2, Whh = _rnn_inputs(2, gamma, V, r, 9, 0.8)
    Uf = np.zeros((2, gamma, V), np.float32)
    Uf[:, 0, 7] = 50.0                                  # x_1 = 7 for both requests
    U = synth.f32_to_bf16_bits(Uf)
    anchor = np.array([3, 40], np.int32)
    Z = np.zeros((r, r), np.uint16)
    x0, l0, _ = oracle_mod.draft_rnn(U, anchor, W1, W2, Z)
    x1, l1, _ = oracle_mod.draft_rnn(U, anchor, W1, W2, Whh)
    assert (x0[:, 0] == 7).all() and (x1[:, 0] == 7).all()
    assert x0[0, 1] == x0[1, 1] and l0[0, 1] == l0[1, 1]           # Markov: no memory
    assert l1[0, 1] != l1[1, 1]                                    # RNN: the anchor persists


def test_rnn_rejects_bad_anchor(oracle_mod):
    U, anchor, W1, W2, Whh = _rnn_inputs(2, 3, 50, 4, 1, 0.1)
    anchor[1] = 50
    with pytest.raises(ValueError):
        oracle_mod.draft_rnn(U, anchor, W1, W2, Whh)


def test_rnn_without_projection_drafts_the_backbone_argmax(oracle_mod):
    # W2 = 0: no bias at all, whatever the state; the draft is the argmax of U per position
    V, r, gamma, nb = 200, 8, 5, 3
    U, anchor, W1, W2, Whh = _rnn_inputs(nb, gamma, V, r, 12, 0.5)
    x, l, _ = oracle_mod.draft_rnn(U, anchor, W1, np.zeros_like(W2), Whh)
    np.testing.assert_array_equal(x, np.argmax(_f(U), axis=2))
    np.testing.assert_array_equal(l, np.max(_f(U), axis=2))


def test_rnn_gumbel_at_low_temperature_is_greedy(oracle_mod):
    # tau -> 0: l / tau dominates the bounded noise, so Gumbel-max selects the argmax
    V, r, gamma, nb = 300, 8, 4, 3
    U, anchor, W1, W2, Whh = _rnn_inputs(nb, gamma, V, r, 13, 0.3)
    xg, _, _ = oracle_mod.draft_rnn(U, anchor, W1, W2, Whh)
    xs, _, _ = oracle_mod.draft_rnn(U, anchor, W1, W2, Whh, mode=1, tau=1e-6, seed=4)
    np.testing.assert_array_equal(xs, xg)


def test_rnn_recurrence_is_row_vector_times_whh(oracle_mod):
    # Hand-computed two-position case that fixes the orientation of the recurrence,
    # s_k[j] = tanh(W1[x_{k-1}][j] + sum_q s_{k-1}[q] Whh[q][j]).  Whh has one entry,
    # Whh[1][2] = a; W2 is the identity on the first r tokens, so the bias at token
    # v < r is bf16(s_k[v]).
    #   position 1: s_1 = tanh(W1[anchor]) = (0, tanh 1, 0, 0); U forces x_1 = 10.
    #   position 2: W1[10] = 0, so s_2 = tanh(s_1 Whh) = (0, 0, tanh(a tanh 1), 0) and
    #   U = 0 on tokens < r (-100 elsewhere): x_2 = 2 with logit bf16(tanh(a tanh 1)).
    # The transposed reading (Whh s) would give s_2 = tanh(a s_1[2]) e_1 = 0, x_2 = 0.
    V, r, a = 64, 4, 0.5
    W1 = np.zeros((V, r), np.float32)
    anchor_tok = 20
    W1[anchor_tok, 1] = 1.0
    W2 = np.zeros((r, V), np.float32)
    W2[np.arange(r), np.arange(r)] = 1.0
    Whh = np.zeros((r, r), np.float32)
    Whh[1, 2] = a
    Uf = np.full((1, 2, V), -100.0, np.float32)
    Uf[0, 0, 10] = 50.0
    Uf[0, 1, :r] = 0.0
    x, l, g = oracle_mod.draft_rnn(_bf16(Uf), np.array([anchor_tok], np.int32), _bf16(W1),
                                   _bf16(W2), _bf16(Whh))
    s2 = math.tanh(a * math.tanh(1.0))
    expect = float(_f(_bf16([s2]))[0])
    assert x[0, 0] == 10 and l[0, 0] == 50.0
    assert x[0, 1] == 2
    assert l[0, 1] == expect
    assert g[0, 1] == expect          # every other token of the first r has logit 0


def test_rnn_forced_on_its_own_tokens_is_the_free_running_draft(oracle_mod):
    V, r, gamma, nb = 300, 8, 6, 3
    U, anchor, W1, W2, Whh = _rnn_inputs(nb, gamma, V, r, 14, 0.4)
    x, l, g = oracle_mod.draft_rnn(U, anchor, W1, W2, Whh, mode=1, tau=0.9, seed=2)
    prev = np.concatenate([anchor[:, None], x[:, :-1]], axis=1)
    xf, lf, gf = oracle_mod.draft_rnn(U, anchor, W1, W2, Whh, mode=1, tau=0.9, seed=2,
                                      forced_prev=prev)
    np.testing.assert_array_equal(xf, x)
    np.testing.assert_array_equal(lf, l)
    np.testing.assert_array_equal(gf, g)
