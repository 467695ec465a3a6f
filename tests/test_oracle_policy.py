"""Pins for the oracle's EMA, recency, score and victim selection (CPU only).

Selection is checked by exhaustive enumeration of subsets on tiny inputs (the
kept set is the unique subset whose every member outranks every evicted
candidate), against the sliding-window and StreamingLLM special cases, and
against its invariants. fp32 expressions are checked against exact rational
evaluation with IEEE round-to-nearest-even.
"""
import itertools
from fractions import Fraction

import numpy as np
import pytest

from oracle import ema_update, recency, composite_score, select_victims
from oracle.segment import Params, prefill_segment


def _f32(fr: Fraction) -> float:
    lo = np.float32(float(fr))
    cands = [np.nextafter(lo, np.float32(-np.inf)), lo, np.nextafter(lo, np.float32(np.inf))]
    return float(min(cands, key=lambda c: (abs(Fraction(float(c)) - fr),
                                           int(np.float32(c).view(np.uint32)) & 1)))


# ---- EMA ------------------------------------------------------------------

def pin_ema_closed_form(upd=ema_update):
    # constant attention a for n steps from 0 gives a (1 - beta^n)
    beta = 0.9
    b = float(np.float32(beta))
    for a in (0.0, 1e-3, 0.25, 1.0):
        ema = np.zeros(3, np.float32)
        w = np.full((4, 3), a)
        for n in range(1, 60):
            ema = upd(ema, w, beta)
            exact = a * (1 - b ** n)
            assert np.all(np.abs(ema - exact) <= 1e-6 * max(a, 1e-30) + 1e-12), (a, n)


def pin_ema_group_mean(upd=ema_update):
    # the update uses the mean over the G query heads of the group
    w = np.array([[0.1, 0.7], [0.3, 0.1], [0.2, 0.0], [0.4, 0.2]])
    ema = upd(np.zeros(2, np.float32), w, 0.5)
    assert np.allclose(ema, 0.5 * w.mean(0), atol=1e-8)


# ---- recency and score --------------------------------------------------------

def pin_recency_exact(rec=recency):
    rng = np.random.default_rng(0)
    for _ in range(200):
        t = int(rng.integers(0, 200000))
        pos = rng.integers(0, t + 1, size=5)
        got = rec(pos, t)
        for p, g in zip(pos, got):
            assert float(g) == _f32(Fraction(int(p) + 1, t + 1))
    assert rec(np.array([41]), 41)[0] == 1.0


def pin_score_exact(score=composite_score):
    rng = np.random.default_rng(1)
    for _ in range(300):
        alpha = float(np.float32(rng.uniform()))
        e = np.float32(rng.uniform() * 0.01)
        r = np.float32(rng.uniform())
        one_minus = _f32(1 - Fraction(alpha))
        left = _f32(Fraction(alpha) * Fraction(float(e)))
        right = _f32(Fraction(one_minus) * Fraction(float(r)))
        exp = _f32(Fraction(left) + Fraction(right))
        assert float(score(np.array([e]), np.array([r]), alpha)[0]) == exp


# ---- selection ----------------------------------------------------------------

def _brute_force_keep(pos, score, t, budget_eff, P, s):
    """Unique kept set: every kept candidate outranks every evicted one."""
    n = len(pos)
    if n <= budget_eff:
        return set(range(n))
    prot = {i for i in range(n) if t - pos[i] < P or pos[i] < s}
    cand = [i for i in range(n) if i not in prot]
    keep_n = budget_eff - len(prot)
    rank = lambda i: (float(score[i]), int(pos[i]))   # noqa: E731
    found = []
    for sub in itertools.combinations(cand, keep_n):
        rest = [i for i in cand if i not in sub]
        if not sub or not rest or min(rank(i) for i in sub) > max(rank(i) for i in rest):
            found.append(set(sub))
    assert len(found) == 1
    return prot | found[0]


def pin_select_brute_force(sel=select_victims):
    rng = np.random.default_rng(2)
    for trial in range(400):
        n = int(rng.integers(1, 13))
        pos = np.sort(rng.choice(40, size=n, replace=False)).astype(np.int64)
        t = int(pos[-1])
        vals = np.float32(rng.choice([0.1, 0.2, 0.2, 0.5, 0.7], size=n))   # many ties
        P = int(rng.integers(0, 4))
        s = int(rng.integers(0, 3))
        n_prot = int(np.sum((t - pos < P) | (pos < s)))
        budget_eff = int(rng.integers(n_prot, n + 2))
        evict = sel(pos, vals, t, budget_eff, P, s)
        keep = set(np.flatnonzero(~evict).tolist())
        assert keep == _brute_force_keep(pos, vals, t, budget_eff, P, s), trial


def pin_select_invariants(sel=select_victims):
    rng = np.random.default_rng(3)
    for trial in range(200):
        n = int(rng.integers(1, 400))
        pos = np.sort(rng.choice(2000, size=n, replace=False)).astype(np.int64)
        t = int(pos[-1]) + int(rng.integers(0, 3))
        vals = np.float32(rng.uniform(size=n))
        P = int(rng.integers(0, 50))
        s = int(rng.integers(0, 5))
        prot = (t - pos < P) | (pos < s)
        budget_eff = int(prot.sum()) + int(rng.integers(0, n + 1))
        evict = sel(pos, vals, t, budget_eff, P, s)
        assert (~evict).sum() == min(n, budget_eff)
        assert not evict[prot].any()
        kept = ~evict & ~prot
        if kept.any() and evict.any():
            kk = min(zip(vals[kept].tolist(), pos[kept].tolist()))
            ee = max(zip(vals[evict].tolist(), pos[evict].tolist()))
            assert kk > ee


def pin_sliding_window(sel=select_victims, score=composite_score, rec=recency):
    # alpha = 0: the score is recency alone, so the most recent tokens stay
    rng = np.random.default_rng(4)
    for _ in range(50):
        n = int(rng.integers(2, 600))
        pos = np.sort(rng.choice(5000, size=n, replace=False)).astype(np.int64)
        t = int(pos[-1])
        ema = np.float32(rng.uniform(size=n))
        sc = score(ema, rec(pos, t), 0.0)
        budget = int(rng.integers(1, n + 1))
        evict = sel(pos, sc, t, budget, 1, 0)
        kept = pos[~evict]
        assert kept.tolist() == pos[-budget:].tolist()


def pin_streaming_llm_layout(sel=select_victims):
    # fixed mode with priority = position keeps the sinks and the newest B - s
    for T, s, w, B in ((100, 4, 8, 20), (5000, 4, 512, 2048), (30, 0, 3, 10), (12, 4, 4, 20)):
        p = Params(mode="fixed", protect_last=w, n_sink=s, fixed_budget=B, int8=False,
                   fp16_window=1)
        k = np.zeros((T, 8), np.float16)
        seg = prefill_segment(k, k, np.arange(T, dtype=np.float32), p)
        if T <= B:
            assert seg.pos.tolist() == list(range(T))
        else:
            exp = list(range(s)) + list(range(T - (B - s), T))
            assert seg.pos.tolist() == exp


ALL_PINS = [pin_ema_closed_form, pin_ema_group_mean, pin_recency_exact, pin_score_exact,
            pin_select_brute_force, pin_select_invariants, pin_sliding_window,
            pin_streaming_llm_layout]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_policy_pins(pin):
    pin()


def test_select_rejects_overprotected():
    with pytest.raises(ValueError):
        select_victims(np.arange(10), np.zeros(10, np.float32), 9, 3, 5, 0)


# ---- planted mistakes ---------------------------------------------------------

def _sel_mutant(kind):
    def sel(pos, score, t, budget_eff, P, s):
        pos = np.asarray(pos, np.int64)
        score = np.asarray(score, np.float32)
        n = pos.size
        ev = np.zeros(n, bool)
        if n <= budget_eff:
            return ev
        if kind == "protect_off_by_one":
            prot = ((t - pos) <= P) | (pos < s)
        else:
            prot = ((t - pos) < P) | (pos < s)
        cand = np.flatnonzero(~prot)
        if kind == "ties_to_older":
            order = np.lexsort((-pos[cand], score[cand]))[::-1]
        else:
            order = np.lexsort((pos[cand], score[cand]))[::-1]
        keep_n = budget_eff if kind == "ignore_protected_count" else budget_eff - int(prot.sum())
        ev[cand[order[keep_n:]]] = True
        return ev
    return sel


@pytest.mark.parametrize("kind", ["protect_off_by_one", "ties_to_older", "ignore_protected_count"])
def test_select_pins_catch_planted_mistakes(kind):
    bad = _sel_mutant(kind)
    caught = 0
    for pin in (pin_select_brute_force, pin_select_invariants, pin_sliding_window):
        try:
            pin(bad)
        except AssertionError:
            caught += 1
    assert caught >= 1, kind


def test_ema_and_score_pins_catch_planted_mistakes():
    def ema_swapped(ema, w, beta):       # decay applied to the new mass instead
        b = float(np.float32(beta))
        return (b * np.asarray(w).mean(0) + (1 - b) * ema).astype(np.float32)

    def ema_sum(ema, w, beta):           # sum over heads instead of mean
        b = float(np.float32(beta))
        return (b * ema + (1 - b) * np.asarray(w).sum(0)).astype(np.float32)

    def score_fma(ema, rec, alpha):      # one fused expression in fp64
        a = float(np.float32(alpha))
        return (a * np.asarray(ema, np.float64) + (1 - a) * np.asarray(rec, np.float64)).astype(np.float32)

    def rec_pos(pos, t):                 # pos / t instead of (pos+1)/(t+1)
        return np.asarray(pos, np.float32) / np.float32(max(t, 1))

    for bad, pins in ((ema_swapped, [pin_ema_closed_form]), (ema_sum, [pin_ema_group_mean]),
                      (score_fma, [pin_score_exact]), (rec_pos, [pin_recency_exact])):
        caught = 0
        for pin in pins:
            try:
                pin(bad)
            except AssertionError:
                caught += 1
        assert caught >= 1, bad.__name__


# ---------------------------------------------------------------------------
# ranker variants: accumulated attention and the static random draw
# ---------------------------------------------------------------------------
import os  # noqa: E402

from oracle.policy import accum_update, random_priority, splitmix64_output  # noqa: E402

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_accum_constant_attention_closed_form():
    # constant attention a = 1/4 on every head for n steps from zero accumulates
    # to n/4 exactly (dyadic values: every fp32 sum is exact)
    acc = np.zeros(5, np.float32)
    w = np.full((4, 5), 0.25)
    for n in range(1, 41):
        acc = accum_update(acc, w)
        assert np.all(acc == np.float32(n / 4))


def test_accum_is_the_running_sum_of_head_means():
    rng = np.random.default_rng(3)
    steps = [rng.random((3, 7)) for _ in range(6)]
    acc = np.zeros(7, np.float32)
    total = np.zeros(7)
    for w in steps:
        acc = accum_update(acc, w)
        total += w.mean(axis=0)
    np.testing.assert_allclose(acc, total, rtol=3e-7 * 6)


def test_splitmix64_reference_outputs():
    lines = open(os.path.join(GOLDEN, "splitmix64_seed0.txt")).read().splitlines()
    want = [int(x, 16) for x in lines if x.strip() and not x.startswith("#")]
    gamma = 0x9E3779B97F4A7C15
    got = [splitmix64_output((k * gamma) & ((1 << 64) - 1)) for k in range(1, 6)]
    assert got == want


def test_random_priority_range_determinism_and_uniformity():
    u = np.array([random_priority(9, 3, 1, 2, p) for p in range(20000)], np.float64)
    assert np.all((u >= 0.0) & (u < 1.0))
    assert np.all(np.float32(u) == u)   # 24-bit fractions: exact in fp32
    assert random_priority(9, 3, 1, 2, 17) == random_priority(9, 3, 1, 2, 17)
    # chi-square over 32 equal bins (31 degrees of freedom; 70 is far in the tail)
    counts = np.bincount(np.minimum((u * 32).astype(int), 31), minlength=32)
    chi2 = float(((counts - len(u) / 32) ** 2 / (len(u) / 32)).sum())
    assert chi2 < 70.0, chi2
    # different segments and seeds give unrelated draws
    v = np.array([random_priority(9, 3, 1, 3, p) for p in range(20000)])
    s2 = np.array([random_priority(10, 3, 1, 2, p) for p in range(20000)])
    assert abs(np.corrcoef(u, v)[0, 1]) < 0.03 and abs(np.corrcoef(u, s2)[0, 1]) < 0.03


def test_random_ranker_segment_uses_its_draws():
    # a prefilled segment under the random ranker carries the draws of its own
    # (layer, seq, kv_head) as its score source
    p = Params(score_source="random", seed=5, fp16_window=4)
    k = np.zeros((12, 8), np.float16)
    seg = prefill_segment(k, k, None, p, (2, 1, 3))
    assert np.array_equal(seg.score_src, np.array([random_priority(5, 2, 1, 3, i) for i in range(12)], np.float32))
