"""Pins for the oracle's confidence, gate and pyramid (CPU only).

Each check compares the oracle with something other than itself: exact closed
forms, hand-derived golden values, scipy's entropy, the one-pass (m, S, T)
identity, invariances the definition implies, and boundary cases of the gate
and the pyramid. The last test plants plausible mistakes in copies of the
oracle function and shows that at least one pin catches each.
"""
import math
import os

import numpy as np
import pytest
import scipy.stats

from oracle import confidence, choose_budget, layer_budgets

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    rows = []
    with open(os.path.join(HERE, "golden", "confidence_closed_forms.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, V, spec, expected, _ = [x.strip() for x in line.split("|")]
            V = int(V)
            parts = [p.strip() for p in spec.split(";")]
            default = float(parts[0].split("=")[1])
            logits = np.full(V, default)
            for p in parts[1:]:
                i, val = p.split(":")
                logits[int(i)] = float(val)
            rows.append((name, logits, float(expected)))
    return rows


# ---- pins, written against an injectable implementation -------------------

def pin_golden(conf=confidence):
    for name, logits, expected in _golden():
        got = conf(logits)["c"]
        assert abs(got - expected) < 1e-12, (name, got, expected)


def pin_uniform(conf=confidence):
    for V in (2, 3, 1024, 50257, 128256):
        got = conf(np.zeros(V))["c"]
        assert abs(got - (0.15 + 0.3 / V)) < 1e-12, (V, got)


def pin_two_level(conf=confidence):
    # one token at logit a, V-1 tokens at 0: every term has a closed form
    for V in (2, 10, 1000, 152064):
        for a in (0.5, 3.0, 12.0):
            l = np.zeros(V)
            l[V // 3] = a
            Z = math.exp(a) + (V - 1)
            p1 = math.exp(a) / Z
            p0 = 1.0 / Z
            H = -(p1 * math.log(p1) + (V - 1) * p0 * math.log(p0))
            margin = a if V > 1 else 0.0
            c = 0.4 * (1 - H / math.log(V)) + 0.3 / (1 + math.exp(-margin)) + 0.3 * p1
            r = conf(l)
            assert abs(r["H"] - H) < 1e-10 * max(1.0, H), (V, a)
            assert abs(r["margin"] - margin) < 1e-9, (V, a)
            assert abs(r["c"] - c) < 1e-12, (V, a, r["c"], c)


def pin_one_hot_limit(conf=confidence):
    for V in (2, 1024, 128256):
        l = np.zeros(V)
        l[7 % V] = 400.0
        assert abs(conf(l)["c"] - 1.0) < 1e-12


def pin_scipy_entropy(conf=confidence):
    rng = np.random.default_rng(1)
    for V in (2, 17, 4096):
        for s in (0.5, 8.0):
            l = rng.standard_normal(V) * s
            p = np.exp(l - l.max())
            p /= p.sum()
            r = conf(l)
            assert abs(r["H"] - scipy.stats.entropy(p)) < 1e-10
            assert abs(r["p_max"] - p.max()) < 1e-14
            top = np.sort(np.log(p))
            assert abs(r["margin"] - (top[-1] - top[-2])) < 1e-9


def pin_invariances(conf=confidence):
    rng = np.random.default_rng(2)
    l = rng.standard_normal(3000) * 4
    c0 = conf(l)["c"]
    assert abs(conf(l + 123.25)["c"] - c0) < 1e-12            # shift
    assert abs(conf(rng.permutation(l))["c"] - c0) < 1e-12     # permutation
    assert 0.0 < c0 <= 1.0


def pin_tied_maximum(conf=confidence):
    l = np.array([1.0, 5.0, 5.0, -2.0])
    r = conf(l)
    assert r["margin"] == 0.0
    assert r["sigmoid_margin"] == 0.5


def pin_one_pass_identity(conf=confidence):
    # H = ln S - T/S with S = sum e^{l-m}, T = sum e^{l-m}(l-m): the identity the
    # GPU reduction uses, checked against the oracle's direct -sum p ln p
    rng = np.random.default_rng(3)
    for V in (2, 100, 50257):
        for s in (0.5, 8.0, 30.0):
            l = rng.standard_normal(V) * s
            m = l.max()
            e = np.exp(l - m)
            S = e.sum()
            T = (e * (l - m)).sum()
            H1 = math.log(S) - T / S
            assert abs(conf(l)["H"] - H1) < 1e-12 * max(1.0, H1) * math.log(V) * 10


ALL_PINS = [pin_golden, pin_uniform, pin_two_level, pin_one_hot_limit, pin_scipy_entropy,
            pin_invariances, pin_tied_maximum, pin_one_pass_identity]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_confidence_pins(pin):
    pin()


def test_gate_boundaries():
    # c == tau takes the >= branch in both polarities
    assert choose_budget(0.6, 0.6, 256, 512, "prose") == 256
    assert choose_budget(0.6, 0.6, 256, 512, "literal") == 512
    assert choose_budget(np.nextafter(0.6, 0), 0.6, 256, 512, "prose") == 512
    assert choose_budget(np.nextafter(0.6, 0), 0.6, 256, 512, "literal") == 256
    with pytest.raises(ValueError):
        choose_budget(0.5, 0.6, 1, 2, "other")


def test_pyramid_endpoints_and_monotone():
    for L in (2, 3, 12, 32, 36, 64):
        for N in (1, 5, 256, 512, 1023, 1024, 2048):
            b = layer_budgets(N, L, True)
            assert b[0] == 2 * N
            assert b[-1] == N // 2
            assert all(b[i] >= b[i + 1] for i in range(L - 1))
            # linear ramp: budget(l) within one of 2N - 1.5 N l / (L-1)
            for l in range(L):
                assert abs(b[l] - (2 * N - 1.5 * N * l / (L - 1))) < 1.0
    assert layer_budgets(700, 1, True) == [700]
    assert layer_budgets(700, 5, False) == [700] * 5
    assert layer_budgets(5, 2, True) == [10, 2]


def test_rejects_bad_input():
    with pytest.raises(ValueError):
        confidence(np.zeros(1))
    with pytest.raises(ValueError):
        confidence(np.array([0.0, np.nan]))


# ---- planted mistakes: each mutant must fail at least one pin ----------------

def _mutant(kind):
    def conf(logits):
        l = np.asarray(logits, dtype=np.float64).ravel()
        V = l.size
        m = l.max()
        log_Z = m + math.log(np.sum(np.exp(l - m)))
        logp = l - log_Z
        p = np.exp(logp)
        nz = p > 0
        H = float(-np.sum(p[nz] * logp[nz]))
        if kind == "log2_entropy":
            H = H / math.log(2)
        if kind == "entropy_sign":
            H = -H
        norm = H / math.log(V)
        if kind == "no_normalise":
            norm = H
        top2 = np.sort(logp)[-2:]
        margin = float(top2[1] - top2[0])
        if kind == "prob_margin":
            top2p = np.sort(p)[-2:]
            margin = float(top2p[1] - top2p[0])
        if kind == "distinct_top2":
            u = np.unique(logp)
            margin = float(u[-1] - u[-2]) if u.size > 1 else 0.0
        sig = 1 / (1 + math.exp(-margin))
        pmax = float(p.max())
        w = (0.4, 0.3, 0.3)
        if kind == "swapped_weights":
            w = (0.3, 0.4, 0.3)
        if kind == "drop_top":
            w = (0.4, 0.3, 0.0)
        c = w[0] * (1 - norm) + w[1] * sig + w[2] * pmax
        return {"c": c, "H": H, "norm_entropy": norm, "margin": margin,
                "sigmoid_margin": sig, "p_max": pmax}
    return conf


@pytest.mark.parametrize("kind", ["log2_entropy", "entropy_sign", "no_normalise", "prob_margin",
                                  "distinct_top2", "swapped_weights", "drop_top"])
def test_pins_catch_planted_mistakes(kind):
    bad = _mutant(kind)
    caught = 0
    for pin in ALL_PINS:
        try:
            pin(bad)
        except AssertionError:
            caught += 1
    assert caught >= 1, kind


def test_unmutated_copy_passes_all_pins():
    good = _mutant("none")
    for pin in ALL_PINS:
        pin(good)
