"""Pins for the oracle's decode attention (CPU only).

Special cases with exact answers, GQA/MHA equivalence, and the library routine
torch.nn.functional.scaled_dot_product_attention evaluated in fp64.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attend


def pin_single_token(att=attend):
    rng = np.random.default_rng(0)
    q = rng.standard_normal((4, 64))
    k = rng.standard_normal((1, 64))
    v = rng.standard_normal((1, 64))
    out, lse, w = att(q, k, v)
    assert np.allclose(out, np.repeat(v, 4, 0), atol=0, rtol=1e-15)
    assert np.allclose(w, 1.0)
    assert np.allclose(lse, (q @ k.T)[:, 0] / 8.0, rtol=1e-14)


def pin_equal_keys_mean(att=attend):
    rng = np.random.default_rng(1)
    q = rng.standard_normal((2, 128))
    k = np.repeat(rng.standard_normal((1, 128)), 50, 0)
    v = rng.standard_normal((50, 128))
    out, lse, _ = att(q, k, v)
    assert np.allclose(out, np.repeat(v.mean(0, keepdims=True), 2, 0), atol=1e-13)
    s0 = (q @ k[0]) / math.sqrt(128)
    assert np.allclose(lse, s0 + math.log(50), atol=1e-12)


def pin_dominant_score(att=attend):
    rng = np.random.default_rng(2)
    D = 64
    k = rng.standard_normal((30, D)) * 0.01
    k[17] = 0
    k[17][3] = 1000.0
    q = np.zeros((1, D))
    q[0][3] = 1.0
    v = rng.standard_normal((30, D))
    out, _, w = att(q, k, v)
    assert abs(w[0, 17] - 1.0) < 1e-12
    assert np.allclose(out[0], v[17], atol=1e-10)


def pin_sdpa(att=attend):
    rng = np.random.default_rng(3)
    for G, D, n in ((1, 64, 7), (4, 128, 300), (5, 128, 1025), (8, 64, 33)):
        q = rng.standard_normal((G, D)) * 2
        k = rng.standard_normal((n, D))
        v = rng.standard_normal((n, D))
        out, lse, w = att(q, k, v)
        tq = torch.tensor(q)[None, :, None, :]
        tk = torch.tensor(k)[None, None].expand(1, G, n, D)
        tv = torch.tensor(v)[None, None].expand(1, G, n, D)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0, :, 0].numpy()
        assert np.abs(out - ref).max() < 1e-12
        s = (q @ k.T) / math.sqrt(D)
        ref_lse = torch.logsumexp(torch.tensor(s), dim=1).numpy()
        assert np.abs(lse - ref_lse).max() < 1e-12
        assert np.allclose(w.sum(1), 1.0, atol=1e-14)


def pin_gqa_equals_replicated(att=attend):
    rng = np.random.default_rng(4)
    G, D, n = 4, 128, 64
    q = rng.standard_normal((G, D))
    k = rng.standard_normal((n, D))
    v = rng.standard_normal((n, D))
    out, lse, _ = att(q, k, v)
    for g in range(G):
        o1, l1, _ = att(q[g:g + 1], k, v)
        assert np.allclose(out[g], o1[0], atol=1e-14)
        assert abs(lse[g] - l1[0]) < 1e-13


ALL_PINS = [pin_single_token, pin_equal_keys_mean, pin_dominant_score, pin_sdpa,
            pin_gqa_equals_replicated]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_attention_pins(pin):
    pin()


def _mutant(kind):
    def att(q, k, v):
        q = np.asarray(q, np.float64)
        k = np.asarray(k, np.float64)
        v = np.asarray(v, np.float64)
        D = q.shape[1]
        s = q @ k.T
        if kind != "no_scale":
            s = s / (D if kind == "scale_D" else math.sqrt(D))
        m = s.max(1, keepdims=True)
        e = np.exp(s - m)
        Z = e.sum(1, keepdims=True)
        w = e / Z
        out = (w @ k) if kind == "keys_as_values" else (w @ v)
        lse = m[:, 0] + np.log(Z[:, 0])
        if kind == "lse_no_max":
            lse = np.log(Z[:, 0])
        return out, lse, w
    return att


@pytest.mark.parametrize("kind", ["no_scale", "scale_D", "keys_as_values", "lse_no_max"])
def test_pins_catch_planted_mistakes(kind):
    bad = _mutant(kind)
    caught = 0
    for pin in ALL_PINS:
        try:
            pin(bad)
        except AssertionError:
            caught += 1
    assert caught >= 1, kind


def test_empty_cache_rejected():
    with pytest.raises(ValueError):
        attend(np.zeros((1, 64)), np.zeros((0, 64)), np.zeros((0, 64)))
