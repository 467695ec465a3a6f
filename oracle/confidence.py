"""Confidence score, budget gate and pyramidal per-layer budgets (oracle).

Test infrastructure: only tests/, the smoke check and the CPU-baseline legs of
bench.py import this module.

What is computed, restated from the sources:

* CONF-KV post, method paragraphs and decode-loop pseudo-code: the next-token
  distribution p = softmax(logits) (temperature 1) is turned into one scalar
  that mixes three signals. With weight 0.4 enters one minus the entropy of p
  normalised by its maximum ln V; with weight 0.3 the logistic sigmoid of the
  gap between the two largest log-probabilities; with weight 0.3 the largest
  probability.
* CONF-KV abstract, and the CONF-KV post's method paragraph and its
  Needle-in-a-Haystack note: a confident step gets the tight budget and an
  uncertain step the loose one. The pseudo-code line of the same post writes
  the opposite polarity (N_high when c >= tau). Both are offered: "prose"
  (default) and "literal".
* CONF-KV abstract and post ("pyramidal variant", after PyramidKV): deeper
  layers get smaller budgets. The ramp is linear from 2N at layer 0 to N/2 at
  the last layer, floored in exact integer arithmetic.

Pins (tests/test_oracle_confidence.py): uniform logits give c = 0.15 + 0.3/V;
two-level logits give a closed form; a one-hot limit gives c -> 1; shift and
permutation invariance; scipy.stats.entropy for H; a tied maximum gives a zero
margin; the one-pass (m, S, T) identity used by the GPU kernel agrees with the
direct entropy to 1e-12; gate boundary cases; pyramid endpoints and
monotonicity.
"""
from __future__ import annotations

import math

import numpy as np

W_ENTROPY = 0.4   # weight of (1 - normalised entropy)
W_MARGIN = 0.3    # weight of sigmoid(top-two log-prob gap)
W_TOP = 0.3       # weight of the top probability


def confidence(logits) -> dict:
    """Confidence of one next-token distribution, in fp64.

    Follows the CONF-KV post's pseudo-code: p = softmax(logits), then
    c = 0.4 (1 - H(p)/ln V) + 0.3 sigmoid(log p_(1) - log p_(2)) + 0.3 max p.

    The entropy is taken directly as -sum p ln p over the nonzero p (zero
    probabilities contribute nothing). The margin is the difference of the two
    largest log-probabilities counted with multiplicity, so a tied maximum gives
    a margin of 0. Requires finite logits and V >= 2.
    """
    l = np.asarray(logits, dtype=np.float64).ravel()
    V = l.size
    if V < 2:
        raise ValueError("vocabulary must hold at least two tokens")
    if not np.all(np.isfinite(l)):
        raise ValueError("logits must be finite")
    # log-softmax, then probabilities
    m = l.max()
    log_Z = m + math.log(np.sum(np.exp(l - m)))
    logp = l - log_Z
    p = np.exp(logp)
    nz = p > 0.0
    H = float(-np.sum(p[nz] * logp[nz]))
    norm_entropy = H / math.log(V)
    top2 = np.sort(logp)[-2:]            # ascending: [second, first]
    margin = float(top2[1] - top2[0])
    sig = 1.0 / (1.0 + math.exp(-margin))
    p_max = float(p.max())
    c = W_ENTROPY * (1.0 - norm_entropy) + W_MARGIN * sig + W_TOP * p_max
    return {"c": c, "H": H, "norm_entropy": norm_entropy, "margin": margin,
            "sigmoid_margin": sig, "p_max": p_max}


def choose_budget(c: float, tau: float, n_low: int, n_high: int,
                  polarity: str = "prose") -> int:
    """Budget gate.

    "prose" (default): confident (c >= tau) -> tight budget n_low, else the
    loose budget n_high, as the CONF-KV abstract and post describe.
    "literal": the pseudo-code line's polarity, n_high when c >= tau.
    The comparison is >= in both, as in the pseudo-code.
    """
    confident = c >= tau
    if polarity == "prose":
        return n_low if confident else n_high
    if polarity == "literal":
        return n_high if confident else n_low
    raise ValueError(f"unknown gate polarity {polarity!r}")


def layer_budgets(N: int, layers: int, pyramidal: bool) -> list[int]:
    """Per-layer budgets for one sequence.

    Without the pyramid every layer gets N. With it, layer l of L gets
    floor(N * (4(L-1) - 3l) / (2(L-1))): 2N at l = 0 falling linearly to
    floor(N/2) at l = L-1 (exact integer arithmetic). A single layer gets N.
    """
    if not pyramidal or layers == 1:
        return [int(N)] * layers
    L1 = layers - 1
    return [(int(N) * (4 * L1 - 3 * l)) // (2 * L1) for l in range(layers)]


def confidence_batch(logits, tau: float, n_low: int, n_high: int, layers: int,
                     pyramidal: bool, polarity: str = "prose"):
    """Per-sequence confidence, budget and per-layer budgets for logits [B, V].

    Each sequence has its own confidence and budget (one budget for all its
    layers and KV heads, or its pyramid).
    Returns (c [B] float64, budget [B] int, budgets [B, layers] int).
    """
    logits = np.asarray(logits)
    B = logits.shape[0]
    c = np.empty(B, dtype=np.float64)
    budget = np.empty(B, dtype=np.int64)
    per_layer = np.empty((B, layers), dtype=np.int64)
    for b in range(B):
        c[b] = confidence(logits[b])["c"]
        budget[b] = choose_budget(c[b], tau, n_low, n_high, polarity)
        per_layer[b] = layer_budgets(int(budget[b]), layers, pyramidal)
    return c, budget, per_layer
