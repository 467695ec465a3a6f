"""Attention-mass EMA, recency, composite score and victim selection (oracle).

Test infrastructure: only tests/, the smoke check and the CPU-baseline legs of
bench.py import this module.

Sources and readings:

* CONF-KV post, method paragraph and decode-loop pseudo-code: every layer
  updates an exponential moving average of the attention mass each token
  receives, ranks tokens by alpha * EMA + (1 - alpha) * recency, and, only
  when its length exceeds the budget, evicts the lowest-ranked tokens while
  the most recent P tokens are never evicted.
* KVpop summary, section 2.1: the first s tokens (sinks) are always kept, the
  w most recent are protected, and the remaining k = B - s - w slots go to the
  highest static priorities. Section 2.4: at inference the k long-range slots
  are maintained with a running threshold over static priorities; for one new
  token per step that is the same select with one victim.

Readings where the pages are silent:

* EMA: ema <- beta * ema + (1 - beta) * a, where a is the token's normalised
  attention probability this step averaged over the G query heads of its KV
  group. New tokens start at 0 and receive their first update in the step they
  arrive. The oracle forms a in fp64 and rounds every update to fp32.
* Recency: rec = float32(pos + 1) / float32(t + 1) (IEEE fp32 division), where
  t is the newest position; the newest token has recency 1.
* Score: fl32(fl32(alpha * ema) + fl32(fl32(1 - alpha) * rec)), no fused
  multiply-add. Fixed-budget mode ranks by the static priority instead.
* Order: the higher (score, position) pair is kept, so equal scores go to the
  newer token. Protected tokens (age t - pos < P, or pos < n_sink) never
  compete.
* Ranker variants (the matched-rate ablation of the hot-path plan): the EMA
  above; the attention mass accumulated over the steps, acc <- acc + a (the
  heavy-hitter score of H2O, which the CONF-KV post lists as related work);
  and a static uniform draw per token. The draw is SplitMix64 (Steele, Lea and
  Flood, 2014, "Fast splittable pseudorandom number generators") used as a
  counter-based generator: the output for state seed + (c + 1) * gamma with
  c = pos | h << 32 | b << 40 | l << 52 (position, KV head, sequence, layer),
  gamma = 0x9E3779B97F4A7C15, and the value (output >> 40) * 2^-24.

Pins (tests/test_oracle_policy.py): constant attention for n steps from zero
gives a (1 - beta^n); exhaustive subset enumeration for n <= 12 equals the
full sort; the length after eviction is min(len, budget); the last P and the
sinks survive; alpha = 0 keeps exactly the most recent tokens (a sliding
window); priority = position in the fixed mode gives the sinks plus the most
recent B - s tokens (the StreamingLLM layout the KVpop summary compares with).
"""
from __future__ import annotations

import numpy as np


def ema_update(ema, w, beta):
    """New EMA after one step.

    ema: fp32 [n]; w: attention probabilities [G, n] (fp64) for the G query
    heads of the group; beta: decay (its fp32 value is used exactly).
    a = mean over the G heads of w; result = fp32(beta * ema + (1 - beta) * a)
    evaluated in fp64.
    """
    beta = float(np.float32(beta))
    a = np.asarray(w, dtype=np.float64).mean(axis=0)
    new = beta * np.asarray(ema, dtype=np.float32).astype(np.float64) + (1.0 - beta) * a
    return new.astype(np.float32)


def accum_update(acc, w):
    """Accumulated attention after one step: fp32(acc + a), a the mean over the
    G heads of w [G, n] (fp64), acc fp32 [n]."""
    a = np.asarray(w, dtype=np.float64).mean(axis=0)
    return (np.asarray(acc, dtype=np.float32).astype(np.float64) + a).astype(np.float32)


_M64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15


def splitmix64_output(state):
    """The SplitMix64 output for a generator state (after its increment)."""
    z = state & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def random_priority(seed, layer, seq, kv_head, pos):
    """Static draw in [0, 1) for token pos of segment (layer, seq, kv_head)."""
    ctr = (int(pos) & 0xFFFFFFFF) | ((int(kv_head) & 0xFF) << 32) | ((int(seq) & 0xFFF) << 40) \
        | ((int(layer) & 0xFFF) << 52)
    out = splitmix64_output(int(seed) + (ctr + 1) * _GAMMA)
    return np.float32((out >> 40) / float(1 << 24))


def recency(pos, t):
    """fp32 (pos + 1) / (t + 1) for positions pos at newest position t."""
    pos = np.asarray(pos, dtype=np.int64)
    return (pos + 1).astype(np.float32) / np.float32(t + 1)


def composite_score(ema, rec, alpha):
    """fp32 alpha * ema + (1 - alpha) * rec, each product rounded, no FMA."""
    a = np.float32(alpha)
    one_minus = np.float32(np.float32(1.0) - a)
    left = (a * np.asarray(ema, dtype=np.float32)).astype(np.float32)
    right = (one_minus * np.asarray(rec, dtype=np.float32)).astype(np.float32)
    return (left + right).astype(np.float32)


def protected_mask(pos, t, protect_last, n_sink):
    """Tokens that may not be evicted: age t - pos < P, or pos < n_sink."""
    pos = np.asarray(pos, dtype=np.int64)
    return ((t - pos) < protect_last) | (pos < n_sink)


def select_victims(pos, score, t, budget_eff, protect_last, n_sink):
    """Boolean mask of the tokens to evict, by a full sort.

    If the segment holds n > budget_eff tokens, the unprotected tokens are
    sorted by (score, position) descending and the first
    budget_eff - |protected| of them are kept; the rest are evicted.
    Otherwise nothing is evicted. Requires budget_eff >= |protected|.
    """
    pos = np.asarray(pos, dtype=np.int64)
    score = np.asarray(score, dtype=np.float32)
    n = pos.size
    evict = np.zeros(n, dtype=bool)
    if n <= budget_eff:
        return evict
    prot = protected_mask(pos, t, protect_last, n_sink)
    n_prot = int(prot.sum())
    if n_prot > budget_eff:
        raise ValueError("more protected tokens than the budget allows")
    cand = np.flatnonzero(~prot)
    # descending by (score, pos): lexsort sorts ascending with the last key primary
    order = np.lexsort((pos[cand], score[cand]))[::-1]
    keep_n = budget_eff - n_prot
    evict[cand[order[keep_n:]]] = True
    return evict
