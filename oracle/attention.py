"""Decode attention over one KV head's cache (oracle).

Test infrastructure: only tests/, the smoke check and the CPU-baseline legs of
bench.py import this module.

The CONF-KV abstract pairs the eviction policy with blockwise online-softmax
attention. Blockwise evaluation is a way to compute the ordinary softmax
attention of one new query over the cache, so the oracle computes that result
directly with a two-pass softmax in fp64:

    s_j   = (q . k_hat_j) / sqrt(D)
    w_j   = exp(s_j - max s) / sum_i exp(s_i - max s)
    out   = sum_j w_j v_hat_j
    lse   = max s + ln sum_j exp(s_j - max s)

The scale 1/sqrt(D) is the standard one; the pages do not state it. k_hat and
v_hat are the stored rows: fp16 rows widened exactly, INT8 rows dequantised as
float(code) * scale in fp32 (so quantisation error is not charged to the
attention kernel). The G query heads of a GQA group share one KV head; query
head h reads KV head h // G.

Pins (tests/test_oracle_attention.py): one cached token gives out = v_hat;
equal keys give the mean of v_hat; one dominant score gives that token's
v_hat; GQA equals MHA with the KV head replicated;
torch.nn.functional.scaled_dot_product_attention in fp64 on random inputs;
the weights sum to 1 and lse equals log-sum-exp of the scores.
"""
from __future__ import annotations

import math

import numpy as np


def attend(q, k_hat, v_hat):
    """Attention of G query rows over n cached rows, in fp64.

    q: [G, D] (any float dtype; widened exactly), k_hat, v_hat: [n, D] float.
    Returns (out [G, D], lse [G], w [G, n]) as float64, where w are the
    normalised attention probabilities.
    """
    q = np.asarray(q).astype(np.float64)
    k = np.asarray(k_hat).astype(np.float64)
    v = np.asarray(v_hat).astype(np.float64)
    G, D = q.shape
    n = k.shape[0]
    if n == 0:
        raise ValueError("attention over an empty cache")
    s = (q @ k.T) / math.sqrt(D)                 # [G, n]
    m = s.max(axis=1, keepdims=True)             # first pass: row maxima
    e = np.exp(s - m)                            # second pass
    Z = e.sum(axis=1, keepdims=True)
    w = e / Z
    out = w @ v
    lse = m[:, 0] + np.log(Z[:, 0])
    return out, lse, w
