"""Pins for three readings of the decode loop that no other pin reaches (CPU).

Each expected result below is derived by hand from the reading it pins, with
recency-only ranking (alpha = 0) where a ranking matters, so that the kept set
is a list of positions written out in the test rather than recomputed with
the oracle's own formulas:

* Effective budget below the protected count. The CONF-KV post's decode-loop
  pseudo-code never evicts the last P tokens and the KVpop summary (section
  2.1) always keeps the sinks, so a budget smaller than P + s cannot be met;
  the reading is budget_eff = max(budget, P + s), and the segment keeps
  exactly the sinks and the last P tokens.
* The budget before the first confidence call. The pseudo-code evicts only
  after the confidence of the step has chosen the budget; a caller that evicts
  before ever calling it gets the larger of the two budgets (per layer, under
  the pyramid), and so does every new batch.
* A step whose eviction is skipped. The pseudo-code converts tokens older than
  the W-token window to INT8 inside the eviction step; when a caller skips
  that step, the next append converts the token that has left the window
  (position t + 1 - W at step t + 1), so that attention still sees FP16 rows
  exactly for ages below W.

The last tests plant plausible mistakes in copies of the oracle and check that
each one fails a pin.
"""
import math

import numpy as np
import pytest
import torch

from confidence_gated_kv_logit_b200 import synth
from oracle import quantize_row
from oracle import segment as oseg
from oracle.segment import OracleCache, Params


# ---------------------------------------------------------------------------
# drivers
# ---------------------------------------------------------------------------

def _confident_logits(B, V=64):
    """Logits whose confidence is ~1 (one token 60 above the rest): c >= tau."""
    lg = np.zeros((B, V), np.float32)
    lg[:, 3] = 60.0
    return lg


def _cache(params_cls, L, Hkv, Hq, D, cache_cls=OracleCache, **kw):
    return cache_cls(L, Hkv, Hq, D, params_cls(**kw))


def _prefill_all(cache, L, B, Hkv, T, D, seed):
    g = synth.generator(seed)
    for l in range(L):
        k, v = synth.prefill_kv(B, Hkv, T, D, g)
        cache.prefill(l, k.numpy(), v.numpy(), [T] * B)
    return g


def _decode_all(cache, L, B, Hq, Hkv, D, g):
    for l in range(L):
        q, kn, vn = synth.step_qkv((B,), Hq, Hkv, D, g)
        cache.decode_attn(l, q.numpy(), kn.numpy(), vn.numpy())


# ---------------------------------------------------------------------------
# (1) budget below P + s
# ---------------------------------------------------------------------------

def pin_budget_below_protected(params_cls=Params):
    T, D = 60, 64
    # (n_sink, P, budget, alpha) -> kept positions after the first step (t = 60)
    cases = [
        (4, 16, 10, 0.5, list(range(4)) + list(range(45, 61))),     # clamp: sinks + last 16
        (4, 16, 10, 0.0, list(range(4)) + list(range(45, 61))),
        (0, 16, 10, 0.5, list(range(45, 61))),                      # clamp to P alone when s = 0
        (4, 16, 20, 0.5, list(range(4)) + list(range(45, 61))),     # budget exactly P + s
        (4, 16, 25, 0.0, list(range(4)) + list(range(40, 61))),     # 5 unprotected slots, by recency
        (2, 0, 1, 0.0, [0, 1]),                                     # P = 0: only the sinks stay
    ]
    for s, P, budget, alpha, kept in cases:
        cache = _cache(params_cls, 1, 2, 4, D, n_low=budget, n_high=budget, protect_last=P, n_sink=s,
                       alpha=alpha, fp16_window=8)
        g = _prefill_all(cache, 1, 1, 2, T, D, seed=1)
        _decode_all(cache, 1, 1, 4, 2, D, g)
        cache.confidence(_confident_logits(1))
        cache.evict_compact(0)
        for h in range(2):
            got = cache.segment(0, 0, h).pos.tolist()
            assert got == kept, (s, P, budget, alpha, got[:8], len(got))
        # the next steps stay at the same length: the newest token in, the
        # oldest unprotected token out
        for step in range(1, 4):
            _decode_all(cache, 1, 1, 4, 2, D, g)
            cache.confidence(_confident_logits(1))
            cache.evict_compact(0)
            t = T + step
            if budget <= s + P:
                want = list(range(s)) + list(range(t - P + 1, t + 1))
            else:
                want = list(range(s)) + list(range(t - (budget - s) + 1, t + 1))
            assert cache.segment(0, 0, 0).pos.tolist() == want, (s, P, budget, step)


def test_budget_below_protected_count():
    pin_budget_below_protected()


# ---------------------------------------------------------------------------
# (2) budget before the first confidence call
# ---------------------------------------------------------------------------

def pin_initial_budget(cache_cls=OracleCache):
    D, T = 64, 400
    # pyramid of the larger budget 160 over 3 layers: floor(160 (8 - 3l) / 4)
    cases = [
        (dict(n_low=64, n_high=160, pyramidal=True), 3, [320, 200, 80]),
        (dict(n_low=160, n_high=64, pyramidal=True), 3, [320, 200, 80]),   # larger = n_low here
        (dict(n_low=64, n_high=160, pyramidal=False), 2, [160, 160]),
        (dict(n_low=64, n_high=160, pyramidal=False, gate="literal"), 2, [160, 160]),
    ]
    for kw, L, eff in cases:
        cache = _cache(Params, L, 1, 2, D, cache_cls=cache_cls, protect_last=16, fp16_window=32, alpha=0.0, **kw)
        g = _prefill_all(cache, L, 2, 1, T, D, seed=2)
        _decode_all(cache, L, 2, 2, 1, D, g)          # t = 400, 401 tokens
        for l in range(L):
            cache.evict_compact(l)                     # no confidence call yet
            for b in range(2):
                got = cache.segment(l, b, 0).pos.tolist()
                assert got == list(range(401 - eff[l], 401)), (kw, l, b, len(got))
    # a confident step then picks n_low (prose gate); a new batch starts over at the larger budget
    cache = _cache(Params, 2, 1, 2, D, cache_cls=cache_cls, n_low=64, n_high=160, protect_last=16,
                   fp16_window=32, alpha=0.0)
    g = _prefill_all(cache, 2, 2, 1, T, D, seed=3)
    _decode_all(cache, 2, 2, 2, 1, D, g)
    cache.confidence(_confident_logits(2))
    for l in range(2):
        cache.evict_compact(l)
        assert len(cache.segment(l, 0, 0)) == 64
    g = _prefill_all(cache, 2, 3, 1, T, D, seed=4)    # batch 3: a new batch
    _decode_all(cache, 2, 3, 2, 1, D, g)
    for l in range(2):
        cache.evict_compact(l)
        for b in range(3):
            assert cache.segment(l, b, 0).pos.tolist() == list(range(241, 401)), (l, b)


def test_budget_before_first_confidence_call():
    pin_initial_budget()


# ---------------------------------------------------------------------------
# (3) conversion on append after a skipped eviction
# ---------------------------------------------------------------------------

def _torch_attention(q, seg):
    """Softmax attention of q [G, D] over the segment's stored rows, with
    torch in fp64 (INT8 rows as code * scale in fp32)."""
    k = torch.from_numpy(seg.k16.astype(np.float32))
    v = torch.from_numpy(seg.v16.astype(np.float32))
    i8 = torch.from_numpy(~seg.is_fp16)
    k[i8] = torch.from_numpy(seg.k8[~seg.is_fp16]).float() * torch.from_numpy(seg.ks[~seg.is_fp16])[:, None]
    v[i8] = torch.from_numpy(seg.v8[~seg.is_fp16]).float() * torch.from_numpy(seg.vs[~seg.is_fp16])[:, None]
    qq = torch.from_numpy(np.asarray(q, np.float32)).double()
    w = torch.softmax(qq @ k.double().T / math.sqrt(qq.shape[1]), dim=1)
    return (w @ v.double()).numpy()


def pin_skipped_eviction_conversion(decode=oseg.decode_attn_segment):
    D, G, T, W = 64, 2, 20, 8
    p = Params(n_low=1000, n_high=1000, protect_last=4, fp16_window=W)
    g = synth.generator(5)
    k, v = synth.prefill_kv(1, 1, T, D, g)
    raw = {i: (k[0, 0, i].numpy(), v[0, 0, i].numpy()) for i in range(T)}
    seg = oseg.prefill_segment(k[0, 0].numpy(), v[0, 0].numpy(), None, p)
    assert seg.pos[seg.is_fp16].tolist() == list(range(13, 20))     # positions <= T - W are INT8
    # step t: (evict after it?, FP16 positions while attention runs, positions converted on append)
    plan = [(20, False, range(13, 21), []),
            (21, False, range(14, 22), [13]),      # eviction of step 20 skipped: 13 converts on append
            (22, True, range(15, 23), [14]),       # skipped again: 14; this step evicts (converts 15)
            (23, True, range(16, 24), []),         # nothing left over
            (24, False, range(17, 25), []),
            (25, True, range(18, 26), [17])]
    for t, evict, fp16, converted in plan:
        before = set(seg.pos[~seg.is_fp16].tolist())
        q, kn, vn = synth.step_qkv((1,), G, 1, D, g)
        raw[t] = (kn[0, 0].numpy(), vn[0, 0].numpy())
        out, _, _ = decode(seg, q[0].numpy(), kn[0, 0].numpy(), vn[0, 0].numpy(), None, p)
        assert seg.pos.tolist() == list(range(t + 1)), t
        assert seg.pos[seg.is_fp16].tolist() == list(fp16), (t, seg.pos[seg.is_fp16].tolist())
        assert sorted(set(seg.pos[~seg.is_fp16].tolist()) - before) == converted, t
        for pos in converted:
            kc, ksc = quantize_row(raw[pos][0])
            vc, vsc = quantize_row(raw[pos][1])
            assert np.array_equal(seg.k8[pos], kc) and seg.ks[pos] == ksc, (t, pos)
            assert np.array_equal(seg.v8[pos], vc) and seg.vs[pos] == vsc, (t, pos)
            assert not seg.k16[pos].any() and not seg.v16[pos].any()
        for pos in fp16:
            assert np.array_equal(seg.k16[pos].view(np.uint16), raw[pos][0].view(np.uint16)), (t, pos)
        np.testing.assert_allclose(out, _torch_attention(q[0].numpy(), seg), rtol=0, atol=1e-12)
        if evict:
            seg = oseg.evict_compact_segment(seg, 1000, p)
            assert seg.pos[seg.is_fp16].tolist() == list(range(t + 2 - W, t + 1)), t


def test_skipped_eviction_converts_on_append():
    pin_skipped_eviction_conversion()


# ---------------------------------------------------------------------------
# planted mistakes
# ---------------------------------------------------------------------------

def _params_mutant(kind):
    class Bad(Params):
        def effective(self, budget):
            if kind == "clamp_to_P":
                return max(int(budget), self.protect_last)
            if kind == "no_clamp":
                return int(budget)
            if kind == "sinks_added":
                return max(int(budget), self.protect_last) + self.n_sink
            return super().effective(budget)
    return Bad


@pytest.mark.parametrize("kind", ["clamp_to_P", "no_clamp", "sinks_added"])
def test_clamp_pin_catches_planted_mistakes(kind):
    pin_budget_below_protected(_params_mutant("none"))
    with pytest.raises((AssertionError, ValueError)):
        pin_budget_below_protected(_params_mutant(kind))


def _cache_mutant(kind):
    class Bad(OracleCache):
        def _initial_budgets(self, B):
            if kind == "n_low":
                N = self.p.n_low
            elif kind == "n_high":
                N = self.p.n_high
            else:
                N = self.p.larger_budget()
            if kind == "flat":
                return np.full((B, self.L), N, np.int64)
            return np.array([self.p.budgets_for(N, self.L)] * B, np.int64)

        def prefill(self, layer, k, v, lens, prio=None):
            B = np.asarray(k).shape[0]
            if kind == "no_reset" and self.budget is not None and self.batch != B:
                # keeps the old batch's budgets (extended row-wise to the new batch)
                self.budget = np.resize(self.budget, (B, self.L))
                self.batch = B
            super().prefill(layer, k, v, lens, prio)
    return Bad


@pytest.mark.parametrize("kind", ["n_low", "n_high", "flat", "no_reset"])
def test_initial_budget_pin_catches_planted_mistakes(kind):
    pin_initial_budget(_cache_mutant("none"))
    with pytest.raises(AssertionError):
        pin_initial_budget(_cache_mutant(kind))


def _decode_mutant(kind):
    def decode(seg, q, k_new, v_new, prio_new, params):
        if kind == "convert_before_append":
            t_old = seg.next_pos - 1
            for i in np.flatnonzero(seg.is_fp16 & (t_old - seg.pos >= params.fp16_window)):
                seg.to_int8(i)
        seg.append(k_new, v_new, oseg.initial_score(params, seg.ident, seg.next_pos))
        t = seg.next_pos - 1
        if kind == "off_by_one":
            sel = seg.is_fp16 & (t - seg.pos > params.fp16_window)
        elif kind == "next_token":
            sel = seg.is_fp16 & (t + 1 - seg.pos >= params.fp16_window)
        elif kind in ("none",):
            sel = seg.is_fp16 & (t - seg.pos >= params.fp16_window)
        else:       # "no_convert", "convert_before_append"
            sel = np.zeros(len(seg), bool)
        for i in np.flatnonzero(sel):
            seg.to_int8(i)
        k_hat, v_hat = seg.rows_hat()
        out, lse, w = oseg.attend(q, k_hat, v_hat)
        seg.score_src = oseg.ema_update(seg.score_src, w, params.ema_decay)
        return out, lse, w
    return decode


@pytest.mark.parametrize("kind", ["no_convert", "off_by_one", "next_token", "convert_before_append"])
def test_conversion_pin_catches_planted_mistakes(kind):
    pin_skipped_eviction_conversion(_decode_mutant("none"))
    with pytest.raises(AssertionError):
        pin_skipped_eviction_conversion(_decode_mutant(kind))
