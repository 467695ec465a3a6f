"""End-to-end invariants of the oracle's decode loop (CPU only).

Drives the oracle cache through prefill and decode steps on a tiny seeded
workload and checks what the method fixes at every step: the length after
eviction, protected survivors, the unique ranking boundary, the FP16 window
by age, that converted rows equal the quantiser applied to the original fp16
row, and that EMA values stay probabilities.
"""
import numpy as np
import pytest
import torch

from confidence_gated_kv_logit_b200 import synth
from oracle import quantize_row
from oracle.segment import OracleCache, Params, segment_scores


def _run(params, L=2, B=2, Hkv=2, Hq=4, D=64, T=150, steps=40, V=256, seed=0, lens=None):
    g = synth.generator(seed)
    cache = OracleCache(L, Hkv, Hq, D, params)
    raw = {}   # (l, b, h, pos) -> (k fp16, v fp16)
    lens = lens or [T] * B
    for l in range(L):
        k, v = synth.prefill_kv(B, Hkv, T, D, g)
        prio = synth.priorities((B, Hkv, T), g).numpy() if params.mode == "fixed" else None
        cache.prefill(l, k.numpy(), v.numpy(), lens, prio)
        for b in range(B):
            for h in range(Hkv):
                for p in range(lens[b]):
                    raw[(l, b, h, p)] = (k[b, h, p].numpy(), v[b, h, p].numpy())
    history = []
    for step in range(steps):
        qs, ks, vs, ps = [], [], [], []
        for l in range(L):
            q, kn, vn = synth.step_qkv((B,), Hq, Hkv, D, g)
            pn = synth.priorities((B, Hkv), g).numpy()
            out, lse = cache.decode_attn(l, q.numpy(), kn.numpy(), vn.numpy(), pn)
            assert np.isfinite(out).all() and np.isfinite(lse).all()
            for b in range(B):
                for h in range(Hkv):
                    raw[(l, b, h, cache.segment(l, b, h).next_pos - 1)] = (kn[b, h].numpy(), vn[b, h].numpy())
        logits = synth.bursty_logits(B, V, g).numpy()
        c, budgets = cache.confidence(logits)
        before = {key: (seg.pos.copy(), segment_scores(seg, params)) for key, seg in cache.segs.items()}
        for l in range(L):
            cache.evict_compact(l)
        history.append((budgets, before))
        yield cache, raw, budgets, before


@pytest.mark.parametrize("params", [
    Params(n_low=40, n_high=90, protect_last=16, fp16_window=32, tau=0.6),
    Params(n_low=40, n_high=90, protect_last=16, fp16_window=32, pyramidal=True, n_sink=3),
    Params(n_low=40, n_high=90, protect_last=40, fp16_window=8, gate="literal", alpha=1.0),
    Params(n_low=30, n_high=30, protect_last=30, alpha=0.0, int8=False),
    Params(mode="fixed", n_sink=4, protect_last=12, fixed_budget=48, int8=False, fp16_window=1),
    Params(mode="fixed", n_sink=4, protect_last=12, fixed_budget=48, int8=True, fp16_window=20),
], ids=["conf", "pyramid_sinks", "literal_attnonly", "sliding_window", "fixed", "fixed_int8"])
def test_decode_loop_invariants(params):
    for cache, raw, budgets, before in _run(params):
        for (l, b, h), seg in cache.segs.items():
            t = seg.next_pos - 1
            pos_before, score_before = before[(l, b, h)]
            budget_eff = params.fixed_budget if params.mode == "fixed" else params.effective(budgets[b, l])
            assert len(seg) == min(pos_before.size, budget_eff)
            assert np.all(np.diff(seg.pos) > 0)
            prot = (t - pos_before < params.protect_last) | (pos_before < params.n_sink)
            assert set(pos_before[prot].tolist()) <= set(seg.pos.tolist())
            kept = np.isin(pos_before, seg.pos)
            cand_k = kept & ~prot
            cand_e = ~kept
            if cand_k.any() and cand_e.any():
                assert (min(zip(score_before[cand_k].tolist(), pos_before[cand_k].tolist()))
                        > max(zip(score_before[cand_e].tolist(), pos_before[cand_e].tolist())))
            if params.int8:
                assert np.array_equal(seg.is_fp16, seg.pos > t + 1 - params.fp16_window)
                for i in np.flatnonzero(~seg.is_fp16)[:5]:
                    k16, v16 = raw[(l, b, h, int(seg.pos[i]))]
                    kc, ksc = quantize_row(k16)
                    assert np.array_equal(seg.k8[i], kc) and seg.ks[i] == ksc
            else:
                assert seg.is_fp16.all()
                i = len(seg) // 2
                k16, _ = raw[(l, b, h, int(seg.pos[i]))]
                assert np.array_equal(seg.k16[i], k16)
            if params.mode != "fixed":
                assert np.all(seg.score_src >= 0) and np.all(seg.score_src <= 1)


def test_ragged_and_empty_prefill():
    p = Params(n_low=20, n_high=40, protect_last=8, fp16_window=16)
    steps = list(_run(p, L=1, B=3, T=60, steps=30, lens=[60, 0, 7]))
    cache, _, budgets, _ = steps[-1]
    assert len(cache.segment(0, 1, 0)) == min(30, p.effective(budgets[1, 0]))
    assert cache.segment(0, 1, 0).next_pos == 30
    assert cache.segment(0, 2, 1).pos[-1] == 36


def test_ema_of_uniform_attention():
    # all keys equal -> every token gets 1/n of the mass each step
    D, T = 64, 10
    p = Params(n_low=1000, n_high=1000, protect_last=4, fp16_window=1000)
    cache = OracleCache(1, 1, 2, D, p)
    k = np.ones((1, 1, T, D), np.float16)
    v = np.zeros((1, 1, T, D), np.float16)
    cache.prefill(0, k, v, [T])
    beta = float(np.float32(0.9))
    expect = np.zeros(T + 3)
    for step in range(3):
        n = T + step + 1
        cache.decode_attn(0, np.ones((1, 2, D), np.float16), np.ones((1, 1, D), np.float16),
                          np.zeros((1, 1, D), np.float16))
        expect[:n] = beta * expect[:n] + (1 - beta) / n
        assert np.allclose(cache.segment(0, 0, 0).score_src, expect[:n], rtol=1e-6)
