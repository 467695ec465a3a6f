"""The eviction kernel's fused EMA pass gives the same cache as the separate pass.

A decode call leaves its attention-mass EMA update to the next eviction of the
same layers, which runs it inside the eviction kernel (one launch, the
candidate keys kept in registers). Anything that reads the cache before that
runs the pass on its own. Two handles with the same prompts and steps are
driven identically except that one is made to run every pass on its own (a
query between attention and eviction); after every eviction their exported
caches must agree bit for bit. The separate pass is the one the parity tests
check against the oracle step by step.
"""
import numpy as np
import pytest
import torch

from confidence_gated_kv_logit_b200 import ALL_LAYERS, ConfKV, build, synth

pytestmark = pytest.mark.gpu

FIELDS = ("pos_c", "sc_c", "ks", "vs", "k_c", "v_c", "pos_r", "sc_r", "k_r", "v_r")


def _equal_caches(ha, hb, L, B, Hkv, where):
    for l in range(L):
        for b in range(B):
            for kvh in range(Hkv):
                ea, eb = ha.export_segment(l, b, kvh), hb.export_segment(l, b, kvh)
                assert ea["n_cold"] == eb["n_cold"] and ea["next_pos"] == eb["next_pos"], (where, l, b, kvh)
                for key in FIELDS:
                    assert np.array_equal(ea[key], eb[key]), (where, l, b, kvh, key)


@pytest.mark.parametrize("profiled", [True, False], ids=["event_brackets", "chained"])
@pytest.mark.parametrize("per_layer", [False, True], ids=["all_layers", "per_layer_calls"])
@pytest.mark.parametrize("G,score,compact", [(4, 0, 0), (5, 0, 0), (1, 1, 0), (4, 2, 0), (4, 0, 2)],
                         ids=["gqa4", "gqa5", "mha_accum", "gqa4_random", "gqa4_linear_window"])
def test_fused_pass_matches_separate_pass(per_layer, G, score, compact, profiled):
    # profiled: per-kernel events sit between the launches, so every kernel
    # waits for the one before; unprofiled, the launches are chained and the
    # fused kernel's EMA pass runs beside the confidence reduction
    build.build()
    dev = torch.device("cuda")
    L, Hkv, D, B, V = 3, 2, 128, 3, 2048
    Hq = Hkv * G
    kw = dict(max_batch=B, max_prefill=3000, n_low=64, n_high=160, protect_last=16, fp16_window=32, n_sink=2,
              pyramidal=1, score_source=score, seed=9, compact=compact)
    ha, hb = ConfKV(L, Hkv, Hq, D, **kw), ConfKV(L, Hkv, Hq, D, **kw)
    g = synth.generator(31, dev)
    lens = [3000, 700, 90]     # the first step evicts thousands from the first sequence (whole-CTA path)
    for l in range(L):
        k, v = synth.prefill_kv(B, Hkv, 3000, D, g, dev)
        for h in (ha, hb):
            h.prefill(k, v, lens, layer=l)
    hb.profile(profiled)
    # per step: which calls run ("a" attention, "c" confidence, "e" eviction)
    schedule = ["ace", "ace", "a", "ace", "ac", "ace", "ace", "a", "a", "ace", "ace", "ace"]
    for step, calls in enumerate(schedule):
        q, kn, vn = synth.step_qkv((L, B), Hq, Hkv, D, g, dev)
        logits = synth.bursty_logits(B, V, g, dev)
        outs = []
        for h in (ha, hb):
            out = torch.empty((L, B, Hq, D), device=dev)
            if "a" in calls:
                if per_layer:
                    for l in range(L):
                        h.decode_attn(q[l], kn[l], vn[l], out[l], l)
                else:
                    h.decode_attn(q, kn, vn, out, ALL_LAYERS)
            outs.append(out)
        ha.query()              # runs ha's deferred EMA passes on their own
        if "c" in calls:
            for h in (ha, hb):
                h.confidence(logits, torch.empty(B, device=dev))
        if "e" in calls:
            for h in (ha, hb):
                h.evict_compact(ALL_LAYERS)
            _equal_caches(ha, hb, L, B, Hkv, step)
        if "a" in calls:
            torch.cuda.synchronize()
            assert torch.equal(outs[0], outs[1]), step
    if profiled:
        prof = hb.profile_read()
        assert prof["ema_evict"]["launches"] > 0      # the fused kernel ran
    assert ha.last_error() == 0 and hb.last_error() == 0
    ha.close()
    hb.close()


def test_fused_bulk_step_at_llama8b_shape():
    # two layers of the Llama-3-8B shape (32q/8kv, D128, batch 16) after a
    # 32768-token prompt: the first eviction drops ~31K tokens per segment
    # through the bulk-shaped fused kernel on one handle, through the separate
    # EMA pass and the eviction kernel on the other; then steady steps
    build.build()
    dev = torch.device("cuda")
    L, Hkv, Hq, D, B, T, V = 2, 8, 32, 128, 16, 32768, 128256
    kw = dict(max_batch=B, max_prefill=T, n_low=1024, n_high=2048, protect_last=128, fp16_window=256)
    ha, hb = ConfKV(L, Hkv, Hq, D, **kw), ConfKV(L, Hkv, Hq, D, **kw)
    g = synth.generator(41, dev)
    for l in range(L):
        k, v = synth.prefill_kv(B, Hkv, T, D, g, dev)
        for h in (ha, hb):
            h.prefill(k, v, [T] * B, layer=l)
        del k, v
    for step in range(6):
        q, kn, vn = synth.step_qkv((L, B), Hq, Hkv, D, g, dev)
        logits = synth.bursty_logits(B, V, g, dev)
        for h in (ha, hb):
            h.decode_attn(q, kn, vn, torch.empty((L, B, Hq, D), device=dev), ALL_LAYERS)
        ha.query()              # ha: the separate EMA pass
        for h in (ha, hb):
            h.confidence(logits, torch.empty(B, device=dev))
            h.evict_compact(ALL_LAYERS)
        _equal_caches(ha, hb, L, B, Hkv, step)
    st = hb.query()
    assert st["max_len"] <= 2048
    assert ha.last_error() == 0 and hb.last_error() == 0
    ha.close()
    hb.close()
