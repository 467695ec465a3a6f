"""Parity of the CUDA library with the CPU oracle on the same seeded inputs.

Per step (step-synchronised): attention outputs within 2e-3 max abs and lse
within 1e-4; EMA within a relative 1e-4; confidence within 1e-5 and budgets
equal (near-tie steps take the GPU's budget on both sides); then, with the
oracle given the GPU's EMA values, the kept set, the compacted cache and the
INT8 codes and scales must be identical bit for bit.
"""
import numpy as np
import pytest
import torch

from oracle.segment import Params
from parity_util import ATOL_C, Pair, run_synced

pytestmark = pytest.mark.gpu


def test_config1_tiny_synced():
    # 1 layer, batch 1, 4 MHA heads, D 64, prefill 600, 32 steps, V 1024
    p = Params(n_low=256, n_high=512, tau=0.6, alpha=0.5, ema_decay=0.9, protect_last=64, fp16_window=128)
    pair = Pair(1, 4, 4, 64, 1, p, max_prefill=600)
    worst = run_synced(pair, [600], 32, 1024)
    assert worst < 1e-4


@pytest.mark.parametrize("case", [
    dict(L=2, Hkv=2, Hq=8, D=128, B=3, lens=[300, 0, 77], p=Params(n_low=64, n_high=160, protect_last=16, fp16_window=32, n_sink=2)),
    dict(L=3, Hkv=2, Hq=10, D=128, B=2, lens=[200, 129], p=Params(n_low=40, n_high=80, protect_last=8, fp16_window=24, pyramidal=True)),
    dict(L=1, Hkv=4, Hq=4, D=64, B=2, lens=[150, 31], p=Params(n_low=30, n_high=70, protect_last=10, fp16_window=48, gate="literal", alpha=1.0)),
    dict(L=2, Hkv=1, Hq=1, D=64, B=1, lens=[90], p=Params(n_low=50, n_high=50, protect_last=50, alpha=0.0, int8=False)),
    dict(L=1, Hkv=2, Hq=4, D=128, B=2, lens=[500, 260], p=Params(n_low=60, n_high=120, protect_last=0, fp16_window=1)),
], ids=["gqa4_ragged_sinks", "gqa5_pyramid", "mha64_literal_attnonly", "sliding_window_int8off", "window1_p0"])
def test_shapes_and_policies_synced(case):
    pair = Pair(case["L"], case["Hkv"], case["Hq"], case["D"], case["B"], case["p"], max_prefill=max(case["lens"]))
    run_synced(pair, case["lens"], 12, 2048)


class ZeroQueryPair(Pair):
    """All-zero queries: every score is 0, attention is uniform, and every
    token of a segment gets the same EMA value."""

    def step_inputs(self, V):
        q, kn, vn, pn, logits = super().step_inputs(V)
        return torch.zeros_like(q), kn, vn, pn, logits


@pytest.mark.parametrize("alpha,zero_q", [(0.5, False), (1.0, True)], ids=["histogram", "all_keys_tied"])
def test_bulk_select_long_prompts_synced(alpha, zero_q):
    # Prompts longer than the 2048 keys the whole-CTA select sorts outright, so
    # the first step's bulk eviction finds its threshold from the key histogram;
    # with uniform attention and alpha 1 every key ties in its score, one bin
    # holds them all and the radix select decides (ties go by position).
    p = Params(n_low=300, n_high=600, alpha=alpha, protect_last=32, fp16_window=64, n_sink=2)
    cls = ZeroQueryPair if zero_q else Pair
    pair = cls(1, 2, 8, 128, 2, p, max_prefill=5000, seed=11)
    run_synced(pair, [5000, 3100], 4, 2048)


class PerLayerPair(Pair):
    """Real-model call pattern: one attention call per layer (as a model's
    layers run one after another), then one eviction call per layer."""

    def gpu_decode_attn(self, q, kn, vn, out, pn, lse):
        for l in range(self.L):
            self.gpu.decode_attn(q[l], kn[l], vn[l], out[l], l, prio_new=None if pn is None else pn[l],
                                 lse_out=lse[l])

    def gpu_evict(self):
        for l in range(self.L):
            self.gpu.evict_compact(l)


@pytest.mark.parametrize("mode", ["confidence", "fixed"])
def test_per_layer_calls_synced(mode):
    if mode == "fixed":
        p = Params(mode="fixed", n_sink=4, protect_last=24, fixed_budget=96, fp16_window=40)
    else:
        p = Params(n_low=64, n_high=160, protect_last=16, fp16_window=32, n_sink=2, pyramidal=True)
    pair = PerLayerPair(3, 2, 8, 128, 2, p, max_prefill=400, seed=12)
    run_synced(pair, [400, 150], 8, 0 if mode == "fixed" else 2048)


@pytest.mark.parametrize("source,alpha", [("accum", 0.5), ("random", 0.5), ("random", 1.0)],
                         ids=["accumulated_attention", "random_blend", "random_only"])
def test_ranker_variants_synced(source, alpha):
    # the ranker variants of the matched-rate ablation, at the same budgets
    p = Params(n_low=80, n_high=160, alpha=alpha, protect_last=16, fp16_window=32, n_sink=2,
               score_source=source, seed=123)
    pair = Pair(2, 2, 8, 128, 2, p, max_prefill=600, seed=13)
    run_synced(pair, [600, 250], 10, 2048)


@pytest.mark.parametrize("int8", [False, True])
def test_fixed_budget_mode_synced(int8):
    p = Params(mode="fixed", n_sink=4, protect_last=24, fixed_budget=96, int8=int8, fp16_window=40)
    pair = Pair(2, 2, 8, 128, 2, p, max_prefill=700)
    run_synced(pair, [700, 50], 10, 0)


@pytest.mark.parametrize("case", [
    dict(L=2, Hkv=2, Hq=8, D=128, B=2, lens=[900, 300], p=Params(n_low=100, n_high=200, protect_last=16, fp16_window=32,
                                                                 n_sink=2)),
    dict(L=3, Hkv=2, Hq=10, D=128, B=2, lens=[700, 129], p=Params(n_low=40, n_high=80, protect_last=8, fp16_window=24,
                                                                  pyramidal=True)),
    dict(L=1, Hkv=4, Hq=4, D=64, B=2, lens=[150, 31], p=Params(n_low=30, n_high=70, protect_last=10, fp16_window=48,
                                                               gate="literal", alpha=1.0)),
], ids=["gqa4_sinks", "gqa5_pyramid", "mha64_window_evictions"])
def test_linear_window_layout_synced(case):
    # no ring: the whole cache stays in position order (checked physically
    # after every eviction), with the same logical content as the oracle
    pair = Pair(case["L"], case["Hkv"], case["Hq"], case["D"], case["B"], case["p"],
                max_prefill=max(case["lens"]), compact="linear", seed=27)
    run_synced(pair, case["lens"], 14, 2048)
    st = pair.gpu.query()
    assert st["moved_window_rows"] > 0


def test_stable_compaction_same_logical_content():
    p = Params(n_low=100, n_high=200, protect_last=16, fp16_window=32)
    pair = Pair(1, 2, 8, 128, 2, p, max_prefill=900, stable=True)
    run_synced(pair, [900, 400], 6, 4096)
    assert pair.gpu.query()["moved_rows"] > 0


def test_free_running_kept_set_agreement():
    # no synchronisation: both sides keep their own EMA; kept sets must agree on >= 99.9% of tokens
    p = Params(n_low=256, n_high=512, protect_last=64, fp16_window=128)
    pair = Pair(2, 2, 8, 128, 2, p, max_prefill=700, seed=3)
    pair.prefill([700, 650])
    agree = total = 0
    for step in range(40):
        q, kn, vn, pn, logits = pair.step_inputs(1024)
        pair.attn(q, kn, vn, pn)
        pair.confidence(logits)
        pair.gpu.evict_compact()
        for l in range(pair.L):
            pair.orc.evict_compact(l)
        for key in pair.segments():
            g = set(pair.gpu_segment(*key)["pos"].tolist())
            o = set(pair.orc.segment(*key).pos.tolist())
            agree += len(g & o)
            total += max(len(g), len(o))
    assert agree / total >= 0.999, agree / total


def test_nonfinite_logits_use_larger_budget_and_flag():
    p = Params(n_low=40, n_high=90, protect_last=8, fp16_window=16)
    pair = Pair(2, 1, 4, 128, 3, p, max_prefill=100)
    pair.prefill([100, 100, 100])
    logits = torch.zeros((3, 500), device="cuda")
    logits[1, 7] = float("nan")
    logits[2, 0] = float("inf")
    c = torch.empty(3, device="cuda")
    bud = torch.empty((3, 2), device="cuda", dtype=torch.int32)
    pair.gpu.confidence(logits, c, bud)
    torch.cuda.synchronize()
    assert abs(c[0].item() - (0.15 + 0.3 / 500)) < 1e-6
    assert np.isnan(c[1].item()) and np.isnan(c[2].item())
    assert bud[1].tolist() == [90, 90] and bud[2].tolist() == [90, 90]
    assert bud[0].tolist() == [90, 90]      # uniform logits: uncertain -> loose budget
    assert pair.gpu.last_error(clear=True) == 4
    assert pair.gpu.last_error() == 0


@pytest.mark.parametrize("V,B", [(1024, 1), (50257, 1), (128256, 16), (152064, 32)])
def test_confidence_parity_vocab_sizes(V, B):
    from oracle import confidence_batch
    from confidence_gated_kv_logit_b200 import ConfKV, synth
    h = ConfKV(4, 1, 1, 64, max_batch=B, max_prefill=8, n_low=512, n_high=1024, pyramidal=1)
    h.prefill(torch.zeros((4, B, 1, 8, 64), dtype=torch.float16, device="cuda"),
              torch.zeros((4, B, 1, 8, 64), dtype=torch.float16, device="cuda"), [8] * B)
    g = synth.generator(11, "cuda")
    for trial in range(3):
        logits = synth.bursty_logits(B, V, g, "cuda")
        if trial == 2:
            logits[0] = 0.0                                      # uniform row: closed form
        c = torch.empty(B, device="cuda")
        bud = torch.empty((B, 4), device="cuda", dtype=torch.int32)
        h.confidence(logits, c, bud)
        torch.cuda.synchronize()
        c_o, N_o, per_layer = confidence_batch(logits.cpu().numpy(), 0.6, 512, 1024, 4, True)
        assert np.abs(c.cpu().numpy() - c_o).max() <= ATOL_C
        near = np.abs(c_o - 0.6) < 1e-5
        assert np.array_equal(bud.cpu().numpy()[~near], per_layer[~near])
        if trial == 2:
            assert abs(c[0].item() - (0.15 + 0.3 / V)) <= 1e-6
    h.close()


# ---- the three decode-loop readings pinned by tests/test_oracle_readings.py ----

def test_budget_below_protected_count_synced():
    # budget n_low = 10 below P + s = 20: the effective budget is P + s, so a
    # segment keeps exactly its sinks and its last P tokens; with n_high = 40
    # the gate moves between the clamp and a real budget
    p = Params(n_low=10, n_high=40, protect_last=16, n_sink=4, fp16_window=8)
    pair = Pair(2, 2, 8, 128, 2, p, max_prefill=300, seed=21)
    run_synced(pair, [300, 90], 12, 2048)
    p = Params(n_low=10, n_high=10, protect_last=16, n_sink=4, fp16_window=8, alpha=0.5)
    pair = Pair(1, 2, 8, 128, 2, p, max_prefill=300, seed=22)
    run_synced(pair, [300, 21], 5, 2048)
    for b, T in ((0, 300), (1, 21)):
        t = T + 4
        for h in range(2):
            got = pair.gpu_segment(0, b, h)["pos"].tolist()
            assert got == list(range(4)) + list(range(t - 15, t + 1)), (b, h, got)


def test_budget_before_first_confidence_call_synced():
    # eviction before any confidence call uses the larger budget, per layer
    # under the pyramid: floor(160 (8 - 3l) / 4) = 320, 200, 80 over 3 layers;
    # recency-only ranking keeps the most recent tokens
    p = Params(n_low=64, n_high=160, protect_last=16, fp16_window=32, pyramidal=True, alpha=0.0)
    pair = Pair(3, 2, 8, 128, 2, p, max_prefill=400, seed=23)
    run_synced(pair, [400, 400], 3, 2048, schedule=["ae", "ace", "ace"])
    p2 = Params(n_low=64, n_high=160, protect_last=16, fp16_window=32, pyramidal=True, alpha=0.0)
    pair = Pair(3, 2, 8, 128, 2, p2, max_prefill=400, seed=24)
    run_synced(pair, [400, 400], 1, 2048, schedule=["ae"])
    for l, eff in enumerate((320, 200, 80)):
        for b in range(2):
            for h in range(2):
                assert pair.gpu_segment(l, b, h)["pos"].tolist() == list(range(401 - eff, 401)), (l, b, h)


@pytest.mark.parametrize("compact", ["hole-fill", "stable", "linear"])
def test_skipped_eviction_converts_on_append_synced(compact):
    # a caller that skips eviction: the next append converts the token that
    # has left the FP16 window (the oracle converts t + 1 - W on append too)
    p = Params(n_low=100, n_high=200, protect_last=16, fp16_window=32, n_sink=2)
    pair = Pair(2, 2, 8, 128, 2, p, max_prefill=400, seed=25, compact=compact)
    schedule = ["a", "a", "ace", "ac", "a", "ace", "ace", "a", "ace"]
    run_synced(pair, [400, 130], 0, 2048, schedule=schedule)
    st = pair.gpu.query()
    assert st["requant_rows"] > 0
