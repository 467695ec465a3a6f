"""Parity at the configurations' full sizes and lengths, on sampled segments.

Every configuration runs at its full shape and for its stated number of
decode steps on the GPU, in the launch configuration the benchmark uses (all
layers per call). The oracle simulates a sample of segments (layers spread
over the depth, sequences at both ends of the batch, several KV heads) from
the same bytes, step-synchronised: attention within 2e-3 and LSE within 1e-4
on every step, EMA within a relative 1e-4, confidence within 1e-5, and the
kept set, compaction and INT8 codes bit-exact given the GPU's EMA (segments
compared every few steps and at the last). The end-to-end criterion -- per
step, kept sets agreeing on at least 99.9% of tokens with both sides running
free -- is checked at the Llama-3-8B shape for its 256 steps.
"""
import numpy as np
import pytest
import torch

from oracle.segment import Params
from parity_util import Pair, run_synced

pytestmark = pytest.mark.gpu


def track(layers, seqs, kv_heads):
    return [(l, b, h) for l in layers for b in seqs for h in kv_heads]


def _close(pair):
    pair.gpu.close()
    torch.cuda.empty_cache()


def test_config2_gpt2_small():
    # 12 layers, 12 MHA heads, D64, batch 1, vocab 50257, 128-token prompt, 4096 steps
    p = Params(n_low=256, n_high=512, protect_last=64, fp16_window=128)
    pair = Pair(12, 12, 12, 64, 1, p, max_prefill=128, track=track([0, 6, 11], [0], [0, 6]), seed=2)
    run_synced(pair, [128], 4096, 50257, check_every=64)
    _close(pair)


def test_config2_sliding_window_512_comparison():
    # the fixed 512-token sliding window in the same harness: alpha 0, P 512, INT8 off, 4096 steps
    p = Params(n_low=512, n_high=512, protect_last=512, alpha=0.0, int8=False, fp16_window=1)
    pair = Pair(12, 12, 12, 64, 1, p, max_prefill=128, track=track([0, 11], [0], [0, 4, 8]), seed=3)
    run_synced(pair, [128], 4096, 50257, check_every=64)
    for key in pair.segments():
        seg = pair.orc.segment(*key)
        assert seg.pos.tolist() == list(range(seg.next_pos - 512, seg.next_pos))
    _close(pair)


def test_config3_llama8b_full_prefill():
    # 32 layers, 32q/8kv, D128, batch 16, prefill 32768: the bulk first step, then all 256 steps
    p = Params(n_low=1024, n_high=2048, protect_last=128, fp16_window=256)
    pair = Pair(32, 8, 32, 128, 16, p, max_prefill=32768, track=track([0, 15, 31], [0, 9], range(8)), seed=4)
    run_synced(pair, [32768] * 16, 256, 128256, check_every=16, all_rows_every=16)
    _close(pair)


def test_config3_llama8b_free_running_kept_sets():
    # no synchronisation: each side keeps its own EMA (fp32 on the GPU, fp64
    # rounded to fp32 per update in the oracle) for all 256 steps; per step the
    # kept sets of the sampled segments must agree on >= 99.9% of tokens
    p = Params(n_low=1024, n_high=2048, protect_last=128, fp16_window=256)
    pair = Pair(32, 8, 32, 128, 16, p, max_prefill=32768, track=track([0, 15, 31], [0, 9], range(8)), seed=7)
    pair.prefill([32768] * 16)
    worst = 1.0
    for step in range(256):
        q, kn, vn, pn, logits = pair.step_inputs(128256)
        pair.attn(q, kn, vn, pn)
        pair.confidence(logits, all_rows=False)
        pair.gpu.evict_compact()
        for l in range(pair.L):
            pair.orc.evict_compact(l)
        agree = total = 0
        for key in pair.segments():
            g = set(pair.gpu_segment(*key)["pos"].tolist())
            o = set(pair.orc.segment(*key).pos.tolist())
            agree += len(g & o)
            total += max(len(g), len(o))
        worst = min(worst, agree / total)
        assert agree / total >= 0.999, (step, agree / total)
    assert pair.gpu.last_error() == 0
    _close(pair)


def test_config4_qwen32b_pyramid():
    # 64 layers, 40q/8kv (G=5), D128, batch 32, vocab 152064, 512-token prompt,
    # 4096 steps with pyramidal budgets: the cache grows past every layer's
    # budget (2N at layer 0 down to N/2 at layer 63), so every tracked layer
    # evicts and requantises
    p = Params(n_low=512, n_high=1024, protect_last=128, fp16_window=256, pyramidal=True)
    pair = Pair(64, 8, 40, 128, 32, p, max_prefill=512, track=track([0, 31, 63], [0, 17], [0, 5]), seed=5)
    run_synced(pair, [512] * 32, 4096, 152064, check_every=64, all_rows_every=256)
    st = pair.gpu.query()
    assert st["max_len"] <= 2048 + 1 and st["min_len"] >= 256
    for (l, b, h) in pair.segments():
        n = len(pair.orc.segment(l, b, h))
        assert n < 512 + 4096, (l, n)        # every tracked layer has evicted
    _close(pair)


@pytest.mark.parametrize("batch", [1, 8, 64])
@pytest.mark.parametrize("ctx", [4096, 32768, 131072])
def test_config5_fixed_budget(batch, ctx):
    # 36 layers, 32q/8kv, D128, B = 2048 = 4 sinks + 512 window + 1532 top-k,
    # static priorities; prefill selects as it ingests, then 256 decode steps
    p = Params(mode="fixed", n_sink=4, protect_last=512, fixed_budget=2048, int8=False, fp16_window=1)
    seqs = [0, batch - 1] if batch > 1 else [0]
    chunk = max(1, (1 << 30) // (8 * ctx * 128))
    pair = Pair(36, 8, 32, 128, batch, p, max_prefill=ctx, track=track([0, 35], seqs, [0, 7]), seed=6,
                gen_chunk=chunk)
    run_synced(pair, [ctx] * batch, 256, 0, check_every=32)
    st = pair.gpu.query()
    assert st["max_len"] == 2048 and st["min_len"] == 2048
    _close(pair)
