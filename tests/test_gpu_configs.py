"""Parity at the configurations' full sizes, on sampled segments.

Every configuration runs at its full shape on the GPU, in the launch
configuration the benchmark uses (all layers per call). The oracle simulates a
sample of segments (layers spread over the depth, two sequences, every KV
head) from the same bytes, step-synchronised: attention within 2e-3, EMA
within a relative 1e-4, confidence within 1e-5, and the kept set, compaction
and INT8 codes bit-exact given the GPU's EMA.
"""
import numpy as np
import pytest
import torch

from oracle.segment import Params
from parity_util import Pair, run_synced

pytestmark = pytest.mark.gpu


def track(layers, seqs, kv_heads):
    return [(l, b, h) for l in layers for b in seqs for h in range(kv_heads)]


def test_config2_gpt2_small():
    # 12 layers, 12 MHA heads, D64, batch 1, vocab 50257, 128-token prompt, 4096 steps
    p = Params(n_low=256, n_high=512, protect_last=64, fp16_window=128)
    pair = Pair(12, 12, 12, 64, 1, p, max_prefill=128, track=track([0, 6, 11], [0], 12)[::6], seed=2)
    run_synced(pair, [128], 4096, 50257, check_every=64)


def test_config2_sliding_window_512_comparison():
    # the fixed 512-token sliding window in the same harness: alpha 0, P 512, INT8 off
    p = Params(n_low=512, n_high=512, protect_last=512, alpha=0.0, int8=False, fp16_window=1)
    pair = Pair(12, 12, 12, 64, 1, p, max_prefill=128, track=track([0, 11], [0], 12)[::4], seed=3)
    run_synced(pair, [128], 1024, 50257, check_every=64)
    for key in pair.segments():
        seg = pair.orc.segment(*key)
        assert seg.pos.tolist() == list(range(seg.next_pos - 512, seg.next_pos))


def test_config3_llama8b_full_prefill():
    # 32 layers, 32q/8kv, D128, batch 16, prefill 32768: bulk first step, then steady steps
    p = Params(n_low=1024, n_high=2048, protect_last=128, fp16_window=256)
    pair = Pair(32, 8, 32, 128, 16, p, max_prefill=32768, track=track([0, 15, 31], [0, 9], 8), seed=4)
    run_synced(pair, [32768] * 16, 12, 128256, check_every=1)


def test_config4_qwen32b_pyramid():
    # 64 layers, 40q/8kv (G=5), D128, batch 32, vocab 152064, 512-token prompt, pyramidal budgets
    p = Params(n_low=512, n_high=1024, protect_last=128, fp16_window=256, pyramidal=True)
    pair = Pair(64, 8, 40, 128, 32, p, max_prefill=512, track=track([0, 31, 63], [0, 17], 8), seed=5)
    run_synced(pair, [512] * 32, 160, 152064, check_every=8)


@pytest.mark.parametrize("batch,ctx", [(8, 32768), (64, 4096), (1, 131072)])
def test_config5_fixed_budget(batch, ctx):
    # 36 layers, 32q/8kv, D128, B = 2048 = 4 sinks + 512 window + 1532 top-k, static priorities
    p = Params(mode="fixed", n_sink=4, protect_last=512, fixed_budget=2048, int8=False, fp16_window=1)
    seqs = [0, batch - 1] if batch > 1 else [0]
    pair = Pair(36, 8, 32, 128, batch, p, max_prefill=ctx, track=track([0, 35], seqs, 8), seed=6)
    run_synced(pair, [ctx] * batch, 16, 0, check_every=1)
    # the kept set after prefill: sinks, window, and the top k by priority (checked by the oracle)
    st = pair.gpu.query()
    assert st["max_len"] == 2048 and st["min_len"] == 2048
