"""The allocation-free confidence entry point agrees with the handle-based one.

confkv_confidence_noalloc serves callers that cannot allocate device memory
(for example code running under an allocator that owns the whole device):
it keeps its scratch in a fixed array inside the library. This test calls it
through the C ABI twice in a row and compares each result with
confkv_confidence on the same logits. It lives in its own file, collected
last, so a failure here never hides the other tests.
"""
import numpy as np
import pytest
import torch

from confidence_gated_kv_logit_b200 import ConfKV, binding, synth
from confidence_gated_kv_logit_b200 import build as _build

pytestmark = pytest.mark.gpu

ATOL_C = 1e-5   # the confidence tolerance used by every parity test


@pytest.mark.parametrize("B,V,L,pyramidal,gate", [(16, 128256, 32, 0, 0), (3, 50257, 12, 1, 1), (256, 1024, 4, 1, 0),
                                                   (2, 262144, 8, 0, 0)])   # the largest vocabulary it accepts
def test_noalloc_matches_handle_on_two_calls(B, V, L, pyramidal, gate):
    _build.build()
    dev = torch.device("cuda")
    pol = dict(n_low=1024, n_high=2048, tau=0.6, pyramidal=pyramidal, gate=gate)
    h = ConfKV(L, 1, 1, 64, max_batch=B, max_prefill=8, **pol)
    h.prefill(torch.zeros((L, B, 1, 8, 64), dtype=torch.float16, device=dev),
              torch.zeros((L, B, 1, 8, 64), dtype=torch.float16, device=dev), [8] * B)
    g = synth.generator(5, dev)
    for call in range(2):
        logits = synth.bursty_logits(B, V, g, dev)
        if call == 1:
            logits[0] = 0.0
        c_ref = torch.empty(B, device=dev)
        b_ref = torch.empty((B, L), dtype=torch.int32, device=dev)
        h.confidence(logits, c_ref, b_ref)
        c_na = torch.full((B,), float("nan"), device=dev)
        b_na = torch.full((B, L), -1, dtype=torch.int32, device=dev)
        binding.confidence_noalloc(logits, L, c_na, b_na, **pol)
        torch.cuda.synchronize()
        assert np.abs(c_na.cpu().numpy() - c_ref.cpu().numpy()).max() <= ATOL_C
        near = np.abs(c_ref.cpu().numpy() - 0.6) < ATOL_C
        assert np.array_equal(b_na.cpu().numpy()[~near], b_ref.cpu().numpy()[~near])
    h.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    _build.build()
    dev = torch.device("cuda")
    c = torch.empty(257, device=dev)
    b = torch.empty((257, 1), dtype=torch.int32, device=dev)
    with pytest.raises(binding.ConfKVError) as e:
        binding.confidence_noalloc(torch.zeros((257, 16), device=dev), 1, c, b)
    assert e.value.status == 2
    # one token past the largest vocabulary whose per-row partials fit the array
    c1 = torch.empty(1, device=dev)
    b1 = torch.empty((1, 1), dtype=torch.int32, device=dev)
    with pytest.raises(binding.ConfKVError) as e:
        binding.confidence_noalloc(torch.zeros((1, 262145), device=dev), 1, c1, b1)
    assert e.value.status == 2
