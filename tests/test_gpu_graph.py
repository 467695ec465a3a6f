"""A decode step captured in a CUDA graph gives the same results as the calls.

With single_stream set, every kernel of a call runs on the caller's stream, so
a whole step (one attention call per layer, the confidence reduction, the
eviction) can be captured and replayed. Two handles with the same prompt run
the same steps, one by direct calls and one by graph replays; outputs,
confidence and the exported caches must agree bit for bit.
"""
import numpy as np
import pytest
import torch

from confidence_gated_kv_logit_b200 import ConfKV, build, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("per_layer", [True, False], ids=["per_layer_calls", "all_layers"])
def test_graph_replay_matches_direct_calls(per_layer):
    build.build()
    dev = torch.device("cuda")
    L, Hkv, Hq, D, B, V = 3, 2, 8, 128, 2, 2048
    kw = dict(max_batch=B, max_prefill=700, n_low=64, n_high=160, protect_last=16, fp16_window=32, n_sink=2,
              single_stream=1)
    handles = [ConfKV(L, Hkv, Hq, D, **kw), ConfKV(L, Hkv, Hq, D, **kw)]
    g = synth.generator(21, dev)
    for l in range(L):
        k, v = synth.prefill_kv(B, Hkv, 700, D, g, dev)
        for h in handles:
            h.prefill(k, v, [700, 410], layer=l)
    steps = [synth.step_qkv((L, B), Hq, Hkv, D, g, dev) + (synth.bursty_logits(B, V, g, dev),) for _ in range(8)]

    def run_step(h, q, kn, vn, lg, out, c):
        if per_layer:
            for l in range(L):
                h.decode_attn(q[l], kn[l], vn[l], out[l], l)
        else:
            h.decode_attn(q, kn, vn, out)
        h.confidence(lg, c)
        h.evict_compact()

    outs = [[], []]
    # direct calls
    for (q, kn, vn, lg) in steps:
        out = torch.empty((L, B, Hq, D), device=dev)
        c = torch.empty(B, device=dev)
        run_step(handles[0], q, kn, vn, lg, out, c)
        outs[0].append((out.clone(), c.clone()))
    # step 0 directly, then a graph of one step replayed on static buffers
    hb = handles[1]
    q0, kn0, vn0, lg0 = steps[0]
    out = torch.empty((L, B, Hq, D), device=dev)
    c = torch.empty(B, device=dev)
    run_step(hb, q0, kn0, vn0, lg0, out, c)
    outs[1].append((out.clone(), c.clone()))
    sq, skn, svn, slg = (x.clone() for x in steps[1])
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run_step(hb, sq, skn, svn, slg, out, c)
    for (q, kn, vn, lg) in steps[1:]:
        sq.copy_(q)
        skn.copy_(kn)
        svn.copy_(vn)
        slg.copy_(lg)
        graph.replay()
        outs[1].append((out.clone(), c.clone()))
    torch.cuda.synchronize()
    for i, ((oa, ca), (ob, cb)) in enumerate(zip(*outs)):
        assert torch.equal(oa, ob), i
        assert torch.equal(ca, cb), i
    for l in range(L):
        for b in range(B):
            for kvh in range(Hkv):
                ea, eb = handles[0].export_segment(l, b, kvh), handles[1].export_segment(l, b, kvh)
                for key in ("pos_c", "sc_c", "ks", "vs", "k_c", "v_c", "pos_r", "sc_r", "k_r", "v_r"):
                    assert np.array_equal(ea[key], eb[key]), (l, b, kvh, key)
    assert handles[0].last_error() == 0 and handles[1].last_error() == 0
    for h in handles:
        h.close()


def test_graph_replays_past_capacity_stop_at_the_device_guard():
    # Replays of a captured decode call do not advance the handle's host-side
    # length bounds, so a caller that replays decode steps without eviction
    # can outgrow the cache. The append kernel's own capacity check then skips
    # the work and sets the device error word; nothing is written out of bounds
    # and the cache stays consistent.
    build.build()
    dev = torch.device("cuda")
    L, Hkv, Hq, D, B = 1, 1, 4, 64, 1
    h = ConfKV(L, Hkv, Hq, D, max_batch=B, max_prefill=100, n_low=32, n_high=48, protect_last=8, fp16_window=16,
               single_stream=1)
    cap_rows = 128                                           # max(100, 48) + 2 rounded up to 64
    g = synth.generator(51, dev)
    k, v = synth.prefill_kv(B, Hkv, 100, D, g, dev)
    h.prefill(k, v, [100], layer=0)
    q, kn, vn = synth.step_qkv((L, B), Hq, Hkv, D, g, dev)
    out = torch.empty((L, B, Hq, D), device=dev)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        h.decode_attn(q, kn, vn, out)
    for _ in range(cap_rows + 20):
        graph.replay()
    torch.cuda.synchronize()
    assert h.last_error(clear=True) == 7                    # CONFKV_ERR_DEVICE: work skipped
    ex = h.export_segment(0, 0, 0)
    assert ex["n_cold"] == cap_rows
    pos = np.concatenate([ex["pos_c"], ex["pos_r"][ex["pos_r"] >= 0]])
    assert len(np.unique(pos)) == len(pos)                   # no token twice
    assert torch.isfinite(out).all()
    del graph
    h.close()
