"""Helpers shared by the GPU parity tests: one workload driven through the
CUDA library and through the CPU oracle on the same seeded bytes."""
from __future__ import annotations

import numpy as np
import torch

from confidence_gated_kv_logit_b200 import ALL_LAYERS, ConfKV, logical_segment, synth
from confidence_gated_kv_logit_b200 import build as _build
from oracle.segment import OracleCache, Params

# Tolerances (stated by the method's acceptance criteria, or derived):
ATOL_OUT = 2e-3     # attention output, max abs (fp32 accumulate vs fp64 over the dequantised cache)
ATOL_C = 1e-5       # confidence
ATOL_LSE = 1e-4     # log-sum-exp: fp32 scores of magnitude <= ~30, relative error ~1e-6
RTOL_EMA = 1e-4     # EMA: fp32 exp(s - lse) per head vs fp64, relative error ~1e-5 at most
ATOL_EMA = 1e-9
NEAR_TIE = 1e-5     # confidence within this of tau: both sides use the GPU's budget


def c_params(p: Params, max_batch: int, max_prefill: int, stable: bool = False) -> dict:
    return dict(mode=1 if p.mode == "fixed" else 0, n_low=p.n_low, n_high=p.n_high, tau=p.tau,
                alpha=p.alpha, ema_decay=p.ema_decay, protect_last=p.protect_last,
                fp16_window=p.fp16_window, n_sink=p.n_sink, fixed_budget=p.fixed_budget,
                pyramidal=int(p.pyramidal), gate=0 if p.gate == "prose" else 1,
                int8_enable=int(p.int8), compact=1 if stable else 0, max_batch=max_batch,
                max_prefill=max_prefill, score_source={"ema": 0, "accum": 1, "random": 2}[p.score_source],
                seed=p.seed)


class Pair:
    """The library and the oracle, fed identical inputs."""

    def __init__(self, L, Hkv, Hq, D, B, params: Params, max_prefill: int, track=None, stable=False,
                 seed=0):
        _build.build()
        self.L, self.Hkv, self.Hq, self.D, self.B, self.p = L, Hkv, Hq, D, B, params
        self.gpu = ConfKV(L, Hkv, Hq, D, **c_params(params, B, max_prefill, stable))
        self.orc = OracleCache(L, Hkv, Hq, D, params, track)
        self.track = track
        self.gen = synth.generator(seed, "cuda")
        self.dev = torch.device("cuda")

    def segments(self):
        if self.track is not None:
            return sorted(self.track)
        return [(l, b, h) for l in range(self.L) for b in range(self.B) for h in range(self.Hkv)]

    def prefill(self, lens, T=None):
        """Prefill every layer on the GPU; the oracle ingests the host copies of
        the tracked segments only (the others are never simulated)."""
        T = T or max(max(lens), 1)
        fixed = self.p.mode == "fixed"
        for l in range(self.L):
            k, v = synth.prefill_kv(self.B, self.Hkv, T, self.D, self.gen, self.dev)
            pr = synth.priorities((self.B, self.Hkv, T), self.gen, self.dev) if fixed else None
            self.gpu.prefill(k, v, lens, layer=l, priority=pr)
            keys = [key for key in self.segments() if key[0] == l]
            if keys:
                kh = np.zeros((self.B, self.Hkv, T, self.D), np.float16)
                vh = np.zeros_like(kh)
                ph = np.zeros((self.B, self.Hkv, T), np.float32) if fixed else None
                for (_, b, h) in keys:
                    kh[b, h] = k[b, h].cpu().numpy()
                    vh[b, h] = v[b, h].cpu().numpy()
                    if fixed:
                        ph[b, h] = pr[b, h].cpu().numpy()
                self.orc.prefill(l, kh, vh, lens, ph)
            del k, v, pr
        torch.cuda.synchronize()

    def step_inputs(self, V):
        q, kn, vn = synth.step_qkv((self.L, self.B), self.Hq, self.Hkv, self.D, self.gen, self.dev)
        pn = synth.priorities((self.L, self.B, self.Hkv), self.gen, self.dev) if self.p.mode == "fixed" else None
        logits = synth.bursty_logits(self.B, V, self.gen, self.dev) if self.p.mode != "fixed" else None
        return q, kn, vn, pn, logits

    def gpu_decode_attn(self, q, kn, vn, out, pn, lse):
        """The library's attention for every layer of the step (one call)."""
        self.gpu.decode_attn(q, kn, vn, out, ALL_LAYERS, prio_new=pn, lse_out=lse)

    def gpu_evict(self):
        self.gpu.evict_compact()

    def attn(self, q, kn, vn, pn):
        out = torch.empty((self.L, self.B, self.Hq, self.D), device=self.dev)
        lse = torch.empty((self.L, self.B, self.Hq), device=self.dev)
        self.gpu_decode_attn(q, kn, vn, out, pn, lse)
        qh, kh, vh = q.cpu().numpy(), kn.cpu().numpy(), vn.cpu().numpy()
        ph = None if pn is None else pn.cpu().numpy()
        o_out = np.zeros((self.L, self.B, self.Hq, self.D))
        o_lse = np.zeros((self.L, self.B, self.Hq))
        for l in range(self.L):
            o, s = self.orc.decode_attn(l, qh[l], kh[l], vh[l], None if ph is None else ph[l])
            o_out[l], o_lse[l] = o, s
        torch.cuda.synchronize()
        return out.cpu().numpy(), lse.cpu().numpy(), o_out, o_lse

    def confidence(self, logits):
        c = torch.empty(self.B, device=self.dev)
        bud = torch.empty((self.B, self.L), device=self.dev, dtype=torch.int32)
        self.gpu.confidence(logits, c, bud)
        torch.cuda.synchronize()
        c_g, bud_g = c.cpu().numpy(), bud.cpu().numpy()
        from oracle import confidence as oconf
        lh = logits.cpu().numpy()
        override = {}
        for b in range(self.B):
            co = oconf(lh[b])["c"]
            if abs(co - self.p.tau) < NEAR_TIE:
                # the GPU's chosen N, read back from its layer-0 budget (2N under the pyramid)
                override[b] = int(bud_g[b, 0]) // (2 if (self.p.pyramidal and self.L > 1) else 1)
        c_o, bud_o = self.orc.confidence(lh, override=override)
        return c_g, bud_g, c_o, bud_o, override

    def gpu_segment(self, l, b, h):
        return logical_segment(self.gpu.export_segment(l, b, h))

    def sync_scores_from_gpu(self):
        """Step-synchronised mode: give the oracle the GPU's EMA values (matched by
        position) so that selection can be compared bit for bit."""
        for key in self.segments():
            g = self.gpu_segment(*key)
            o = self.orc.segment(*key)
            assert np.array_equal(g["pos"], o.pos), key
            o.score_src = g["score_src"].astype(np.float32).copy()


def assert_segment_equal(g: dict, o, key, exact_scores=True):
    assert g["next_pos"] == o.next_pos, key
    assert np.array_equal(g["pos"], o.pos), (key, g["pos"][:10], o.pos[:10])
    assert np.array_equal(g["is_fp16"], o.is_fp16), key
    f = o.is_fp16
    assert np.array_equal(g["k16"][f].view(np.uint16), o.k16[f].view(np.uint16)), key
    assert np.array_equal(g["v16"][f].view(np.uint16), o.v16[f].view(np.uint16)), key
    i = ~f
    assert np.array_equal(g["k8"][i], o.k8[i]), key
    assert np.array_equal(g["v8"][i], o.v8[i]), key
    assert np.array_equal(g["ks"][i].view(np.uint32), o.ks[i].view(np.uint32)), key
    assert np.array_equal(g["vs"][i].view(np.uint32), o.vs[i].view(np.uint32)), key
    if exact_scores:
        assert np.array_equal(g["score_src"].view(np.uint32), o.score_src.astype(np.float32).view(np.uint32)), key
    else:
        np.testing.assert_allclose(g["score_src"], o.score_src, rtol=RTOL_EMA, atol=ATOL_EMA, err_msg=str(key))


def run_synced(pair: Pair, lens, steps, V, T=None, check_every=1):
    """Step-synchronised parity run: per step, attention (tolerance), EMA
    (tolerance), confidence and budgets, then -- with the oracle given the
    GPU's EMA -- the kept set, compaction and INT8 codes bit for bit."""
    pair.prefill(lens, T)
    for key in pair.segments():
        assert_segment_equal(pair.gpu_segment(*key), pair.orc.segment(*key), key)
    worst = 0.0
    for step in range(steps):
        check = (step % check_every == 0) or step == steps - 1
        q, kn, vn, pn, logits = pair.step_inputs(V)
        out_g, lse_g, out_o, lse_o = pair.attn(q, kn, vn, pn)
        for (l, b, h) in pair.segments():
            sl = slice(h * pair.orc.G, (h + 1) * pair.orc.G)
            err = float(np.abs(out_g[l, b, sl] - out_o[l, b, sl]).max())
            worst = max(worst, err)
            assert err <= ATOL_OUT, (step, l, b, h, err)
            assert np.abs(lse_g[l, b, sl] - lse_o[l, b, sl]).max() <= ATOL_LSE
            if check:
                assert_segment_equal(pair.gpu_segment(l, b, h), pair.orc.segment(l, b, h), (step, l, b, h),
                                     exact_scores=pair.p.mode == "fixed" or pair.p.score_source == "random")
        if logits is not None:
            c_g, bud_g, c_o, bud_o, override = pair.confidence(logits)
            assert np.abs(c_g - c_o).max() <= ATOL_C, (c_g, c_o)
            assert np.array_equal(bud_g, bud_o), (step, bud_g, bud_o, override)
        pair.sync_scores_from_gpu()
        pair.gpu_evict()
        for l in range(pair.L):
            pair.orc.evict_compact(l)
        if check:
            for key in pair.segments():
                assert_segment_equal(pair.gpu_segment(*key), pair.orc.segment(*key), (step,) + key)
    assert pair.gpu.last_error() == 0
    return worst
