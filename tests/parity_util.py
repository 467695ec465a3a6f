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


COMPACT = {"hole-fill": 0, "stable": 1, "linear": 2}


def c_params(p: Params, max_batch: int, max_prefill: int, stable: bool = False, compact: str = None) -> dict:
    return dict(mode=1 if p.mode == "fixed" else 0, n_low=p.n_low, n_high=p.n_high, tau=p.tau,
                alpha=p.alpha, ema_decay=p.ema_decay, protect_last=p.protect_last,
                fp16_window=p.fp16_window, n_sink=p.n_sink, fixed_budget=p.fixed_budget,
                pyramidal=int(p.pyramidal), gate=0 if p.gate == "prose" else 1,
                int8_enable=int(p.int8), compact=COMPACT[compact or ("stable" if stable else "hole-fill")],
                max_batch=max_batch,
                max_prefill=max_prefill, score_source={"ema": 0, "accum": 1, "random": 2}[p.score_source],
                seed=p.seed)


class Pair:
    """The library and the oracle, fed identical inputs."""

    def __init__(self, L, Hkv, Hq, D, B, params: Params, max_prefill: int, track=None, stable=False,
                 seed=0, gen_chunk=None, compact=None):
        _build.build()
        self.L, self.Hkv, self.Hq, self.D, self.B, self.p = L, Hkv, Hq, D, B, params
        # prompt K/V are drawn this many sequences at a time (bounds the fp32
        # temporaries of the generator at the largest shapes)
        self.gen_chunk = gen_chunk or B
        self.compact = compact or ("stable" if stable else "hole-fill")
        self.gpu = ConfKV(L, Hkv, Hq, D, **c_params(params, B, max_prefill, compact=self.compact))
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
            if self.gen_chunk >= self.B:
                k, v = synth.prefill_kv(self.B, self.Hkv, T, self.D, self.gen, self.dev)
            else:
                k = torch.empty((self.B, self.Hkv, T, self.D), dtype=torch.float16, device=self.dev)
                v = torch.empty_like(k)
                for b0 in range(0, self.B, self.gen_chunk):
                    b1 = min(self.B, b0 + self.gen_chunk)
                    k[b0:b1], v[b0:b1] = synth.prefill_kv(b1 - b0, self.Hkv, T, self.D, self.gen, self.dev)
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

    def tracked_layers(self):
        return sorted({l for (l, _, _) in self.segments()})

    def attn(self, q, kn, vn, pn):
        """One attention step on both sides. Only the tracked layers are copied
        to the host and simulated: returns (GPU out, GPU lse, oracle out, oracle
        lse), each a dict from a tracked layer to its [B, Hq, ...] array."""
        out = torch.empty((self.L, self.B, self.Hq, self.D), device=self.dev)
        lse = torch.empty((self.L, self.B, self.Hq), device=self.dev)
        self.gpu_decode_attn(q, kn, vn, out, pn, lse)
        ls = self.tracked_layers()
        idx = torch.tensor(ls, device=self.dev)
        qh, kh, vh = (x.index_select(0, idx).cpu().numpy() for x in (q, kn, vn))
        ph = None if pn is None else pn.index_select(0, idx).cpu().numpy()
        o_out, o_lse = {}, {}
        for i, l in enumerate(ls):
            o_out[l], o_lse[l] = self.orc.decode_attn(l, qh[i], kh[i], vh[i], None if ph is None else ph[i])
        torch.cuda.synchronize()
        go = out.index_select(0, idx).cpu().numpy()
        gl = lse.index_select(0, idx).cpu().numpy()
        g_out = {l: go[i] for i, l in enumerate(ls)}
        g_lse = {l: gl[i] for i, l in enumerate(ls)}
        return g_out, g_lse, o_out, o_lse

    def tracked_seqs(self):
        return sorted({b for (_, b, _) in self.segments()})

    def confidence(self, logits, all_rows=True):
        """Confidence on both sides. With all_rows False the oracle evaluates
        only the tracked sequences (the other rows of c_o are NaN and their
        budgets are not compared)."""
        c = torch.empty(self.B, device=self.dev)
        bud = torch.empty((self.B, self.L), device=self.dev, dtype=torch.int32)
        self.gpu.confidence(logits, c, bud)
        torch.cuda.synchronize()
        c_g, bud_g = c.cpu().numpy(), bud.cpu().numpy()
        from oracle import confidence as oconf
        rows = list(range(self.B)) if all_rows else self.tracked_seqs()
        lh = logits.index_select(0, torch.tensor(rows, device=self.dev)).cpu().numpy()
        full = np.zeros((self.B, lh.shape[1]), np.float32)
        full[rows] = lh
        override = {}
        for i, b in enumerate(rows):
            co = oconf(lh[i])["c"]
            if abs(co - self.p.tau) < NEAR_TIE:
                # the GPU's chosen N, read back from its layer-0 budget (2N under the pyramid)
                override[b] = int(bud_g[b, 0]) // (2 if (self.p.pyramidal and self.L > 1) else 1)
        c_o, bud_o = self.orc.confidence(full, override=override, rows=rows)
        return c_g[rows], bud_g[rows], c_o[rows], bud_o[rows], override

    def gpu_segment(self, l, b, h):
        return logical_segment(self.gpu.export_segment(l, b, h))

    def exact_scores(self):
        """Whether both sides hold the same score sources bit for bit without
        synchronisation (static priorities or static draws)."""
        return self.p.mode == "fixed" or self.p.score_source == "random"

    def sync_scores_from_gpu(self):
        """Step-synchronised mode: give the oracle the GPU's EMA values (matched by
        position) so that selection can be compared bit for bit."""
        if self.exact_scores():
            return
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


def assert_linear_layout(ex: dict, key):
    """The linear layout's physical order: the INT8 region in increasing
    position, the window in slots [0, n) in increasing position, every later
    slot empty, and every window position above every INT8 one."""
    pc = ex["pos_c"].astype(np.int64)
    pr = ex["pos_r"].astype(np.int64)
    assert np.all(np.diff(pc) > 0), key
    n = int((pr >= 0).sum())
    assert np.all(pr[:n] >= 0) and np.all(pr[n:] == -1), (key, pr[:8], n)
    assert np.all(np.diff(pr[:n]) > 0), key
    if n and pc.size:
        assert pr[0] > pc[-1], key


def run_synced(pair: Pair, lens, steps, V, T=None, check_every=1, schedule=None, all_rows_every=None):
    """Step-synchronised parity run: per step, attention (tolerance), EMA
    (tolerance), confidence and budgets, then -- with the oracle given the
    GPU's EMA -- the kept set, compaction and INT8 codes bit for bit.

    ``schedule`` lists, per step, which calls run: "a" attention, "c"
    confidence, "e" eviction (default "ace" every step; fixed mode has no
    confidence). Segments are compared every ``check_every`` steps and at the
    last step. The oracle's confidence covers every row every
    ``all_rows_every`` steps (default: every step), otherwise only the tracked
    sequences."""
    if schedule is None:
        schedule = ["ace"] * steps
    steps = len(schedule)
    all_rows_every = all_rows_every or 1
    pair.prefill(lens, T)
    for key in pair.segments():
        assert_segment_equal(pair.gpu_segment(*key), pair.orc.segment(*key), key)
    worst = 0.0
    for step, calls in enumerate(schedule):
        check = (step % check_every == 0) or step == steps - 1
        q, kn, vn, pn, logits = pair.step_inputs(V)
        if "a" in calls:
            out_g, lse_g, out_o, lse_o = pair.attn(q, kn, vn, pn)
            for (l, b, h) in pair.segments():
                sl = slice(h * pair.orc.G, (h + 1) * pair.orc.G)
                err = float(np.abs(out_g[l][b, sl] - out_o[l][b, sl]).max())
                worst = max(worst, err)
                assert err <= ATOL_OUT, (step, l, b, h, err)
                assert np.abs(lse_g[l][b, sl] - lse_o[l][b, sl]).max() <= ATOL_LSE
                if check:
                    assert_segment_equal(pair.gpu_segment(l, b, h), pair.orc.segment(l, b, h), (step, l, b, h),
                                         exact_scores=pair.exact_scores())
        if "c" in calls and logits is not None:
            c_g, bud_g, c_o, bud_o, override = pair.confidence(logits, all_rows=step % all_rows_every == 0)
            assert np.abs(c_g - c_o).max() <= ATOL_C, (c_g, c_o)
            assert np.array_equal(bud_g, bud_o), (step, bud_g, bud_o, override)
        if "e" in calls:
            pair.sync_scores_from_gpu()
            pair.gpu_evict()
            for l in range(pair.L):
                pair.orc.evict_compact(l)
            if check:
                for key in pair.segments():
                    assert_segment_equal(pair.gpu_segment(*key), pair.orc.segment(*key), (step,) + key)
                    if pair.compact == "linear":
                        assert_linear_layout(pair.gpu.export_segment(*key), (step,) + key)
    assert pair.gpu.last_error() == 0
    return worst
