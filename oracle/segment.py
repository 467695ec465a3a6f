"""Cache segments and the decode-step driver (oracle).

Test infrastructure: only tests/, the smoke check and the CPU-baseline legs of
bench.py import this module.

A segment is the cache of one (layer, sequence, KV head). The oracle keeps it
as its logical content: a list of tokens sorted by position, each with its
precision (FP16 or INT8), payload, scales and EMA (or static priority). The
physical layout of the CUDA library is free; parity is on this content.

One decode step follows the order of the CONF-KV post's decode-loop
pseudo-code: the new token is appended (the model call that produces
attention), attention runs over the cache including the new token, the
confidence of the step's logits picks the budget, every layer updates its EMA,
evicts the lowest-ranked tokens if it is over budget, and converts tokens that
leave the FP16 window to INT8.

Readings where the pages are silent (each restated where it is used):

* FP16 window by absolute age: while attention runs at step t, a token is FP16
  exactly when t - pos < W. The token that the next step's append would push
  out of the window (pos = t + 1 - W) is converted to INT8 as the last action
  of step t. Prefill of T tokens treats its end as the end of step T - 1, so
  positions <= T - W are stored INT8.
* Budget: one budget per sequence from its own logits, applied to every layer
  (or its pyramid) and KV head. The effective budget is max(budget, P + s),
  since protected tokens cannot be evicted. Before the first confidence
  evaluation, and for non-finite logits, the larger of the two budgets is used.
* Fixed-budget mode (KVpop summary, section 2.1): the cache never holds more
  than B = s + w + k tokens between steps, so prefill applies the selection
  (sinks, the last w, the top k by priority) as it ingests. INT8 is off by
  default in this mode since the KVpop summary says nothing of quantisation.

Pins: tests/test_oracle_segment.py (decode-loop invariants on seeded runs)
and tests/test_oracle_readings.py, whose expected kept sets are written out
by hand for a budget below P + s (sinks and the last P stay), for eviction
before the first confidence call and after a new batch (the larger budget,
per layer under the pyramid), and for a skipped eviction (the next append
converts position t + 1 - W); planted mistakes in copies of each fail them.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .attention import attend
from .confidence import confidence, choose_budget, layer_budgets
from .policy import accum_update, composite_score, ema_update, random_priority, recency, select_victims
from .quant import dequantize_rows, quantize_row, quantize_rows


@dataclass
class Params:
    """Policy parameters; mirrors the knobs the pages name."""
    mode: str = "conf"            # "conf" (CONF-KV) or "fixed" (B = s + w + k)
    n_low: int = 256
    n_high: int = 512
    tau: float = 0.6
    alpha: float = 0.5
    ema_decay: float = 0.9
    protect_last: int = 64        # P (fixed mode: w)
    fp16_window: int = 128        # W
    n_sink: int = 0               # s
    fixed_budget: int = 0         # B (fixed mode)
    pyramidal: bool = False
    gate: str = "prose"           # "prose" or "literal"
    int8: bool = True
    score_source: str = "ema"     # conf mode ranking source: "ema", "accum" or "random"
    seed: int = 0                 # "random": seed of the static draws

    def budgets_for(self, budget: int, layers: int) -> list[int]:
        return layer_budgets(budget, layers, self.pyramidal)

    def larger_budget(self) -> int:
        return max(self.n_low, self.n_high)

    def effective(self, budget: int) -> int:
        return max(int(budget), self.protect_last + self.n_sink)


@dataclass
class Segment:
    """Logical content of one (layer, sequence, KV head) cache."""
    head_dim: int
    pos: np.ndarray = None        # int64 [n], strictly increasing
    is_fp16: np.ndarray = None    # bool [n]
    k16: np.ndarray = None        # float16 [n, D] (zero rows for INT8 tokens)
    v16: np.ndarray = None
    k8: np.ndarray = None         # int8 [n, D] (zero rows for FP16 tokens)
    v8: np.ndarray = None
    ks: np.ndarray = None         # float32 [n] (0 for FP16 tokens)
    vs: np.ndarray = None
    score_src: np.ndarray = None  # float32 [n]: EMA (conf mode) or priority (fixed)
    next_pos: int = 0
    ident: tuple = (0, 0, 0)      # (layer, seq, kv_head), for the random ranker's draws

    def __post_init__(self):
        D = self.head_dim
        if self.pos is None:
            self.pos = np.zeros(0, np.int64)
            self.is_fp16 = np.zeros(0, bool)
            self.k16 = np.zeros((0, D), np.float16)
            self.v16 = np.zeros((0, D), np.float16)
            self.k8 = np.zeros((0, D), np.int8)
            self.v8 = np.zeros((0, D), np.int8)
            self.ks = np.zeros(0, np.float32)
            self.vs = np.zeros(0, np.float32)
            self.score_src = np.zeros(0, np.float32)

    def __len__(self):
        return int(self.pos.size)

    def take(self, idx) -> "Segment":
        return Segment(self.head_dim, self.pos[idx], self.is_fp16[idx], self.k16[idx],
                       self.v16[idx], self.k8[idx], self.v8[idx], self.ks[idx], self.vs[idx],
                       self.score_src[idx], self.next_pos, self.ident)

    def rows_hat(self):
        """(k_hat, v_hat) as fp32 [n, D]: fp16 rows widened, INT8 rows dequantised."""
        k = self.k16.astype(np.float32)
        v = self.v16.astype(np.float32)
        i8 = ~self.is_fp16
        if i8.any():
            k[i8] = dequantize_rows(self.k8[i8], self.ks[i8])
            v[i8] = dequantize_rows(self.v8[i8], self.vs[i8])
        return k, v

    def append(self, k, v, prio):
        """Append the new token at position next_pos, FP16, EMA 0 (or its priority)."""
        D = self.head_dim
        self.pos = np.append(self.pos, np.int64(self.next_pos))
        self.is_fp16 = np.append(self.is_fp16, True)
        self.k16 = np.vstack([self.k16, np.asarray(k, np.float16).reshape(1, D)])
        self.v16 = np.vstack([self.v16, np.asarray(v, np.float16).reshape(1, D)])
        self.k8 = np.vstack([self.k8, np.zeros((1, D), np.int8)])
        self.v8 = np.vstack([self.v8, np.zeros((1, D), np.int8)])
        self.ks = np.append(self.ks, np.float32(0))
        self.vs = np.append(self.vs, np.float32(0))
        self.score_src = np.append(self.score_src, np.float32(0 if prio is None else prio))
        self.next_pos += 1

    def to_int8(self, i):
        """Convert token i (FP16) to INT8 in place: K and V quantised separately."""
        self.k8[i], self.ks[i] = quantize_row(self.k16[i])
        self.v8[i], self.vs[i] = quantize_row(self.v16[i])
        self.k16[i] = 0
        self.v16[i] = 0
        self.is_fp16[i] = False


def initial_score(params: Params, ident, pos) -> np.float32:
    """Score source of a token entering the cache in confidence mode: 0, or its
    static draw for the random ranker."""
    if params.score_source == "random":
        return random_priority(params.seed, *ident, pos)
    return np.float32(0)


def prefill_segment(k16, v16, prio, params: Params, ident=(0, 0, 0)) -> Segment:
    """Ingest T prompt tokens (positions 0..T-1) of one segment.

    Confidence mode evicts nothing at prefill. Fixed mode keeps the sinks, the
    last w and the top k = B - s - w of the rest by (priority, position). With
    INT8 on, positions <= T - W are stored INT8 (see the module notes).
    """
    k16 = np.asarray(k16, np.float16)
    v16 = np.asarray(v16, np.float16)
    T, D = k16.shape
    seg = Segment(D)
    seg.ident = tuple(ident)
    seg.pos = np.arange(T, dtype=np.int64)
    seg.is_fp16 = np.ones(T, bool)
    seg.k16 = k16.copy()
    seg.v16 = v16.copy()
    seg.k8 = np.zeros((T, D), np.int8)
    seg.v8 = np.zeros((T, D), np.int8)
    seg.ks = np.zeros(T, np.float32)
    seg.vs = np.zeros(T, np.float32)
    if params.mode == "fixed":
        seg.score_src = np.asarray(prio, np.float32).copy()
    else:
        seg.score_src = np.array([initial_score(params, seg.ident, p) for p in range(T)], np.float32)
    seg.next_pos = T
    if params.mode == "fixed" and T > 0:
        evict = select_victims(seg.pos, seg.score_src, T - 1, params.fixed_budget,
                               params.protect_last, params.n_sink)
        seg = seg.take(np.flatnonzero(~evict))
    if params.int8:
        old = np.flatnonzero(seg.pos <= T - params.fp16_window)
        if old.size:
            seg.k8[old], seg.ks[old] = quantize_rows(seg.k16[old])
            seg.v8[old], seg.vs[old] = quantize_rows(seg.v16[old])
            seg.k16[old] = 0
            seg.v16[old] = 0
            seg.is_fp16[old] = False
    return seg


def decode_attn_segment(seg: Segment, q, k_new, v_new, prio_new, params: Params):
    """Append the new token, attend with the G query heads, update the EMA.

    While attention runs at step t a token is FP16 exactly when t - pos < W;
    normally eviction of the previous step has already converted the token
    leaving the window, and this only acts when a step skipped eviction.
    Returns (out [G, D], lse [G], w [G, n]) in fp64.
    """
    seg.append(k_new, v_new, prio_new if params.mode == "fixed" else initial_score(params, seg.ident, seg.next_pos))
    if params.int8:
        t = seg.next_pos - 1
        for i in np.flatnonzero(seg.is_fp16 & (t - seg.pos >= params.fp16_window)):
            seg.to_int8(i)
    k_hat, v_hat = seg.rows_hat()
    out, lse, w = attend(q, k_hat, v_hat)
    if params.mode != "fixed":
        if params.score_source == "ema":
            seg.score_src = ema_update(seg.score_src, w, params.ema_decay)
        elif params.score_source == "accum":
            seg.score_src = accum_update(seg.score_src, w)
        elif params.score_source != "random":   # random: the static draws stand
            raise ValueError(f"unknown score source {params.score_source!r}")
    return out, lse, w


def segment_scores(seg: Segment, params: Params) -> np.ndarray:
    """Ranking score per token: the composite score, or the priority (fixed)."""
    if params.mode == "fixed":
        return seg.score_src.astype(np.float32)
    t = seg.next_pos - 1
    return composite_score(seg.score_src, recency(seg.pos, t), params.alpha)


def evict_compact_segment(seg: Segment, budget: int, params: Params) -> Segment:
    """Evict to the effective budget, compact, convert the leaving token to INT8.

    The newest position is t = next_pos - 1. Compaction on logical content is
    the filter of the token list by the keep set.
    """
    t = seg.next_pos - 1
    budget_eff = params.fixed_budget if params.mode == "fixed" else params.effective(budget)
    evict = select_victims(seg.pos, segment_scores(seg, params), t, budget_eff,
                           params.protect_last, params.n_sink)
    seg = seg.take(np.flatnonzero(~evict))
    if params.int8:
        leaving = np.flatnonzero((seg.pos == t + 1 - params.fp16_window) & seg.is_fp16)
        for i in leaving:
            seg.to_int8(i)
    return seg


class OracleCache:
    """All segments of a model, driven like the C-ABI library.

    Tensors use the library's layouts: prefill k/v [B, Hkv, T, D] for one layer,
    q [B, Hq, D], k_new/v_new [B, Hkv, D], logits [B, V]. ``track`` restricts
    the simulation to a set of (layer, seq, kv_head) triples (the rest are
    skipped and their outputs are NaN).
    """

    def __init__(self, layers, kv_heads, q_heads, head_dim, params: Params, track=None):
        if q_heads % kv_heads:
            raise ValueError("q_heads must be a multiple of kv_heads")
        self.L, self.Hkv, self.Hq, self.D = layers, kv_heads, q_heads, head_dim
        self.G = q_heads // kv_heads
        self.p = params
        self.track = None if track is None else set(map(tuple, track))
        self.segs: dict = {}
        self.batch = 0
        self.budget = None       # [B, L]

    def tracked(self, l, b, h) -> bool:
        return self.track is None or (l, b, h) in self.track

    def _initial_budgets(self, B):
        if self.p.mode == "fixed":
            return np.full((B, self.L), self.p.fixed_budget, np.int64)
        return np.array([self.p.budgets_for(self.p.larger_budget(), self.L)] * B, np.int64)

    def prefill(self, layer, k, v, lens, prio=None):
        k = np.asarray(k)
        B = k.shape[0]
        if self.budget is None or self.batch != B:
            self.batch = B
            self.budget = self._initial_budgets(B)
        for b in range(B):
            T = int(lens[b])
            for h in range(self.Hkv):
                if not self.tracked(layer, b, h):
                    continue
                pr = None if prio is None else np.asarray(prio)[b, h, :T]
                self.segs[(layer, b, h)] = prefill_segment(k[b, h, :T], np.asarray(v)[b, h, :T], pr, self.p,
                                                           (layer, b, h))

    def decode_attn(self, layer, q, k_new, v_new, prio_new=None):
        q = np.asarray(q)
        B = q.shape[0]
        out = np.full((B, self.Hq, self.D), np.nan)
        lse = np.full((B, self.Hq), np.nan)
        for b in range(B):
            for h in range(self.Hkv):
                if not self.tracked(layer, b, h):
                    continue
                seg = self.segs[(layer, b, h)]
                g0 = h * self.G
                pn = None if prio_new is None else float(np.asarray(prio_new)[b, h])
                o, s, _ = decode_attn_segment(seg, q[b, g0:g0 + self.G], np.asarray(k_new)[b, h],
                                              np.asarray(v_new)[b, h], pn, self.p)
                out[b, g0:g0 + self.G] = o
                lse[b, g0:g0 + self.G] = s
        return out, lse

    def confidence(self, logits, override=None, rows=None):
        """Per-sequence confidence and budgets. ``override`` maps a sequence to a
        budget to use instead of the gate's (near-tie steps). ``rows`` limits
        the work to those sequences (the others keep their budgets and get
        c = NaN), for runs that simulate only a few sequences."""
        logits = np.asarray(logits)
        B = logits.shape[0]
        c = np.full(B, np.nan)
        for b in (range(B) if rows is None else rows):
            c[b] = confidence(logits[b])["c"]
            N = choose_budget(c[b], self.p.tau, self.p.n_low, self.p.n_high, self.p.gate)
            if override is not None and b in override:
                N = int(override[b])
            self.budget[b] = self.p.budgets_for(N, self.L)
        return c, self.budget.copy()

    def evict_compact(self, layer):
        for b in range(self.batch):
            for h in range(self.Hkv):
                if not self.tracked(layer, b, h):
                    continue
                key = (layer, b, h)
                self.segs[key] = evict_compact_segment(self.segs[key], int(self.budget[b, layer]), self.p)

    def segment(self, layer, seq, kvh) -> Segment:
        return self.segs[(layer, seq, kvh)]
