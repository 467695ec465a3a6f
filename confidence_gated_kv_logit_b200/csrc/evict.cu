// Eviction, compaction and conversion of the token leaving the FP16 window,
// one warp per segment in the common step, the whole CTA for large evictions
// (CONF-KV post, decode-loop pseudo-code: evict only when
// the layer holds more than its budget, rank by alpha*EMA + (1-alpha)*recency,
// never evict the last P tokens, then convert tokens older than the window to
// INT8; the post's implementation note names contiguous compaction as the hard
// part. KVpop summary 2.1 / 2.4: sinks always kept, fixed budget, running
// threshold over static priorities).
//
// Per segment:
//   1. n = cold tokens + occupied window slots; budget_eff = max(budget, P + s)
//      (fixed mode: B); e = n - budget_eff victims if positive.
//   2. keys (ordered score bits << 32 | position) of unprotected tokens; the e
//      smallest are the victims. Up to 16 victims (the steady state: one new
//      token per step) by one warp, from this step's candidate record or a
//      warp scan; more (budget drops, step 1) by the whole CTA, from the e-th
//      smallest key found by a histogram of the keys (select.cuh).
//   3. victims in the window ring free their slot; victims in the cold region
//      are recorded in a bitmask and the region is compacted: hole-fill moves
//      the survivors above the new end into the holes below it (bytes
//      proportional to e), stable compaction shifts every survivor after the
//      first hole down in order. Both leave the same logical content.
//   4. the token that the next append would push out of the window
//      (position t+1-W) is quantised into the end of the cold region.
//
// The fused variant (the steady decode step in confidence mode) first runs
// the step's attention-mass EMA pass over the warp's segment (ema_warp.cuh)
// and takes the victims of step 2 from the keys that pass merged, in
// registers; segments with more victims go to the whole-CTA path as above,
// which reads the EMA values the pass has just written.
#include "common.cuh"
#include "kernels.h"
#include "ema_warp.cuh"
#include "select.cuh"
#include "warp_select.cuh"

namespace confkv {

namespace {

constexpr int NT = 256;

template <int D, bool CI8>
struct Rows {
  static constexpr int ROWB = CI8 ? D : 2 * D;    // bytes of one K (or V) row in the cold region
  static constexpr int KP = ROWB / 16;            // K parts: 16-byte chunks
  static constexpr int VP = CI8 ? D / 4 : ROWB / 16;   // V parts: four codes (dims 4q..4q+3), or 16-byte chunks
  static constexpr int NP = KP + VP;              // parts of one token's K and V
};

// Part p of cold token i's K/V data (placement in layout.cuh). An INT8 V part
// carries its four codes in .x.
template <int D, bool CI8>
__device__ __forceinline__ uint4 load_part(const Cache& c, int s, int i, int p) {
  using R = Rows<D, CI8>;
  const size_t base = (size_t)s * c.cap * D;
  if (p < R::KP) {
    const unsigned char* k = CI8 ? reinterpret_cast<const unsigned char*>(c.k8 + base)
                                 : reinterpret_cast<const unsigned char*>(c.kc + base);
    return *reinterpret_cast<const uint4*>(k + (CI8 ? k8_off(i, 16 * p, D) : h_off(i, 16 * p, D)));
  }
  const int q = p - R::KP;
  if constexpr (CI8) {
    const unsigned char* v = reinterpret_cast<const unsigned char*>(c.v8 + base);
    uint32_t w = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) w |= (uint32_t)v[v8_off(i, 4 * q + e, D)] << (8 * e);
    return make_uint4(w, 0u, 0u, 0u);
  } else {
    const unsigned char* v = reinterpret_cast<const unsigned char*>(c.vc + base);
    return *reinterpret_cast<const uint4*>(v + h_off(i, 16 * q, D));
  }
}

template <int D, bool CI8>
__device__ __forceinline__ void store_part(const Cache& c, int s, int i, int p, uint4 val) {
  using R = Rows<D, CI8>;
  const size_t base = (size_t)s * c.cap * D;
  if (p < R::KP) {
    unsigned char* k = CI8 ? reinterpret_cast<unsigned char*>(c.k8 + base) : reinterpret_cast<unsigned char*>(c.kc + base);
    *reinterpret_cast<uint4*>(k + (CI8 ? k8_off(i, 16 * p, D) : h_off(i, 16 * p, D))) = val;
    return;
  }
  const int q = p - R::KP;
  if constexpr (CI8) {
    unsigned char* v = reinterpret_cast<unsigned char*>(c.v8 + base);
#pragma unroll
    for (int e = 0; e < 4; ++e) v[v8_off(i, 4 * q + e, D)] = (unsigned char)(val.x >> (8 * e));
  } else {
    unsigned char* v = reinterpret_cast<unsigned char*>(c.vc + base);
    *reinterpret_cast<uint4*>(v + h_off(i, 16 * q, D)) = val;
  }
}

// Move cold row `src` to `dst` (both < cap), part `part` of Rows::NP; part 0
// also moves the metadata.
template <int D, bool CI8>
__device__ __forceinline__ void move_cold_row(const Cache& c, int s, int src, int dst, int part) {
  store_part<D, CI8>(c, s, dst, part, load_part<D, CI8>(c, s, src, part));
  if (part == 0) {
    const size_t so = (size_t)s * c.cap + src, dO = (size_t)s * c.cap + dst;
    c.pos_c[dO] = c.pos_c[so];
    c.sc_c[dO] = c.sc_c[so];
    if (CI8) {
      c.ks[dO] = c.ks[so];
      c.vs[dO] = c.vs[so];
    }
  }
}

constexpr int kSegsPerCta = NT / 32;     // the fast path gives each warp one segment
struct WarpCounts {
  int scanned = 0, moved = 0, requant = 0, moved_win = 0;
};

// One segment by one warp. Handles the common decode step (at most
// kWarpMaxVictims victims, hole-fill order) with shuffles only: one pass over
// the keys in which every lane keeps its own few smallest, a warp merge of the
// lane lists, the same hole-fill pairing as the whole-CTA path (the k-th
// hole below the new end gets the k-th survivor above it) and the conversion
// of the token leaving the window. Returns false, having written nothing,
// when the segment needs the whole-CTA path (more victims, stable order, or
// a lane list that may have dropped a victim). ws_pairs: 2*kWarpMaxVictims
// ints of shared memory owned by this warp.
template <int D, bool CI8>
__device__ bool evict_segment_warp(const Cache& c, const Policy& pol, const EvictLaunch& a, int item, int lane,
                                   WarpCounts* wc, int* ws_pairs, const EmaOut* fused = nullptr) {
  using R = Rows<D, CI8>;
  int l, b, h;
  const int s = seg_of(c, a.r, item, &l, &b, &h);
  const int t = c.next_pos[s] - 1;
  const int n_cold = c.n_cold[s];
  const int W = c.W;
  if (!(n_cold >= 0 && n_cold <= c.cap && t >= -1)) {
    if (lane == 0) record_violation(c.err, kSiteEvictSeg, s, n_cold);
    return true;
  }
  const int32_t* pos_c = c.pos_c + (size_t)s * c.cap;
  const float* sc_c = c.sc_c + (size_t)s * c.cap;
  int32_t* pos_r = c.pos_r + (size_t)s * c.Wst;
  const float* sc_r = c.sc_r + (size_t)s * c.Wst;

  const int budget_eff = pol.mode == 1 ? pol.fixed_budget
                                       : max(a.budget[(size_t)b * c.L + l], pol.P + pol.n_sink);
  auto rank = [&](int pos, float sc) -> unsigned long long {
    if (t - pos < pol.P || pos < pol.n_sink) return kNoKey;
    return rank_key(pol, sc, pos, t);
  };
  // Everything the conversion of the window's leaving token needs is loaded
  // now, in parallel with the candidate record (it does not depend on the
  // victims, except that the token may itself be one: checked below).
  const int leaving = t + 1 - W;
  const bool may_req = CI8 && W > 0 && leaving >= 0;
  // ring: the slot the next append takes; linear window: the oldest slot
  const int rq_slot = may_req && !c.linear ? (t + 1) % W : 0;
  int rq_pos = -1;
  float rq_sc = 0.0f;
  uint32_t rq_k[D / 64], rq_v[D / 64];
  if (may_req) {
    rq_pos = pos_r[rq_slot];
    rq_sc = sc_r[rq_slot];
    row_load_h<D>(c.kr + (size_t)s * c.Wst * D, rq_slot, lane, rq_k);
    row_load_h<D>(c.vr + (size_t)s * c.Wst * D, rq_slot, lane, rq_v);
  }
  bool leaving_evicted = false;

  // This step's EMA pass may have left the segment's smallest keys and its
  // window slot count (confidence mode): then nothing needs rescanning.
  // The record is read whole and unconditionally (one round trip, next to the
  // segment counters); whether it applies is decided afterwards.
  EvictCand* cd = a.cand != nullptr ? a.cand + s : nullptr;
  int4 hdr = make_int4(0, 0, -1, -1);                 // n_ring, safe, stamp, n_cold
  unsigned long long rec_key = kNoKey;
  int rec_idx = -1;
  if (cd != nullptr && fused == nullptr) {
    hdr = *reinterpret_cast<const int4*>(&cd->n_ring);
    if (lane < kCandMax) {
      rec_key = cd->key[lane];
      rec_idx = cd->idx[lane];
    }
  }
  bool have = false;
  int n_ring = 0, count = 0, safe = 0;
  unsigned long long my_key = kNoKey;
  int my_idx = -1;
  if (fused != nullptr) {
    // this kernel's own EMA pass over the segment has just merged its keys
    have = true;
    n_ring = fused->n_ring;
    safe = fused->safe;
    my_key = lane < kCandMax ? fused->key : kNoKey;
    my_idx = lane < kCandMax ? fused->idx : -1;
    count = fused->count;
  } else if (cd != nullptr && pol.mode == 0 && !a.stable && hdr.z == t + 1 && hdr.w == n_cold) {
    have = true;
    n_ring = hdr.x;
    safe = hdr.y;
    my_key = rec_key;
    my_idx = rec_idx;
    count = __popc(__ballot_sync(0xffffffffu, lane < kCandMax && my_key != kNoKey));
  }
  // Otherwise one pass over the segment counts the occupied window slots and
  // keeps each lane's kLaneKeep smallest keys; the keys are computed before
  // the victim count is known (it needs the slot count) and are simply
  // unused when nothing is evicted. Loads are 16 bytes (four tokens) per lane.
  LaneBest best;
  best.init();
  if (!have) {
    const bool use_bound = pol.mode == 0 && pol.one_minus_alpha >= 0x1p-60f;
    const float t1_over_oma = use_bound ? (float)(t + 1) / pol.one_minus_alpha : 0.0f;
    int ring_here = 0;
    for (int s0 = 4 * lane; s0 < W; s0 += 128) {   // the ring stride is a multiple of 64 slots
      const int4 p4 = *reinterpret_cast<const int4*>(pos_r + s0);
      const float4 f4 = *reinterpret_cast<const float4*>(sc_r + s0);
      const int pp[4] = {p4.x, p4.y, p4.z, p4.w};
      const float ff[4] = {f4.x, f4.y, f4.z, f4.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (s0 + q < W && pp[q] >= 0) {
          ++ring_here;
          if (pp[q] + 1 <= best.pos_bound) {
            best.offer(rank(pp[q], ff[q]), n_cold + s0 + q);
            if (use_bound) best.update_bound(t1_over_oma);
          }
        }
      }
    }
    for (int base = 0; base < n_cold; base += 256) {   // cap is a multiple of 64 tokens
      int4 P[2];
      float4 F[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int i0 = base + 128 * u + 4 * lane;
        P[u] = make_int4(-1, -1, -1, -1);
        F[u] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (i0 < n_cold) {
          P[u] = *reinterpret_cast<const int4*>(pos_c + i0);
          F[u] = *reinterpret_cast<const float4*>(sc_c + i0);
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int pp[4] = {P[u].x, P[u].y, P[u].z, P[u].w};
        const float ff[4] = {F[u].x, F[u].y, F[u].z, F[u].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = base + 128 * u + 4 * lane + q;
          if (i < n_cold && pp[q] + 1 <= best.pos_bound) {
            best.offer(rank(pp[q], ff[q]), i);
            if (use_bound) best.update_bound(t1_over_oma);
          }
        }
      }
    }
    n_ring = __reduce_add_sync(0xffffffffu, ring_here);
  }
  const int n = n_cold + n_ring;
  const int e = n - budget_eff;
  int n_cold_new = n_cold;
  int moved = 0;

  if (e > 0 && t >= 0) {
    if (e > kWarpMaxVictims || a.stable) return false;
    // the e smallest keys: victim j's index in lane j; nothing is written
    // before the completeness check (see warp_merge_smallest)
    if (!have) warp_merge_smallest(best, lane, e, &my_key, &my_idx, &count, &safe);
    if (count < e || safe < e) return false;
    const int my_victim = lane < e ? my_idx : -1;

    const bool is_v = my_victim >= 0;
    if (is_v && my_victim >= n_cold) pos_r[my_victim - n_cold] = -1;   // window victims free their slot
    leaving_evicted = __any_sync(0xffffffffu, may_req && is_v && my_victim == n_cold + rq_slot);
    const bool cold_v = is_v && my_victim < n_cold;
    const int ec = __popc(__ballot_sync(0xffffffffu, cold_v));
    if (ec > 0) {
      const int n_keep = n_cold - ec;
      // holes: cold victims below n_keep; movers: survivors in [n_keep, n_cold).
      // Pair p moves the p-th mover (ascending) into the p-th hole (ascending).
      const bool hole = cold_v && my_victim < n_keep;
      int hole_rank = 0;
      bool idx_is_victim = false;
      const int idx = n_keep + lane;                  // mover candidate of this lane (lane < ec)
#pragma unroll
      for (int q = 0; q < kWarpMaxVictims; ++q) {
        const int vq = __shfl_sync(0xffffffffu, my_victim, q);
        const bool cq = __shfl_sync(0xffffffffu, cold_v, q);
        hole_rank += (cq && vq < n_keep && vq < my_victim) ? 1 : 0;
        idx_is_victim |= cq && vq == idx;
      }
      const bool mover = lane < ec && !idx_is_victim;
      const unsigned mb = __ballot_sync(0xffffffffu, mover);
      const int np = __popc(mb);
      int* holes = ws_pairs;
      int* movers = ws_pairs + kWarpMaxVictims;
      if (hole) holes[hole_rank] = my_victim;
      if (mover) movers[__popc(mb & ((1u << lane) - 1u))] = idx;
      __syncwarp();
      for (int w = lane; w < np * R::NP; w += 32) {
        const int pr = w / R::NP;
        const int src = movers[pr], dst = holes[pr];
        if (kChecked && !guard(dst >= 0 && dst < n_keep && src >= n_keep && src < n_cold, c.err, kSiteEvictPair,
                               s, src))
          continue;
        move_cold_row<D, CI8>(c, s, src, dst, w - pr * R::NP);
      }
      moved = np;
      n_cold_new = n_keep;
    }
  }
  if (cd != nullptr && lane == 0) cd->stamp = -1;   // the record described the segment before this call
  __syncwarp();   // ring slots freed and rows moved above are visible to every lane

  // the token that the next append would push out of the window becomes INT8
  int requant = 0;
  if (may_req && rq_pos == leaving && !leaving_evicted) {
    const size_t rs = (size_t)s * c.Wst + rq_slot;
    const int idx = n_cold_new;
    if (idx >= c.cap || idx < 0) {
      if (lane == 0) record_violation(c.err, kSiteEvictRequant, s, idx);
    } else {
      const size_t cb = (size_t)s * c.cap * D, cs = (size_t)s * c.cap + idx;
      uint32_t pk;
      const float ksc = row_quantize<D>(rq_k, &pk);
      row_store_k8<D>(c.k8 + cb, idx, lane, pk);
      const float vsc = row_quantize<D>(rq_v, &pk);
      row_store_v8<D>(c.v8 + cb, idx, lane, pk);
      if (lane == 0) {
        c.ks[cs] = ksc;
        c.vs[cs] = vsc;
        c.pos_c[cs] = leaving;
        c.sc_c[cs] = rq_sc;
        c.pos_r[rs] = -1;
      }
      n_cold_new = idx + 1;
      requant = 1;
    }
  }
  int moved_win = 0;
  if (c.linear && requant) {
    // the window's oldest slot has been converted: the rest moves down one
    // (no eviction ran here, so the window is slots [0, n_ring))
    __syncwarp();
    warp_window_shift<D>(c, s, 1, n_ring, lane);
    moved_win = max(0, n_ring - 1);
  }
  if (lane == 0) c.n_cold[s] = n_cold_new;
  wc->scanned = have ? 0 : n;   // tokens whose keys this call read
  wc->moved = moved;
  wc->requant = requant;
  wc->moved_win = moved_win;
  return true;
}

// Pairs p in [0, np): move cold row movers[p] into holes[p] (all holes are
// below n_keep, all movers at or above it, so no move reads a row another
// writes). Called by every thread of the CTA.
template <int D, bool CI8>
__device__ __forceinline__ void move_pairs_warp(const Cache& c, int s, const int* __restrict__ holes,
                                                const int* __restrict__ movers, int np, int n_keep, int n_cold) {
  using R = Rows<D, CI8>;
  const int lane = threadIdx.x & 31;
  const size_t base = (size_t)s * c.cap * D;
  for (int p0 = threadIdx.x & ~31; p0 < np; p0 += NT) {
    const int p = p0 + lane;
    const bool on = p < np;
    const int src = on ? movers[p] : 0, dst = on ? holes[p] : 0;
    if (kChecked && on && !guard(dst >= 0 && dst < n_keep && src >= n_keep && src < n_cold, c.err, kSiteEvictPair,
                                 s, src))
      continue;
    // K (or fp16 K and V) rows as 16-byte chunks, with the row's metadata:
    // every load of the round in flight before any store
    constexpr int CH = CI8 ? R::KP : R::NP;   // fp16 rows move K and V by chunks
    constexpr int RND = CH < 4 ? CH : 4;
    const size_t so = (size_t)s * c.cap + src, dO = (size_t)s * c.cap + dst;
    int pv = 0;
    float sv = 0.0f, kv = 0.0f, vv = 0.0f;
    if (on) {
      pv = c.pos_c[so];
      sv = c.sc_c[so];
      if (CI8) {
        kv = c.ks[so];
        vv = c.vs[so];
      }
    }
#pragma unroll
    for (int c0 = 0; c0 < CH; c0 += RND) {
      uint4 v[RND];
#pragma unroll
      for (int u = 0; u < RND; ++u)
        if (on && c0 + u < CH) v[u] = load_part<D, CI8>(c, s, src, c0 + u);
#pragma unroll
      for (int u = 0; u < RND; ++u)
        if (on && c0 + u < CH) store_part<D, CI8>(c, s, dst, c0 + u, v[u]);
    }
    if (on) {
      c.pos_c[dO] = pv;
      c.sc_c[dO] = sv;
      if (CI8) {
        c.ks[dO] = kv;
        c.vs[dO] = vv;
      }
    }
    if constexpr (CI8) {
      // V codes: dimension-major, one byte per dimension. With the placement
      // of layout.cuh, the byte of token i, dimension d sits at
      //   blk(i) + ((32d + r) ^ X(d)),  r = i % 32, X(d) = ((d >> 2) & 7) << 4,
      // which splits into a compile-time part (32d) ^ (X & 0x60) and one of
      // two per-token bases (r or r ^ 16): every access below is a single
      // load or store at an immediate offset.
      const unsigned char* vsrc = reinterpret_cast<const unsigned char*>(c.v8 + base);
      unsigned char* vdst = reinterpret_cast<unsigned char*>(c.v8 + base);
      const unsigned char* sb0 = vsrc + (size_t)(src >> 5) * 32 * D + (src & 31);
      const unsigned char* sb1 = vsrc + (size_t)(src >> 5) * 32 * D + ((src & 31) ^ 16);
      unsigned char* db0 = vdst + (size_t)(dst >> 5) * 32 * D + (dst & 31);
      unsigned char* db1 = vdst + (size_t)(dst >> 5) * 32 * D + ((dst & 31) ^ 16);
#pragma unroll
      for (int d0 = 0; d0 < D; d0 += 32) {
        unsigned char bv[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const int d = d0 + u;
          const int X = ((d >> 2) & 7) << 4;
          const int off = (32 * d) ^ (X & 0x60);
          bv[u] = on ? ((X & 0x10) ? sb1 : sb0)[off] : 0;
        }
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const int d = d0 + u;
          const int X = ((d >> 2) & 7) << 4;
          const int off = (32 * d) ^ (X & 0x60);
          if (on) ((X & 0x10) ? db1 : db0)[off] = bv[u];
        }
      }
    }
  }
}

struct EvictSmem {
  SelectSmem<NT> sm;
  int list_h[NT];
  int list_m[NT];
  __align__(16) unsigned char stage[16384];
  int stage_meta[4][64];
};

// One segment by the whole CTA (all NT threads call it with the same item):
// any number of victims, both compaction orders.
// Linear window layout: move the occupied window slots of segment s, in
// order, to slots [0, n) and empty the rest; the whole CTA, staging up to 64
// slots at a time through shared memory (every destination is at or below
// its source, and a chunk is read whole before any of it is written).
// Returns the number of slots that moved (in every thread).
template <int D>
__device__ int block_window_compact(const Cache& c, int s, EvictSmem& es) {
  constexpr int RB = 4 * D;                       // bytes of one slot: fp16 K and V rows
  constexpr int CH = 16384 / RB < 64 ? 16384 / RB : 64;
  constexpr int HP = RB / 32;                     // 16-byte parts of one row
  unsigned char* kr = reinterpret_cast<unsigned char*>(c.kr + (size_t)s * c.Wst * D);
  unsigned char* vr = reinterpret_cast<unsigned char*>(c.vr + (size_t)s * c.Wst * D);
  int32_t* pr = c.pos_r + (size_t)s * c.Wst;
  float* sr = c.sc_r + (size_t)s * c.Wst;
  uint4* stage = reinterpret_cast<uint4*>(es.stage);
  int dst_base = 0, moved = 0;
  for (int base = 0; base < c.W; base += CH) {
    const int slot = base + (int)threadIdx.x;
    const bool live = threadIdx.x < CH && slot < c.W && pr[slot] >= 0;
    int total;
    const int r = block_scan_flag<NT>(live, es.sm, &total);
    for (int w = threadIdx.x; w < CH * 2 * HP; w += NT) {
      const int rr = w / (2 * HP), part = w - rr * 2 * HP;
      const int sl = base + rr;
      if (sl < c.W) {
        const unsigned char* src = part < HP ? kr : vr;
        stage[w] = *reinterpret_cast<const uint4*>(src + h_off(sl, 16 * (part % HP), D));
      }
    }
    if (live) {
      es.stage_meta[0][threadIdx.x] = pr[slot];
      es.stage_meta[1][threadIdx.x] = __float_as_int(sr[slot]);
      es.list_m[threadIdx.x] = dst_base + r;
    }
    if (threadIdx.x < CH) es.list_h[threadIdx.x] = live ? 1 : 0;
    __syncthreads();
    for (int w = threadIdx.x; w < CH * 2 * HP; w += NT) {
      const int rr = w / (2 * HP), part = w - rr * 2 * HP;
      if (base + rr < c.W && es.list_h[rr]) {
        unsigned char* dst = part < HP ? kr : vr;
        *reinterpret_cast<uint4*>(dst + h_off(es.list_m[rr], 16 * (part % HP), D)) = stage[w];
      }
    }
    if (live) {
      const int d = es.list_m[threadIdx.x];
      pr[d] = es.stage_meta[0][threadIdx.x];
      sr[d] = __int_as_float(es.stage_meta[1][threadIdx.x]);
      moved += d != slot ? 1 : 0;
    }
    dst_base += total;
    __syncthreads();
  }
  for (int j = dst_base + (int)threadIdx.x; j < c.W; j += NT) pr[j] = -1;
  return block_sum_int<NT>(moved, es.sm);
}

// Keys already in this CTA's scratch (the bulk variant's EMA pass wrote
// them): the occupied window slots and this thread's range of counted keys.
// A bin map of key high halves fixed before the keys exist (confidence
// mode): high halves at or below `lo` fall in bin 0, the rest in steps of
// 2^shift, the last bin taking everything above; monotone in the key. With
// `lo` below every score's bits and the steps sized to reach a score of 2,
// the bins cover the scores' range at 2^(23 - shift) bins per octave.
struct KeyBins {
  uint32_t lo;
  int shift;
  __device__ __forceinline__ int operator()(uint32_t hv) const {
    return hv <= lo ? 0 : (int)min((uint32_t)(kSelBins - 1), (hv - lo) >> shift);
  }
};

struct BlockKeys {
  int n_ring;
  uint32_t kmn, kmx;
  bool binned;    // the keys' histogram over `bins` is in the select buffer
  KeyBins bins;
};

template <int D, bool CI8>
__device__ void evict_segment_block(const Cache& c, const Policy& pol, const EvictLaunch& a, int item,
                                    EvictSmem& es, const BlockKeys* pre = nullptr) {
  using R = Rows<D, CI8>;
  SelectSmem<NT>& sm = es.sm;
  int* list_h = es.list_h;
  int* list_m = es.list_m;
  unsigned char* stage = es.stage;
  int (*stage_meta)[64] = es.stage_meta;

  int l, b, h;
  const int s = seg_of(c, a.r, item, &l, &b, &h);
  const int t = c.next_pos[s] - 1;
  const int n_cold = c.n_cold[s];
  const int W = c.W;
  if (!guard(n_cold >= 0 && n_cold <= c.cap && t >= -1, c.err, kSiteEvictSeg, s, n_cold)) return;
  const int32_t* pos_c = c.pos_c + (size_t)s * c.cap;
  const float* sc_c = c.sc_c + (size_t)s * c.cap;
  int32_t* pos_r = c.pos_r + (size_t)s * c.Wst;
  const float* sc_r = c.sc_r + (size_t)s * c.Wst;

  int n_ring;
  if (pre != nullptr) {
    n_ring = pre->n_ring;
  } else {
    int ring_here = 0;
    for (int slot = threadIdx.x; slot < W; slot += NT) ring_here += pos_r[slot] >= 0;
    n_ring = block_sum_int<NT>(ring_here, sm);
  }
  const int n = n_cold + n_ring;
  const int budget_eff = pol.mode == 1 ? pol.fixed_budget
                                       : max(a.budget[(size_t)b * c.L + l], pol.P + pol.n_sink);
  const int e = n - budget_eff;
  int n_cold_new = n_cold;
  int moved = 0;

  if (e > 0 && t >= 0) {
    auto pos_of = [&](int i) -> int { return i < n_cold ? pos_c[i] : pos_r[i - n_cold]; };
    auto key = [&](int i) -> unsigned long long {
      int pos;
      float sc;
      if (i < n_cold) {
        pos = pos_c[i];
        sc = sc_c[i];
      } else {
        pos = pos_r[i - n_cold];
        if (pos < 0) return kNoKey;
        sc = sc_r[i - n_cold];
      }
      if (t - pos < pol.P || pos < pol.n_sink) return kNoKey;
      return rank_key(pol, sc, pos, t);
    };
    const int span = n_cold + W;
    uint32_t* vm = a.vmask + (size_t)s * a.mask_words;
    auto victim = [&](int i) -> bool { return (vm[i >> 5] >> (i & 31)) & 1u; };
    if (e == 1 && !a.stable) {
      // one victim; its index comes with the argmin, and at most one row (the
      // last cold row) moves into its place
      int vi;
      block_argmin_idx<NT>(key, span, sm, &vi);
      if (vi >= n_cold) {
        if (threadIdx.x == 0) pos_r[vi - n_cold] = -1;
      } else if (vi >= 0) {
        const int last = n_cold - 1;
        if (vi != last) {
          for (int w = threadIdx.x; w < R::NP; w += NT) move_cold_row<D, CI8>(c, s, last, vi, w);
          moved = 1;
        }
        n_cold_new = n_cold - 1;
      }
      __syncthreads();
    } else {
    // High halves of the keys (ordered score bits; 0xFFFFFFFF = never a
    // victim) into this CTA's scratch, four tokens per thread in flight.
    uint32_t* __restrict__ khi = a.kscratch + (size_t)blockIdx.x * a.scratch_stride;
    auto hi_of = [&](int pos, float sc) -> uint32_t {
      const bool none = pos < 0 || t - pos < pol.P || pos < pol.n_sink;
      return none ? 0xFFFFFFFFu : (uint32_t)(rank_key(pol, sc, pos, t) >> 32);
    };
    // cold region: 8 tokens per thread per step in two 16-byte loads each of
    // positions and EMA values (the region is a multiple of 64 tokens long);
    // each thread also keeps the range of its counted keys for the select
    uint32_t kmn = 0xFFFFFFFFu, kmx = 0u;
    auto track = [&](uint32_t hv) {
      if (hv != 0xFFFFFFFFu) {
        kmn = min(kmn, hv);
        kmx = max(kmx, hv);
      }
    };
    if (pre != nullptr) {
      kmn = pre->kmn;
      kmx = pre->kmx;
    }
    for (int i0 = 8 * threadIdx.x; pre == nullptr && i0 < n_cold; i0 += 8 * NT) {
      const int4 p0 = reinterpret_cast<const int4*>(pos_c + i0)[0];
      const int4 p1 = reinterpret_cast<const int4*>(pos_c + i0)[1];
      const float4 f0 = reinterpret_cast<const float4*>(sc_c + i0)[0];
      const float4 f1 = reinterpret_cast<const float4*>(sc_c + i0)[1];
      const int pp[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
      const float ff[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
      uint32_t hv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        hv[j] = i0 + j < n_cold ? hi_of(pp[j], ff[j]) : 0xFFFFFFFFu;
        track(hv[j]);
      }
      if (i0 + 8 <= n_cold) {
        reinterpret_cast<uint4*>(khi + i0)[0] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        reinterpret_cast<uint4*>(khi + i0)[1] = make_uint4(hv[4], hv[5], hv[6], hv[7]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (i0 + j < n_cold) khi[i0 + j] = hv[j];
      }
    }
    for (int slot = threadIdx.x; pre == nullptr && slot < W; slot += NT) {
      const uint32_t hv = hi_of(pos_r[slot], sc_r[slot]);
      khi[n_cold + slot] = hv;
      track(hv);
    }
    __syncthreads();
    // the e-th smallest key: the victims are the keys up to it
    unsigned long long* selbuf = reinterpret_cast<unsigned long long*>(es.stage);
    const unsigned long long thr =
        pre != nullptr && pre->binned
            ? select_in_hist<NT>(khi, pos_of, span, e, sm, selbuf, pre->bins)
            : block_select_threshold<NT>(khi, pos_of, span, e, sm, selbuf, true, kmn, kmx);
    const uint32_t thr_hi = (uint32_t)(thr >> 32), thr_lo = (uint32_t)thr;
    auto below_thr = [&](uint32_t hv, int i) -> bool {   // the position only matters on a tie of the high half
      return hv != 0xFFFFFFFFu && (hv < thr_hi || (hv == thr_hi && (uint32_t)pos_of(i) <= thr_lo));
    };
    auto is_victim = [&](int i) -> bool { return below_thr(khi[i], i); };

    // victim bitmask of the cold region: each thread builds whole 32-token
    // words from eight 16-byte loads of the key scratch
    int ecold_here = 0;
    for (int w = threadIdx.x; w < ((n_cold + 31) >> 5); w += NT) {
      uint4 q[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) q[u] = reinterpret_cast<const uint4*>(khi + 32 * w)[u];
      uint32_t bits = 0u;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t hv[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = 32 * w + 4 * u + j;
          if (i < n_cold && below_thr(hv[j], i)) bits |= 1u << (4 * u + j);
        }
      }
      vm[w] = bits;
      ecold_here += __popc(bits);
    }
    // window victims free their slot (each thread reads and writes only its own slots)
    for (int slot = threadIdx.x; slot < W; slot += NT)
      if (is_victim(n_cold + slot)) pos_r[slot] = -1;
    const int e_cold = block_sum_int<NT>(ecold_here, sm);   // includes a block barrier: vm is visible
    const int n_keep = n_cold - e_cold;

    if (e_cold == 0) {
      // every victim was in the window ring: the cold region is unchanged
    } else if (!a.stable) {
      // Hole-fill: the k-th hole below n_keep receives the k-th survivor at or
      // above it. Both lists come from one pass over the mask words (popcount
      // and a block scan) into this CTA's scratch.
      int* __restrict__ holes = reinterpret_cast<int*>(khi + a.scratch_keys);
      int* __restrict__ movers = holes + c.cap;
      const int words = (n_cold + 31) >> 5;
      int hole_base = 0, mover_base = 0;
      for (int w0 = 0; w0 < words; w0 += NT) {
        const int w = w0 + (int)threadIdx.x;
        uint32_t hb = 0u, mb = 0u;
        const int lo_i = w << 5;
        if (w < words) {
          const uint32_t bits = vm[w];
          const uint32_t valid = lo_i + 32 <= n_cold ? 0xffffffffu : ((1u << (n_cold - lo_i)) - 1u);
          const uint32_t below = lo_i + 32 <= n_keep ? 0xffffffffu
                                 : (lo_i >= n_keep ? 0u : ((1u << (n_keep - lo_i)) - 1u));
          hb = bits & below & valid;
          mb = ~bits & ~below & valid;
        }
        int htot, mtot;
        int ho = hole_base + block_excl_scan_int<NT>(__popc(hb), sm, &htot);
        int mo = mover_base + block_excl_scan_int<NT>(__popc(mb), sm, &mtot);
        while (hb) {
          holes[ho++] = lo_i + __ffs(hb) - 1;
          hb &= hb - 1u;
        }
        while (mb) {
          movers[mo++] = lo_i + __ffs(mb) - 1;
          mb &= mb - 1u;
        }
        hole_base += htot;
        mover_base += mtot;
      }
      __syncthreads();   // the lists are complete and visible
      const int np = min(hole_base, mover_base);
      // moves: each warp takes 32 consecutive pairs, lane j the j-th; K rows
      // move as 16-byte chunks, and V codes one dimension at a time, so that
      // a warp instruction reads and writes 32 neighbouring bytes of a
      // dimension-major row whenever the holes and the movers run in order
      // (as they do in bulk evictions).
      move_pairs_warp<D, CI8>(c, s, holes, movers, np, n_keep, n_cold);
      moved = np;
      __syncthreads();
    } else {
      // stable: from the first hole on, every survivor moves down by the number
      // of victims before it, in chunks staged through shared memory
      constexpr int CH = 16384 / (16 * R::NP) < 64 ? 16384 / (16 * R::NP) : 64;
      int dst_base = 0;
      for (int base = 0; base < n_cold; base += CH) {
        const int i = base + (int)threadIdx.x;
        const bool live = threadIdx.x < CH && i < n_cold && !victim(i);
        int total;
        const int r = block_scan_flag<NT>(live, sm, &total);
        // stage this chunk's survivors (rows and metadata), then write them back
        for (int w = threadIdx.x; w < CH * R::NP; w += NT) {
          const int rr = w / R::NP, part = w - rr * R::NP;
          const int src = base + rr;
          if (src < n_cold) reinterpret_cast<uint4*>(stage)[w] = load_part<D, CI8>(c, s, src, part);
        }
        if (live) {
          const size_t so = (size_t)s * c.cap + i;
          stage_meta[0][threadIdx.x] = pos_c[i];
          stage_meta[1][threadIdx.x] = __float_as_int(sc_c[i]);
          stage_meta[2][threadIdx.x] = CI8 ? __float_as_int(c.ks[so]) : 0;
          stage_meta[3][threadIdx.x] = CI8 ? __float_as_int(c.vs[so]) : 0;
          list_m[threadIdx.x] = dst_base + r;
        }
        if (threadIdx.x < CH) list_h[threadIdx.x] = live ? 1 : 0;
        __syncthreads();
        for (int w = threadIdx.x; w < CH * R::NP; w += NT) {
          const int rr = w / R::NP, part = w - rr * R::NP;
          if (base + rr < n_cold && list_h[rr]) {
            const size_t dO = (size_t)s * c.cap + list_m[rr];
            store_part<D, CI8>(c, s, list_m[rr], part, reinterpret_cast<const uint4*>(stage)[w]);
            if (part == 0) {
              c.pos_c[dO] = stage_meta[0][rr];
              c.sc_c[dO] = __int_as_float(stage_meta[1][rr]);
              if (CI8) {
                c.ks[dO] = __int_as_float(stage_meta[2][rr]);
                c.vs[dO] = __int_as_float(stage_meta[3][rr]);
              }
            }
          }
        }
        if (threadIdx.x < CH && live && list_m[threadIdx.x] != i) ++moved;
        dst_base += total;
        __syncthreads();
      }
      moved = block_sum_int<NT>(moved, sm);
    }
    n_cold_new = n_keep;
    }
  }

  // the token that the next append would push out of the window becomes INT8
  __syncthreads();
  const int leaving = t + 1 - W;
  int conv_slot = W > 0 ? (t + 1) % W : 0;
  if (c.linear) {
    // linear window: the oldest occupied slot (the window is in position order)
    int f = W;
    for (int slot = threadIdx.x; slot < W; slot += NT)
      if (pos_r[slot] >= 0) f = min(f, slot);
    f = __reduce_min_sync(0xffffffffu, f);
    if ((threadIdx.x & 31) == 0) sm.warp_tot[threadIdx.x >> 5] = f;
    __syncthreads();
    f = W;
#pragma unroll
    for (int i = 0; i < NT / 32; ++i) f = min(f, sm.warp_tot[i]);
    __syncthreads();
    conv_slot = f < W ? f : 0;
  }
  if (W > 0 && leaving >= 0 && threadIdx.x < 32) {
    const int slot = conv_slot;
    const size_t rs = (size_t)s * c.Wst + slot;
    if (c.pos_r[rs] == leaving) {
      const int idx = n_cold_new;
      if (idx >= c.cap || idx < 0) {
        if (threadIdx.x == 0) record_violation(c.err, kSiteEvictRequant, s, idx);
      } else {
        const size_t cs = (size_t)s * c.cap + idx;
        warp_requant<D>(c, s, slot, idx, threadIdx.x);
        __syncwarp();
        if (threadIdx.x == 0) {
          c.pos_c[cs] = leaving;
          c.sc_c[cs] = c.sc_r[rs];
          c.pos_r[rs] = -1;
          atomicAdd(&c.counters[kCntRequant], 1ull);
        }
        n_cold_new = idx + 1;
      }
    }
  }
  int moved_win = 0;
  if (c.linear) {
    __syncthreads();   // the conversion above has emptied its slot
    moved_win = block_window_compact<D>(c, s, es);
  }
  if (threadIdx.x == 0) {
    c.n_cold[s] = n_cold_new;
    if (moved_win > 0) atomicAdd(&c.counters[kCntMovedWin], (unsigned long long)moved_win);
    atomicAdd(&c.counters[kCntEvictBlock], 1ull);
    if (a.cand != nullptr) a.cand[s].stamp = -1;
    // tokens whose keys this path read from the cache (precomputed keys came
    // with the EMA pass's own reads)
    if (pre == nullptr || (e == 1 && !a.stable)) atomicAdd(&c.counters[kCntEvictScanned], (unsigned long long)n);
    if (moved > 0) atomicAdd(&c.counters[kCntMovedRows], (unsigned long long)moved);
  }
}

// GMAX > 0: the fused variant. Each warp first runs the step's EMA pass over
// its segment (ema_warp.cuh, the same code as the EMA kernel, for G <= GMAX
// query heads per KV head) and evicts from the merged keys it leaves in
// registers: no candidate record, and no separate EMA launch.
template <int D, bool CI8, int GMAX>
__global__ void __launch_bounds__(NT, GMAX > 4 ? 3 : 4) evict_kernel(Cache c, Policy pol, EvictLaunch a, EmaIn ein,
                                                                      int items) {
  // The fused variant's EMA pass reads only what attention and the kernels
  // before it wrote. When the previous kernel is the confidence reduction
  // (a.ema_early), which releases its successor only once everything before
  // it has completed and which touches none of the pass's data, the pass runs
  // before the wait, beside that reduction; the budgets it writes are read
  // after the wait.
  const bool early = GMAX > 0 && a.ema_early != 0;
  if (!early) chain_enter();
  __shared__ EvictSmem es;
  __shared__ int slow_items[kSegsPerCta];
  __shared__ int n_slow;
  __shared__ unsigned long long cnt[4];
  __shared__ int pairs[kSegsPerCta][2 * kWarpMaxVictims];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) n_slow = 0;
  if (threadIdx.x < 4) cnt[threadIdx.x] = 0;
  __syncthreads();
  // Segments are dealt to warps through a multiplicative bijection of
  // [0, items) (the multiplier is a prime above any item count), so that the
  // segments of one sequence, which share a budget and so need the whole-CTA
  // path at the same steps, land in different CTAs.
  const int slot = blockIdx.x * kSegsPerCta + warp;
  const int item = slot < items ? (int)(((unsigned long long)slot * 2654435761ull) % (unsigned long long)items) : items;
  EmaOut eo;
  if constexpr (GMAX > 0) {
    if (item < items) {
      int l, b, h;
      const int s = seg_of(c, a.r, item, &l, &b, &h);
      ema_segment_warp<GMAX>(c, ein, pol, s, lane, &eo);
    }
  }
  if (early) chain_enter();
  if (item < items) {
    WarpCounts wc;
    bool done;
    if constexpr (GMAX > 0) {
      // a corrupt segment was recorded by the pass; eviction skips it likewise
      done = !eo.ok || evict_segment_warp<D, CI8>(c, pol, a, item, lane, &wc, pairs[warp], &eo);
    } else {
      done = evict_segment_warp<D, CI8>(c, pol, a, item, lane, &wc, pairs[warp]);
    }
    if (!done) {
      if (lane == 0) slow_items[atomicAdd(&n_slow, 1)] = item;
    } else if (lane == 0) {
      if (wc.scanned) atomicAdd(&cnt[0], (unsigned long long)wc.scanned);
      if (wc.moved) atomicAdd(&cnt[1], (unsigned long long)wc.moved);
      if (wc.requant) atomicAdd(&cnt[2], (unsigned long long)wc.requant);
      if (wc.moved_win) atomicAdd(&cnt[3], (unsigned long long)wc.moved_win);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (cnt[0]) atomicAdd(&c.counters[kCntEvictScanned], cnt[0]);
    if (cnt[1]) atomicAdd(&c.counters[kCntMovedRows], cnt[1]);
    if (cnt[2]) atomicAdd(&c.counters[kCntRequant], cnt[2]);
    if (cnt[3]) atomicAdd(&c.counters[kCntMovedWin], cnt[3]);
  }
  const int ns = n_slow;
  for (int k = 0; k < ns; ++k) {
    __syncthreads();   // the previous segment's shared-memory use is over
    evict_segment_block<D, CI8>(c, pol, a, slow_items[k], es);
  }
}

// The step's EMA pass over segment s by the whole CTA (the same arithmetic
// per token as ema_segment_warp), also writing every token's key high half
// into this CTA's scratch as the whole-CTA eviction path wants it, with each
// thread's range of counted keys and the occupied window slots. Returns false
// (recorded) for a corrupt segment.
template <int GMAX>
__device__ bool cta_ema_keys(const Cache& c, const EmaIn& in, const Policy& pol, int s, uint32_t* __restrict__ khi,
                             BlockKeys* bk, SelectSmem<NT>& sm, uint32_t* __restrict__ hist) {
  constexpr float kLog2eF = 1.4426950408889634f;
  const int G = c.G;
  const float invG = 1.0f / (float)G;
  float lse[GMAX];
#pragma unroll
  for (int g = 0; g < GMAX; ++g) lse[g] = g < G ? in.lse_ws[(size_t)s * G + g] * kLog2eF : 0.0f;   // log2 units
  const int n_cold = c.n_cold[s];
  const int t = c.next_pos[s] - 1;
  if (!(n_cold >= 0 && n_cold <= c.cap && t >= -1)) {   // the same answer in every thread
    if (threadIdx.x == 0) record_violation(c.err, kSiteEmaSeg, s, n_cold);
    return false;
  }
  const float* sb = in.scores + (size_t)s * G * in.score_stride;
  float* scc = c.sc_c + (size_t)s * c.cap;
  const int32_t* pc = c.pos_c + (size_t)s * c.cap;
  // Confidence mode: every score is at least (1 - alpha)/(t + 1) (a recency
  // term of at least 1/(t + 1), an EMA of probabilities >= 0), so a fixed bin
  // map from half that up to 2 is known now and the select's histogram is
  // built here, as the keys are computed (kSelBins 32-bit counts in `hist`).
  KeyBins bins{0u, 0};
  const bool binned = pol.mode == 0 && pol.one_minus_alpha > 0.0f && t >= 0;
  if (binned) {
    bins.lo = ordered_bits(0.5f * pol.one_minus_alpha / (float)(t + 1));
    const uint32_t span = ordered_bits(2.0f) - bins.lo;
    while ((span >> bins.shift) >= (uint32_t)kSelBins) ++bins.shift;
    for (int i = threadIdx.x; i < kSelBins; i += NT) hist[i] = 0u;
    __syncthreads();
  }
  // four consecutive keys (nq of them valid) into the histogram, runs of one
  // bin added at once
  auto hist_add = [&](uint32_t h0, uint32_t h1, uint32_t h2, uint32_t h3, int nq) {
    const uint32_t hh[4] = {h0, h1, h2, h3};
    int cur = -1;
    uint32_t cnt = 0u;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (q < nq && hh[q] != 0xFFFFFFFFu) {
        const int bq = bins(hh[q]);
        if (bq != cur) {
          if (cnt) atomicAdd(&hist[cur], cnt);
          cur = bq;
          cnt = 0u;
        }
        ++cnt;
      }
    }
    if (cnt) atomicAdd(&hist[cur], cnt);
  };
  auto hi_of = [&](int pos, float sc) -> uint32_t {
    const bool none = pos < 0 || t - pos < pol.P || pos < pol.n_sink;
    return none ? 0xFFFFFFFFu : (uint32_t)(rank_key(pol, sc, pos, t) >> 32);
  };
  uint32_t kmn = 0xFFFFFFFFu, kmx = 0u;
  auto track = [&](uint32_t hv) {
    if (hv != 0xFFFFFFFFu) {
      kmn = min(kmn, hv);
      kmx = max(kmx, hv);
    }
  };
  // cold region: four consecutive tokens per thread, two groups in flight
  for (int base = 0; base < n_cold; base += 8 * NT) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i0 = base + 4 * NT * u + 4 * (int)threadIdx.x;
      if (i0 + 3 < n_cold) {
        const float4 e =
            ema_update4<GMAX>(sb, in.score_stride, i0, *reinterpret_cast<const float4*>(scc + i0), lse, G, invG, pol);
        const int4 p4 = *reinterpret_cast<const int4*>(pc + i0);
        *reinterpret_cast<float4*>(scc + i0) = e;
        const uint4 hv = make_uint4(hi_of(p4.x, e.x), hi_of(p4.y, e.y), hi_of(p4.z, e.z), hi_of(p4.w, e.w));
        *reinterpret_cast<uint4*>(khi + i0) = hv;
        track(hv.x);
        track(hv.y);
        track(hv.z);
        track(hv.w);
        if (binned) hist_add(hv.x, hv.y, hv.z, hv.w, 4);
      } else if (i0 < n_cold) {   // the last, partial group
        const float4 e =
            ema_update4<GMAX>(sb, in.score_stride, i0, *reinterpret_cast<const float4*>(scc + i0), lse, G, invG, pol);
        const int4 p4 = *reinterpret_cast<const int4*>(pc + i0);
        const int pp[3] = {p4.x, p4.y, p4.z};
        const float ee[3] = {e.x, e.y, e.z};
        uint32_t hq[3] = {0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu};
#pragma unroll
        for (int q = 0; q < 3; ++q)
          if (i0 + q < n_cold) {
            scc[i0 + q] = ee[q];
            const uint32_t h = hi_of(pp[q], ee[q]);
            khi[i0 + q] = h;
            track(h);
            hq[q] = h;
          }
        if (binned) hist_add(hq[0], hq[1], hq[2], 0xFFFFFFFFu, 3);
      }
    }
  }
  // window ring: occupied slots only (the ring stride is a multiple of 64)
  const int32_t* pr = c.pos_r + (size_t)s * c.Wst;
  float* scr = c.sc_r + (size_t)s * c.Wst;
  int ring_here = 0;
  for (int s0 = 4 * (int)threadIdx.x; s0 < c.W; s0 += 4 * NT) {
    const int4 p4 = *reinterpret_cast<const int4*>(pr + s0);
    const float4 e = ema_update4<GMAX>(sb, in.score_stride, c.cap + s0, *reinterpret_cast<const float4*>(scr + s0),
                                       lse, G, invG, pol);
    const int pp[4] = {p4.x, p4.y, p4.z, p4.w};
    const float ee[4] = {e.x, e.y, e.z, e.w};
    uint32_t hq[4] = {0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (s0 + q < c.W) {
        uint32_t h = 0xFFFFFFFFu;
        if (pp[q] >= 0) {
          scr[s0 + q] = ee[q];
          ++ring_here;
          h = hi_of(pp[q], ee[q]);
        }
        khi[n_cold + s0 + q] = h;
        track(h);
        hq[q] = h;
      }
    }
    if (binned) hist_add(hq[0], hq[1], hq[2], hq[3], 4);
  }
  bk->n_ring = block_sum_int<NT>(ring_here, sm);   // includes a block barrier: the keys are visible
  bk->kmn = kmn;
  bk->kmx = kmx;
  bk->binned = binned;
  bk->bins = bins;
  return true;
}

// The bulk variant of the fused kernel: a persistent grid whose CTAs claim
// one segment at a time, run its EMA pass with every thread (writing the
// keys), then evict it by the whole-CTA path. Claiming lets the CTAs of an
// SM drift apart, so that one streams its segment while another selects.
template <int D, bool CI8, int GMAX>
__global__ void __launch_bounds__(NT, 3) evict_bulk_kernel(Cache c, Policy pol, EvictLaunch a, EmaIn ein,
                                                           int items) {
  chain_enter();
  __shared__ EvictSmem es;
  __shared__ int claimed;
  uint32_t* khi = a.kscratch + (size_t)blockIdx.x * a.scratch_stride;
  while (true) {
    if (threadIdx.x == 0) claimed = atomicAdd(a.bulk_sched, 1);
    __syncthreads();
    const int item = claimed;
    __syncthreads();   // every thread has read it before the next claim
    if (item >= items) break;
    int l, b, h;
    const int s = seg_of(c, a.r, item, &l, &b, &h);
    BlockKeys bk;
    if (!cta_ema_keys<GMAX>(c, ein, pol, s, khi, &bk, es.sm, reinterpret_cast<uint32_t*>(es.stage))) continue;
    evict_segment_block<D, CI8>(c, pol, a, item, es, &bk);
    __syncthreads();
  }
  // the last CTA to finish resets the counters for the next launch
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(a.bulk_sched + 1, 1) == (int)gridDim.x - 1) {
      a.bulk_sched[0] = 0;
      a.bulk_sched[1] = 0;
    }
  }
}

template <int D, bool CI8, int GMAX>
cudaError_t run_bulk(const Cache& c, const Policy& pol, const EvictLaunch& a, const EmaIn& ema, int num_sms,
                     cudaStream_t st) {
  const int items = a.r.items(c.Hkv);
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, evict_bulk_kernel<D, CI8, GMAX>, NT, 0);
  if (e != cudaSuccess) return e;
  // the key scratch exists for evict_grid(items) CTAs (or more)
  const int grid = max(1, min(evict_grid(items), max(1, per_sm) * num_sms));
  (void)launch_chained(evict_bulk_kernel<D, CI8, GMAX>, grid, NT, 0, st, c, pol, a, ema, items);
  return cudaGetLastError();
}

// One segment per CTA by the whole-CTA path (calls over few segments).
template <int D, bool CI8>
__global__ void __launch_bounds__(NT) evict_block_kernel(Cache c, Policy pol, EvictLaunch a, int items) {
  chain_enter();
  __shared__ EvictSmem es;
  if ((int)blockIdx.x < items) evict_segment_block<D, CI8>(c, pol, a, (int)blockIdx.x, es);
}

template <int D, bool CI8>
cudaError_t run(const Cache& c, const Policy& pol, const EvictLaunch& a, const EmaIn* ema, cudaStream_t st,
                long long* launches, Prof* prof) {
  const int items = a.r.items(c.Hkv);
  const int grid = evict_grid(items);
  if (ema == nullptr) {
    ProfScope ps(prof, kKEvict, st);
    (void)launch_chained(evict_kernel<D, CI8, 0>, grid, NT, 0, st, c, pol, a, EmaIn{}, items);
  } else {
    ProfScope ps(prof, kKEmaEvict, st);
    if (c.G <= 4)
      (void)launch_chained(evict_kernel<D, CI8, 4>, grid, NT, 0, st, c, pol, a, *ema, items);
    else
      (void)launch_chained(evict_kernel<D, CI8, 8>, grid, NT, 0, st, c, pol, a, *ema, items);
  }
  ++*launches;
  return cudaGetLastError();
}

}  // namespace

int evict_grid(int items) { return (items + kSegsPerCta - 1) / kSegsPerCta; }

int few_segment_limit(int num_sms) { return 2 * num_sms; }

cudaError_t launch_evict_compact(const Cache& c, const Policy& pol, const EvictLaunch& a, const EmaIn* ema,
                                 bool bulk, int num_sms, cudaStream_t st, long long* launches, Prof* prof) {
  const int items = a.r.items(c.Hkv);
  if (items == 0) return cudaSuccess;
  if (ema != nullptr && (pol.mode != 0 || c.G < 1 || c.G > 8)) return cudaErrorInvalidValue;
  const bool few = items <= few_segment_limit(num_sms) && items <= a.scratch_ctas;
  if (ema == nullptr && few) {
    // too few segments to fill the GPU one warp each: one CTA per segment
    ProfScope ps(prof, kKEvict, st);
    if (c.D == 128)
      (void)(c.cold_int8 ? launch_chained(evict_block_kernel<128, true>, items, NT, 0, st, c, pol, a, items)
                         : launch_chained(evict_block_kernel<128, false>, items, NT, 0, st, c, pol, a, items));
    else
      (void)(c.cold_int8 ? launch_chained(evict_block_kernel<64, true>, items, NT, 0, st, c, pol, a, items)
                         : launch_chained(evict_block_kernel<64, false>, items, NT, 0, st, c, pol, a, items));
    ++*launches;
    return cudaGetLastError();
  }
  if (ema != nullptr && bulk) {
    ProfScope ps(prof, kKEmaEvict, st);
    cudaError_t e;
    if (c.D == 128)
      e = c.cold_int8 ? (c.G <= 4 ? run_bulk<128, true, 4>(c, pol, a, *ema, num_sms, st)
                                  : run_bulk<128, true, 8>(c, pol, a, *ema, num_sms, st))
                      : (c.G <= 4 ? run_bulk<128, false, 4>(c, pol, a, *ema, num_sms, st)
                                  : run_bulk<128, false, 8>(c, pol, a, *ema, num_sms, st));
    else
      e = c.cold_int8 ? (c.G <= 4 ? run_bulk<64, true, 4>(c, pol, a, *ema, num_sms, st)
                                  : run_bulk<64, true, 8>(c, pol, a, *ema, num_sms, st))
                      : (c.G <= 4 ? run_bulk<64, false, 4>(c, pol, a, *ema, num_sms, st)
                                  : run_bulk<64, false, 8>(c, pol, a, *ema, num_sms, st));
    ++*launches;
    return e;
  }
  if (c.D == 128)
    return c.cold_int8 ? run<128, true>(c, pol, a, ema, st, launches, prof)
                       : run<128, false>(c, pol, a, ema, st, launches, prof);
  return c.cold_int8 ? run<64, true>(c, pol, a, ema, st, launches, prof)
                     : run<64, false>(c, pol, a, ema, st, launches, prof);
}

}  // namespace confkv
