// Eviction, compaction and conversion of the token leaving the FP16 window,
// one CTA per segment (CONF-KV post, decode-loop pseudo-code: evict only when
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
//      smallest are the victims: argmin when e = 1 (the steady state: one new
//      token per step), MSD radix select otherwise (budget drops, step 1).
//   3. victims in the window ring free their slot; victims in the cold region
//      are recorded in a bitmask and the region is compacted: hole-fill moves
//      the survivors above the new end into the holes below it (bytes
//      proportional to e), stable compaction shifts every survivor after the
//      first hole down in order. Both leave the same logical content.
//   4. the token that the next append would push out of the window
//      (position t+1-W) is quantised into the end of the cold region.
#include "common.cuh"
#include "kernels.h"
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
  int scanned = 0, moved = 0, requant = 0;
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
                                   WarpCounts* wc, int* ws_pairs) {
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
  // This step's EMA pass may have left the segment's smallest keys and its
  // window slot count (confidence mode): then nothing needs rescanning.
  EvictCand* cd = a.cand != nullptr ? a.cand + s : nullptr;
  bool have = false;
  int n_ring = 0, count = 0, safe = 0;
  unsigned long long my_key = kNoKey;
  int my_idx = -1;
  if (cd != nullptr && pol.mode == 0 && !a.stable && cd->stamp == t + 1 && cd->n_cold == n_cold) {
    have = true;
    n_ring = cd->n_ring;
    safe = cd->safe;
    if (lane < kCandMax) {
      my_key = cd->key[lane];
      my_idx = cd->idx[lane];
    }
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
  const int leaving = t + 1 - W;
  if (CI8 && W > 0 && leaving >= 0) {
    const int slot = (t + 1) % W;
    const size_t rs = (size_t)s * c.Wst + slot;
    if (c.pos_r[rs] == leaving) {
      const int idx = n_cold_new;
      if (idx >= c.cap || idx < 0) {
        if (lane == 0) record_violation(c.err, kSiteEvictRequant, s, idx);
      } else {
        const size_t cs = (size_t)s * c.cap + idx;
        warp_requant<D>(c, s, slot, idx, lane);
        __syncwarp();
        if (lane == 0) {
          c.pos_c[cs] = leaving;
          c.sc_c[cs] = c.sc_r[rs];
          c.pos_r[rs] = -1;
        }
        n_cold_new = idx + 1;
        requant = 1;
      }
    }
  }
  if (lane == 0) c.n_cold[s] = n_cold_new;
  wc->scanned = have ? 0 : n;   // tokens whose keys this call read
  wc->moved = moved;
  wc->requant = requant;
  return true;
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
template <int D, bool CI8>
__device__ void evict_segment_block(const Cache& c, const Policy& pol, const EvictLaunch& a, int item,
                                    EvictSmem& es) {
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

  int ring_here = 0;
  for (int slot = threadIdx.x; slot < W; slot += NT) ring_here += pos_r[slot] >= 0;
  const int n_ring = block_sum_int<NT>(ring_here, sm);
  const int n = n_cold + n_ring;
  const int budget_eff = pol.mode == 1 ? pol.fixed_budget
                                       : max(a.budget[(size_t)b * c.L + l], pol.P + pol.n_sink);
  const int e = n - budget_eff;
  int n_cold_new = n_cold;
  int moved = 0;

  if (e > 0 && t >= 0) {
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
      // steady state: one victim; its index comes with the argmin, and at most
      // one row (the last cold row) moves into its place
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
    const SelectResult sel = block_select_smallest<NT>(key, span, e, sm);

    // victim bitmask of the cold region (one ballot per 32 tokens), and count
    int ecold_here = 0;
    for (int base = 0; base < n_cold; base += NT) {
      const int i = base + (int)threadIdx.x;
      const bool v = i < n_cold && is_selected(key(i), sel);
      const unsigned bal = __ballot_sync(0xffffffffu, v);
      if ((threadIdx.x & 31) == 0 && i < n_cold) {
        vm[i >> 5] = bal;
        ecold_here += __popc(bal);
      }
    }
    // window victims free their slot (each thread reads and writes only its own slots)
    for (int slot = threadIdx.x; slot < W; slot += NT)
      if (is_selected(key(n_cold + slot), sel)) pos_r[slot] = -1;
    const int e_cold = block_sum_int<NT>(ecold_here, sm);   // includes a block barrier: vm is visible
    const int n_keep = n_cold - e_cold;

    if (e_cold == 0) {
      // every victim was in the window ring: the cold region is unchanged
    } else if (!a.stable) {
      // hole-fill: pair the k-th hole below n_keep with the k-th survivor above it
      int hcur = 0, mcur = n_keep;
      while (true) {
        const int nh = block_collect<NT, NT>([&](int i) { return victim(i); }, &hcur, n_keep, list_h, sm);
        const int nm = block_collect<NT, NT>([&](int i) { return !victim(i); }, &mcur, n_cold, list_m, sm);
        const int np = min(nh, nm);
        if (np == 0) break;
        for (int w = threadIdx.x; w < np * R::NP; w += NT) {
          const int p = w / R::NP;
          if (kChecked && !guard(list_h[p] >= 0 && list_h[p] < n_keep && list_m[p] >= n_keep && list_m[p] < n_cold,
                                 c.err, kSiteEvictPair, s, list_m[p]))
            continue;
          move_cold_row<D, CI8>(c, s, list_m[p], list_h[p], w - p * R::NP);
        }
        moved += np;
        __syncthreads();
      }
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
  if (W > 0 && leaving >= 0 && threadIdx.x < 32) {
    const int slot = (t + 1) % W;
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
  if (threadIdx.x == 0) {
    c.n_cold[s] = n_cold_new;
    atomicAdd(&c.counters[kCntEvictBlock], 1ull);
    if (a.cand != nullptr) a.cand[s].stamp = -1;
    atomicAdd(&c.counters[kCntEvictScanned], (unsigned long long)n);
    if (moved > 0) atomicAdd(&c.counters[kCntMovedRows], (unsigned long long)moved);
  }
}

template <int D, bool CI8>
__global__ void __launch_bounds__(NT, 4) evict_kernel(Cache c, Policy pol, EvictLaunch a, int items) {
  __shared__ EvictSmem es;
  __shared__ int slow_items[kSegsPerCta];
  __shared__ int n_slow;
  __shared__ unsigned long long cnt[3];
  __shared__ int pairs[kSegsPerCta][2 * kWarpMaxVictims];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) n_slow = 0;
  if (threadIdx.x < 3) cnt[threadIdx.x] = 0;
  __syncthreads();
  // Segments are dealt to warps through a multiplicative bijection of
  // [0, items) (the multiplier is a prime above any item count), so that the
  // segments of one sequence, which share a budget and so need the whole-CTA
  // path at the same steps, land in different CTAs.
  const int slot = blockIdx.x * kSegsPerCta + warp;
  const int item = slot < items ? (int)(((unsigned long long)slot * 2654435761ull) % (unsigned long long)items) : items;
  if (item < items) {
    WarpCounts wc;
    if (!evict_segment_warp<D, CI8>(c, pol, a, item, lane, &wc, pairs[warp])) {
      if (lane == 0) slow_items[atomicAdd(&n_slow, 1)] = item;
    } else if (lane == 0) {
      if (wc.scanned) atomicAdd(&cnt[0], (unsigned long long)wc.scanned);
      if (wc.moved) atomicAdd(&cnt[1], (unsigned long long)wc.moved);
      if (wc.requant) atomicAdd(&cnt[2], (unsigned long long)wc.requant);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (cnt[0]) atomicAdd(&c.counters[kCntEvictScanned], cnt[0]);
    if (cnt[1]) atomicAdd(&c.counters[kCntMovedRows], cnt[1]);
    if (cnt[2]) atomicAdd(&c.counters[kCntRequant], cnt[2]);
  }
  const int ns = n_slow;
  for (int k = 0; k < ns; ++k) {
    __syncthreads();   // the previous segment's shared-memory use is over
    evict_segment_block<D, CI8>(c, pol, a, slow_items[k], es);
  }
}

template <int D, bool CI8>
cudaError_t run(const Cache& c, const Policy& pol, const EvictLaunch& a, cudaStream_t st, long long* launches,
                Prof* prof) {
  const int items = a.r.items(c.Hkv);
  ProfScope ps(prof, kKEvict, st);
  evict_kernel<D, CI8><<<(items + kSegsPerCta - 1) / kSegsPerCta, NT, 0, st>>>(c, pol, a, items);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_evict_compact(const Cache& c, const Policy& pol, const EvictLaunch& a, cudaStream_t st,
                                 long long* launches, Prof* prof) {
  if (a.r.items(c.Hkv) == 0) return cudaSuccess;
  if (c.D == 128)
    return c.cold_int8 ? run<128, true>(c, pol, a, st, launches, prof) : run<128, false>(c, pol, a, st, launches, prof);
  return c.cold_int8 ? run<64, true>(c, pol, a, st, launches, prof) : run<64, false>(c, pol, a, st, launches, prof);
}

}  // namespace confkv
