// The attention-mass EMA of one segment by one warp (the second pass of
// decode attention, with the saved log-sum-exp): per token, the mean over the
// G query heads of exp(s - lse) enters the EMA (CONF-KV post, pseudo-code
// update_ema), the token's eviction key is computed from the new value, and
// the segment's kCandMax smallest keys are merged across the warp.
//
// Used by the EMA kernel (which stores the merged keys as the segment's
// candidate record for a later eviction call) and by the eviction kernel's
// fused variant (which runs this pass and then evicts from the merged keys
// directly), so that both give the same EMA values and keys bit for bit.
#pragma once

#include "common.cuh"
#include "kernels.h"
#include "warp_select.cuh"

namespace confkv {

// The merged candidates of one segment: lane j < count holds the j-th
// smallest key and its index (cold index, or n_cold + ring slot); `safe` of
// them are certainly the segment's smallest; the occupied window slots; and
// the segment counters the pass saw.
struct EmaOut {
  unsigned long long key;
  int idx;
  int count, safe, n_ring;
  int n_cold, t;
  bool ok;   // false: the segment's counters were corrupt (recorded, nothing written)
};

// fl(beta*e + (1-beta)*(mean over the first G of GMAX score rows of
// 2^(s - lse))) for four consecutive tokens; runtime G <= GMAX, rows summed
// in order.
template <int GMAX>
__device__ __forceinline__ float4 ema_update4(const float* __restrict__ sb, int stride, int col, float4 e,
                                              const float (&lse)[GMAX], int G, float invG, const Policy& pol) {
  float sum[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int g = 0; g < GMAX; ++g) {
    if (g < G) {
      const float4 v = *reinterpret_cast<const float4*>(sb + (size_t)g * stride + col);   // log2 units
      sum[0] += ex2(v.x - lse[g]);
      sum[1] += ex2(v.y - lse[g]);
      sum[2] += ex2(v.z - lse[g]);
      sum[3] += ex2(v.w - lse[g]);
    }
  }
  e.x = fmaf(pol.beta, e.x, pol.one_minus_beta * (sum[0] * invG));
  e.y = fmaf(pol.beta, e.y, pol.one_minus_beta * (sum[1] * invG));
  e.z = fmaf(pol.beta, e.z, pol.one_minus_beta * (sum[2] * invG));
  e.w = fmaf(pol.beta, e.w, pol.one_minus_beta * (sum[3] * invG));
  return e;
}

// The pass over segment s by one warp. Every lane returns the same counts.
template <int GMAX>
__device__ __forceinline__ void ema_segment_warp(const Cache& c, const EmaIn& in, const Policy& pol, int s, int lane,
                                                 EmaOut* o) {
  constexpr float kLog2eF = 1.4426950408889634f;
  const int G = c.G;
  const float invG = 1.0f / (float)G;
  float lse[GMAX];
#pragma unroll
  for (int g = 0; g < GMAX; ++g) lse[g] = g < G ? in.lse_ws[(size_t)s * G + g] * kLog2eF : 0.0f;   // log2 units
  const int n_cold = c.n_cold[s];
  const int t = c.next_pos[s] - 1;
  o->n_cold = n_cold;
  o->t = t;
  o->ok = n_cold >= 0 && n_cold <= c.cap;
  if (!o->ok) {
    if (lane == 0) record_violation(c.err, kSiteEmaSeg, s, n_cold);
    return;
  }
  const float* sb = in.scores + (size_t)s * G * in.score_stride;
  float* scc = c.sc_c + (size_t)s * c.cap;
  const int32_t* pc = c.pos_c + (size_t)s * c.cap;
  LaneBest best;
  best.init();
  const bool use_bound = pol.one_minus_alpha >= 0x1p-60f;
  const float t1_over_oma = use_bound ? (float)(t + 1) / pol.one_minus_alpha : 0.0f;
  auto offer = [&](int pos, float ema, int idx) {
    if (pos + 1 > best.pos_bound) return;
    if (t - pos < pol.P || pos < pol.n_sink) return;   // protected: never a victim
    best.offer(rank_key(pol, ema, pos, t), idx);
    if (use_bound) best.update_bound(t1_over_oma);
  };
  // cold region [0, n_cold): the region and the score rows are multiples of 64
  // long. Each lane takes four tokens per 128, two such groups in flight. A
  // group of four whose smallest position is past the lane's bound offers
  // nothing (one test for the group: the common case once the list is full).
  for (int base = 0; base < n_cold; base += 256) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i0 = base + 128 * u + 4 * lane;
      if (i0 + 3 < n_cold) {
        const float4 e =
            ema_update4<GMAX>(sb, in.score_stride, i0, *reinterpret_cast<const float4*>(scc + i0), lse, G, invG, pol);
        const int4 p4 = *reinterpret_cast<const int4*>(pc + i0);
        *reinterpret_cast<float4*>(scc + i0) = e;
        if (min(min(p4.x, p4.y), min(p4.z, p4.w)) + 1 <= best.pos_bound) {
          offer(p4.x, e.x, i0);
          offer(p4.y, e.y, i0 + 1);
          offer(p4.z, e.z, i0 + 2);
          offer(p4.w, e.w, i0 + 3);
        }
      } else if (i0 < n_cold) {   // the last, partial group
        const float4 e =
            ema_update4<GMAX>(sb, in.score_stride, i0, *reinterpret_cast<const float4*>(scc + i0), lse, G, invG, pol);
        const int4 p4 = *reinterpret_cast<const int4*>(pc + i0);
        scc[i0] = e.x;
        offer(p4.x, e.x, i0);
        if (i0 + 1 < n_cold) {
          scc[i0 + 1] = e.y;
          offer(p4.y, e.y, i0 + 1);
        }
        if (i0 + 2 < n_cold) {
          scc[i0 + 2] = e.z;
          offer(p4.z, e.z, i0 + 2);
        }
      }
    }
  }
  // window ring: occupied slots only (the ring stride is a multiple of 64)
  const int32_t* pr = c.pos_r + (size_t)s * c.Wst;
  float* scr = c.sc_r + (size_t)s * c.Wst;
  int ring_here = 0;
  for (int s0 = 4 * lane; s0 < c.W; s0 += 128) {
    const int4 p4 = *reinterpret_cast<const int4*>(pr + s0);
    const float4 e = ema_update4<GMAX>(sb, in.score_stride, c.cap + s0, *reinterpret_cast<const float4*>(scr + s0),
                                       lse, G, invG, pol);
    const int pp[4] = {p4.x, p4.y, p4.z, p4.w};
    const float ee[4] = {e.x, e.y, e.z, e.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (s0 + q < c.W && pp[q] >= 0) {
        scr[s0 + q] = ee[q];
        ++ring_here;
        offer(pp[q], ee[q], n_cold + s0 + q);
      }
    }
  }
  o->n_ring = __reduce_add_sync(0xffffffffu, ring_here);
  warp_merge_smallest(best, lane, kCandMax, &o->key, &o->idx, &o->count, &o->safe);
}

}  // namespace confkv
