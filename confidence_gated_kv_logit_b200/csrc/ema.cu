// Attention-mass EMA: the second pass of decode attention, with the saved
// log-sum-exp. Per token, the mean over the G query heads of exp(s - lse)
// enters the EMA (CONF-KV post, pseudo-code update_ema); every token's
// eviction key is computed from the new value, and the segment's kCandMax
// smallest keys go to its candidate record for the eviction kernel.
//
// In the steady decode step the pass runs inside the eviction kernel (its
// fused variant, evict.cu), which evicts straight from the merged keys. The
// kernels here run it on its own, when something needs the EMA values before
// the next eviction (or a handle runs every pass inside its decode call):
//
//   ema_kernel     : one warp per segment, eight segments per CTA (calls over
//                    many segments, e.g. all layers at once): the pass of
//                    ema_warp.cuh, whose merged keys become the segment's
//                    candidate record.
//   ema_cta_kernel : one CTA of four warps per segment (calls over few
//                    segments, e.g. one layer: four warps each still fit in
//                    one wave and shorten the longest segment's chain of
//                    round trips fourfold), with a two-level candidate merge.
#include <math_constants.h>

#include "common.cuh"
#include "kernels.h"
#include "ema_warp.cuh"
#include "warp_select.cuh"

namespace confkv {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// One warp per segment; the pass itself is ema_segment_warp (ema_warp.cuh).
// Its merged keys become the segment's candidate record for the eviction
// kernel (which then need not rescan the segment).
template <int GMAX>
__global__ void __launch_bounds__(256) ema_kernel(Cache c, AttnLaunch a, Policy pol) {
  chain_enter();
  const int lane = threadIdx.x & 31;
  const int item = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (item >= a.r.items(c.Hkv)) return;
  int l, b, h;
  const int s = seg_of(c, a.r, item, &l, &b, &h);
  EmaOut o;
  ema_segment_warp<GMAX>(c, EmaIn{a.lse_ws, a.scores, a.score_stride}, pol, s, lane, &o);
  if (!o.ok || a.cand == nullptr) return;
  EvictCand* cd = a.cand + s;
  if (lane < kCandMax) {
    cd->key[lane] = o.key;
    cd->idx[lane] = o.idx;
  }
  if (lane == 0) {
    cd->n_ring = o.n_ring;
    cd->safe = o.safe;
    cd->n_cold = o.n_cold;
    cd->stamp = o.t + 1;
  }
}

// Two-level candidate merge, used by the CTA variant: each warp merges its
// lanes' lists into its kWarpWant smallest keys (with a bound: every key of
// the warp's tokens <= bound is in its list); warp 0 ranks the 32 keys. Every
// key of the segment <= the smallest bound is among the 32, so a ranked key up
// to that bound is certainly the segment's key of that rank.
constexpr int kCtaWarps = 4;
constexpr int kCtaThreads = 32 * kCtaWarps;
constexpr int kWarpWant = 8;
static_assert(kCtaWarps * kWarpWant == 32, "the final merge holds one key per lane");

template <int GMAX>
__global__ void __launch_bounds__(kCtaThreads, 8) ema_cta_kernel(Cache c, AttnLaunch a, Policy pol) {
  chain_enter();
  __shared__ unsigned long long w_key[kCtaWarps * kWarpWant];
  __shared__ int w_idx[kCtaWarps * kWarpWant];
  __shared__ unsigned long long w_bound[kCtaWarps];
  __shared__ int w_ring[kCtaWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int l, b, h;
  const int s = seg_of(c, a.r, blockIdx.x, &l, &b, &h);
  const int G = c.G;
  const float invG = 1.0f / (float)G;
  float lse[GMAX];
#pragma unroll
  for (int g = 0; g < GMAX; ++g) lse[g] = g < G ? a.lse_ws[(size_t)s * G + g] * kLog2e : 0.0f;   // log2 units
  const int n_cold = c.n_cold[s];
  const int t = c.next_pos[s] - 1;
  if (!(n_cold >= 0 && n_cold <= c.cap)) {   // the same answer in every thread of the CTA
    if (tid == 0) record_violation(c.err, kSiteEmaSeg, s, n_cold);
    return;
  }
  const float* sb = a.scores + (size_t)s * G * a.score_stride;
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
  // cold region: thread k takes four tokens per 512, two groups per round
  for (int base = 0; base < n_cold; base += 8 * kCtaThreads) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i0 = base + 4 * kCtaThreads * u + 4 * tid;
      if (i0 + 3 < n_cold) {
        const float4 e = ema_update4<GMAX>(sb, a.score_stride, i0, *reinterpret_cast<const float4*>(scc + i0), lse, G, invG, pol);
        const int4 p4 = *reinterpret_cast<const int4*>(pc + i0);
        *reinterpret_cast<float4*>(scc + i0) = e;
        if (min(min(p4.x, p4.y), min(p4.z, p4.w)) + 1 <= best.pos_bound) {
          offer(p4.x, e.x, i0);
          offer(p4.y, e.y, i0 + 1);
          offer(p4.z, e.z, i0 + 2);
          offer(p4.w, e.w, i0 + 3);
        }
      } else if (i0 < n_cold) {   // the last, partial group
        const float4 e = ema_update4<GMAX>(sb, a.score_stride, i0, *reinterpret_cast<const float4*>(scc + i0), lse, G, invG, pol);
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
  for (int s0 = 4 * tid; s0 < c.W; s0 += 4 * kCtaThreads) {
    const int4 p4 = *reinterpret_cast<const int4*>(pr + s0);
    const float4 e = ema_update4<GMAX>(sb, a.score_stride, c.cap + s0, *reinterpret_cast<const float4*>(scr + s0), lse, G, invG, pol);
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
  if (a.cand == nullptr) return;   // the same answer in every thread
  {
    const int ring_w = __reduce_add_sync(0xffffffffu, ring_here);
    unsigned long long mk, bound;
    int mi, cnt, safe_w;
    warp_merge_smallest(best, lane, kWarpWant, &mk, &mi, &cnt, &safe_w, &bound);
    if (lane < kWarpWant) {
      w_key[warp * kWarpWant + lane] = lane < cnt ? mk : kNoKey;
      w_idx[warp * kWarpWant + lane] = mi;
    }
    if (lane == 0) {
      w_bound[warp] = bound;
      w_ring[warp] = ring_w;
    }
  }
  __syncthreads();
  if (warp != 0) return;
  const unsigned long long k = w_key[lane];
  const int ix = w_idx[lane];
  unsigned long long lim = w_bound[0];
  int n_ring = w_ring[0];
#pragma unroll
  for (int w = 1; w < kCtaWarps; ++w) {
    lim = w_bound[w] < lim ? w_bound[w] : lim;
    n_ring += w_ring[w];
  }
  // rank among the valid keys (keys are distinct: the position is their low half)
  int rank = 0;
#pragma unroll 8
  for (int j = 0; j < 32; ++j) rank += w_key[j] < k ? 1 : 0;
  const bool valid = k != kNoKey;
  const int n = __popc(__ballot_sync(0xffffffffu, valid));
  const int safe = __popc(__ballot_sync(0xffffffffu, valid && rank < kCandMax && k <= lim));
  EvictCand* cd = a.cand + s;
  if (valid && rank < kCandMax) {
    cd->key[rank] = k;
    cd->idx[rank] = ix;
  }
  if (lane >= n && lane < kCandMax) {   // the slots past the n candidates
    cd->key[lane] = kNoKey;
    cd->idx[lane] = -1;
  }
  if (lane == 0) {
    cd->n_ring = n_ring;
    cd->safe = safe;
    cd->n_cold = n_cold;
    cd->stamp = t + 1;
  }
}

template <int GMAX>
void launch_ema(const Cache& c, const Policy& pol, const AttnLaunch& a, cudaStream_t st) {
  const int items = a.r.items(c.Hkv);
  // four warps per segment while they fit in one wave (about 32 warps per SM)
  if ((long long)items * kCtaWarps <= (long long)a.num_sms * 32)
    (void)launch_chained(ema_cta_kernel<GMAX>, items, kCtaThreads, 0, st, c, a, pol);
  else
    (void)launch_chained(ema_kernel<GMAX>, (items + 7) / 8, 256, 0, st, c, a, pol);
}

}  // namespace

cudaError_t run_ema(const Cache& c, const Policy& pol, const AttnLaunch& a, cudaStream_t st) {
  if (c.G < 1 || c.G > 8) return cudaErrorInvalidValue;
  if (c.G <= 4) launch_ema<4>(c, pol, a, st);
  else launch_ema<8>(c, pol, a, st);
  return cudaGetLastError();
}

}  // namespace confkv
