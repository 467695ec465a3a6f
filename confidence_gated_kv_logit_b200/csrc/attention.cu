// Decode attention over the mixed FP16/INT8 cache (CONF-KV abstract: the
// policy is combined with blockwise online-softmax attention and mixed
// FP16/INT8 storage; CONF-KV post, implementation note: INT8 is dequantised
// inside the attention kernel).
//
//   append_kernel     : writes the new token into the FP16 window ring (or the
//                       cold region when INT8 is off)
//   attn_kernel       : persistent, warp-specialised split-K attention. One
//                       producer warp streams K/V tiles and their scales or
//                       positions into a 3-stage shared-memory ring with 1-D
//                       TMA bulk copies; four consumer warps compute scores,
//                       an online softmax with lazy rescaling, and P.V with the
//                       INT8 codes converted in registers (byte permute into
//                       the fp32 mantissa) and packed f32x2 FMAs. The per-token
//                       scale of K multiplies the dot product; the scale of V
//                       is folded into the probability. No tensor cores: one
//                       query row per KV head is a GEMV.
//   combine_kernel    : merges split partials into out and lse
//   ema_kernel        : second pass with the saved log-sum-exp: per token the
//                       mean over the G query heads of exp(s - lse) enters the
//                       attention-mass EMA (CONF-KV post, pseudo-code update_ema)
#include <math_constants.h>

#include "common.cuh"
#include "kernels.h"
#include "tma.cuh"

namespace confkv {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------------------
// append: one warp per segment. If the window slot of the new position still
// holds a token (a caller skipped eviction), that token is converted to INT8
// first, exactly as eviction would have done.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) append_kernel(Cache c, Range r, const __half* __restrict__ k_new,
                                                     const __half* __restrict__ v_new,
                                                     const float* __restrict__ prio_new, int fixed_mode) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= r.items(c.Hkv)) return;
  int l, b, h;
  const int s = seg_of(c, r, warp, &l, &b, &h);
  const int t = c.next_pos[s];
  if (!guard(t >= 0 && c.n_cold[s] >= 0 && c.n_cold[s] <= c.cap, c.err, kSiteAppendSeg, s, t)) return;
  const size_t in_row = ((size_t)((l - r.l0) * r.B + b) * c.Hkv + h);
  const __half* kn = k_new + in_row * D;
  const __half* vn = v_new + in_row * D;
  const float sc_new = fixed_mode ? prio_new[in_row] : 0.0f;
  if (c.W > 0) {
    const int slot = t % c.W;
    const size_t rs = (size_t)s * c.Wst + slot;
    const int old = c.pos_r[rs];
    if (old >= 0) {
      const int idx = c.n_cold[s];
      if (idx >= c.cap) {
        if (lane == 0) set_error(c.err, kErrDevice);
        return;
      }
      const size_t cs = (size_t)s * c.cap + idx;
      warp_quantize_row<D>(c.kr + rs * D, c.k8 + cs * D, c.ks + cs, lane);
      warp_quantize_row<D>(c.vr + rs * D, c.v8 + cs * D, c.vs + cs, lane);
      if (lane == 0) {
        c.pos_c[cs] = old;
        c.sc_c[cs] = c.sc_r[rs];
        c.n_cold[s] = idx + 1;
        atomicAdd(&c.counters[kCntRequant], 1ull);
      }
      __syncwarp();
    }
    warp_copy_row_h<D>(kn, c.kr + rs * D, lane);
    warp_copy_row_h<D>(vn, c.vr + rs * D, lane);
    if (lane == 0) {
      c.pos_r[rs] = t;
      c.sc_r[rs] = sc_new;
    }
  } else {
    const int idx = c.n_cold[s];
    if (idx >= c.cap) {
      if (lane == 0) set_error(c.err, kErrDevice);
      return;
    }
    const size_t cs = (size_t)s * c.cap + idx;
    warp_copy_row_h<D>(kn, c.kc + cs * D, lane);
    warp_copy_row_h<D>(vn, c.vc + cs * D, lane);
    if (lane == 0) {
      c.pos_c[cs] = t;
      c.sc_c[cs] = sc_new;
      c.n_cold[s] = idx + 1;
    }
  }
  if (lane == 0) c.next_pos[s] = t + 1;
}

// ---------------------------------------------------------------------------
// attention
// ---------------------------------------------------------------------------
template <int D, int G, bool CI8>
struct Cfg {
  static constexpr int LPT = D / 16;              // lanes per token in the score phase (16 dims each)
  static constexpr int NG = 32 / LPT;             // tokens per warp per score step
  static constexpr int E = D / 32;                // dims per lane in the value phase
  static constexpr int ROWB_C = CI8 ? D : 2 * D;  // bytes of one cold row
  static constexpr int ROWB_R = 2 * D;            // bytes of one window row
  static constexpr int KV_BYTES = 8192;           // bytes of K (and of V) per stage
  static constexpr int TT_C = KV_BYTES / ROWB_C;  // tokens per cold tile
  static constexpr int TT_R = KV_BYTES / ROWB_R;  // tokens per window tile
  static constexpr int NCW = 4;                   // consumer warps
  static constexpr int TW_C = TT_C / NCW;         // tokens per consumer warp per tile
  static constexpr int TW_R = TT_R / NCW;
  static constexpr int TW_MAX = TW_C > TW_R ? TW_C : TW_R;
  static constexpr int MAX_STEPS = TW_MAX / NG;   // score steps per warp per tile
  static constexpr int MINB = G >= 4 ? 2 : 3;     // CTAs per SM the register budget is sized for
  static constexpr int NSTAGE = MINB == 2 ? 4 : 3;
  static constexpr int AUX_BYTES = 2 * (TT_C > TT_R ? TT_C : TT_R) * 4;
  static constexpr int STAGE_BYTES = 2 * KV_BYTES + AUX_BYTES;
  static constexpr int PS_BYTES = NCW * TW_MAX * 8 * 4;          // probabilities, padded to 8 heads
  static constexpr int MERGE_BYTES = NCW * G * (D + 2) * 4;
  static constexpr int SMEM_BYTES = NSTAGE * STAGE_BYTES + PS_BYTES + MERGE_BYTES + 2 * NSTAGE * 8 + 16;
  static_assert(G <= LPT, "at most head_dim/16 query heads per KV head");
  static_assert(TW_C % NG == 0 && TW_R % NG == 0, "tile split");
  static_assert(TW_MAX <= 32, "validity mask is one word");
};

struct Unit {
  int s, l, b, h;
  int n_cold;
  int tiles_c, t0, t1;
};

template <int D, int G, bool CI8>
__device__ __forceinline__ Unit make_unit(const Cache& c, const Range& r, int splits, int unit) {
  using C = Cfg<D, G, CI8>;
  Unit u;
  const int item = unit / splits;
  const int split = unit - item * splits;
  u.s = seg_of(c, r, item, &u.l, &u.b, &u.h);
  u.n_cold = c.n_cold[u.s];
  if (u.n_cold < 0 || u.n_cold > c.cap) {   // corrupt segment: record once (by its split 0) and skip
    if (split == 0 && threadIdx.x == 0) record_violation(c.err, kSiteAttnSeg, u.s, u.n_cold);
    u.n_cold = 0;
    u.tiles_c = 0;
    u.t0 = u.t1 = 0;
    return u;
  }
  u.tiles_c = (u.n_cold + C::TT_C - 1) / C::TT_C;
  const int tiles_r = (c.W + C::TT_R - 1) / C::TT_R;
  const int tiles = u.tiles_c + tiles_r;
  const int per = (tiles + splits - 1) / splits;
  u.t0 = min(tiles, split * per);
  u.t1 = min(tiles, u.t0 + per);
  return u;
}

template <int D, int G, bool CI8>
__global__ void __launch_bounds__(160, (G >= 4 ? 2 : 3)) attn_kernel(Cache c, AttnLaunch a, int splits, int units,
                                                                  float qscale) {
  using C = Cfg<D, G, CI8>;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* stages = smem;
  float* ps_all = reinterpret_cast<float*>(smem + C::NSTAGE * C::STAGE_BYTES);
  float* merge = reinterpret_cast<float*>(smem + C::NSTAGE * C::STAGE_BYTES + C::PS_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::NSTAGE * C::STAGE_BYTES + C::PS_BYTES + C::MERGE_BYTES);
  uint64_t* empty = full + C::NSTAGE;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + C::NSTAGE);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::NCW);
    }
    abort_flag[0] = 0;
    abort_flag[1] = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == C::NCW) {
    // ------------------------------ producer -------------------------------
    // One lane issues every copy; the other lanes go straight to the final
    // barrier. On a timed-out wait the copies already issued are waited for
    // (bounded) so that none lands after the CTA has exited.
    if (lane == 0) {
      int ctr = 0;
      bool stop = false;
      for (int unit = blockIdx.x; unit < units && !stop; unit += gridDim.x) {
        const Unit u = make_unit<D, G, CI8>(c, a.r, splits, unit);
        for (int t = u.t0; t < u.t1; ++t) {
          const int st = ctr % C::NSTAGE;
          if (ctr >= C::NSTAGE && !mbar_wait_bounded(&empty[st], ((ctr / C::NSTAGE) - 1) & 1)) {
            set_error(c.err, kErrDevice);
            *abort_flag = 1;
          }
          if (*abort_flag) {
            stop = true;
            break;
          }
          unsigned char* sb = stages + st * C::STAGE_BYTES;
          const bool cold = t < u.tiles_c;
          if (kChecked) {
            const int j0 = cold ? t * C::TT_C : (t - u.tiles_c) * C::TT_R;
            const int cnt = cold ? min(C::TT_C, u.n_cold - j0) : min(C::TT_R, c.W - j0);
            const int lim = cold ? c.cap : c.Wst;
            if (!guard(cnt >= 1 && j0 >= 0 && j0 + ((cnt + 3) & ~3) <= lim, c.err, kSiteAttnTile, u.s, j0)) {
              *abort_flag = 1;   // consumers give up on their bounded wait for this tile
              stop = true;
              break;
            }
          }
          if (cold) {
            const int j0 = t * C::TT_C;
            const int cnt = min(C::TT_C, u.n_cold - j0);
            const int cnt4 = (cnt + 3) & ~3;
            const uint32_t kvb = (uint32_t)cnt * C::ROWB_C;
            const uint32_t aux = CI8 ? 2u * cnt4 * 4u : 0u;
            mbar_arrive_expect_tx(&full[st], 2 * kvb + aux);
            const size_t row0 = (size_t)u.s * c.cap + j0;
            if (CI8) {
              bulk_g2s(sb, c.k8 + row0 * D, kvb, &full[st]);
              bulk_g2s(sb + C::KV_BYTES, c.v8 + row0 * D, kvb, &full[st]);
              bulk_g2s(sb + 2 * C::KV_BYTES, c.ks + row0, cnt4 * 4, &full[st]);
              bulk_g2s(sb + 2 * C::KV_BYTES + C::TT_C * 4, c.vs + row0, cnt4 * 4, &full[st]);
            } else {
              bulk_g2s(sb, c.kc + row0 * D, kvb, &full[st]);
              bulk_g2s(sb + C::KV_BYTES, c.vc + row0 * D, kvb, &full[st]);
            }
          } else {
            const int j0 = (t - u.tiles_c) * C::TT_R;
            const int cnt = min(C::TT_R, c.W - j0);
            const int cnt4 = (cnt + 3) & ~3;
            const uint32_t kvb = (uint32_t)cnt * C::ROWB_R;
            mbar_arrive_expect_tx(&full[st], 2 * kvb + cnt4 * 4);
            const size_t row0 = (size_t)u.s * c.Wst + j0;
            bulk_g2s(sb, c.kr + row0 * D, kvb, &full[st]);
            bulk_g2s(sb + C::KV_BYTES, c.vr + row0 * D, kvb, &full[st]);
            bulk_g2s(sb + 2 * C::KV_BYTES, c.pos_r + row0, cnt4 * 4, &full[st]);
          }
          ++ctr;
        }
      }
      if (stop) {
        for (int k = max(0, ctr - C::NSTAGE); k < ctr; ++k)
          (void)mbar_wait_bounded(&full[k % C::NSTAGE], (k / C::NSTAGE) & 1, 1000000000ll);
      }
    }
    __syncthreads();
    return;
  }

  // -------------------------------- consumers --------------------------------
  const int sub = lane % C::LPT;       // which 16-dim slice of a row this lane scores
  const int gi = lane / C::LPT;        // which token of a score step this lane's group takes
  float* ps = ps_all + warp * C::TW_MAX * 8;
  volatile int* stop_snapshot = abort_flag + 1;
  int ctr = 0;

  for (int unit = blockIdx.x; unit < units; unit += gridDim.x) {
    const Unit u = make_unit<D, G, CI8>(c, a.r, splits, unit);
    // query slice of this lane, scaled by 1/sqrt(D)
    float2 q2[G][8];
    {
      const size_t qrow = (size_t)((u.l - a.r.l0) * a.r.B + u.b) * c.Hq + u.h * G;
      if (kChecked) guard(qrow + G <= (size_t)a.r.items(c.Hkv) * G, c.err, kSiteAttnQ, u.s, (int)qrow);
      const __half* qp = a.q + qrow * D + sub * 16;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const uint4 w0 = *reinterpret_cast<const uint4*>(qp + g * D);
        const uint4 w1 = *reinterpret_cast<const uint4*>(qp + g * D + 8);
        const uint32_t ww[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float2 f = h2_to_f2(ww[i]);
          q2[g][i] = make_float2(f.x * qscale, f.y * qscale);
        }
      }
    }
    float m[G], lsum[G];
    float2 acc[G][C::E / 2];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = -CUDART_INF_F;
      lsum[g] = 0.0f;
#pragma unroll
      for (int e = 0; e < C::E / 2; ++e) acc[g][e] = make_float2(0.0f, 0.0f);
    }
    unsigned long long n_rows_c = 0, n_rows_r = 0;
    float* sc_base = a.scores + (size_t)u.s * G * a.score_stride;

    for (int t = u.t0; t < u.t1; ++t) {
      const int st = ctr % C::NSTAGE;
      const bool ok = mbar_wait_bounded(&full[st], (ctr / C::NSTAGE) & 1);
      if (!ok) {
        set_error(c.err, kErrDevice);
        *abort_flag = 1;
      }
      if (*abort_flag) break;   // every consumer warp still reaches the merge barriers
      const unsigned char* sb = stages + st * C::STAGE_BYTES;
      const bool cold = t < u.tiles_c;
      const int tw = cold ? C::TW_C : C::TW_R;
      const int j0 = cold ? t * C::TT_C : (t - u.tiles_c) * C::TT_R;
      const int cnt = cold ? min(C::TT_C, u.n_cold - j0) : min(C::TT_R, c.W - j0);
      const int wb = warp * tw;         // first token of this warp in the tile
      uint32_t vmask = 0;               // tokens of this warp that are valid
      const int steps = tw / C::NG;
      // scores of this warp's tokens (log2 units); the maximum is updated once
      // per tile so that every probability of the tile uses the same reference
      float u2s[C::MAX_STEPS][G];
      float vsc[C::MAX_STEPS];
      bool up = false;
#pragma unroll
      for (int stp = 0; stp < C::MAX_STEPS; ++stp) {
        if (stp >= steps) break;
        const int tl = stp * C::NG + gi;      // token index within this warp's share
        const int tok = wb + tl;              // token index within the tile
        bool valid = tok < cnt;
        if (!cold && valid) valid = reinterpret_cast<const int32_t*>(sb + 2 * C::KV_BYTES)[tok] >= 0;
        float part[G];
#pragma unroll
        for (int g = 0; g < G; ++g) part[g] = 0.0f;
        if (valid) {
          float2 x2[8];
          if (cold && CI8) {
            const uint4 w = *reinterpret_cast<const uint4*>(sb + tok * D + sub * 16);
            i8x4_to_f2x2(w.x, x2[0], x2[1]);
            i8x4_to_f2x2(w.y, x2[2], x2[3]);
            i8x4_to_f2x2(w.z, x2[4], x2[5]);
            i8x4_to_f2x2(w.w, x2[6], x2[7]);
          } else {
            const uint4 w0 = *reinterpret_cast<const uint4*>(sb + tok * (2 * D) + sub * 32);
            const uint4 w1 = *reinterpret_cast<const uint4*>(sb + tok * (2 * D) + sub * 32 + 16);
            x2[0] = h2_to_f2(w0.x); x2[1] = h2_to_f2(w0.y); x2[2] = h2_to_f2(w0.z); x2[3] = h2_to_f2(w0.w);
            x2[4] = h2_to_f2(w1.x); x2[5] = h2_to_f2(w1.y); x2[6] = h2_to_f2(w1.z); x2[7] = h2_to_f2(w1.w);
          }
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float2 s2 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < 8; ++i) s2 = __ffma2_rn(q2[g][i], x2[i], s2);
            part[g] = s2.x + s2.y;
          }
        }
#pragma unroll
        for (int o = 1; o < C::LPT; o <<= 1) {
#pragma unroll
          for (int g = 0; g < G; ++g) part[g] += __shfl_xor_sync(0xffffffffu, part[g], o);
        }
        const float kscale = (cold && CI8 && valid) ? reinterpret_cast<const float*>(sb + 2 * C::KV_BYTES)[tok] : 1.0f;
        vsc[stp] = (cold && CI8 && valid) ? reinterpret_cast<const float*>(sb + 2 * C::KV_BYTES + C::TT_C * 4)[tok]
                                          : 1.0f;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float sg = part[g] * kscale;
          if (valid && sub == g) {
            const int col = (cold ? 0 : c.cap) + j0 + tok;
            if (!kChecked || guard(col >= 0 && col < a.score_stride, c.err, kSiteAttnScore, u.s, col))
              sc_base[(size_t)g * a.score_stride + col] = sg;
          }
          u2s[stp][g] = valid ? sg * kLog2e : -CUDART_INF_F;
          up |= u2s[stp][g] > m[g];
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, valid && sub == 0);
        // bit gi of the ballot (taken from lane gi*LPT) -> token tl = stp*NG + gi
#pragma unroll
        for (int k = 0; k < C::NG; ++k)
          if (bal & (1u << (k * C::LPT))) vmask |= 1u << (stp * C::NG + k);
      }
      if (__any_sync(0xffffffffu, up)) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float tmax = -CUDART_INF_F;
#pragma unroll
          for (int stp = 0; stp < C::MAX_STEPS; ++stp)
            if (stp < steps) tmax = fmaxf(tmax, u2s[stp][g]);
          const float nm = fmaxf(m[g], warp_max(tmax));
          if (nm > m[g]) {
            const float corr = exp2f(m[g] - nm);
            lsum[g] *= corr;
#pragma unroll
            for (int e = 0; e < C::E / 2; ++e) acc[g][e] = __fmul2_rn(acc[g][e], make_float2(corr, corr));
            m[g] = nm;
          }
        }
      }
#pragma unroll
      for (int stp = 0; stp < C::MAX_STEPS; ++stp) {
        if (stp >= steps) break;
        const int tl = stp * C::NG + gi;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float u = u2s[stp][g];
          const float p = u == -CUDART_INF_F ? 0.0f : exp2f(u - m[g]);   // invalid tokens carry nothing
          lsum[g] += p;
          if (sub == g) ps[tl * 8 + g] = p * vsc[stp];
        }
      }
      if (lane == 0) {
        if (cold) n_rows_c += __popc(vmask);
        else n_rows_r += __popc(vmask);
      }
      __syncwarp();
      // ---- P.V over this warp's tokens: lanes over the head dimension ----
      uint32_t mk = vmask;
      while (mk) {
        const int tl = __ffs(mk) - 1;
        mk &= mk - 1;
        const int tok = wb + tl;
        float2 x2[C::E / 2];
        if (cold && CI8) {
          if constexpr (C::E == 4) {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(sb + C::KV_BYTES + tok * D + lane * 4);
            i8x4_to_f2x2(w, x2[0], x2[1]);
          } else {
            const uint32_t w = *reinterpret_cast<const uint16_t*>(sb + C::KV_BYTES + tok * D + lane * 2);
            float2 hi;
            i8x4_to_f2x2(w, x2[0], hi);
          }
        } else {
          if constexpr (C::E == 4) {
            const uint2 w = *reinterpret_cast<const uint2*>(sb + C::KV_BYTES + tok * (2 * D) + lane * 8);
            x2[0] = h2_to_f2(w.x);
            x2[1] = h2_to_f2(w.y);
          } else {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(sb + C::KV_BYTES + tok * (2 * D) + lane * 4);
            x2[0] = h2_to_f2(w);
          }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float p = ps[tl * 8 + g];
#pragma unroll
          for (int e = 0; e < C::E / 2; ++e) acc[g][e] = __ffma2_rn(make_float2(p, p), x2[e], acc[g][e]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      ++ctr;
    }

    // ---- merge the four consumer warps of this unit ----
    float* mg = merge;                                  // [NCW][G] maxima
    float* lg = merge + C::NCW * G;                     // [NCW][G] sums
    float* ag = merge + 2 * C::NCW * G;                 // [NCW][G][D] accumulators
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float ls = warp_sum(lsum[g]) * (1.0f / C::LPT);   // every lane of a group added the same p
      if (lane == 0) {
        mg[warp * G + g] = m[g];
        lg[warp * G + g] = ls;
      }
#pragma unroll
      for (int e = 0; e < C::E / 2; ++e) {
        ag[(warp * G + g) * D + lane * C::E + 2 * e] = acc[g][e].x;
        ag[(warp * G + g) * D + lane * C::E + 2 * e + 1] = acc[g][e].y;
      }
    }
    if (lane == 0) {
      atomicAdd(&c.counters[kCntAttnInt8], CI8 ? n_rows_c : 0ull);
      atomicAdd(&c.counters[kCntAttnFp16], n_rows_r + (CI8 ? 0ull : n_rows_c));
    }
    named_barrier_sync(1, C::NCW * 32);
    if (threadIdx.x == 0) *stop_snapshot = *abort_flag;
    const int item = unit / splits;
    const int split = unit - item * splits;
    for (int idx = threadIdx.x; idx < G * D; idx += C::NCW * 32) {
      const int g = idx / D, d = idx - g * D;
      float M = -CUDART_INF_F;
#pragma unroll
      for (int w = 0; w < C::NCW; ++w) M = fmaxf(M, mg[w * G + g]);
      float L = 0.0f, A = 0.0f;
      if (M != -CUDART_INF_F) {
#pragma unroll
        for (int w = 0; w < C::NCW; ++w) {
          const float mw = mg[w * G + g];
          if (mw == -CUDART_INF_F) continue;
          const float f = exp2f(mw - M);
          L += lg[w * G + g] * f;
          A += ag[(w * G + g) * D + d] * f;
        }
      }
      if (splits == 1) {
        const size_t orow = (size_t)((u.l - a.r.l0) * a.r.B + u.b) * c.Hq + u.h * G + g;
        if (kChecked && !guard(orow < (size_t)a.r.items(c.Hkv) * G, c.err, kSiteAttnOut, u.s, (int)orow)) continue;
        a.out[orow * D + d] = A / L;
        if (d == 0) {
          const float lse = (M + __log2f(L)) * kLn2;
          a.lse_ws[(size_t)u.s * G + g] = lse;
          if (a.lse_out) a.lse_out[orow] = lse;
        }
      } else {
        float* pp = a.part + ((size_t)(item * splits + split) * G + g) * (D + 2);
        pp[d] = A;
        if (d == 0) {
          pp[D] = M;
          pp[D + 1] = L;
        }
      }
    }
    named_barrier_sync(1, C::NCW * 32);
    if (*stop_snapshot) break;        // same value for every consumer thread
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// combine split partials: one warp per (item, head)
// ---------------------------------------------------------------------------
template <int D, int G>
__global__ void __launch_bounds__(256) combine_kernel(Cache c, AttnLaunch a, int splits) {
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int items = a.r.items(c.Hkv);
  if (wid >= items * G) return;
  const int item = wid / G, g = wid - item * G;
  int l, b, h;
  const int s = seg_of(c, a.r, item, &l, &b, &h);
  float M = -CUDART_INF_F;
  for (int sp = 0; sp < splits; ++sp)
    M = fmaxf(M, a.part[((size_t)(item * splits + sp) * G + g) * (D + 2) + D]);
  float L = 0.0f;
  float A[D / 32];
#pragma unroll
  for (int e = 0; e < D / 32; ++e) A[e] = 0.0f;
  for (int sp = 0; sp < splits; ++sp) {
    const float* pp = a.part + ((size_t)(item * splits + sp) * G + g) * (D + 2);
    const float ms = pp[D];
    if (ms == -CUDART_INF_F) continue;
    const float f = exp2f(ms - M);
    L += pp[D + 1] * f;
#pragma unroll
    for (int e = 0; e < D / 32; ++e) A[e] += pp[lane + 32 * e] * f;
  }
  const size_t orow = (size_t)((l - a.r.l0) * a.r.B + b) * c.Hq + h * G + g;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) a.out[orow * D + lane + 32 * e] = A[e] / L;
  if (lane == 0) {
    const float lse = (M + __log2f(L)) * kLn2;
    a.lse_ws[(size_t)s * G + g] = lse;
    if (a.lse_out) a.lse_out[orow] = lse;
  }
}

// ---------------------------------------------------------------------------
// attention-mass EMA: one CTA per segment
// ---------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(256) ema_kernel(Cache c, AttnLaunch a, Policy pol) {
  const int item = blockIdx.x;
  int l, b, h;
  const int s = seg_of(c, a.r, item, &l, &b, &h);
  float lse[G];
#pragma unroll
  for (int g = 0; g < G; ++g) lse[g] = a.lse_ws[(size_t)s * G + g];
  const int n_cold = c.n_cold[s];
  if (!guard(n_cold >= 0 && n_cold <= c.cap, c.err, kSiteEmaSeg, s, n_cold)) return;
  const float* sb = a.scores + (size_t)s * G * a.score_stride;
  const float invG = 1.0f / G;
  for (int i = threadIdx.x; i < n_cold + c.W; i += blockDim.x) {
    float* scp;
    int col;
    if (i < n_cold) {
      scp = c.sc_c + (size_t)s * c.cap + i;
      col = i;
    } else {
      const int slot = i - n_cold;
      if (c.pos_r[(size_t)s * c.Wst + slot] < 0) continue;
      scp = c.sc_r + (size_t)s * c.Wst + slot;
      col = c.cap + slot;
    }
    float sum = 0.0f;
#pragma unroll
    for (int g = 0; g < G; ++g) sum += __expf(sb[(size_t)g * a.score_stride + col] - lse[g]);
    *scp = fmaf(pol.beta, *scp, pol.one_minus_beta * (sum * invG));
  }
}

template <int D, int G, bool CI8>
cudaError_t run_attn(const Cache& c, const Policy& pol, const AttnLaunch& a, cudaStream_t st, long long* launches,
                     Prof* prof) {
  using C = Cfg<D, G, CI8>;
  const int items = a.r.items(c.Hkv);
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, G, CI8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  int ctas_per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ctas_per_sm, attn_kernel<D, G, CI8>, 160, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  ctas_per_sm = max(1, ctas_per_sm);
  const int resident = a.num_sms * ctas_per_sm;
  const int tiles_ub = (a.max_cold_tokens + C::TT_C - 1) / C::TT_C + (c.W + C::TT_R - 1) / C::TT_R;
  int splits = 1;
  if (items < 2 * resident) {
    // few segments: split the token axis so that every SM has work
    splits = (2 * resident + items - 1) / items;
    splits = min(splits, max(1, tiles_ub / 2));
  } else if (tiles_ub >= 64) {
    // long segments: finer units even out the last wave
    splits = min((16 * resident + items - 1) / items, tiles_ub / 16);
    splits = max(1, splits);
  }
  while (splits > 1 && (long long)items * splits > a.part_units) --splits;
  const int units = items * splits;
  const int grid = min(units, resident);
  {
    ProfScope ps(prof, kKAttention, st);
    attn_kernel<D, G, CI8><<<grid, 160, C::SMEM_BYTES, st>>>(c, a, splits, units, rsqrtf((float)D));
  }
  ++*launches;
  if (splits > 1) {
    const int warps = items * G;
    ProfScope ps(prof, kKCombine, st);
    combine_kernel<D, G><<<(warps * 32 + 255) / 256, 256, 0, st>>>(c, a, splits);
    ++*launches;
  }
  if (pol.mode == 0) {
    ProfScope ps(prof, kKEma, st);
    ema_kernel<G><<<items, 256, 0, st>>>(c, a, pol);
    ++*launches;
  }
  return cudaGetLastError();
}

template <int D, int G>
cudaError_t run_attn_g(const Cache& c, const Policy& pol, const AttnLaunch& a, cudaStream_t st, long long* n,
                       Prof* prof) {
  return c.cold_int8 ? run_attn<D, G, true>(c, pol, a, st, n, prof) : run_attn<D, G, false>(c, pol, a, st, n, prof);
}

}  // namespace

cudaError_t launch_decode_attn(const Cache& c, const Policy& pol, const AttnLaunch& a, cudaStream_t st,
                               long long* launches, Prof* prof) {
  const int items = a.r.items(c.Hkv);
  if (items == 0) return cudaSuccess;
  const int blocks = (items * 32 + 255) / 256;
  {
    ProfScope ps(prof, kKAppend, st);
    if (c.D == 128)
      append_kernel<128><<<blocks, 256, 0, st>>>(c, a.r, a.k_new, a.v_new, a.prio_new, pol.mode == 1);
    else
      append_kernel<64><<<blocks, 256, 0, st>>>(c, a.r, a.k_new, a.v_new, a.prio_new, pol.mode == 1);
  }
  ++*launches;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (c.D == 128) {
    switch (c.G) {
      case 1: return run_attn_g<128, 1>(c, pol, a, st, launches, prof);
      case 2: return run_attn_g<128, 2>(c, pol, a, st, launches, prof);
      case 4: return run_attn_g<128, 4>(c, pol, a, st, launches, prof);
      case 5: return run_attn_g<128, 5>(c, pol, a, st, launches, prof);
      case 8: return run_attn_g<128, 8>(c, pol, a, st, launches, prof);
    }
  } else {
    switch (c.G) {
      case 1: return run_attn_g<64, 1>(c, pol, a, st, launches, prof);
      case 2: return run_attn_g<64, 2>(c, pol, a, st, launches, prof);
      case 4: return run_attn_g<64, 4>(c, pol, a, st, launches, prof);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace confkv
