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

// CTAs per SM the register budget of the G >= 4 attention kernels targets.
#ifndef CONFKV_G4_MINB
#define CONFKV_G4_MINB 2
#endif

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
  // Score reduction across the LPT lanes of a token: when G divides LPT, each
  // lane group scores TPG = LPT/G tokens at once and a transposed (reduce-
  // scatter) butterfly leaves exactly one (token, head) score in every lane;
  // otherwise one token per group and a plain butterfly, lanes sub < G keep
  // one head each.
  static constexpr bool XPOSE = (LPT % G) == 0;
  static constexpr int TPG = XPOSE ? LPT / G : 1;
  static constexpr int STEP_TOK = NG * TPG;       // tokens per warp per score step
  static constexpr int SPT_C = (TW_C + STEP_TOK - 1) / STEP_TOK;
  static constexpr int SPT_R = (TW_R + STEP_TOK - 1) / STEP_TOK;
  static constexpr int MAX_STEPS = SPT_C > SPT_R ? SPT_C : SPT_R;
  static constexpr int MINB = G >= 4 ? CONFKV_G4_MINB : 3;   // CTAs per SM the register budget is sized for
  static constexpr int NSTAGE = MINB == 2 ? 4 : 3;
  static constexpr int AUX_BYTES = 2 * (TT_C > TT_R ? TT_C : TT_R) * 4;
  static constexpr int STAGE_BYTES = 2 * KV_BYTES + AUX_BYTES;
  static constexpr int PS_BYTES = NCW * TW_MAX * 8 * 4;          // probabilities [8 heads][TW_MAX] per warp
  static constexpr int MERGE_BYTES = NCW * G * (D + 2) * 4;
  static constexpr int SMEM_BYTES = NSTAGE * STAGE_BYTES + PS_BYTES + MERGE_BYTES + 2 * NSTAGE * 8 + 16;
  static_assert(G <= LPT, "at most head_dim/16 query heads per KV head");
  static_assert(TW_MAX <= 32, "a warp's share of a tile is at most 32 tokens");
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


// Per-warp online-softmax state of one unit.
template <int D, int G>
struct WarpState {
  float m[G];                // running maximum per head (log2 units), uniform in the warp
  float2 acc[G][D / 32];     // P.V partial sums: .x over even tokens, .y over odd tokens of a pair
  float l_own;               // this lane's share of the softmax sum of its own head
};

enum TileKind { kTileCold8 = 0, kTileCold16 = 1, kTileRing = 2 };

// One warp's share of one staged tile: scores (with the lane-group reduction),
// the once-per-tile maximum update, probabilities, then P.V over token pairs.
// Loops have compile-time trip counts; rows outside the tile are loaded
// predicated to zero instead of branching.
template <int D, int G, bool CI8, int KIND>
__device__ __forceinline__ void consume_tile(const Cache& c, const AttnLaunch& a, const unsigned char* sb,
                                             const float2 (&q2)[G][8], WarpState<D, G>& ws, float* ps,
                                             float* sc_base, int s_id, int j0, int cnt, int warp, int lane,
                                             unsigned long long& n_rows) {
  using C = Cfg<D, G, CI8>;
  constexpr bool COLD = KIND != kTileRing;
  constexpr bool I8 = KIND == kTileCold8;
  constexpr int TW = COLD ? C::TW_C : C::TW_R;
  constexpr int ROWB = I8 ? D : 2 * D;
  constexpr int STEPS = (TW + C::STEP_TOK - 1) / C::STEP_TOK;
  constexpr int E = D / 32;
  const int sub = lane % C::LPT;
  const int gi = lane / C::LPT;
  const bool own = C::XPOSE || sub < G;
  const int g_own = C::XPOSE ? sub % G : (sub < G ? sub : 0);
  const int t_own = C::XPOSE ? sub / G : 0;
  const int wb = warp * TW;
  const float* aux = reinterpret_cast<const float*>(sb + 2 * C::KV_BYTES);
  const unsigned char* kb = sb;
  const unsigned char* vb = sb + C::KV_BYTES;

  float u_own[STEPS];
  int tl_own[STEPS];
  float lmax = -CUDART_INF_F;
#pragma unroll
  for (int stp = 0; stp < STEPS; ++stp) {
    float v[C::XPOSE ? C::LPT : G];
#pragma unroll
    for (int tg = 0; tg < C::TPG; ++tg) {
      // rows past the tile's end are staged rows of earlier tiles (or zeros): their
      // scores are computed and discarded below, never masked per element
      const int row = wb + min(stp * C::STEP_TOK + tg * C::NG + gi, TW - 1);
      float2 x2[8];
      if constexpr (I8) {
        const uint4 w = *reinterpret_cast<const uint4*>(kb + row * ROWB + sub * 16);
        i8x4_to_f2x2(w.x, x2[0], x2[1]);
        i8x4_to_f2x2(w.y, x2[2], x2[3]);
        i8x4_to_f2x2(w.z, x2[4], x2[5]);
        i8x4_to_f2x2(w.w, x2[6], x2[7]);
      } else {
        const uint4 w0 = *reinterpret_cast<const uint4*>(kb + row * ROWB + sub * 32);
        const uint4 w1 = *reinterpret_cast<const uint4*>(kb + row * ROWB + sub * 32 + 16);
        x2[0] = h2_to_f2(w0.x); x2[1] = h2_to_f2(w0.y); x2[2] = h2_to_f2(w0.z); x2[3] = h2_to_f2(w0.w);
        x2[4] = h2_to_f2(w1.x); x2[5] = h2_to_f2(w1.y); x2[6] = h2_to_f2(w1.z); x2[7] = h2_to_f2(w1.w);
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float2 sa = make_float2(0.0f, 0.0f), sb2 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          sa = __ffma2_rn(q2[g][i], x2[i], sa);
          sb2 = __ffma2_rn(q2[g][i + 1], x2[i + 1], sb2);
        }
        const float2 t2 = __fadd2_rn(sa, sb2);
        v[tg * G + g] = t2.x + t2.y;
      }
    }
    float mine;
    if constexpr (C::XPOSE) {
#pragma unroll
      for (int o = C::LPT / 2; o >= 1; o >>= 1) {
        const bool upper = (sub & o) != 0;
#pragma unroll
        for (int k = 0; k < o; ++k) {
          const float send = upper ? v[k] : v[k + o];
          const float keep = upper ? v[k + o] : v[k];
          v[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      mine = v[0];                       // value index sub = (token t_own, head g_own)
    } else {
#pragma unroll
      for (int o = 1; o < C::LPT; o <<= 1) {
#pragma unroll
        for (int g = 0; g < G; ++g) v[g] += __shfl_xor_sync(0xffffffffu, v[g], o);
      }
      mine = v[0];
#pragma unroll
      for (int g = 1; g < G; ++g) mine = (sub == g) ? v[g] : mine;
    }
    const int tl = stp * C::STEP_TOK + t_own * C::NG + gi;
    const int tok = wb + tl;
    const bool in_own = own && tl < TW && tok < cnt;
    bool valid = in_own;
    if constexpr (!COLD) valid = valid && reinterpret_cast<const int32_t*>(aux)[in_own ? tok : 0] >= 0;
    const float kscale = I8 ? aux[in_own ? tok : 0] : 1.0f;
    const float sg = mine * kscale;
    if (valid) {
      const int col = (COLD ? 0 : c.cap) + j0 + tok;
      if (!kChecked || guard(col >= 0 && col < a.score_stride, c.err, kSiteAttnScore, s_id, col))
        sc_base[(size_t)g_own * a.score_stride + col] = sg;
    }
    u_own[stp] = valid ? sg * kLog2e : -CUDART_INF_F;
    tl_own[stp] = (own && tl < TW) ? tl : -1;   // every token < TW gets a probability (0 if invalid)
    lmax = fmaxf(lmax, u_own[stp]);
    if constexpr (!COLD) {
      const uint32_t bal = __ballot_sync(0xffffffffu, valid && g_own == 0);
      if (lane == 0) n_rows += __popc(bal);
    }
  }

  // ---- running maximum: updated once per tile, only when it grows ----
  float m_own = ws.m[0];
#pragma unroll
  for (int g = 1; g < G; ++g) m_own = (g_own == g) ? ws.m[g] : m_own;
  if (__any_sync(0xffffffffu, lmax > m_own)) {
    float l_scale = 1.0f;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float hm = warp_max(g_own == g ? lmax : -CUDART_INF_F);
      if (hm > ws.m[g]) {
        const float corr = exp2f(ws.m[g] - hm);
#pragma unroll
        for (int e = 0; e < E; ++e) ws.acc[g][e] = __fmul2_rn(ws.acc[g][e], make_float2(corr, corr));
        if (g_own == g) l_scale = corr;
        ws.m[g] = hm;
      }
    }
    ws.l_own *= l_scale;
    m_own = ws.m[0];
#pragma unroll
    for (int g = 1; g < G; ++g) m_own = (g_own == g) ? ws.m[g] : m_own;
  }
  // probabilities, head-major: ps[g * TW_MAX + token]; the V scale is folded in
#pragma unroll
  for (int stp = 0; stp < STEPS; ++stp) {
    const float uu = u_own[stp];
    const float p = uu == -CUDART_INF_F ? 0.0f : exp2f(uu - m_own);   // invalid tokens carry nothing
    ws.l_own += p;
    const int tl = tl_own[stp];
    if (tl >= 0) {
      const float vscale = (I8 && p != 0.0f) ? aux[C::TT_C + wb + tl] : 1.0f;
      ps[g_own * C::TW_MAX + tl] = p * vscale;
    }
  }
  if (COLD && lane == 0) n_rows += max(0, min(TW, cnt - wb));   // this warp's valid rows
  __syncwarp();

  // ---- P.V over token pairs: lanes over the head dimension ----
  // Rows past the tile's end carry probability 0 and finite staged data.
#pragma unroll
  for (int pp = 0; pp < TW / 2; ++pp) {
    const int t0 = 2 * pp;
    float2 x2[E];                     // (token t0, token t0+1) value pairs per dimension
    if constexpr (I8) {
      uint32_t w0, w1;
      if constexpr (E == 4) {
        w0 = *reinterpret_cast<const uint32_t*>(vb + (wb + t0) * ROWB + lane * 4);
        w1 = *reinterpret_cast<const uint32_t*>(vb + (wb + t0 + 1) * ROWB + lane * 4);
      } else {
        w0 = *reinterpret_cast<const uint16_t*>(vb + (wb + t0) * ROWB + lane * 2);
        w1 = *reinterpret_cast<const uint16_t*>(vb + (wb + t0 + 1) * ROWB + lane * 2);
      }
      const uint32_t u0 = w0 ^ 0x80808080u, u1 = w1 ^ 0x80808080u;
      const float2 bias = make_float2(-8388736.0f, -8388736.0f);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const uint32_t sel = 0x7540u + (uint32_t)e;    // byte e of the word into 2^23's mantissa
        float2 f;
        f.x = __uint_as_float(__byte_perm(u0, 0x4B000000u, sel));
        f.y = __uint_as_float(__byte_perm(u1, 0x4B000000u, sel));
        x2[e] = __fadd2_rn(f, bias);
      }
    } else {
      uint32_t w0[E / 2], w1[E / 2];
      if constexpr (E == 4) {
        const uint2 a0 = *reinterpret_cast<const uint2*>(vb + (wb + t0) * ROWB + lane * 8);
        const uint2 a1 = *reinterpret_cast<const uint2*>(vb + (wb + t0 + 1) * ROWB + lane * 8);
        w0[0] = a0.x; w0[1] = a0.y; w1[0] = a1.x; w1[1] = a1.y;
      } else {
        w0[0] = *reinterpret_cast<const uint32_t*>(vb + (wb + t0) * ROWB + lane * 4);
        w1[0] = *reinterpret_cast<const uint32_t*>(vb + (wb + t0 + 1) * ROWB + lane * 4);
      }
#pragma unroll
      for (int k = 0; k < E / 2; ++k) {
        x2[2 * k] = h2_to_f2(__byte_perm(w0[k], w1[k], 0x5410));       // (t0 dim 2k,   t1 dim 2k)
        x2[2 * k + 1] = h2_to_f2(__byte_perm(w0[k], w1[k], 0x7632));   // (t0 dim 2k+1, t1 dim 2k+1)
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float2 p2 = *reinterpret_cast<const float2*>(ps + g * C::TW_MAX + t0);
#pragma unroll
      for (int e = 0; e < E; ++e) ws.acc[g][e] = __ffma2_rn(p2, x2[e], ws.acc[g][e]);
    }
  }
  __syncwarp();
}

template <int D, int G, bool CI8>
__global__ void __launch_bounds__(160, (G >= 4 ? CONFKV_G4_MINB : 3)) attn_kernel(Cache c, AttnLaunch a, int splits, int units,
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
  // Zero the stage ring once: rows a tile does not fill then hold zeros or an
  // earlier tile's finite data, so the tile loops need no per-row masks.
  for (int i = threadIdx.x; i < C::NSTAGE * C::STAGE_BYTES / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(stages)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_shared();
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
  const bool own = C::XPOSE || sub < G;
  const int g_own = C::XPOSE ? sub % G : (sub < G ? sub : 0);
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
    WarpState<D, G> ws;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      ws.m[g] = -CUDART_INF_F;
#pragma unroll
      for (int e = 0; e < C::E; ++e) ws.acc[g][e] = make_float2(0.0f, 0.0f);
    }
    ws.l_own = 0.0f;
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
      if (t < u.tiles_c) {
        const int j0 = t * C::TT_C;
        const int cnt = min(C::TT_C, u.n_cold - j0);
        if constexpr (CI8)
          consume_tile<D, G, CI8, kTileCold8>(c, a, sb, q2, ws, ps, sc_base, u.s, j0, cnt, warp, lane, n_rows_c);
        else
          consume_tile<D, G, CI8, kTileCold16>(c, a, sb, q2, ws, ps, sc_base, u.s, j0, cnt, warp, lane, n_rows_c);
      } else {
        const int j0 = (t - u.tiles_c) * C::TT_R;
        const int cnt = min(C::TT_R, c.W - j0);
        consume_tile<D, G, CI8, kTileRing>(c, a, sb, q2, ws, ps, sc_base, u.s, j0, cnt, warp, lane, n_rows_r);
      }
      if (lane == 0) mbar_arrive(&empty[st]);
      ++ctr;
    }
    // fold the (even token, odd token) halves of the P.V sums
    float acc[G][C::E];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < C::E; ++e) acc[g][e] = ws.acc[g][e].x + ws.acc[g][e].y;
    const float* m = ws.m;
    const float l_own = ws.l_own;

    // ---- merge the four consumer warps of this unit ----
    float* mg = merge;                                  // [NCW][G] maxima
    float* lg = merge + C::NCW * G;                     // [NCW][G] sums
    float* ag = merge + 2 * C::NCW * G;                 // [NCW][G][D] accumulators
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float ls = warp_sum((own && g_own == g) ? l_own : 0.0f);
      if (lane == 0) {
        mg[warp * G + g] = m[g];
        lg[warp * G + g] = ls;
      }
#pragma unroll
      for (int e = 0; e < C::E; ++e) ag[(warp * G + g) * D + lane * C::E + e] = acc[g][e];
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
