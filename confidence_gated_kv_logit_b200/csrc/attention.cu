// Decode attention over the mixed FP16/INT8 cache (CONF-KV abstract: the
// policy is combined with blockwise online-softmax attention and mixed
// FP16/INT8 storage; CONF-KV post, implementation note: INT8 is dequantised
// inside the attention kernel).
//
//   append_kernel  : writes the new token into the FP16 window ring (or the
//                    cold region when INT8 is off) and prepares the segment's
//                    query operands for the tensor cores
//   attn_kernel    : persistent, warp-specialised split-K attention. One
//                    producer warp streams K/V tiles with their scales or
//                    positions into a shared-memory ring with 1-D TMA bulk
//                    copies; four consumer warps run both contractions on the
//                    tensor cores (mma.sync) and keep one online softmax per
//                    CTA.
//   combine_kernel : merges split partials into out and lse
// The second pass with the saved log-sum-exp (the attention-mass EMA) runs in
// the eviction kernel's fused variant, or on its own (ema.cu).
//
// Arithmetic. The G query heads of one KV head (padded to GP = 4 or 8) make
// both products small GEMMs:
//   * INT8 scores S = K8 . q: each query head is written as an integer
//     Q = q * 2^(27-ex) (ex from the head's max |q|; exact for every fp16 q
//     above 2^-16 of the maximum) and split into four balanced base-128 digit
//     planes, so one s8 x s8 MMA with exact int32 accumulation per plane gives
//     S exactly; the planes are recombined in fp32 and scaled by the token's K
//     scale and the head's 2^(ex-27)/sqrt(D).
//   * INT8 P.V: the probabilities times the token's V scale, P' = p * vs, are
//     written as 31-bit integers relative to the tile's largest V scale and
//     split into four byte planes (u8 x s8 MMA, exact int32 per tile), then
//     folded into fp32 accumulators with weights 2^(8k - E).
//   * FP16 tiles: K and q are fp16, so S comes from an f16 MMA with fp32
//     accumulation; for P.V each probability is split into fp16 hi + lo
//     (about 22 significant bits) and multiplied with fp16 V on the f16 MMA.
// The V codes are stored dimension-major in blocks of 32 tokens so that the
// token axis (the reduction axis of P.V) is contiguous per dimension.
#include <math_constants.h>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"
#include "tma.cuh"

namespace confkv {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// 2^k for -126 <= k <= 127
__device__ __forceinline__ float pow2i(int k) { return __int_as_float((k + 127) << 23); }


// Exponent ex with v in [2^(ex-1), 2^ex) for a normal v > 0; 0 for v = 0.
__device__ __forceinline__ int exp_of(float v) {
  return v > 0.0f ? (int)((__float_as_uint(v) >> 23) & 0xffu) - 126 : 0;
}

template <int N>
__device__ __forceinline__ float sel(const float (&v)[N], int i) {
  float r = 1.0f;
#pragma unroll
  for (int k = 0; k < N; ++k) r = (i == k) ? v[k] : r;
  return r;
}

// ---------------------------------------------------------------------------
// Prepared query operands of one segment (written by append_kernel):
//   I8 : B fragments of the int8 score MMA, [kb][nb][lane] x 2 words. Column
//        n of n-block nb is head n/2 + 4*(nb/2), digit plane 2*(nb%2) + n%2.
//   H  : B fragments of the f16 score MMA, [ks][lane] x 2 words, column = head.
//   CQ : per head, 2^(ex-27) / sqrt(D) (the int8 scores' scale).
// ---------------------------------------------------------------------------
template <int D, int GP>
struct QF {
  static constexpr int KB = D / 32, KS = D / 16, NB = GP / 2;
  static constexpr int I8_OFF = 0;
  static constexpr int H_OFF = KB * NB * 32 * 8;
  static constexpr int CQ_OFF = H_OFF + KS * 32 * 8;
  static constexpr int BYTES = (CQ_OFF + GP * 4 + 255) / 256 * 256;
};

// The balanced base-128 digits of Q (least significant first):
// Q = d0 + 128 d1 + 128^2 d2 + 128^3 d3 with |d_k| <= 64 for |Q| < 2^27.
__device__ __forceinline__ void q_digits(int Q, int (&d)[4]) {
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    d[k] = ((Q + 64) & 127) - 64;
    Q = (Q - d[k]) >> 7;
  }
  d[3] = Q;
}

template <int D, int GP>
__device__ __forceinline__ void prepare_query(const Cache& c, const AttnLaunch& a, int s, int l, int b, int h,
                                              int lane, float qscale) {
  using Q = QF<D, GP>;
  const int G = c.G;
  const __half* qb = a.q + ((size_t)((l - a.r.l0) * a.r.B + b) * c.Hq + (size_t)h * G) * D;
  unsigned char* out = a.qfrag + (size_t)s * a.qf_stride;
  const int g = lane >> 2, t = lane & 3;
  // Every load is issued first. Lane (g, t) holds, for head g/2 + 4*hs, the
  // 8 dims kb*32 + half*16 + 4t .. +3 of every k-block (32 values), which are
  // also what its digit planes need; the eight lanes of one head (t and g&1)
  // cover all D dims, so three shuffles give the head's max |q|.
  uint2 w[GP / 4][Q::KB][2];
#pragma unroll
  for (int hs = 0; hs < GP / 4; ++hs) {
    const int hh = g / 2 + 4 * hs;
#pragma unroll
    for (int kb = 0; kb < Q::KB; ++kb)
#pragma unroll
      for (int half = 0; half < 2; ++half)
        w[hs][kb][half] = hh < G ? *reinterpret_cast<const uint2*>(qb + (size_t)hh * D + kb * 32 + half * 16 + 4 * t)
                                 : make_uint2(0u, 0u);
  }
  uint32_t hq[Q::KS][2];
#pragma unroll
  for (int ks = 0; ks < Q::KS; ++ks) {
    hq[ks][0] = g < G ? *reinterpret_cast<const uint32_t*>(qb + (size_t)g * D + ks * 16 + 2 * t) : 0u;
    hq[ks][1] = g < G ? *reinterpret_cast<const uint32_t*>(qb + (size_t)g * D + ks * 16 + 8 + 2 * t) : 0u;
  }
#pragma unroll
  for (int ks = 0; ks < Q::KS; ++ks)
    reinterpret_cast<uint2*>(out + Q::H_OFF)[ks * 32 + lane] = make_uint2(hq[ks][0], hq[ks][1]);

#pragma unroll
  for (int hs = 0; hs < GP / 4; ++hs) {
    const int hh = g / 2 + 4 * hs;
    float mx = 0.0f;
#pragma unroll
    for (int kb = 0; kb < Q::KB; ++kb)
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const float2 f01 = h2_to_f2(w[hs][kb][half].x), f23 = h2_to_f2(w[hs][kb][half].y);
        mx = fmaxf(fmaxf(mx, fmaxf(fabsf(f01.x), fabsf(f01.y))), fmaxf(fabsf(f23.x), fabsf(f23.y)));
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    const int ex = exp_of(mx);
    const float sc = mx > 0.0f ? pow2i(27 - ex) : 1.0f;
    if ((lane & 7) == 0) reinterpret_cast<float*>(out + Q::CQ_OFF)[hh] = mx > 0.0f ? qscale * pow2i(ex - 27) : 0.0f;
    // column g of n-block nb = 2*hs + p2 is head g/2 + 4*hs, digit plane 2*p2 + g%2
#pragma unroll
    for (int kb = 0; kb < Q::KB; ++kb) {
      uint32_t r[2][2] = {{0u, 0u}, {0u, 0u}};   // [p2][half]
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const float2 f01 = h2_to_f2(w[hs][kb][half].x), f23 = h2_to_f2(w[hs][kb][half].y);
        const float qv[4] = {f01.x, f01.y, f23.x, f23.y};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int d[4];
          q_digits(__float2int_rn(qv[e] * sc), d);
          const int lo = (g & 1) ? d[1] : d[0], hi = (g & 1) ? d[3] : d[2];
          r[0][half] |= (uint32_t)(lo & 0xff) << (8 * e);
          r[1][half] |= (uint32_t)(hi & 0xff) << (8 * e);
        }
      }
#pragma unroll
      for (int p2 = 0; p2 < 2; ++p2)
        reinterpret_cast<uint2*>(out + Q::I8_OFF)[(kb * Q::NB + 2 * hs + p2) * 32 + lane] =
            make_uint2(r[p2][0], r[p2][1]);
    }
  }
}

// ---------------------------------------------------------------------------
// append: one warp per segment. If the window slot of the new position still
// holds a token (a caller skipped eviction), that token is converted to INT8
// first, exactly as eviction would have done. Then the segment's query
// operands are prepared.
// ---------------------------------------------------------------------------
template <int D, int GP>
__global__ void __launch_bounds__(256) append_kernel(Cache c, AttnLaunch a, Policy pol, float qscale) {
  chain_enter();
  const bool fixed_mode = pol.mode == 1;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const Range r = a.r;
  if (warp >= r.items(c.Hkv)) return;
  int l, b, h;
  const int s = seg_of(c, r, warp, &l, &b, &h);
  // Every load that depends on nothing but the segment is issued first (the
  // query work below stores, and the compiler keeps loads after stores):
  // the counters and the new K/V row travel with the query's loads.
  const int t = c.next_pos[s];
  const int n_cold0 = c.n_cold[s];
  const size_t in_row = ((size_t)((l - r.l0) * r.B + b) * c.Hkv + h);
  const __half* kn = a.k_new + in_row * D;
  const __half* vn = a.v_new + in_row * D;
  const float sc_new = fixed_mode ? a.prio_new[in_row] : initial_score(pol, l, b, h, t);
  uint32_t kw[D / 64], vw[D / 64];
  row_load_plain<D>(kn, lane, kw);
  row_load_plain<D>(vn, lane, vw);
  prepare_query<D, GP>(c, a, s, l, b, h, lane, qscale);   // independent of the cache state
  if (!guard(t >= 0 && n_cold0 >= 0 && n_cold0 <= c.cap, c.err, kSiteAppendSeg, s, t)) return;
  if (c.W > 0 && c.linear) {
    // Linear window: slots [0, n16) hold the window in position order. If
    // its oldest token has reached age W (a caller skipped eviction), it is
    // converted to INT8 as eviction would have done and the window moves
    // down by one slot; the new token goes after the last occupied slot.
    const int32_t* pr = c.pos_r + (size_t)s * c.Wst;
    int occ = 0;
    for (int sl = lane; sl < c.W; sl += 32) occ += pr[sl] >= 0;
    int n16 = __reduce_add_sync(0xffffffffu, occ);
    const int oldest = n16 > 0 ? pr[0] : -1;
    if (n16 > 0 && t - oldest >= c.W) {
      const int idx = n_cold0;
      if (idx >= c.cap) {
        if (lane == 0) set_error(c.err, kErrDevice);
        return;
      }
      warp_requant<D>(c, s, 0, idx, lane);
      if (lane == 0) {
        const size_t cs = (size_t)s * c.cap + idx;
        c.pos_c[cs] = oldest;
        c.sc_c[cs] = c.sc_r[(size_t)s * c.Wst];
        c.n_cold[s] = idx + 1;
        atomicAdd(&c.counters[kCntRequant], 1ull);
        if (n16 > 1) atomicAdd(&c.counters[kCntMovedWin], (unsigned long long)(n16 - 1));
      }
      __syncwarp();
      warp_window_shift<D>(c, s, 1, n16, lane);
      --n16;
    }
    if (n16 >= c.W) {   // cannot happen: a full window's oldest token has age W
      if (lane == 0) set_error(c.err, kErrDevice);
      return;
    }
    row_store_h<D>(c.kr + (size_t)s * c.Wst * D, n16, lane, kw);
    row_store_h<D>(c.vr + (size_t)s * c.Wst * D, n16, lane, vw);
    if (lane == 0) {
      c.pos_r[(size_t)s * c.Wst + n16] = t;
      c.sc_r[(size_t)s * c.Wst + n16] = sc_new;
    }
  } else if (c.W > 0) {
    const int slot = t % c.W;
    const size_t rs = (size_t)s * c.Wst + slot;
    const int old = c.pos_r[rs];
    if (old >= 0) {
      const int idx = n_cold0;
      if (idx >= c.cap) {
        if (lane == 0) set_error(c.err, kErrDevice);
        return;
      }
      warp_requant<D>(c, s, slot, idx, lane);
      if (lane == 0) {
        const size_t cs = (size_t)s * c.cap + idx;
        c.pos_c[cs] = old;
        c.sc_c[cs] = c.sc_r[rs];
        c.n_cold[s] = idx + 1;
        atomicAdd(&c.counters[kCntRequant], 1ull);
      }
      __syncwarp();
    }
    row_store_h<D>(c.kr + (size_t)s * c.Wst * D, slot, lane, kw);
    row_store_h<D>(c.vr + (size_t)s * c.Wst * D, slot, lane, vw);
    if (lane == 0) {
      c.pos_r[rs] = t;
      c.sc_r[rs] = sc_new;
    }
  } else {
    const int idx = n_cold0;
    if (idx >= c.cap) {
      if (lane == 0) set_error(c.err, kErrDevice);
      return;
    }
    const size_t cs = (size_t)s * c.cap + idx;
    row_store_h<D>(c.kc + (size_t)s * c.cap * D, idx, lane, kw);
    row_store_h<D>(c.vc + (size_t)s * c.cap * D, idx, lane, vw);
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
template <int D, int GP, bool CI8>
struct Cfg {
  static constexpr int NCW = 4;                 // consumer warps
  static constexpr int TTC = CI8 ? 128 : 64;    // tokens per cold tile
  static constexpr int TTR = 64;                // tokens per window tile
  static constexpr int KVB = 128 * D;           // bytes of K (and of V) per stage, either kind
  static constexpr int AUXB = 1024;             // K and V scales (int8) or positions (window)
  static constexpr int STAGE = 2 * KVB + AUXB;
  static constexpr int NSTAGE = D == 128 ? 3 : 4;
  static constexpr int KB = D / 32;             // k-blocks of the int8 score MMA
  static constexpr int KS = D / 16;             // k-steps of the f16 score MMA
  static constexpr int NB = GP / 2;             // n-blocks of the int8 score MMA (GP heads x 4 planes)
  static constexpr int MB = GP / 4;             // 16-row blocks of the P.V rows
  static constexpr int NBW = D / 32;            // 8-dimension n-blocks of P.V per consumer warp
  static constexpr int HPL = GP / 4;            // heads per lane in the int8 score layout
  static constexpr int PS_OFF = NSTAGE * STAGE;
  static constexpr int PSTR = 40;               // floats per probability row (conflict-free stores)
  static constexpr int PS_BYTES = NCW * GP * PSTR * 4;
  static constexpr int FB_OFF = PS_OFF + PS_BYTES;
  static constexpr int FB_ONE = 4 * MB * 32;    // uint4 per buffer
  static constexpr int FB_BYTES = 2 * FB_ONE * 16;
  static constexpr int WM_OFF = FB_OFF + FB_BYTES;
  static constexpr int LS_OFF = WM_OFF + NCW * GP * 4;
  static constexpr int BAR_OFF = LS_OFF + NCW * GP * 4;
  static constexpr int FLAG_OFF = BAR_OFF + 2 * NSTAGE * 8;
  static constexpr int UQ = 8;                  // unit-id queue entries (> NSTAGE)
  static constexpr int UQ_OFF = FLAG_OFF + 16;
  static constexpr int UN_OFF = UQ_OFF + UQ * 4;  // each queued unit's cold-token count
  // The query operands of the next unit are staged in shared memory when a
  // slot fits beside two CTAs per SM (GP = 4); otherwise the consumers read
  // them from global memory.
  static constexpr bool QSM = GP == 4;
  static constexpr int QBAR_OFF = UN_OFF + UQ * 4;                 // qfull, qempty mbarriers
  static constexpr int QS_OFF = (QBAR_OFF + 16 + 127) / 128 * 128;
  static constexpr int SMEM = QSM ? QS_OFF + QF<D, GP>::BYTES : QBAR_OFF + 16;
};

struct Unit {
  int s, l, b, h;
  int n_cold;
  int tiles_c, t0, t1;
};

// n_cold < -1: read the segment's count from global memory (the producer);
// otherwise the count the producer read (the consumers, from the unit queue).
template <int D, int GP, bool CI8>
__device__ __forceinline__ Unit make_unit(const Cache& c, const Range& r, int splits, int unit, int n_cold = -2) {
  using C = Cfg<D, GP, CI8>;
  Unit u;
  const int item = unit / splits;
  const int split = unit - item * splits;
  u.s = seg_of(c, r, item, &u.l, &u.b, &u.h);
  u.n_cold = n_cold < -1 ? c.n_cold[u.s] : n_cold;
  if (u.n_cold < 0 || u.n_cold > c.cap) {   // corrupt segment: record once (by its split 0) and skip
    if (split == 0 && threadIdx.x == 0) record_violation(c.err, kSiteAttnSeg, u.s, u.n_cold);
    u.n_cold = 0;
    u.tiles_c = 0;
    u.t0 = u.t1 = 0;
    return u;
  }
  u.tiles_c = (u.n_cold + C::TTC - 1) / C::TTC;
  const int tiles_r = (c.W + C::TTR - 1) / C::TTR;
  const int tiles = u.tiles_c + tiles_r;
  const int per = (tiles + splits - 1) / splits;
  u.t0 = min(tiles, split * per);
  u.t1 = min(tiles, u.t0 + per);
  return u;
}

// Online-softmax state of one unit, shared by the four consumer warps: the
// maxima m (log2 units) are the same in every lane. acc holds this lane's
// rows of the P.V accumulator: rows g and g+8 of each 16-row block, where
// GP = 4: row r is head r % 4 (int8 digit plane r / 4, or fp16 hi/lo part);
// GP = 8: row r of block mb is head r % 8 (plane 2 mb + r / 8, or hi/lo in
// block 0). A head's output is the sum of its rows. lp8 / lp16 are this
// lane's shares of the softmax sums of the heads it scores in the int8
// layout (t + 4j) and in the fp16 layout (2t, 2t+1).
template <int D, int GP>
struct SoftmaxState {
  float m[GP];
  float acc[GP / 4][D / 32][4];
  float lp8[GP / 4];
  float lp16[2];
};

// New running maxima from the four warps' tile maxima; rescale when they grow.
template <int D, int GP>
__device__ __forceinline__ void update_max(SoftmaxState<D, GP>& st, const float* wmax, int lane) {
  float mn[GP];
  bool grow = false;
#pragma unroll
  for (int h = 0; h < GP; ++h) {
    float v = st.m[h];
#pragma unroll
    for (int w = 0; w < 4; ++w) v = fmaxf(v, wmax[w * GP + h]);
    mn[h] = v;
    grow |= v > st.m[h];
  }
  if (grow) {
    const int g = lane >> 2, t = lane & 3;
    float corr[GP];
#pragma unroll
    for (int h = 0; h < GP; ++h) corr[h] = mn[h] > st.m[h] ? ex2(st.m[h] - mn[h]) : 1.0f;
    const float ca = sel(corr, GP == 4 ? (g & 3) : g);
#pragma unroll
    for (int mb = 0; mb < GP / 4; ++mb)
#pragma unroll
      for (int nb = 0; nb < D / 32; ++nb)
#pragma unroll
        for (int k = 0; k < 4; ++k) st.acc[mb][nb][k] *= ca;
#pragma unroll
    for (int j = 0; j < GP / 4; ++j) st.lp8[j] *= sel(corr, t + 4 * j);
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) st.lp16[cc] *= sel(corr, 2 * t + cc);
#pragma unroll
    for (int h = 0; h < GP; ++h) st.m[h] = mn[h];
  }
}

// Floats per row of a warp's probability buffer: 40 (not 32) puts the rows of
// the four heads a lane group writes at once in different banks.
constexpr int kPstr = 40;

// Byte `k` of each of four words, packed into one word (w0 lowest).
__device__ __forceinline__ uint32_t pack_plane(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, int k) {
  const uint32_t s = (uint32_t)k | ((uint32_t)(k + 4) << 4);
  return __byte_perm(__byte_perm(w0, w1, s), __byte_perm(w2, w3, s), 0x5410);
}

// Per-lane offsets of the ldmatrix row addresses within a staged tile; they
// depend only on the lane and the warp, so they are computed once. With rows
// starting at multiples of 8 and the placement of layout.cuh, the chunk XOR of
// a row is (lane & 7) for every tile.
struct LaneOffsets {
  uint32_t k8_row;     // INT8 K: row (warp*32 + r0) * D, r0 = (lane&7) + 8*((lane>>3)&1)
  uint32_t kx;         // chunk bits (lane>>4) XOR (lane&7), as a byte offset
  uint32_t h_row;      // fp16 K: row (warp*16 + r0) * 2D
  uint32_t v8[2];      // INT8 V: offset of this lane's 16 bytes for n-block pair 0/1, k-step 0
  uint32_t hv[2];      // fp16 V (.trans): offset for n-block pair 0/1, k-step 0
};

template <int D>
__device__ __forceinline__ LaneOffsets lane_offsets(int warp, int lane) {
  LaneOffsets o;
  const int r0 = (lane & 7) + 8 * ((lane >> 3) & 1);
  o.k8_row = (uint32_t)((warp * 32 + r0) * D);
  o.kx = (uint32_t)((((lane >> 4) ^ (lane & 7)) & 7) << 4);
  o.h_row = (uint32_t)((warp * 16 + r0) * 2 * D);
#pragma unroll
  for (int nbp = 0; nbp < 2; ++nbp) {
    const int d = warp * (D / 4) + nbp * 16 + (lane & 7) + 8 * (lane >> 4);
    o.v8[nbp] = (uint32_t)swz128((size_t)d * 32 + 16 * ((lane >> 3) & 1));
    const int dh = warp * (D / 4) + nbp * 16 + 8 * (lane >> 4);
    o.hv[nbp] = (uint32_t)h_off(r0, 2 * dh, D);
  }
  return o;
}

struct TileCtx {
  const unsigned char* sb;   // the staged tile
  int j0, cnt;               // first row of the tile in its region; rows present
  bool ok;                   // the tile arrived
  float* ps;                 // this warp's probability rows [GP][kPstr]
  uint4* fb;                 // A operands of P.V for this tile, [k-step][mb][lane]
  float* wmax;               // [4][GP]
  volatile int* abort_flag;
  float* sc_base;            // scores of this segment, [G][score_stride]
  int warp, lane;
  LaneOffsets lo;
  uint64_t keep_policy;      // L2 policy of the score stores (read again by the EMA pass)
};

// One INT8 tile (128 tokens): warp w scores tokens 32w..32w+31 and builds the
// P.V operand of k-step w; every warp then multiplies all four k-steps into
// its D/4 output dimensions. Returns false when the CTA is aborting.
template <int D, int GP>
__device__ __forceinline__ bool consume_i8(const Cache& c, const AttnLaunch& a, const TileCtx& x,
                                           SoftmaxState<D, GP>& st, const uint2 (&qi)[D / 32][GP / 2],
                                           const float (&cq8)[GP / 4], unsigned long long& n_rows) {
  constexpr int KB = D / 32, NB = GP / 2, MB = GP / 4, NBW = D / 32, HPL = GP / 4;
  const int lane = x.lane, warp = x.warp;
  const int g = lane >> 2, t = lane & 3;
  const int G = c.G;
  const uint32_t kt = smem_addr(x.sb), vt = kt + 128 * D;
  const float* ksc = reinterpret_cast<const float*>(x.sb + 2 * 128 * D);
  const float* vsc = ksc + 128;

  // ---- scores: two 16-row blocks, KB k-blocks, NB n-blocks ----
  float u[2][2][HPL];
#pragma unroll
  for (int mb2 = 0; mb2 < 2; ++mb2) {
    int sacc[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int k = 0; k < 4; ++k) sacc[nb][k] = 0;
    const int rb = warp * 32 + mb2 * 16;
    if constexpr (GP == 8) {
      // twice the MMAs per chain: a second accumulator set over the odd
      // k-blocks halves the dependency chains (the integer sums add exactly)
      int sodd[NB][4];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int k = 0; k < 4; ++k) sodd[nb][k] = 0;
#pragma unroll
      for (int kb = 0; kb < KB; ++kb) {
        uint32_t af[4];
        if constexpr (D == 128)
          ldsm_x4(af, kt + x.lo.k8_row + mb2 * 16 * D + (((uint32_t)kb << 5) ^ x.lo.kx));
        else
          ldsm_x4(af, kt + (uint32_t)k8_off(rb + (lane & 7) + ((lane >> 3) & 1) * 8, kb * 32 + (lane >> 4) * 16, D));
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) mma_s8s8((kb & 1) ? sodd[nb] : sacc[nb], af, qi[kb][nb].x, qi[kb][nb].y);
      }
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int k = 0; k < 4; ++k) sacc[nb][k] += sodd[nb][k];
    } else {
#pragma unroll
      for (int kb = 0; kb < KB; ++kb) {
        uint32_t af[4];
        if constexpr (D == 128)   // 128-byte rows: the chunk XOR is the row index mod 8 = lane & 7
          ldsm_x4(af, kt + x.lo.k8_row + mb2 * 16 * D + (((uint32_t)kb << 5) ^ x.lo.kx));
        else
          ldsm_x4(af, kt + (uint32_t)k8_off(rb + (lane & 7) + ((lane >> 3) & 1) * 8, kb * 32 + (lane >> 4) * 16, D));
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) mma_s8s8(sacc[nb], af, qi[kb][nb].x, qi[kb][nb].y);
      }
    }
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int r = rb + g + 8 * hr;
      const bool in = r < x.cnt;
      const float ksr = ksc[r];
#pragma unroll
      for (int j = 0; j < HPL; ++j) {
        const int* p01 = sacc[2 * j];
        const int* p23 = sacc[2 * j + 1];
        const float S = fmaf((float)p23[2 * hr + 1], 2097152.0f,
                             fmaf((float)p23[2 * hr], 16384.0f, fmaf((float)p01[2 * hr + 1], 128.0f, (float)p01[2 * hr])));
        const float sg = S * (ksr * cq8[j]);
        const int head = t + 4 * j;
        const bool valid = in && head < G;
        const float ul = sg * kLog2e;
        if (valid) {
          const int col = x.j0 + r;
          if (!kChecked || guard(col < a.score_stride, c.err, kSiteAttnScore, 0, col)) {
            float* dst = x.sc_base + (size_t)head * a.score_stride + col;   // scores are kept in log2 units
            st_f32_policy(dst, ul, x.keep_policy);
          }
        }
        u[mb2][hr][j] = valid ? ul : -CUDART_INF_F;
      }
    }
  }
  // ---- tile maxima, the tile's largest V scale, then the CTA-wide update ----
#pragma unroll
  for (int j = 0; j < HPL; ++j) {
    float lm = fmaxf(fmaxf(u[0][0][j], u[0][1][j]), fmaxf(u[1][0][j], u[1][1][j]));
    lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, 4));
    lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, 8));
    lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, 16));
    if (g == 0) x.wmax[warp * GP + t + 4 * j] = lm;
  }
  float vm;
  {
    const int i0 = lane * 4;
    const float4 v4 = *reinterpret_cast<const float4*>(vsc + i0);
    vm = fmaxf(fmaxf(i0 < x.cnt ? v4.x : 0.0f, i0 + 1 < x.cnt ? v4.y : 0.0f),
               fmaxf(i0 + 2 < x.cnt ? v4.z : 0.0f, i0 + 3 < x.cnt ? v4.w : 0.0f));
    vm = warp_max(vm);
  }
  if (named_barrier_or(1, 128, !x.ok || *x.abort_flag != 0)) return false;
  update_max<D, GP>(st, x.wmax, lane);

  // ---- probabilities times V scale, into this warp's rows ----
#pragma unroll
  for (int j = 0; j < HPL; ++j) {
    const int head = t + 4 * j;
    const float mh = sel(st.m, head);
#pragma unroll
    for (int mb2 = 0; mb2 < 2; ++mb2)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int rl = mb2 * 16 + g + 8 * hr;
        const float uu = u[mb2][hr][j];
        const float p = uu == -CUDART_INF_F ? 0.0f : ex2(uu - mh);
        st.lp8[j] += p;
        x.ps[head * kPstr + rl] = p == 0.0f ? 0.0f : p * vsc[warp * 32 + rl];
      }
  }
  if (lane == 0) n_rows += max(0, min(32, x.cnt - warp * 32));
  __syncwarp();

  // ---- P.V operand of k-step `warp`: P' * 2^E as four byte planes ----
  // P' <= vm < 2^(31 - E), so P' * 2^E < 2^31.
  const int E = 31 - exp_of(vm);
  const float sP = pow2i(E);
  const int ha = GP == 4 ? (g & 3) : g;
  {
    const float4 v0 = *reinterpret_cast<const float4*>(x.ps + ha * kPstr + 4 * t);
    const float4 v1 = *reinterpret_cast<const float4*>(x.ps + ha * kPstr + 16 + 4 * t);
    const uint32_t P0 = __float2uint_rn(v0.x * sP), P1 = __float2uint_rn(v0.y * sP);
    const uint32_t P2 = __float2uint_rn(v0.z * sP), P3 = __float2uint_rn(v0.w * sP);
    const uint32_t P4 = __float2uint_rn(v1.x * sP), P5 = __float2uint_rn(v1.y * sP);
    const uint32_t P6 = __float2uint_rn(v1.z * sP), P7 = __float2uint_rn(v1.w * sP);
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
      const int pl_lo = GP == 4 ? (g >> 2) : 2 * mb;
      const int pl_hi = pl_lo + (GP == 4 ? 2 : 1);
      uint4 f;
      f.x = pack_plane(P0, P1, P2, P3, pl_lo);
      f.y = pack_plane(P0, P1, P2, P3, pl_hi);
      f.z = pack_plane(P4, P5, P6, P7, pl_lo);
      f.w = pack_plane(P4, P5, P6, P7, pl_hi);
      x.fb[(warp * MB + mb) * 32 + lane] = f;
    }
  }
  named_barrier_sync(1, 128);

  // ---- P.V: four k-steps of 32 tokens, NBW n-blocks of this warp ----
  int ia[MB][NBW][4];
#pragma unroll
  for (int mb = 0; mb < MB; ++mb)
#pragma unroll
    for (int nb = 0; nb < NBW; ++nb)
#pragma unroll
      for (int k = 0; k < 4; ++k) ia[mb][nb][k] = 0;
  if constexpr (GP == 8) {
    // a second accumulator set over the odd k-steps halves the dependency
    // chains (exact integer sums)
    int iodd[MB][NBW][4];
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
      for (int nb = 0; nb < NBW; ++nb)
#pragma unroll
        for (int k = 0; k < 4; ++k) iodd[mb][nb][k] = 0;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t af[MB][4];
#pragma unroll
      for (int mb = 0; mb < MB; ++mb) {
        const uint4 f = x.fb[(ks * MB + mb) * 32 + lane];
        af[mb][0] = f.x;
        af[mb][1] = f.y;
        af[mb][2] = f.z;
        af[mb][3] = f.w;
      }
#pragma unroll
      for (int nbp = 0; nbp < NBW / 2; ++nbp) {
        uint32_t bf[4];
        ldsm_x4(bf, vt + (uint32_t)(ks * 32 * D) + x.lo.v8[nbp]);
#pragma unroll
        for (int mb = 0; mb < MB; ++mb) {
          mma_u8s8((ks & 1) ? iodd[mb][2 * nbp] : ia[mb][2 * nbp], af[mb], bf[0], bf[1]);
          mma_u8s8((ks & 1) ? iodd[mb][2 * nbp + 1] : ia[mb][2 * nbp + 1], af[mb], bf[2], bf[3]);
        }
      }
    }
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
      for (int nb = 0; nb < NBW; ++nb)
#pragma unroll
        for (int k = 0; k < 4; ++k) ia[mb][nb][k] += iodd[mb][nb][k];
  } else {
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t af[MB][4];
#pragma unroll
      for (int mb = 0; mb < MB; ++mb) {
        const uint4 f = x.fb[(ks * MB + mb) * 32 + lane];
        af[mb][0] = f.x;
        af[mb][1] = f.y;
        af[mb][2] = f.z;
        af[mb][3] = f.w;
      }
#pragma unroll
      for (int nbp = 0; nbp < NBW / 2; ++nbp) {
        uint32_t bf[4];
        ldsm_x4(bf, vt + (uint32_t)(ks * 32 * D) + x.lo.v8[nbp]);   // ks*32*D is a multiple of 2 KB
#pragma unroll
        for (int mb = 0; mb < MB; ++mb) {
          mma_u8s8(ia[mb][2 * nbp], af[mb], bf[0], bf[1]);
          mma_u8s8(ia[mb][2 * nbp + 1], af[mb], bf[2], bf[3]);
        }
      }
    }
  }
  const float inv = pow2i(-E);
#pragma unroll
  for (int mb = 0; mb < MB; ++mb) {
    const int pl_lo = GP == 4 ? (g >> 2) : 2 * mb;
    const int pl_hi = pl_lo + (GP == 4 ? 2 : 1);
    const float wl = inv * pow2i(8 * pl_lo), wh = inv * pow2i(8 * pl_hi);
#pragma unroll
    for (int nb = 0; nb < NBW; ++nb) {
      st.acc[mb][nb][0] = fmaf((float)ia[mb][nb][0], wl, st.acc[mb][nb][0]);
      st.acc[mb][nb][1] = fmaf((float)ia[mb][nb][1], wl, st.acc[mb][nb][1]);
      st.acc[mb][nb][2] = fmaf((float)ia[mb][nb][2], wh, st.acc[mb][nb][2]);
      st.acc[mb][nb][3] = fmaf((float)ia[mb][nb][3], wh, st.acc[mb][nb][3]);
    }
  }
  return true;
}

// One FP16 tile (64 tokens of the window ring, or of the cold region when
// INT8 is off): warp w scores tokens 16w..16w+15 and builds k-step w.
template <int D, int GP, bool RING>
__device__ __forceinline__ bool consume_h(const Cache& c, const AttnLaunch& a, const TileCtx& x,
                                          SoftmaxState<D, GP>& st, const uint2 (&qh)[D / 16], float qscale,
                                          unsigned long long& n_rows) {
  constexpr int KS = D / 16, MB = GP / 4, NBW = D / 32;
  const int lane = x.lane, warp = x.warp;
  const int g = lane >> 2, t = lane & 3;
  const int G = c.G;
  const uint32_t kt = smem_addr(x.sb), vt = kt + 128 * D;
  const int32_t* pos = reinterpret_cast<const int32_t*>(x.sb + 2 * 128 * D);
  const int rb = warp * 16;

  float f[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  if constexpr (GP == 8) {
    // a second accumulator over the odd k-steps halves the MMA dependency chain
    float fo[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t af[4];
      ldsm_x4(af, kt + x.lo.h_row + (((uint32_t)ks << 5) ^ x.lo.kx));
      mma_f16((ks & 1) ? fo : f, af, qh[ks].x, qh[ks].y);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) f[k] += fo[k];
  } else {
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t af[4];
      ldsm_x4(af, kt + x.lo.h_row + (((uint32_t)ks << 5) ^ x.lo.kx));
      mma_f16(f, af, qh[ks].x, qh[ks].y);
    }
  }
  float u[2][2];
  bool tok_valid[2];
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int r = rb + g + 8 * hr;
    bool tv = r < x.cnt;
    if (RING) tv = tv && pos[r] >= 0;
    tok_valid[hr] = tv;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int head = 2 * t + cc;
      const bool valid = tv && head < G;
      const float ul = f[2 * hr + cc] * qscale * kLog2e;
      if (valid) {
        const int col = (RING ? c.cap : 0) + x.j0 + r;
        if (!kChecked || guard(col < a.score_stride, c.err, kSiteAttnScore, 1, col)) {
          float* dst = x.sc_base + (size_t)head * a.score_stride + col;   // scores are kept in log2 units
          st_f32_policy(dst, ul, x.keep_policy);
        }
      }
      u[hr][cc] = valid ? ul : -CUDART_INF_F;
    }
  }
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    float lm = fmaxf(u[0][cc], u[1][cc]);
    lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, 4));
    lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, 8));
    lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, 16));
    if (g == 0 && 2 * t + cc < GP) x.wmax[warp * GP + 2 * t + cc] = lm;
  }
  if (named_barrier_or(1, 128, !x.ok || *x.abort_flag != 0)) return false;
  update_max<D, GP>(st, x.wmax, lane);

#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const int head = 2 * t + cc;
    if (head < GP) {
      const float mh = sel(st.m, head);
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const float uu = u[hr][cc];
        const float p = uu == -CUDART_INF_F ? 0.0f : ex2(uu - mh);
        st.lp16[cc] += p;
        x.ps[head * kPstr + g + 8 * hr] = p;
      }
    }
  }
  {
    const unsigned bal0 = __ballot_sync(0xffffffffu, t == 0 && tok_valid[0]);
    const unsigned bal1 = __ballot_sync(0xffffffffu, t == 0 && tok_valid[1]);
    if (lane == 0) n_rows += __popc(bal0) + __popc(bal1);
  }
  __syncwarp();

  // ---- P.V operand of k-step `warp`: p = hi + lo in fp16 ----
  {
    const int ha = GP == 4 ? (g & 3) : g;
    const float2 pa = *reinterpret_cast<const float2*>(x.ps + ha * kPstr + 2 * t);
    const float2 pb = *reinterpret_cast<const float2*>(x.ps + ha * kPstr + 8 + 2 * t);
    const __half2 ha2 = __float22half2_rn(pa), hb2 = __float22half2_rn(pb);
    const float2 fa = __half22float2(ha2), fb2 = __half22float2(hb2);
    const __half2 la2 = __float22half2_rn(make_float2(pa.x - fa.x, pa.y - fa.y));
    const __half2 lb2 = __float22half2_rn(make_float2(pb.x - fb2.x, pb.y - fb2.y));
    const uint32_t uha = *reinterpret_cast<const uint32_t*>(&ha2), uhb = *reinterpret_cast<const uint32_t*>(&hb2);
    const uint32_t ula = *reinterpret_cast<const uint32_t*>(&la2), ulb = *reinterpret_cast<const uint32_t*>(&lb2);
    uint4 fr;
    if (GP == 4) {
      const bool lo_part = g >= 4;          // rows 0-3: hi parts, rows 4-7: lo parts, rows 8-15: zero
      fr = make_uint4(lo_part ? ula : uha, 0u, lo_part ? ulb : uhb, 0u);
    } else {
      fr = make_uint4(uha, ula, uhb, ulb);  // row g: hi, row g+8: lo
    }
    x.fb[(warp * MB) * 32 + lane] = fr;
  }
  named_barrier_sync(1, 128);

#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    const uint4 fr = x.fb[(ks * MB) * 32 + lane];
    const uint32_t af[4] = {fr.x, fr.y, fr.z, fr.w};
#pragma unroll
    for (int nbp = 0; nbp < NBW / 2; ++nbp) {
      uint32_t bf[4];
      ldsm_x4_t(bf, vt + (uint32_t)(ks * 16 * 2 * D) + x.lo.hv[nbp]);   // 16 rows: a multiple of the XOR period
      mma_f16(st.acc[0][2 * nbp], af, bf[0], bf[1]);
      mma_f16(st.acc[0][2 * nbp + 1], af, bf[2], bf[3]);
    }
  }
  return true;
}

template <int D, int GP, bool CI8>
__global__ void __launch_bounds__(160, 2) attn_kernel(Cache c, AttnLaunch a, int splits, int units, float qscale) {
  chain_enter();
  using C = Cfg<D, GP, CI8>;
  using Q = QF<D, GP>;
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* stages = smem;
  float* ps_all = reinterpret_cast<float*>(smem + C::PS_OFF);
  uint4* fb_all = reinterpret_cast<uint4*>(smem + C::FB_OFF);
  float* wmax = reinterpret_cast<float*>(smem + C::WM_OFF);
  float* lsum = reinterpret_cast<float*>(smem + C::LS_OFF);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + C::NSTAGE;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::FLAG_OFF);
  volatile int* uq = reinterpret_cast<volatile int*>(smem + C::UQ_OFF);
  volatile int* uqn = reinterpret_cast<volatile int*>(smem + C::UN_OFF);
  uint64_t* qfull = reinterpret_cast<uint64_t*>(smem + C::QBAR_OFF);
  uint64_t* qempty = qfull + 1;
  unsigned char* qsm = smem + C::QS_OFF;   // valid when C::QSM

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Zero the stage ring once: rows a tile does not fill then hold zeros or an
  // earlier tile's data, never uninitialised bits.
  for (int i = threadIdx.x; i < C::NSTAGE * C::STAGE / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(stages)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_shared();
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::NCW);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, C::NCW);
    abort_flag[0] = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == C::NCW) {
    // ------------------------------ producer -------------------------------
    // One lane issues every copy. On a timed-out wait the copies already
    // issued are waited for (bounded) so that none lands after the CTA exits.
    if (lane == 0) {
      // Units are claimed one at a time from a launch-wide counter, so CTAs
      // that drew short segments take more of them (no static tail). Each
      // claimed unit id goes into the queue uq before the unit's first stage
      // is published; a unit without tiles, and the end, are published as a
      // stage without data.
      int ctr = 0;
      int nq = 0;   // query-operand copies issued
      // K/V tiles are read once per step: they go first when L2 needs room
      const uint64_t stream_policy = l2_evict_first_policy();
      auto copy = [&](void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
        bulk_g2s_hint(dst, src, bytes, bar, stream_policy);
      };
      bool stop = false;
      auto next_stage = [&]() -> int {
        const int st = ctr % C::NSTAGE;
        if (ctr >= C::NSTAGE && !mbar_wait_bounded(&empty[st], ((ctr / C::NSTAGE) - 1) & 1)) {
          set_error(c.err, kErrDevice);
          *abort_flag = 1;
        }
        if (*abort_flag) stop = true;
        return st;
      };
      for (int k = 0; !stop; ++k) {
        const int unit = atomicAdd(a.sched, 1);
        if (unit >= units) {
          const int st = next_stage();
          uq[k % C::UQ] = -1;                       // the end
          if (!stop) {
            mbar_arrive(&full[st]);
            ++ctr;
          }
          break;
        }
        const Unit u = make_unit<D, GP, CI8>(c, a.r, splits, unit);
        uq[k % C::UQ] = unit;
        uqn[k % C::UQ] = u.n_cold;
        // the consumers load the unit's query operands when they reach it (up
        // to NSTAGE tiles from now)
        if constexpr (C::QSM) {
          // into the one shared slot, once the consumers have read the previous unit's
          if (k > 0 && !mbar_wait_bounded(qempty, (k - 1) & 1)) {
            set_error(c.err, kErrDevice);
            *abort_flag = 1;
            stop = true;
            break;
          }
          mbar_arrive_expect_tx(qfull, (uint32_t)Q::BYTES);
          bulk_g2s(qsm, a.qfrag + (size_t)u.s * a.qf_stride, (uint32_t)Q::BYTES, qfull);
          ++nq;
        }
        if (u.t0 == u.t1) {
          const int st = next_stage();
          if (stop) break;
          mbar_arrive(&full[st]);                   // no data: the consumers only close the unit
          ++ctr;
          continue;
        }
        for (int t = u.t0; t < u.t1; ++t) {
          const int st = next_stage();
          if (stop) break;
          unsigned char* sb = stages + st * C::STAGE;
          const bool cold = t < u.tiles_c;
          const int j0 = cold ? t * C::TTC : (t - u.tiles_c) * C::TTR;
          if (kChecked) {
            const int cnt = cold ? min(C::TTC, u.n_cold - j0) : C::TTR;
            const int lim = cold ? c.cap : c.Wst;
            if (!guard(cnt >= 1 && j0 >= 0 && j0 + (cold && CI8 ? ((cnt + 31) & ~31) : C::TTR) <= lim, c.err,
                       kSiteAttnTile, u.s, j0)) {
              *abort_flag = 1;
              stop = true;
              break;
            }
          }
          if (cold && CI8) {
            const int cnt = min(C::TTC, u.n_cold - j0);
            const int cnt4 = (cnt + 3) & ~3;
            const uint32_t kbytes = (uint32_t)(D == 64 ? ((cnt + 1) & ~1) : cnt) * D;   // whole 128-byte lines
            const uint32_t vbytes = (uint32_t)((cnt + 31) >> 5) * 32 * D;                // whole 32-token blocks
            mbar_arrive_expect_tx(&full[st], kbytes + vbytes + 2u * cnt4 * 4u);
            const size_t row0 = (size_t)u.s * c.cap + j0;
            copy(sb, c.k8 + row0 * D, kbytes, &full[st]);
            copy(sb + C::KVB, c.v8 + row0 * D, vbytes, &full[st]);
            copy(sb + 2 * C::KVB, c.ks + row0, cnt4 * 4, &full[st]);
            copy(sb + 2 * C::KVB + 512, c.vs + row0, cnt4 * 4, &full[st]);
          } else if (cold) {
            // fp16 cold rows: the whole 64-row tile (rows past n_cold hold finite older data or zeros)
            const uint32_t kvb = (uint32_t)C::TTR * 2 * D;
            mbar_arrive_expect_tx(&full[st], 2 * kvb);
            const size_t row0 = (size_t)u.s * c.cap + j0;
            copy(sb, c.kc + row0 * D, kvb, &full[st]);
            copy(sb + C::KVB, c.vc + row0 * D, kvb, &full[st]);
          } else {
            // window ring: the whole 64-slot tile (the ring stride is a multiple of 64)
            const uint32_t kvb = (uint32_t)C::TTR * 2 * D;
            mbar_arrive_expect_tx(&full[st], 2 * kvb + C::TTR * 4);
            const size_t row0 = (size_t)u.s * c.Wst + j0;
            copy(sb, c.kr + row0 * D, kvb, &full[st]);
            copy(sb + C::KVB, c.vr + row0 * D, kvb, &full[st]);
            copy(sb + 2 * C::KVB, c.pos_r + row0, C::TTR * 4, &full[st]);
          }
          ++ctr;
        }
      }
      if (stop) {
        for (int k = max(0, ctr - C::NSTAGE); k < ctr; ++k)
          (void)mbar_wait_bounded(&full[k % C::NSTAGE], (k / C::NSTAGE) & 1, 1000000000ll);
        if (C::QSM && nq > 0) (void)mbar_wait_bounded(qfull, (nq - 1) & 1, 1000000000ll);
      }
    }
    __syncthreads();
    return;
  }

  // -------------------------------- consumers --------------------------------
  const int g = lane >> 2, t = lane & 3;
  const LaneOffsets lane_offs = lane_offsets<D>(warp, lane);
  // scores: evict-last, so that their lines are not written back while the K/V tiles stream
  const uint64_t keep_policy = l2_evict_last_policy();
  int ctr = 0;
  for (int k = 0;; ++k) {
    // the next unit: its id is published with its first stage
    {
      const bool ok = mbar_wait_bounded(&full[ctr % C::NSTAGE], (ctr / C::NSTAGE) & 1);
      if (!ok) {
        set_error(c.err, kErrDevice);
        *abort_flag = 1;
      }
    }
    const int unit = uq[k % C::UQ];
    if (named_barrier_or(2, 128, unit < 0 || *abort_flag != 0)) break;   // the end, or an abort
    const Unit u = make_unit<D, GP, CI8>(c, a.r, splits, unit, uqn[k % C::UQ]);
    const unsigned char* qf = a.qfrag + (size_t)u.s * a.qf_stride;
    if constexpr (C::QSM) {
      if (!mbar_wait_bounded(qfull, k & 1)) {
        set_error(c.err, kErrDevice);
        *abort_flag = 1;
      }
      qf = qsm;
    }
    uint2 qi[C::KB][C::NB];
    float cq8[C::HPL];
    if constexpr (CI8) {
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
        for (int nb = 0; nb < C::NB; ++nb)
          qi[kb][nb] = reinterpret_cast<const uint2*>(qf + Q::I8_OFF)[(kb * C::NB + nb) * 32 + lane];
#pragma unroll
      for (int j = 0; j < C::HPL; ++j) cq8[j] = reinterpret_cast<const float*>(qf + Q::CQ_OFF)[t + 4 * j];
    }
    uint2 qh[C::KS];
#pragma unroll
    for (int ks = 0; ks < C::KS; ++ks) qh[ks] = reinterpret_cast<const uint2*>(qf + Q::H_OFF)[ks * 32 + lane];
    if constexpr (C::QSM) {
      __syncwarp();   // every lane of the warp has read the slot
      if (lane == 0) mbar_arrive(qempty);
    }

    SoftmaxState<D, GP> st;
#pragma unroll
    for (int h = 0; h < GP; ++h) st.m[h] = -CUDART_INF_F;
#pragma unroll
    for (int mb = 0; mb < C::MB; ++mb)
#pragma unroll
      for (int nb = 0; nb < C::NBW; ++nb)
#pragma unroll
        for (int k = 0; k < 4; ++k) st.acc[mb][nb][k] = 0.0f;
#pragma unroll
    for (int j = 0; j < C::HPL; ++j) st.lp8[j] = 0.0f;
    st.lp16[0] = st.lp16[1] = 0.0f;
    unsigned long long n_rows_c = 0, n_rows_r = 0;

    TileCtx x;
    x.ps = ps_all + warp * GP * kPstr;
    x.wmax = wmax;
    x.abort_flag = abort_flag;
    x.sc_base = a.scores + (size_t)u.s * c.G * a.score_stride;
    x.warp = warp;
    x.lane = lane;
    x.lo = lane_offs;
    x.keep_policy = keep_policy;
    bool aborted = false;
    if (u.t0 == u.t1) {   // a stage without data: release it and close the unit
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[ctr % C::NSTAGE]);
      ++ctr;
    }
    for (int tt = u.t0; tt < u.t1; ++tt) {
      const int stg = ctr % C::NSTAGE;
      x.ok = mbar_wait_bounded(&full[stg], (ctr / C::NSTAGE) & 1);
      if (!x.ok) {
        set_error(c.err, kErrDevice);
        *abort_flag = 1;
      }
      x.sb = stages + stg * C::STAGE;
      x.fb = fb_all + (ctr & 1) * C::FB_ONE;
      bool go;
      if (tt < u.tiles_c) {
        x.j0 = tt * C::TTC;
        x.cnt = min(C::TTC, u.n_cold - x.j0);
        if constexpr (CI8) go = consume_i8<D, GP>(c, a, x, st, qi, cq8, n_rows_c);
        else go = consume_h<D, GP, false>(c, a, x, st, qh, qscale, n_rows_c);
      } else {
        x.j0 = (tt - u.tiles_c) * C::TTR;
        x.cnt = min(C::TTR, c.W - x.j0);
        go = consume_h<D, GP, true>(c, a, x, st, qh, qscale, n_rows_r);
      }
      if (!go) {
        aborted = true;
        break;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stg]);
      ++ctr;
    }

    // ---- softmax sums over the CTA, then this unit's output ----
#pragma unroll
    for (int h = 0; h < GP; ++h) {
      float v = 0.0f;
#pragma unroll
      for (int j = 0; j < C::HPL; ++j) v += (t + 4 * j == h) ? st.lp8[j] : 0.0f;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) v += (2 * t + cc == h) ? st.lp16[cc] : 0.0f;
      v = warp_sum(v);
      if (lane == 0) lsum[warp * GP + h] = v;
    }
    if (lane == 0) {
      atomicAdd(&c.counters[kCntAttnInt8], CI8 ? n_rows_c : 0ull);
      atomicAdd(&c.counters[kCntAttnFp16], n_rows_r + (CI8 ? 0ull : n_rows_c));
    }
    named_barrier_sync(2, 128);
    float L[GP];
#pragma unroll
    for (int h = 0; h < GP; ++h) L[h] = lsum[h] + lsum[GP + h] + lsum[2 * GP + h] + lsum[3 * GP + h];
    const int item = unit / splits;
    const int split = unit - item * splits;
    const int ha = GP == 4 ? (g & 3) : g;
    const bool writer = (GP == 4 ? g < 4 : true) && ha < c.G;
    const float Lh = sel(L, ha), Mh = sel(st.m, ha);
    const size_t orow = (size_t)((u.l - a.r.l0) * a.r.B + u.b) * c.Hq + (size_t)u.h * c.G + ha;
    float* pp = a.part + ((size_t)(item * splits + split) * c.G + ha) * (D + 2);
#pragma unroll
    for (int nb = 0; nb < C::NBW; ++nb) {
      float o0, o1;
      if constexpr (GP == 4) {
        o0 = st.acc[0][nb][0] + st.acc[0][nb][2];
        o1 = st.acc[0][nb][1] + st.acc[0][nb][3];
        o0 += __shfl_xor_sync(0xffffffffu, o0, 16);
        o1 += __shfl_xor_sync(0xffffffffu, o1, 16);
      } else {
        o0 = (st.acc[0][nb][0] + st.acc[0][nb][2]) + (st.acc[1][nb][0] + st.acc[1][nb][2]);
        o1 = (st.acc[0][nb][1] + st.acc[0][nb][3]) + (st.acc[1][nb][1] + st.acc[1][nb][3]);
      }
      const int d = warp * (D / 4) + nb * 8 + 2 * t;
      if (writer && !aborted) {
        if (splits == 1) {
          if (kChecked && !guard(orow < (size_t)a.r.items(c.Hkv) * c.G, c.err, kSiteAttnOut, u.s, (int)orow)) continue;
          *reinterpret_cast<float2*>(a.out + orow * D + d) = make_float2(o0 / Lh, o1 / Lh);
        } else {
          *reinterpret_cast<float2*>(pp + d) = make_float2(o0, o1);
        }
      }
    }
    if (writer && !aborted && warp == 0 && t == 0) {
      if (splits == 1) {
        const float lse = (Mh + __log2f(Lh)) * kLn2;
        a.lse_ws[(size_t)u.s * c.G + ha] = lse;
        if (a.lse_out) a.lse_out[orow] = lse;
      } else {
        pp[D] = Mh;
        pp[D + 1] = Lh;
      }
    }
    // leave together when any warp saw an abort (same answer in every consumer thread)
    if (named_barrier_or(2, 128, aborted || *abort_flag != 0)) break;
  }
  __syncthreads();
  // the last CTA to finish resets the unit counter for the next launch
  if (threadIdx.x == 0 && atomicAdd(a.sched + 1, 1) == (int)gridDim.x - 1) {
    a.sched[0] = 0;
    a.sched[1] = 0;
  }
}

// ---------------------------------------------------------------------------
// combine split partials: one warp per (item, head)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) combine_kernel(Cache c, AttnLaunch a, int splits) {
  chain_enter();
  const int G = c.G;
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

template <int D, int GP, bool CI8>
cudaError_t run_attn(const Cache& c, const Policy& pol, const AttnLaunch& a, cudaStream_t st, long long* launches,
                     Prof* prof) {
  using C = Cfg<D, GP, CI8>;
  const int items = a.r.items(c.Hkv);
  const float qscale = rsqrtf((float)D);
  {
    ProfScope ps(prof, kKAppend, st);
    (void)launch_chained(append_kernel<D, GP>, (items * 32 + 255) / 256, 256, 0, st, c, a, pol, qscale);
  }
  ++*launches;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_kernel<D, GP, CI8>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  int ctas_per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ctas_per_sm, attn_kernel<D, GP, CI8>, 160, C::SMEM);
  if (e != cudaSuccess) return e;
  ctas_per_sm = max(1, ctas_per_sm);
  const int resident = a.num_sms * ctas_per_sm;
  const int tiles_ub = (a.max_cold_tokens + C::TTC - 1) / C::TTC + (c.W + C::TTR - 1) / C::TTR;
  int splits = 1;
  if (items < 2 * resident) {
    // few segments: split the token axis so that every SM has work
    splits = (2 * resident + items - 1) / items;
    splits = min(splits, max(1, tiles_ub / 2));
  } else if (tiles_ub >= 32) {
    // long segments: finer units even out the last wave
    splits = min((16 * resident + items - 1) / items, tiles_ub / 8);
    splits = max(1, splits);
  }
  while (splits > 1 && (long long)items * splits > a.part_units) --splits;
  const int units = items * splits;
  const int grid = min(units, resident);
  {
    ProfScope ps(prof, kKAttention, st);
    (void)launch_chained(attn_kernel<D, GP, CI8>, grid, 160, C::SMEM, st, c, a, splits, units, qscale);
  }
  ++*launches;
  if (splits > 1) {
    const int warps = items * c.G;
    ProfScope ps(prof, kKCombine, st);
    (void)launch_chained(combine_kernel<D>, (warps * 32 + 255) / 256, 256, 0, st, c, a, splits);
    ++*launches;
  }
  if (pol.mode == 0 && a.run_ema) {
    ProfScope ps(prof, kKEma, st);
    e = run_ema(c, pol, a, st);
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  return cudaGetLastError();
}

template <int D, int GP>
cudaError_t run_attn_gp(const Cache& c, const Policy& pol, const AttnLaunch& a, cudaStream_t st, long long* n,
                        Prof* prof) {
  return c.cold_int8 ? run_attn<D, GP, true>(c, pol, a, st, n, prof) : run_attn<D, GP, false>(c, pol, a, st, n, prof);
}

}  // namespace

int qfrag_bytes(int D, int G) {
  if (D == 128) return G <= 4 ? QF<128, 4>::BYTES : QF<128, 8>::BYTES;
  return G <= 4 ? QF<64, 4>::BYTES : QF<64, 8>::BYTES;
}

cudaError_t launch_decode_attn(const Cache& c, const Policy& pol, const AttnLaunch& a, cudaStream_t st,
                               long long* launches, Prof* prof) {
  if (a.r.items(c.Hkv) == 0) return cudaSuccess;
  if (c.G < 1 || c.G > 8) return cudaErrorInvalidValue;
  if (c.D == 128)
    return c.G <= 4 ? run_attn_gp<128, 4>(c, pol, a, st, launches, prof)
                    : run_attn_gp<128, 8>(c, pol, a, st, launches, prof);
  if (c.D == 64)
    return c.G <= 4 ? run_attn_gp<64, 4>(c, pol, a, st, launches, prof)
                    : run_attn_gp<64, 8>(c, pol, a, st, launches, prof);
  return cudaErrorInvalidValue;
}

}  // namespace confkv
