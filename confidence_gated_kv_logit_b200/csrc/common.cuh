// Device-side view of a CONF-KV cache and helpers shared by the kernels.
//
// Layout in HBM (one "segment" = the cache of one (layer, sequence, KV head)):
//   segment id s = (layer * max_batch + seq) * kv_heads + kv_head
//   cold region  (older tokens, a hole-free prefix [0, n_cold) of `cap` rows)
//       INT8 codes k8/v8 [S][cap][D] + fp32 scales ks/vs [S][cap]   (INT8 on)
//       or fp16 rows  kc/vc [S][cap][D]                              (INT8 off)
//       int32 pos_c [S][cap], fp32 sc_c [S][cap] (EMA, or priority in fixed mode)
//   FP16 window ring (INT8 on only): W slots per segment, slot = pos mod W,
//       allocated with a stride Wst = W rounded up to 4 slots (the linear
//       layout keeps no ring: slots [0, n) hold the window in position order)
//       fp16 kr/vr [S][Wst][D], int32 pos_r [S][Wst] (-1 = empty), fp32 sc_r [S][Wst]
//   int32 n_cold [S], next_pos [S]
// Rows are 64 or 128 B (INT8) and 128 or 256 B (fp16), so every row starts on a
// 16-byte boundary and moves as 128-bit words.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "layout.cuh"

namespace confkv {

// sticky device error codes (values match confkv_status)
constexpr int kErrNonfinite = 4;
constexpr int kErrDevice = 7;

// cumulative counters (confkv_stats)
enum Counter {
  kCntAttnInt8 = 0,
  kCntAttnFp16 = 1,
  kCntEvictScanned = 2,
  kCntMovedRows = 3,
  kCntRequant = 4,
  kCntEvictBlock = 5,
  kCntMovedWin = 6,
  kNumCounters = 8
};

struct Cache {
  int L, Bmax, Hkv, Hq, G, D, W, cap;
  int Wst;            // ring allocation stride per segment: W rounded up to 4 slots
  int cold_int8;
  int linear;         // window without a ring: slots [0, n) hold the FP16 tokens in position order
  int8_t* k8;
  int8_t* v8;
  __half* kc;
  __half* vc;
  float* ks;
  float* vs;
  int32_t* pos_c;
  float* sc_c;
  __half* kr;
  __half* vr;
  int32_t* pos_r;
  float* sc_r;
  int32_t* n_cold;
  int32_t* next_pos;
  int32_t* err;
  unsigned long long* counters;
};

struct Policy {
  int mode;           // 0 confidence, 1 fixed budget
  int n_low, n_high;
  float tau;
  float alpha, one_minus_alpha;   // (1 - alpha) rounded once to fp32
  float beta, one_minus_beta;
  int P;              // protect_last
  int n_sink;
  int fixed_budget;
  int gate;           // 0 prose, 1 literal
  int pyramidal;
  int score_source;   // confkv.h CONFKV_SCORE_*
  uint32_t seed;      // static draws (CONFKV_SCORE_RANDOM)
};

constexpr int kScoreEma = 0, kScoreAccum = 1, kScoreRandom = 2;   // confkv.h CONFKV_SCORE_*

// The static draw of the random ranker for token `pos` of segment (l, b, h):
// SplitMix64 (Steele, Lea and Flood, 2014) at counter pos | h << 32 | b << 40 |
// l << 52, i.e. its output for state seed + (counter + 1) * 0x9E3779B97F4A7C15,
// top 24 bits as a fraction in [0, 1) (exact in fp32).
__host__ __device__ __forceinline__ float random_priority(uint32_t seed, int l, int b, int h, int pos) {
  const unsigned long long ctr = (unsigned long long)(uint32_t)pos | ((unsigned long long)(h & 0xff) << 32) |
                                 ((unsigned long long)(b & 0xfff) << 40) | ((unsigned long long)(l & 0xfff) << 52);
  unsigned long long z = (unsigned long long)seed + (ctr + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  return (float)(z >> 40) * 0x1p-24f;
}

// The initial score source of a token entering the cache (prefill or append)
// in confidence mode: 0 for the EMA and the accumulated mass, the draw for the
// random ranker.
__device__ __forceinline__ float initial_score(const Policy& pol, int l, int b, int h, int pos) {
  return pol.score_source == kScoreRandom ? random_priority(pol.seed, l, b, h, pos) : 0.0f;
}

// A call covers layers [l0, l0 + nl) and sequences [0, B) of every KV head.
struct Range {
  int l0, nl, B;
  __host__ __device__ int items(int Hkv) const { return nl * B * Hkv; }
};

__device__ __forceinline__ int seg_of(const Cache& c, const Range& r, int item, int* l_out, int* b_out,
                                      int* h_out) {
  int per_layer = r.B * c.Hkv;
  int l = r.l0 + item / per_layer;
  int rem = item % per_layer;
  int b = rem / c.Hkv;
  int h = rem % c.Hkv;
  *l_out = l;
  *b_out = b;
  *h_out = h;
  return (l * c.Bmax + b) * c.Hkv + h;
}

__device__ __forceinline__ void set_error(int32_t* err, int code) { atomicCAS(err, 0, code); }

// A global store with an L2 eviction-priority policy (createpolicy).
__device__ __forceinline__ void st_f32_policy(float* p, float v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol) : "memory");
}

// err[0] is the sticky status word; err[1..3] describe the first failed device
// check: (site, segment, offending value).
__device__ __forceinline__ void record_violation(int32_t* err, int site, int seg, int val) {
  if (atomicCAS(err, 0, kErrDevice) == 0) {
    err[1] = site;
    err[2] = seg;
    err[3] = val;
  }
}

// Returns ok; records the first failure. Used for checks that are always on
// (per segment) and, in builds with CONFKV_CHECKED, for every data-dependent index.
__device__ __forceinline__ bool guard(bool ok, int32_t* err, int site, int seg, int val) {
  if (!ok) record_violation(err, site, seg, val);
  return ok;
}

#ifdef CONFKV_CHECKED
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif

// Check sites (value of err[1]).
enum Site {
  kSiteAppendSeg = 101, kSiteAppendSlot = 102,
  kSiteAttnSeg = 201, kSiteAttnTile = 202, kSiteAttnScore = 203, kSiteAttnOut = 204, kSiteAttnQ = 205,
  kSiteEmaSeg = 301, kSiteEmaCol = 302,
  kSiteEvictSeg = 401, kSiteEvictPair = 402, kSiteEvictRequant = 403, kSiteEvictWord = 404,
  kSitePrefillRow = 501, kSiteCombine = 601
};

// ---------------------------------------------------------------------------
// Exact int8 -> fp32 conversion without the conversion unit: the biased byte
// u = x + 128 is permuted into the low mantissa byte of 2^23 (bit pattern
// 0x4B0000uu, value 2^23 + u), and one fp32 subtraction of 2^23 + 128 leaves
// x exactly. Four bytes of one word give two float2 pairs; the subtraction is
// a packed f32x2 add.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void i8x4_to_f2x2(uint32_t w, float2& lo, float2& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const float2 bias = make_float2(-8388736.0f, -8388736.0f);
  float2 a, b;
  a.x = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540));
  a.y = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541));
  b.x = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542));
  b.y = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543));
  lo = __fadd2_rn(a, bias);
  hi = __fadd2_rn(b, bias);
}

// 2^x with the SFU's approximation (relative error about 2^-22; results below
// 2^-126 flush to zero): the softmax weights and the EMA terms.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float2 h2_to_f2(uint32_t w) {
  return __half22float2(*reinterpret_cast<const __half2*>(&w));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Order-preserving map of an fp32 score to uint32 (-0 is folded onto +0).
__device__ __forceinline__ uint32_t ordered_bits(float f) {
  uint32_t u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Ranking score of one token: fixed mode ranks by the stored priority;
// confidence mode by fl(fl(alpha*ema) + fl((1-alpha)*rec)), rec = (pos+1)/(t+1),
// every operation an IEEE fp32 operation with no contraction.
__device__ __forceinline__ float rank_score(const Policy& p, float sc, int pos, int t) {
  if (p.mode == 1) return sc;
  const float rec = __fdiv_rn((float)(pos + 1), (float)(t + 1));
  return __fadd_rn(__fmul_rn(p.alpha, sc), __fmul_rn(p.one_minus_alpha, rec));
}

__device__ __forceinline__ unsigned long long rank_key(const Policy& p, float sc, int pos, int t) {
  return ((unsigned long long)ordered_bits(rank_score(p, sc, pos, t)) << 32) | (uint32_t)pos;
}

constexpr unsigned long long kNoKey = ~0ull;

// ---------------------------------------------------------------------------
// Row access by one warp: lane l holds the E = D/32 consecutive dimensions
// E*l .. E*l+E-1 of a row, as D/64 words of fp16 pairs. "region" arguments are
// the start of one segment's rows; the placement formulas are in layout.cuh.
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void row_load_plain(const __half* __restrict__ row, int lane, uint32_t (&w)[D / 64]) {
  if constexpr (D == 128) {
    const uint2 v = reinterpret_cast<const uint2*>(row)[lane];
    w[0] = v.x;
    w[1] = v.y;
  } else {
    w[0] = reinterpret_cast<const uint32_t*>(row)[lane];
  }
}

template <int D>
__device__ __forceinline__ void row_load_h(const __half* __restrict__ region, int i, int lane, uint32_t (&w)[D / 64]) {
  const unsigned char* p = reinterpret_cast<const unsigned char*>(region) + h_off(i, lane * (D / 16), D);
  if constexpr (D == 128) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x;
    w[1] = v.y;
  } else {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  }
}

template <int D>
__device__ __forceinline__ void row_store_h(__half* __restrict__ region, int i, int lane, const uint32_t (&w)[D / 64]) {
  unsigned char* p = reinterpret_cast<unsigned char*>(region) + h_off(i, lane * (D / 16), D);
  if constexpr (D == 128) {
    *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
  } else {
    *reinterpret_cast<uint32_t*>(p) = w[0];
  }
}

// Symmetric per-row INT8 quantisation: amax = max |x| over the row, scale =
// amax / 127 and code = clamp(rint_half_even(x / scale), +-127), both
// divisions IEEE fp32; a zero row gets scale 0 and codes 0. Returns the scale
// (the same in every lane) and the lane's E codes packed little-endian.
template <int D>
__device__ __forceinline__ float row_quantize(const uint32_t (&w)[D / 64], uint32_t* packed) {
  constexpr int E = D / 32;
  float x[E];
#pragma unroll
  for (int k = 0; k < D / 64; ++k) {
    const float2 f = h2_to_f2(w[k]);
    x[2 * k] = f.x;
    x[2 * k + 1] = f.y;
  }
  float amax = 0.0f;
#pragma unroll
  for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(x[e]));
  amax = warp_max(amax);
  const float scale = __fdiv_rn(amax, 127.0f);
  uint32_t pk = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    int q = 0;
    if (scale != 0.0f) {
      q = __float2int_rn(__fdiv_rn(x[e], scale));
      q = max(-127, min(127, q));
    }
    pk |= ((uint32_t)(q & 0xff)) << (8 * e);
  }
  *packed = pk;
  return scale;
}

template <int D>
__device__ __forceinline__ void row_store_k8(int8_t* __restrict__ region, int i, int lane, uint32_t packed) {
  int8_t* p = region + k8_off(i, lane * (D / 32), D);
  if constexpr (D == 128) *reinterpret_cast<uint32_t*>(p) = packed;
  else *reinterpret_cast<uint16_t*>(p) = (uint16_t)packed;
}

template <int D>
__device__ __forceinline__ void row_store_v8(int8_t* __restrict__ region, int i, int lane, uint32_t packed) {
#pragma unroll
  for (int e = 0; e < D / 32; ++e) region[v8_off(i, lane * (D / 32) + e, D)] = (int8_t)(packed >> (8 * e));
}

// Quantise fp16 row `src_i` of a permuted fp16 region (K and V) into cold
// row `dst_i` (codes and scales); one warp.
template <int D>
__device__ __forceinline__ void warp_requant(const Cache& c, int s, int ring_slot, int cold_i, int lane) {
  const size_t rb = (size_t)s * c.Wst * D, cb = (size_t)s * c.cap * D, cs = (size_t)s * c.cap + cold_i;
  uint32_t w[D / 64], pk;
  row_load_h<D>(c.kr + rb, ring_slot, lane, w);
  float sc = row_quantize<D>(w, &pk);
  row_store_k8<D>(c.k8 + cb, cold_i, lane, pk);
  if (lane == 0) c.ks[cs] = sc;
  row_load_h<D>(c.vr + rb, ring_slot, lane, w);
  sc = row_quantize<D>(w, &pk);
  row_store_v8<D>(c.v8 + cb, cold_i, lane, pk);
  if (lane == 0) c.vs[cs] = sc;
}

// Linear window layout: move window slots [from, n) of segment s down to
// [0, n - from), positions and score sources with them, and empty the slots
// left behind; one warp. Rows are loaded four at a time before any is stored
// (every destination is below its source, so no row is overwritten before it
// has been read).
template <int D>
__device__ __forceinline__ void warp_window_shift(const Cache& c, int s, int from, int n, int lane) {
  if (from <= 0 || n <= from) {
    if (lane == 0)
      for (int j = max(0, n - from); j < n; ++j) c.pos_r[(size_t)s * c.Wst + j] = -1;
    return;
  }
  __half* kr = c.kr + (size_t)s * c.Wst * D;
  __half* vr = c.vr + (size_t)s * c.Wst * D;
  int32_t* pr = c.pos_r + (size_t)s * c.Wst;
  float* sr = c.sc_r + (size_t)s * c.Wst;
  for (int j = from; j < n; j += 4) {
    uint32_t k[4][D / 64], v[4][D / 64];
    int pp[4];
    float ss[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (j + u < n) {
        row_load_h<D>(kr, j + u, lane, k[u]);
        row_load_h<D>(vr, j + u, lane, v[u]);
        pp[u] = pr[j + u];
        ss[u] = sr[j + u];
      }
    __syncwarp();
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (j + u < n) {
        row_store_h<D>(kr, j + u - from, lane, k[u]);
        row_store_h<D>(vr, j + u - from, lane, v[u]);
        if (lane == 0) {
          pr[j + u - from] = pp[u];
          sr[j + u - from] = ss[u];
        }
      }
    __syncwarp();
  }
  if (lane == 0)
    for (int j = n - from; j < n; ++j) pr[j] = -1;
  __syncwarp();
}

// ---------------------------------------------------------------------------
// Chained launches (programmatic dependent launch). The kernels of one decode
// step follow one another on the caller's stream; each is launched with
// programmatic stream serialisation, so its CTAs may be scheduled while the
// previous kernel is still finishing. Every chained kernel starts with
// chain_enter(): it waits until the previous kernel has completed and its
// writes are visible (so nothing is read or written early), then lets the next
// kernel of the stream begin launching. Because each kernel waits before it
// releases its successor, at most two kernels of the chain are resident at a
// time and completion stays transitive: a kernel that has passed
// chain_enter() knows every earlier kernel of the stream has completed. A
// kernel launched without the attribute passes straight through.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void chain_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... P, typename... A>
cudaError_t launch_chained(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, A&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<A&&>(args)...);
}

}  // namespace confkv
