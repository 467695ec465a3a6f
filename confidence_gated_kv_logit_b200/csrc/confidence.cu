// Confidence of the next-token distribution and the per-layer budget
// (CONF-KV post, decode-loop pseudo-code and method paragraphs; CONF-KV
// abstract for the gate polarity and the pyramidal variant).
//
// One pass over each row of logits keeps, per thread, the running maximum m,
// S = sum exp(l - m), T = sum exp(l - m) (l - m) and the two largest logits
// counted with multiplicity. Partials are merged with
//   m = max(m_a, m_b),  S = S_a e^(m_a-m) + S_b e^(m_b-m),
//   T = e^(m_a-m) (T_a + (m_a-m) S_a) + e^(m_b-m) (T_b + (m_b-m) S_b),
// which follows from the definitions. Then
//   H = ln S - T/S,  max p = 1/S,  margin = l_(1) - l_(2)  (= log p_(1) - log p_(2)),
//   c = 0.4 (1 - H / ln V) + 0.3 sigmoid(margin) + 0.3 / S.
// A row is split over several CTAs; each writes its partial and takes a ticket
// from an atomic counter, and the CTA that takes the last ticket merges the
// partials and writes c and the budgets (no CTA waits on another).
#include <math_constants.h>

#include "common.cuh"
#include "kernels.h"

namespace confkv {

namespace {

constexpr int NT = 256;

__device__ __forceinline__ void top2_insert(float x, float& t1, float& t2) {
  if (x > t1) {
    t2 = t1;
    t1 = x;
  } else if (x > t2) {
    t2 = x;
  }
}

__device__ __forceinline__ void merge(ConfPartial& a, const ConfPartial& b) {
  a.bad |= b.bad;
  top2_insert(b.top1, a.top1, a.top2);
  top2_insert(b.top2, a.top1, a.top2);
  if (b.S == 0.0f) return;
  if (a.S == 0.0f) {
    a.m = b.m;
    a.S = b.S;
    a.T = b.T;
    return;
  }
  const float m = fmaxf(a.m, b.m);
  const float da = a.m - m, db = b.m - m;
  const float fa = __expf(da), fb = __expf(db);
  a.T = fa * fmaf(da, a.S, a.T) + fb * fmaf(db, b.S, b.T);
  a.S = fa * a.S + fb * b.S;
  a.m = m;
}

__device__ __forceinline__ ConfPartial shfl_partial(const ConfPartial& p, int o) {
  ConfPartial q;
  q.m = __shfl_xor_sync(0xffffffffu, p.m, o);
  q.S = __shfl_xor_sync(0xffffffffu, p.S, o);
  q.T = __shfl_xor_sync(0xffffffffu, p.T, o);
  q.top1 = __shfl_xor_sync(0xffffffffu, p.top1, o);
  q.top2 = __shfl_xor_sync(0xffffffffu, p.top2, o);
  q.bad = __shfl_xor_sync(0xffffffffu, p.bad, o);
  return q;
}

__global__ void __launch_bounds__(NT) confidence_kernel(ConfLaunch a, Policy pol) {
  chain_enter();
  __shared__ ConfPartial wpart[NT / 32];
  __shared__ int is_last;
  const int row = blockIdx.y;
  const int chunk = (a.V + a.cpr - 1) / a.cpr;
  const int v0 = blockIdx.x * chunk;
  const int v1 = min(a.V, v0 + chunk);
  const float* lg = a.logits + (size_t)row * a.V;

  // Each pass loads U logits per thread into registers (a CTA's whole chunk
  // in one pass when the row is split vocab/4096 ways). The CTA first agrees on
  // the pass maximum M, so every thread sums S = sum e^(l-M) and
  // T = sum e^(l-M)(l-M) against the same M and the block reductions are plain
  // sums; the top two are kept branch-free, counted with multiplicity
  // (t2 = max(t2, min(t1, x)), t1 = max(t1, x)).
  __shared__ float red[NT / 32][4];
  __shared__ int red_bad[NT / 32];
  constexpr int U = 16;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  ConfPartial cta;   // meaningful in thread 0
  cta.m = -CUDART_INF_F;
  cta.S = 0.0f;
  cta.T = 0.0f;
  cta.top1 = -CUDART_INF_F;
  cta.top2 = -CUDART_INF_F;
  cta.bad = 0;
  for (int base = v0; base < v1; base += NT * U) {
    float x[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * NT + threadIdx.x;
      x[u] = i < v1 ? __ldcs(lg + i) : -CUDART_INF_F;
    }
    float mx = -CUDART_INF_F, t1 = -CUDART_INF_F, t2 = -CUDART_INF_F;
    bool bad = false;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * NT + threadIdx.x;
      const bool finite = fabsf(x[u]) <= 3.402823466e38f;
      bad |= i < v1 && !finite;
      if (!finite) x[u] = -CUDART_INF_F;        // out of range or non-finite: no contribution
      mx = fmaxf(mx, x[u]);
      t2 = fmaxf(t2, fminf(t1, x[u]));
      t1 = fmaxf(t1, x[u]);
    }
    mx = warp_max(mx);
    if (lane == 0) red[wid][0] = mx;
    __syncthreads();
    float M = red[0][0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) M = fmaxf(M, red[w][0]);
    float S = 0.0f, T = 0.0f;
    if (M != -CUDART_INF_F) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float d = x[u] - M;                 // -inf for the excluded elements
        const float ev = __expf(d);               // 0 for them
        S += ev;
        T = fmaf(ev, ev > 0.0f ? d : 0.0f, T);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      S += __shfl_xor_sync(0xffffffffu, S, o);
      T += __shfl_xor_sync(0xffffffffu, T, o);
      const float o1 = __shfl_xor_sync(0xffffffffu, t1, o), o2 = __shfl_xor_sync(0xffffffffu, t2, o);
      t2 = fmaxf(fminf(t1, o1), fmaxf(t2, o2));
      t1 = fmaxf(t1, o1);
    }
    const bool wbad = __any_sync(0xffffffffu, bad);
    __syncthreads();   // every thread has read red[.][0]
    if (lane == 0) {
      red[wid][0] = S;
      red[wid][1] = T;
      red[wid][2] = t1;   // the warp's top two
      red[wid][3] = t2;
      red_bad[wid] = wbad ? 1 : 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      ConfPartial q;
      q.m = M;
      q.S = 0.0f;
      q.T = 0.0f;
      q.top1 = -CUDART_INF_F;
      q.top2 = -CUDART_INF_F;
      q.bad = 0;
      for (int w = 0; w < NT / 32; ++w) {
        q.S += red[w][0];
        q.T += red[w][1];
        q.bad |= red_bad[w];
        q.top2 = fmaxf(fminf(q.top1, red[w][2]), fmaxf(q.top2, red[w][3]));
        q.top1 = fmaxf(q.top1, red[w][2]);
      }
      if (M == -CUDART_INF_F) q.S = 0.0f;
      merge(cta, q);
    }
    __syncthreads();   // red is reused by the next pass
  }
  if (threadIdx.x == 0) {
    a.part[(size_t)row * a.cpr + blockIdx.x] = cta;
    __threadfence();
    const unsigned prev = atomicAdd(&a.tickets[row], 1u);
    is_last = (prev == (unsigned)a.cpr - 1u);
  }
  __syncthreads();
  if (!is_last) return;

  // last CTA of this row: every thread loads one partial (read past L1), then
  // the same warp and block merge as above
  __threadfence();
  ConfPartial acc;
  acc.m = -CUDART_INF_F;
  acc.S = 0.0f;
  acc.T = 0.0f;
  acc.top1 = -CUDART_INF_F;
  acc.top2 = -CUDART_INF_F;
  acc.bad = 0;
  const ConfPartial* pp = a.part + (size_t)row * a.cpr;
  for (int k = threadIdx.x; k < a.cpr; k += NT) {
    ConfPartial q;
    q.m = __ldcg(&pp[k].m);
    q.S = __ldcg(&pp[k].S);
    q.T = __ldcg(&pp[k].T);
    q.top1 = __ldcg(&pp[k].top1);
    q.top2 = __ldcg(&pp[k].top2);
    q.bad = __ldcg(&pp[k].bad);
    merge(acc, q);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const ConfPartial q = shfl_partial(acc, o);
    merge(acc, q);
  }
  __syncthreads();   // every thread is done with wpart from the first merge
  if ((threadIdx.x & 31) == 0) wpart[threadIdx.x >> 5] = acc;
  __syncthreads();
  __shared__ int n_sh;
  if (threadIdx.x == 0) {
    acc = wpart[0];
    for (int w = 1; w < NT / 32; ++w) merge(acc, wpart[w]);
    a.tickets[row] = 0u;   // ready for the next launch
    float c;
    int N;
    const int larger = max(pol.n_low, pol.n_high);
    if (acc.bad || !(acc.S > 0.0f)) {
      c = CUDART_NAN_F;
      N = larger;
      set_error(a.err, kErrNonfinite);
    } else {
      const float H = logf(acc.S) - acc.T / acc.S;
      const float norm_entropy = H / logf((float)a.V);
      const float margin = acc.top1 - acc.top2;
      const float sig = 1.0f / (1.0f + expf(-margin));
      const float p_max = 1.0f / acc.S;
      c = 0.4f * (1.0f - norm_entropy) + 0.3f * sig + 0.3f * p_max;
      const bool confident = c >= pol.tau;
      if (pol.gate == 0) N = confident ? pol.n_low : pol.n_high;
      else N = confident ? pol.n_high : pol.n_low;
    }
    a.c_ws[row] = c;
    if (a.c_out) a.c_out[row] = c;
    n_sh = N;
  }
  __syncthreads();
  // the per-layer budgets, one layer per thread
  const int N = n_sh;
  for (int l = threadIdx.x; l < a.L; l += NT) {
    int bl = N;
    if (pol.pyramidal && a.L > 1) {
      const long long L1 = a.L - 1;
      bl = (int)(((long long)N * (4 * L1 - 3 * (long long)l)) / (2 * L1));
    }
    a.budget_ws[(size_t)row * a.L + l] = bl;
    if (a.budget_out) a.budget_out[(size_t)row * a.L + l] = bl;
  }
}

}  // namespace

cudaError_t launch_confidence(const ConfLaunch& a, const Policy& pol, cudaStream_t st, long long* launches,
                              Prof* prof, bool chained) {
  dim3 grid(a.cpr, a.B);
  ProfScope ps(prof, kKConfidence, st);
  if (chained)
    (void)launch_chained(confidence_kernel, grid, NT, 0, st, a, pol);
  else
    confidence_kernel<<<grid, NT, 0, st>>>(a, pol);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace confkv
