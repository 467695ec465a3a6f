// Prompt ingest (positions 0..len-1 of every segment of the call).
//
// Confidence mode keeps every prompt token (eviction only runs inside the
// decode loop of the CONF-KV post's pseudo-code). Fixed-budget mode (KVpop
// summary, section 2.1) keeps the s sinks, the last w and the top k of the
// rest by (priority, position) as it ingests, with the same segmented select
// as eviction. With INT8 on, tokens that are already older than the window at
// the next step (positions <= len - W) are quantised on the way in; the rest
// go to the FP16 window ring at slot pos mod W.
#include "common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace confkv {

namespace {

constexpr int NT = 256;

// Confidence mode: segment metadata (window slots emptied first).
__global__ void __launch_bounds__(NT) prefill_meta_kernel(Cache c, PrefillLaunch a) {
  const int item = blockIdx.x;
  int l, b, h;
  const int s = seg_of(c, a.r, item, &l, &b, &h);
  const int len = a.lens[b];
  for (int slot = threadIdx.x; slot < c.Wst; slot += NT) {
    c.pos_r[(size_t)s * c.Wst + slot] = -1;
    c.sc_r[(size_t)s * c.Wst + slot] = 0.0f;
  }
  if (threadIdx.x == 0) {
    c.n_cold[s] = c.W > 0 ? max(0, len - c.W + 1) : len;
    c.next_pos[s] = len;
    if (a.cand) a.cand[s].stamp = -1;
  }
}

// Fixed mode: select the kept positions of each segment from its priorities
// and write them in increasing order; also the segment metadata.
__global__ void __launch_bounds__(NT) prefill_select_kernel(Cache c, Policy pol, PrefillLaunch a) {
  __shared__ SelectSmem<NT> sm;
  const int item = blockIdx.x;
  int l, b, h;
  const int s = seg_of(c, a.r, item, &l, &b, &h);
  const int len = a.lens[b];
  const float* prio = a.prio + ((size_t)((l - a.r.l0) * a.r.B + b) * c.Hkv + h) * a.t_stride;
  const int t = len - 1;
  for (int slot = threadIdx.x; slot < c.Wst; slot += NT) {
    c.pos_r[(size_t)s * c.Wst + slot] = -1;
    c.sc_r[(size_t)s * c.Wst + slot] = 0.0f;
  }
  auto key = [&](int p) -> unsigned long long {
    if (t - p < pol.P || p < pol.n_sink) return kNoKey;
    return ((unsigned long long)ordered_bits(prio[p]) << 32) | (uint32_t)p;
  };
  const int e = len - pol.fixed_budget;
  SelectResult sel{0ull, 0ull};
  bool any = false;
  if (e > 0) {
    any = true;
    sel = (e == 1) ? block_argmin<NT>(key, len, sm) : block_select_smallest<NT>(key, len, e, sm);
  }
  int32_t* list = a.keep_list + (size_t)item * pol.fixed_budget;
  int kept = 0, cold = 0;
  for (int base = 0; base < len; base += NT) {
    const int p = base + threadIdx.x;
    const bool keep = p < len && !(any && is_selected(key(p), sel));
    int total;
    const int r = kept + block_scan_flag<NT>(keep, sm, &total);
    if (keep && r < pol.fixed_budget) list[r] = p;
    const bool is_cold = keep && (c.W == 0 || p <= len - c.W);
    cold += block_sum_int<NT>(is_cold ? 1 : 0, sm);
    kept += total;
  }
  if (threadIdx.x == 0) {
    a.keep_count[item] = min(kept, pol.fixed_budget);
    c.n_cold[s] = cold;
    c.next_pos[s] = len;
    if (a.cand) a.cand[s].stamp = -1;
  }
}

// One warp per (segment, token): copy or quantise the K and V rows.
template <int D>
__global__ void __launch_bounds__(NT) prefill_ingest_kernel(Cache c, Policy pol, PrefillLaunch a, int fixed_mode,
                                                            int per_item) {
  const long long gw = ((long long)blockIdx.x * NT + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int item = (int)(gw / per_item);
  const int i = (int)(gw - (long long)item * per_item);
  if (item >= a.r.items(c.Hkv)) return;
  int l, b, h;
  const int s = seg_of(c, a.r, item, &l, &b, &h);
  const int len = a.lens[b];
  int p;
  if (fixed_mode) {
    if (i >= a.keep_count[item]) return;
    p = a.keep_list[(size_t)item * per_item + i];
  } else {
    if (i >= len) return;
    p = i;
  }
  const size_t in_row = (((size_t)((l - a.r.l0) * a.r.B + b) * c.Hkv + h) * a.t_stride + p);
  const __half* ksrc = a.k + in_row * D;
  const __half* vsrc = a.v + in_row * D;
  const float sc = fixed_mode ? a.prio[in_row] : initial_score(pol, l, b, h, p);
  uint32_t w[D / 64];
  if (c.W > 0 && p > len - c.W) {
    // ring: slot pos mod W; linear window: the kept list's window part in
    // order (it follows the n_cold cold tokens)
    const int slot = c.linear ? i - c.n_cold[s] : p % c.W;
    if (c.linear && (slot < 0 || slot >= c.W)) {
      if (lane == 0) set_error(c.err, kErrDevice);
      return;
    }
    const size_t rs = (size_t)s * c.Wst + slot;
    row_load_plain<D>(ksrc, lane, w);
    row_store_h<D>(c.kr + (size_t)s * c.Wst * D, slot, lane, w);
    row_load_plain<D>(vsrc, lane, w);
    row_store_h<D>(c.vr + (size_t)s * c.Wst * D, slot, lane, w);
    if (lane == 0) {
      c.pos_r[rs] = p;
      c.sc_r[rs] = sc;
    }
    return;
  }
  const int idx = i;   // cold rows are a prefix of the kept list (in position order)
  if (idx >= c.cap) {
    if (lane == 0) set_error(c.err, kErrDevice);
    return;
  }
  const size_t cs = (size_t)s * c.cap + idx;
  const size_t cb = (size_t)s * c.cap * D;
  if (c.cold_int8) {
    uint32_t pk;
    row_load_plain<D>(ksrc, lane, w);
    float scale = row_quantize<D>(w, &pk);
    row_store_k8<D>(c.k8 + cb, idx, lane, pk);
    if (lane == 0) c.ks[cs] = scale;
    row_load_plain<D>(vsrc, lane, w);
    scale = row_quantize<D>(w, &pk);
    row_store_v8<D>(c.v8 + cb, idx, lane, pk);
    if (lane == 0) c.vs[cs] = scale;
  } else {
    row_load_plain<D>(ksrc, lane, w);
    row_store_h<D>(c.kc + cb, idx, lane, w);
    row_load_plain<D>(vsrc, lane, w);
    row_store_h<D>(c.vc + cb, idx, lane, w);
  }
  if (lane == 0) {
    c.pos_c[cs] = p;
    c.sc_c[cs] = sc;
  }
}

}  // namespace

cudaError_t launch_prefill(const Cache& c, const Policy& pol, const PrefillLaunch& a, cudaStream_t st,
                           long long* launches, Prof* prof) {
  ProfScope ps(prof, kKPrefill, st);
  const int items = a.r.items(c.Hkv);
  if (items == 0) return cudaSuccess;
  const bool fixed = pol.mode == 1;
  if (fixed) prefill_select_kernel<<<items, NT, 0, st>>>(c, pol, a);
  else prefill_meta_kernel<<<items, NT, 0, st>>>(c, a);
  ++*launches;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int per_item = fixed ? pol.fixed_budget : a.t_stride;
  const long long warps = (long long)items * per_item;
  if (warps == 0) return cudaSuccess;
  const long long blocks = (warps * 32 + NT - 1) / NT;
  if (c.D == 128) prefill_ingest_kernel<128><<<(unsigned)blocks, NT, 0, st>>>(c, pol, a, fixed ? 1 : 0, per_item);
  else prefill_ingest_kernel<64><<<(unsigned)blocks, NT, 0, st>>>(c, pol, a, fixed ? 1 : 0, per_item);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace confkv
