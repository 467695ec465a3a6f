// Block-wide building blocks for the segmented top-k select (one CTA per
// segment): flag scans, ordered collection, argmin, MSD radix select and a
// histogram threshold select on 64-bit keys (score bits, position) that are
// unique within a segment.
#pragma once

#include "common.cuh"

namespace confkv {

template <int NT>
struct SelectSmem {
  unsigned hist[256];
  unsigned long long prefix, mask;
  int rem, done;
  int warp_tot[NT / 32];
  unsigned long long wmin[NT / 32];
  int widx[NT / 32];
  int next;
  int misc[4];
};

// Exclusive prefix of a 0/1 flag over the block; *total receives the count.
template <int NT>
__device__ __forceinline__ int block_scan_flag(bool f, SelectSmem<NT>& sm, int* total) {
  const unsigned bal = __ballot_sync(0xffffffffu, f);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (lane == 0) sm.warp_tot[w] = __popc(bal);
  __syncthreads();
  int off = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) {
    const int v = sm.warp_tot[i];
    off += (i < w) ? v : 0;
    tot += v;
  }
  __syncthreads();
  *total = tot;
  return off + __popc(bal & ((1u << lane) - 1u));
}

template <int NT>
__device__ __forceinline__ int block_sum_int(int v, SelectSmem<NT>& sm) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) sm.warp_tot[threadIdx.x >> 5] = v;
  __syncthreads();
  int tot = 0;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) tot += sm.warp_tot[i];
  __syncthreads();
  return tot;
}

// Collect, in increasing order, up to CAP indices i in [*cur, end) with
// pred(i), into list[] (shared memory). Advances *cur past the last collected
// index (or to end). Every thread returns the same count and cursor, and the
// list is complete and visible to all threads on return.
template <int NT, int CAP, class Pred>
__device__ int block_collect(Pred pred, int* cur, int end, int* list, SelectSmem<NT>& sm) {
  int count = 0;
  int c0 = *cur;
  while (count < CAP && c0 < end) {
    const int i = c0 + threadIdx.x;
    const bool f = i < end && pred(i);
    int total;
    const int r = count + block_scan_flag<NT>(f, sm, &total);
    if (f && r < CAP) list[r] = i;
    if (count + total > CAP) {
      if (f && r == CAP - 1) sm.next = i + 1;
      __syncthreads();
      c0 = sm.next;
      count = CAP;
      __syncthreads();
      break;
    }
    count += total;
    c0 += NT;
  }
  *cur = min(c0, end);
  __syncthreads();   // list[] entries written by other threads are visible to every caller thread
  return count;
}

struct SelectResult {
  unsigned long long prefix, mask;   // selected: key != kNoKey && (key & mask) <= prefix
};

// Smallest key among kf(0..n-1) (absent keys are kNoKey).
template <int NT, class KeyFn>
__device__ SelectResult block_argmin(KeyFn kf, int n, SelectSmem<NT>& sm) {
  unsigned long long best = kNoKey;
  for (int i = threadIdx.x; i < n; i += NT) {
    const unsigned long long k = kf(i);
    best = k < best ? k : best;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
    best = other < best ? other : best;
  }
  if ((threadIdx.x & 31) == 0) sm.wmin[threadIdx.x >> 5] = best;
  __syncthreads();
  unsigned long long m = kNoKey;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) m = sm.wmin[i] < m ? sm.wmin[i] : m;
  __syncthreads();
  return SelectResult{m, ~0ull};
}

// Smallest key among kf(0..n-1) and the index that holds it (-1 if none).
template <int NT, class KeyFn>
__device__ unsigned long long block_argmin_idx(KeyFn kf, int n, SelectSmem<NT>& sm, int* idx_out) {
  unsigned long long best = kNoKey;
  int bi = -1;
  for (int i = threadIdx.x; i < n; i += NT) {
    const unsigned long long k = kf(i);
    if (k < best) {
      best = k;
      bi = i;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (other < best) {
      best = other;
      bi = oi;
    }
  }
  if ((threadIdx.x & 31) == 0) {
    sm.wmin[threadIdx.x >> 5] = best;
    sm.widx[threadIdx.x >> 5] = bi;
  }
  __syncthreads();
  unsigned long long m = kNoKey;
  int mi = -1;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i)
    if (sm.wmin[i] < m) {
      m = sm.wmin[i];
      mi = sm.widx[i];
    }
  __syncthreads();
  *idx_out = mi;
  return m;
}

// The k smallest keys (1 <= k <= number of present keys), by MSD radix select
// with 8-bit digits. Stops early once the bucket holding the k-th key is
// entirely selected.
template <int NT, class KeyFn>
__device__ SelectResult block_select_smallest(KeyFn kf, int n, int k, SelectSmem<NT>& sm) {
  if (threadIdx.x == 0) {
    sm.prefix = 0;
    sm.mask = 0;
    sm.rem = k;
    sm.done = 0;
  }
  __syncthreads();
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += NT) sm.hist[i] = 0;
    __syncthreads();
    const unsigned long long prefix = sm.prefix, mask = sm.mask;
    for (int i = threadIdx.x; i < n; i += NT) {
      const unsigned long long key = kf(i);
      if (key != kNoKey && (key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      unsigned cnt[8];
      unsigned tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = sm.hist[lane * 8 + j];
        tot += cnt[j];
      }
      unsigned incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const unsigned excl = incl - tot;
      const unsigned rem = (unsigned)sm.rem;
      __syncwarp();
      if (excl < rem && rem <= incl) {
        unsigned below = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (below + cnt[j] >= rem) {
            const unsigned nrem = rem - below;
            sm.prefix = prefix | ((unsigned long long)(lane * 8 + j) << shift);
            sm.mask = mask | (0xffull << shift);
            sm.rem = (int)nrem;
            sm.done = (cnt[j] == nrem) ? 1 : 0;
            break;
          }
          below += cnt[j];
        }
      }
    }
    __syncthreads();
    if (sm.done) break;
  }
  SelectResult r{sm.prefix, sm.mask};
  __syncthreads();
  return r;
}

// Exclusive prefix of an int over the block; *total receives the sum.
template <int NT>
__device__ __forceinline__ int block_excl_scan_int(int v, SelectSmem<NT>& sm, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) sm.warp_tot[w] = incl;
  __syncthreads();
  int off = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) {
    const int x = sm.warp_tot[i];
    off += (i < w) ? x : 0;
    tot += x;
  }
  __syncthreads();
  *total = tot;
  return off + incl - v;
}

// The k smallest of the 64-bit keys (hi[i] << 32) | lo(i), i < n, where
// hi[i] == 0xFFFFFFFF marks an absent key (1 <= k <= number of present
// keys): MSD radix select with 8-bit digits, stopping once the bucket holding
// the k-th key is entirely selected. The high halves come from memory the
// caller filled once; lo(i) is evaluated only in the passes over the low half
// (when the high halves alone do not separate the k-th key). Histograms take
// one shared-memory atomic per distinct digit of a warp (__match_any_sync).
template <int NT, class LoFn>
__device__ SelectResult block_select_smallest_hi(const uint32_t* __restrict__ hi, LoFn lo, int n, int k,
                                                 SelectSmem<NT>& sm) {
  if (threadIdx.x == 0) {
    sm.prefix = 0;
    sm.mask = 0;
    sm.rem = k;
    sm.done = 0;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int wbase = threadIdx.x & ~31;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += NT) sm.hist[i] = 0;
    __syncthreads();
    const unsigned long long prefix = sm.prefix, mask = sm.mask;
    const bool need_lo = shift < 32;
    // eight keys per thread per step, all loaded before any is counted
    for (int base = wbase * 8; base < n; base += NT * 8) {   // whole warps step together
      uint32_t hv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = base + u * 32 + lane;
        hv[u] = i < n ? hi[i] : 0xFFFFFFFFu;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = base + u * 32 + lane;
        unsigned bin = 256u;
        if (hv[u] != 0xFFFFFFFFu) {
          unsigned long long key = (unsigned long long)hv[u] << 32;
          if (need_lo) key |= (uint32_t)lo(i);
          if ((key & mask) == prefix) bin = (unsigned)((key >> shift) & 255u);
        }
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin != 256u && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[bin], (unsigned)__popc(peers));
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      unsigned cnt[8];
      unsigned tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = sm.hist[lane * 8 + j];
        tot += cnt[j];
      }
      unsigned incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const unsigned excl = incl - tot;
      const unsigned rem = (unsigned)sm.rem;
      __syncwarp();
      if (excl < rem && rem <= incl) {
        unsigned below = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (below + cnt[j] >= rem) {
            const unsigned nrem = rem - below;
            sm.prefix = prefix | ((unsigned long long)(lane * 8 + j) << shift);
            sm.mask = mask | (0xffull << shift);
            sm.rem = (int)nrem;
            sm.done = (cnt[j] == nrem) ? 1 : 0;
            break;
          }
          below += cnt[j];
        }
      }
    }
    __syncthreads();
    if (sm.done) break;
  }
  SelectResult r{sm.prefix, sm.mask};
  __syncthreads();
  return r;
}

__device__ __forceinline__ bool is_selected(unsigned long long key, const SelectResult& r) {
  return key != kNoKey && (key & r.mask) <= r.prefix;
}

// Sort m (a power of two, at most 8*NT) keys of shared memory ascending with
// a bitonic network; all NT threads call it; ends with a barrier. Each thread
// loads two pairs of a stage before comparing either.
template <int NT, typename K>
__device__ __forceinline__ void block_bitonic_sort(K* buf, int m) {
  for (int size = 2; size <= m; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i0 = (int)threadIdx.x; i0 < (m >> 1); i0 += 2 * NT) {
        const int i1 = i0 + NT;
        const int a0 = 2 * i0 - (i0 & (stride - 1)), a1 = 2 * i1 - (i1 & (stride - 1));
        const bool two = i1 < (m >> 1);
        const K x0 = buf[a0], y0 = buf[a0 + stride];
        K x1 = x0, y1 = y0;
        if (two) {
          x1 = buf[a1];
          y1 = buf[a1 + stride];
        }
        if ((x0 > y0) == ((a0 & size) == 0)) {
          buf[a0] = y0;
          buf[a0 + stride] = x0;
        }
        if (two && (x1 > y1) == ((a1 & size) == 0)) {
          buf[a1] = y1;
          buf[a1 + stride] = x1;
        }
      }
      __syncthreads();
    }
  }
}

constexpr int kSelBuf = 2048;   // 64-bit entries of the shared buffer block_select_threshold uses
constexpr int kSelBins = 2048;  // histogram bins (the first half of the buffer, as 32-bit counts)
constexpr int kSelCand = (kSelBuf * 8 - kSelBins * 4) / 8;   // keys of one bin the rest of the buffer holds

// The k-th smallest of the keys of block_select_threshold, given the
// histogram of the counted high halves (first kSelBins 32-bit words of buf,
// complete and visible) over a bin map `bin_of` that is monotone in the high
// half: the bin holding the k-th key is located, its keys collected and
// sorted; when that bin is too full for the buffer, the radix select decides.
template <int NT, typename LoFn, typename BinFn>
__device__ unsigned long long select_in_hist(const uint32_t* __restrict__ hi, LoFn lo, int n, int k,
                                             SelectSmem<NT>& sm, unsigned long long* buf, BinFn bin_of) {
  const uint4* hi4 = reinterpret_cast<const uint4*>(hi);
  const int n4 = (n + 3) >> 2;
  auto key_at = [&](const uint4& q, int j) { return j == 0 ? q.x : j == 1 ? q.y : j == 2 ? q.z : q.w; };
  uint32_t* hist = reinterpret_cast<uint32_t*>(buf);
  // the bin holding the k-th key: each thread sums its kSelBins/NT bins, a
  // block scan places them
  constexpr int BPT = kSelBins / NT;
  uint32_t cnt[BPT];
  uint32_t tot = 0u;
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    cnt[j] = hist[threadIdx.x * BPT + j];
    tot += cnt[j];
  }
  int all;
  const int excl = block_excl_scan_int<NT>((int)tot, sm, &all);
  if (threadIdx.x == 0) sm.misc[2] = -1;
  __syncthreads();
  if (excl < k && k <= excl + (int)tot) {
    int below = excl;
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      if (below + (int)cnt[j] >= k) {
        sm.misc[2] = threadIdx.x * BPT + j;   // the bin
        sm.misc[3] = below;                   // counted keys in lower bins
        sm.misc[0] = (int)cnt[j];
        break;
      }
      below += (int)cnt[j];
    }
  }
  __syncthreads();
  const int bstar = sm.misc[2], nbelow = sm.misc[3], ncand = sm.misc[0];
  if (bstar >= 0 && ncand <= kSelCand) {
    // pass 3: the keys of that bin into the second half of the buffer
    unsigned long long* cand = buf + kSelBins / 2;
    __syncthreads();   // every thread has read the bin
    if (threadIdx.x == 0) sm.misc[1] = 0;
    __syncthreads();
    for (int v0 = threadIdx.x; v0 < n4; v0 += 4 * NT) {
      uint4 q[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) q[r] = v0 + r * NT < n4 ? hi4[v0 + r * NT] : make_uint4(~0u, ~0u, ~0u, ~0u);
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = 4 * (v0 + r * NT) + j;
          const uint32_t hv = key_at(q[r], j);
          if (i < n && hv != 0xFFFFFFFFu && bin_of(hv) == bstar) {
            const int slot = atomicAdd(&sm.misc[1], 1);
            cand[slot] = ((unsigned long long)hv << 32) | (uint32_t)i;   // index for now
          }
        }
    }
    __syncthreads();
    // the low halves, all loads of a thread in flight together
    for (int j0 = (int)threadIdx.x; j0 < ncand; j0 += 4 * NT) {
      int idx[4];
      uint32_t lov[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = j0 + r * NT;
        idx[r] = j < ncand ? (int)(uint32_t)cand[j] : -1;
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) lov[r] = idx[r] >= 0 ? (uint32_t)lo(idx[r]) : 0u;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = j0 + r * NT;
        if (j < ncand) cand[j] = (cand[j] & 0xFFFFFFFF00000000ull) | lov[r];
      }
    }
    int m = 1;
    while (m < ncand) m <<= 1;
    for (int i = ncand + threadIdx.x; i < m; i += NT) cand[i] = kNoKey;
    __syncthreads();
    block_bitonic_sort<NT>(cand, m);
    const unsigned long long r = cand[k - nbelow - 1];
    __syncthreads();
    return r;
  }
  __syncthreads();
  const SelectResult r = block_select_smallest_hi<NT>(hi, lo, n, k, sm);
  return r.prefix | ~r.mask;
}

// The k-th smallest (1-based) of the n 64-bit keys (hi[i] << 32) | lo(i),
// where hi[i] == 0xFFFFFFFF marks an entry that is never counted (k must not
// exceed the counted entries): every counted key <= the result is one of the
// k smallest. hi must be 16-byte aligned and readable up to n rounded up to
// 4. Up to kSelBuf keys are sorted outright. Otherwise three passes over the
// high halves: their range; a histogram of kSelBins bins, monotone in the
// key, which locates the bin holding the k-th key; the keys of that bin,
// which are sorted. When that bin is too full for the buffer, the radix
// select above decides (its result, as a threshold, is prefix | ~mask).
// buf: kSelBuf 64-bit entries of shared memory.
// A caller that has just written the high halves may pass its threads' own
// minimum and maximum of the counted ones (range_given): the range pass is
// then skipped.
template <int NT, typename LoFn>
__device__ unsigned long long block_select_threshold(const uint32_t* __restrict__ hi, LoFn lo, int n, int k,
                                                     SelectSmem<NT>& sm, unsigned long long* buf,
                                                     bool range_given = false, uint32_t my_mn = 0xFFFFFFFFu,
                                                     uint32_t my_mx = 0u) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (n <= kSelBuf) {
    int m = 1;
    while (m < n) m <<= 1;
    for (int i = threadIdx.x; i < m; i += NT) {
      unsigned long long key = kNoKey;
      if (i < n) {
        const uint32_t hv = hi[i];
        if (hv != 0xFFFFFFFFu) key = ((unsigned long long)hv << 32) | (uint32_t)lo(i);
      }
      buf[i] = key;
    }
    __syncthreads();
    block_bitonic_sort<NT>(buf, m);
    const unsigned long long r = buf[k - 1];
    __syncthreads();
    return r;
  }
  const uint4* hi4 = reinterpret_cast<const uint4*>(hi);
  const int n4 = (n + 3) >> 2;
  auto key_at = [&](const uint4& q, int j) { return j == 0 ? q.x : j == 1 ? q.y : j == 2 ? q.z : q.w; };
  // pass 1: the range of the counted high halves
  uint32_t mn = my_mn, mx = my_mx;
  for (int v0 = threadIdx.x; !range_given && v0 < n4; v0 += 4 * NT) {
    uint4 q[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) q[r] = v0 + r * NT < n4 ? hi4[v0 + r * NT] : make_uint4(~0u, ~0u, ~0u, ~0u);
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = 4 * (v0 + r * NT) + j;
        const uint32_t hv = key_at(q[r], j);
        if (i < n && hv != 0xFFFFFFFFu) {
          mn = min(mn, hv);
          mx = max(mx, hv);
        }
      }
  }
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  uint32_t* hist = reinterpret_cast<uint32_t*>(buf);
  if (lane == 0) {
    sm.hist[wid] = mn;
    sm.hist[32 + wid] = mx;
  }
  for (int b = threadIdx.x; b < kSelBins; b += NT) hist[b] = 0u;
  __syncthreads();
  mn = sm.hist[0];
  mx = sm.hist[32];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) {
    mn = min(mn, sm.hist[w]);
    mx = max(mx, sm.hist[32 + w]);
  }
  // bin(h) = floor((h - mn) * M / 2^32): monotone in h and below kSelBins
  const unsigned long long range = (unsigned long long)(mx - mn) + 1ull;
  const uint32_t M = range <= kSelBins ? 0u : (uint32_t)(((unsigned long long)kSelBins << 32) / range);
  auto bin_of = [&](uint32_t hv) -> int {
    const uint32_t d = hv - mn;
    return range <= kSelBins ? (int)d : (int)__umulhi(d, M);
  };
  // pass 2: histogram
  for (int v0 = threadIdx.x; v0 < n4; v0 += 4 * NT) {
    uint4 q[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) q[r] = v0 + r * NT < n4 ? hi4[v0 + r * NT] : make_uint4(~0u, ~0u, ~0u, ~0u);
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = 4 * (v0 + r * NT) + j;
        const uint32_t hv = key_at(q[r], j);
        if (i < n && hv != 0xFFFFFFFFu) atomicAdd(&hist[bin_of(hv)], 1u);
      }
  }
  __syncthreads();
  return select_in_hist<NT>(hi, lo, n, k, sm, buf, bin_of);
}

}  // namespace confkv
