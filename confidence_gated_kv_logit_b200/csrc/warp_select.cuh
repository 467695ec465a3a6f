// Warp-level selection of the smallest eviction keys of one segment, shared
// by the eviction kernel and the EMA pass (which computes the same keys right
// after updating the EMA values and hands the smallest ones to eviction).
#pragma once

#include <stddef.h>

#include "common.cuh"

namespace confkv {

constexpr int kCandMax = 16;    // smallest keys kept per segment (and victims one warp handles)
constexpr int kWarpMaxVictims = kCandMax;
constexpr int kLaneKeep = 4;              // smallest keys each lane keeps during the scan


// Minimum over the warp of a 64-bit key: the smallest high half, then the
// smallest low half among the lanes that hold it (two warp reductions).
__device__ __forceinline__ unsigned long long warp_min_u64(unsigned long long v) {
  const unsigned hi = (unsigned)(v >> 32);
  const unsigned mh = __reduce_min_sync(0xffffffffu, hi);
  const unsigned ml = __reduce_min_sync(0xffffffffu, hi == mh ? (unsigned)v : 0xffffffffu);
  return ((unsigned long long)mh << 32) | ml;
}

// Keeps the kLaneKeep smallest (key, index) pairs seen by this lane, ascending.
//
// pos_bound lets the scan skip a token without computing its key. In
// confidence mode score = RN(RN(alpha*ema) + RN((1-alpha)*rec)) with
// ema >= 0 and rec = RN((pos+1)/(t+1)); with every rounding at most 2^-24
// relative, score >= (1-alpha)*(pos+1)/(t+1) * (1 - 2^-23). Once the list is
// full with largest kept score thr, a token with
//   pos + 1 > thr * (t+1) / (1-alpha) * (1 + 2^-19)
// therefore has score > thr and cannot enter (1 + 2^-19 exceeds
// 1 / (1 - 2^-23) plus the three fp32 roundings of computing the bound).
struct LaneBest {
  unsigned long long k[kLaneKeep];
  int i[kLaneKeep];
  int pos_bound;   // tokens with pos + 1 > pos_bound cannot enter
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int j = 0; j < kLaneKeep; ++j) {
      k[j] = kNoKey;
      i[j] = -1;
    }
    pos_bound = 0x7fffffff;
  }
  __device__ __forceinline__ void offer(unsigned long long key, int idx) {
    if (key < k[kLaneKeep - 1]) {
      k[kLaneKeep - 1] = key;
      i[kLaneKeep - 1] = idx;
#pragma unroll
      for (int j = kLaneKeep - 1; j > 0; --j) {
        if (k[j] < k[j - 1]) {
          const unsigned long long tk = k[j];
          k[j] = k[j - 1];
          k[j - 1] = tk;
          const int ti = i[j];
          i[j] = i[j - 1];
          i[j - 1] = ti;
        }
      }
    }
  }
  // Recompute pos_bound after an insertion (confidence mode with 1-alpha >= 2^-60).
  __device__ __forceinline__ void update_bound(float t1_over_oma) {
    if (k[kLaneKeep - 1] == kNoKey) return;
    const uint32_t o = (uint32_t)(k[kLaneKeep - 1] >> 32);
    const float thr = __uint_as_float(o & 0x7fffffffu);   // scores are >= 0: ordered bits = bits | 2^31
    const float b = ceilf(thr * t1_over_oma * (1.0f + 0x1p-19f));
    pos_bound = b >= 2147483647.0f ? 0x7fffffff : (int)b;
  }
  __device__ __forceinline__ void pop() {
#pragma unroll
    for (int j = 0; j < kLaneKeep - 1; ++j) {
      k[j] = k[j + 1];
      i[j] = i[j + 1];
    }
    k[kLaneKeep - 1] = kNoKey;
    i[kLaneKeep - 1] = -1;
  }
};


// Eviction candidates of one segment, written by the EMA pass: the smallest
// keys (ascending) with their indices (cold index, or n_cold + ring slot, as
// of that pass), the number of occupied window slots, how many of the keys
// are certainly the segment's smallest (`safe`), and the next position the
// segment had then (`stamp`); -1 marks a record that must not be used.
struct EvictCand {
  unsigned long long key[kCandMax];
  int idx[kCandMax];
  int n_ring, safe, stamp, n_cold;   // read as one 16-byte word
};
static_assert(sizeof(EvictCand) == 208, "candidate record layout");
static_assert(offsetof(EvictCand, n_ring) % 16 == 0, "the record header is one aligned 16-byte word");

// Merge every lane's list into the segment's smallest keys: lane j < count
// receives the j-th smallest key and its index. Also returns (in every lane)
// how many of them are certainly the segment's smallest: a lane whose list
// was full dropped only keys above its largest kept key k3, so the merged
// keys up to the smallest such k3 are exact.
// If `complete_below` is given it receives a key B such that every key <= B
// that this warp saw is in the merged list (the smallest full-list k3, or the
// last merged key when the list was cut at `want`).
__device__ __forceinline__ void warp_merge_smallest(LaneBest& best, int lane, int want, unsigned long long* my_key,
                                                    int* my_idx, int* count, int* safe,
                                                    unsigned long long* complete_below = nullptr) {
  const unsigned long long k3 = best.k[kLaneKeep - 1];
  const unsigned long long lim = warp_min_u64(k3);   // kNoKey when no list is full
  unsigned long long mk = kNoKey;
  int mi = -1, n = 0;
  for (int j = 0; j < want; ++j) {
    const unsigned long long m = warp_min_u64(best.k[0]);
    if (m == kNoKey) break;
    const unsigned own = __ballot_sync(0xffffffffu, best.k[0] == m);
    const int src = __ffs(own) - 1;
    const int vi = __shfl_sync(0xffffffffu, best.i[0], src);
    if (lane == src) best.pop();
    if (lane == j) {
      mk = m;
      mi = vi;
    }
    ++n;
  }
  *my_key = mk;
  *my_idx = mi;
  *count = n;
  *safe = __popc(__ballot_sync(0xffffffffu, lane < n && mk <= lim));
  if (complete_below != nullptr) {
    const unsigned long long last = n == want && n > 0 ? __shfl_sync(0xffffffffu, mk, n - 1) : kNoKey;
    *complete_below = last < lim ? last : lim;
  }
}

}  // namespace confkv
