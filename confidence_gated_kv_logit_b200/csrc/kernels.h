// Host-side launch interface of the CONF-KV kernels (internal to libconfkv).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"
#include "prof.h"
#include "warp_select.cuh"

namespace confkv {

struct ConfPartial {
  float m, S, T, top1, top2;
  int bad;
};

// K1: confidence reduction over logits [B][V] -> c[B], budget[B][L].
struct ConfLaunch {
  const float* logits;
  int B, V, L;
  ConfPartial* part;      // [B][cpr]
  unsigned* tickets;      // [B], zero between launches
  int cpr;                // CTAs per row
  float* c_ws;            // [B]
  int32_t* budget_ws;     // [B][L]
  float* c_out;           // optional
  int32_t* budget_out;    // optional
  int32_t* err;
};
// chained: launched as the next kernel of the step's chain (set false when
// the previous operation on the stream is not one of the library's kernels)
cudaError_t launch_confidence(const ConfLaunch& a, const Policy& pol, cudaStream_t st, long long* launches,
                              Prof* prof, bool chained = true);

// K2: prefill ingest.
struct PrefillLaunch {
  Range r;
  const int32_t* lens;    // device [B]
  int t_stride;
  const __half* k;        // [nl][B][Hkv][t_stride][D]
  const __half* v;
  const float* prio;      // [nl][B][Hkv][t_stride] (fixed mode) or null
  int32_t* keep_list;     // fixed mode: [items][fixed_budget] positions kept (ascending)
  int32_t* keep_count;    // fixed mode: [items]
  EvictCand* cand;        // [S] eviction candidates, invalidated for the segments ingested
};
cudaError_t launch_prefill(const Cache& c, const Policy& pol, const PrefillLaunch& a, cudaStream_t st,
                           long long* launches, Prof* prof);

// K3 + K3c + EMA: decode attention.
struct AttnLaunch {
  Range r;
  const __half* q;        // [nl][B][Hq][D]
  const __half* k_new;    // [nl][B][Hkv][D]
  const __half* v_new;
  const float* prio_new;  // [nl][B][Hkv] (fixed mode) or null
  float* out;             // [nl][B][Hq][D]
  float* lse_out;         // [nl][B][Hq] or null
  float* lse_ws;          // [S][G]
  float* scores;          // [S][G][score_stride]
  int score_stride;
  float* part;            // [units][G][D+2]
  int part_units;         // capacity of part in (item, split) units
  int max_cold_tokens;    // host upper bound of n_cold over the call's segments
  int num_sms;
  unsigned char* qfrag;   // [S][qf_stride] query operands prepared by the append kernel
  int qf_stride;
  EvictCand* cand;        // [S] eviction candidates written by the EMA pass (confidence mode)
  int* sched;             // [2] unit counter and finished-CTA counter of the attention kernel (zero between launches)
  int run_ema;            // confidence mode: 1 runs the EMA pass after attention, 0 leaves it to the caller
};
cudaError_t launch_decode_attn(const Cache& c, const Policy& pol, const AttnLaunch& a, cudaStream_t st,
                               long long* launches, Prof* prof);
// Bytes of the prepared query operands of one segment (qfrag stride).
int qfrag_bytes(int D, int G);
// The EMA pass of a decode call (after attention and, with splits, the
// combine), on stream st.
cudaError_t run_ema(const Cache& c, const Policy& pol, const AttnLaunch& a, cudaStream_t st);

// K4 + K5 + K6: select, compaction, conversion of the token leaving the window.
struct EvictLaunch {
  Range r;
  const int32_t* budget;  // [Bmax][L]
  uint32_t* vmask;        // [S][mask_words] victim bitmask scratch
  int mask_words;
  int stable;             // 1: order-preserving compaction
  EvictCand* cand;        // [S] candidates from this step's EMA pass (used when their stamp matches)
  uint32_t* kscratch;     // per CTA of the evict grid: key high halves [cap + Wst], then hole and mover lists [cap] each
  int scratch_stride;     // uint32 words per CTA
  int scratch_keys;       // offset of the hole list (= cap + Wst)
  int* bulk_sched;        // [2] segment counter and finished-CTA counter of the bulk variant (zero between launches)
  // 1: the previous kernel on the stream is the confidence reduction, so the
  // fused variant may run its EMA pass before waiting for it (see evict_kernel)
  int ema_early = 0;
  int scratch_ctas = 0;   // CTAs kscratch covers (no launch uses more)
};
// Where an EMA pass reads the step's attention results.
struct EmaIn {
  const float* lse_ws;   // [S][G] natural-log LSE of the step
  const float* scores;   // [S][G][score_stride] scaled scores, log2 units
  int score_stride;
};
// With `ema` set, the eviction kernel first runs the step's EMA pass over
// each segment (the fused variant; confidence mode only). `bulk` selects the
// variant for evictions of thousands of tokens per segment (the first step
// after a long prompt): one segment at a time per CTA, claimed from a
// counter, the EMA pass spread over the whole CTA and writing the keys the
// select needs.
cudaError_t launch_evict_compact(const Cache& c, const Policy& pol, const EvictLaunch& a, const EmaIn* ema,
                                 bool bulk, int num_sms, cudaStream_t st, long long* launches, Prof* prof);
// CTAs the evict kernel uses for `items` segments (the scratch is per CTA).
int evict_grid(int items);
// Calls over at most this many segments evict with one CTA per segment (the
// whole-CTA path) when the EMA pass has already run: too few segments to fill
// the GPU one warp each. The key scratch covers that many CTAs. (With the EMA
// pass fused in, the per-warp kernel stays faster: measured on the GPT-2
// shape.)
int few_segment_limit(int num_sms);

}  // namespace confkv
