/*
 * confkv.h — C ABI of the B200 CONF-KV decode-step library (libconfkv.so).
 *
 * CONF-KV ("Conf-KV: confidence-aware KV-cache eviction with mixed ..."
 * rcap.io post, and the chatpaper.ai abstract "CONF-KV: Confidence-Aware KV
 * Cache Eviction with Mixed-Precision Storage for Long-Horizon LLMs") is a
 * KV-cache manager: every decode step it turns the next-token distribution
 * into a confidence score, picks a token budget from it, keeps the tokens with
 * the highest blend of attention-mass EMA and recency inside that budget
 * (never the most recent P), stores older tokens in INT8 and the recent window
 * in FP16, and keeps the cache contiguous. The same select also runs the
 * fixed-budget B = s + w + k mode of the KVpop summary (gist.science,
 * sections 2.1 and 2.4): sinks + protected window + top-k static priorities.
 *
 * One decode step, in the order of the CONF-KV post's decode-loop pseudo-code:
 *   confkv_decode_attn   (append the new token, attention, attention-mass EMA)
 *   confkv_confidence    (confidence of the step's logits -> budget per layer)
 *   confkv_evict_compact (select victims, compact, convert the token leaving
 *                         the FP16 window to INT8)
 *
 * Conventions shared by every entry point:
 *  - Pointers named *_host are host memory; every other array pointer is
 *    device memory of the current CUDA device, owned by the caller, never
 *    freed or retained by the library after the call's work completes.
 *  - fp16 arrays are IEEE binary16 passed as `const void*`; fp32 as float.
 *    K/V/q/out arrays must start on a 16-byte boundary (ERR_ARG otherwise).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). Every call is asynchronous on that stream unless documented as
 *    synchronising. One handle must not be used from two streams at once: the
 *    cache and the scratch belong to the handle. The library's kernels are
 *    launched with programmatic stream serialisation: each starts by waiting
 *    for the work before it on the stream to complete, so the next one's
 *    launch overlaps its end; work of the caller in between is ordered as
 *    usual.
 *  - Errors the host can detect (bad arguments, capacity, wrong state) are
 *    returned before anything is launched, and the call has no effect.
 *    Conditions only the device can see (non-finite logits, a failed device
 *    check) set a sticky device error word read by confkv_last_error.
 *  - No call traps, asserts on the device, or throws across the ABI.
 */
#ifndef CONFKV_H
#define CONFKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CONFKV_API __attribute__((visibility("default")))
#else
#define CONFKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct confkv_handle confkv_handle;

typedef enum {
  CONFKV_OK = 0,
  CONFKV_ERR_ARG = 1,        /* invalid argument (null pointer, out of range, inconsistent) */
  CONFKV_ERR_CAPACITY = 2,   /* the call could exceed the cache capacity sized at create */
  CONFKV_ERR_STATE = 3,      /* wrong call order (e.g. decode before prefill) or destroyed handle */
  CONFKV_ERR_NONFINITE = 4,  /* device word: a logit row held NaN/Inf (that row used the larger budget) */
  CONFKV_ERR_CUDA = 5,       /* a CUDA runtime call failed */
  CONFKV_ERR_OOM = 6,        /* device allocation failed at create */
  CONFKV_ERR_DEVICE = 7      /* device word: a kernel's own bounds check fired (work skipped) */
} confkv_status;

enum { CONFKV_MODE_CONF = 0, CONFKV_MODE_FIXED = 1 };
/* Budget gate polarity. PROSE (default): confident (c >= tau) -> n_low, else
 * n_high, as the CONF-KV abstract and post describe. LITERAL: the
 * pseudo-code line's polarity, n_high when c >= tau. */
enum { CONFKV_GATE_PROSE = 0, CONFKV_GATE_LITERAL = 1 };
/* Compaction variant and window layout; all give the same logical cache
 * content (the tokens, their precision, payload, scales and EMA):
 *   HOLEFILL  survivors above the new end of the INT8 region move into the
 *             holes below it (bytes in proportion to the victims); the FP16
 *             window is a ring, slot = position mod W;
 *   STABLE    order-preserving compaction of the INT8 region (every survivor
 *             after the first hole moves down); the window is a ring;
 *   LINEAR    no ring: the INT8 region is compacted in order and the FP16
 *             window occupies slots [0, n) in position order, so the whole
 *             cache is position-ordered; every conversion or window eviction
 *             moves the window's later slots down. Confidence mode with INT8
 *             on only. */
enum { CONFKV_COMPACT_HOLEFILL = 0, CONFKV_COMPACT_STABLE = 1, CONFKV_COMPACT_LINEAR = 2 };
/* Score source of the confidence mode's ranking (score = alpha*source +
 * (1-alpha)*recency):
 *   EMA    ema <- beta*ema + (1-beta)*a (the CONF-KV post's EMA; the default);
 *   ACCUM  acc <- acc + a, the attention mass accumulated over the steps (the
 *          heavy-hitter score the CONF-KV post's related work, H2O, uses);
 *   RANDOM a static per-token draw u in [0, 1), from SplitMix64 (Steele, Lea
 *          and Flood, 2014) at counter pos | h << 32 | b << 40 | l << 52
 *          (position, KV head, sequence, layer): state seed + (counter + 1) *
 *          0x9E3779B97F4A7C15, mixed, u = (mix >> 40) * 2^-24.
 * a is the token's attention probability this step, averaged over the G query
 * heads. These are the ranker variants of the matched-rate ablation. */
enum { CONFKV_SCORE_EMA = 0, CONFKV_SCORE_ACCUM = 1, CONFKV_SCORE_RANDOM = 2 };

#define CONFKV_ALL_LAYERS (-1)

typedef struct {
  int32_t mode;          /* CONFKV_MODE_CONF or CONFKV_MODE_FIXED */
  int32_t n_low;         /* tight budget (tokens per KV head), >= 1 */
  int32_t n_high;        /* loose budget, >= 1 */
  float tau;             /* confidence threshold, compared with >= */
  float alpha;           /* score = alpha*EMA + (1-alpha)*recency, in [0, 1] */
  float ema_decay;       /* beta in ema <- beta*ema + (1-beta)*a, in [0, 1] */
  int32_t protect_last;  /* P: tokens with age t-pos < P are never evicted (fixed mode: w) */
  int32_t fp16_window;   /* W: tokens with age < W are FP16 while attention runs; >= 1 when int8_enable */
  int32_t n_sink;        /* s: positions < s are never evicted */
  int32_t fixed_budget;  /* B = s + w + k (fixed mode only), >= s + w */
  int32_t pyramidal;     /* nonzero: layer l gets floor(N(4(L-1)-3l)/(2(L-1))) */
  int32_t gate;          /* CONFKV_GATE_PROSE or CONFKV_GATE_LITERAL */
  int32_t int8_enable;   /* nonzero: tokens older than the window are stored INT8 */
  int32_t compact;       /* CONFKV_COMPACT_HOLEFILL or CONFKV_COMPACT_STABLE */
  int32_t max_batch;     /* sequences the cache is sized for */
  int32_t max_prefill;   /* longest prompt confkv_prefill accepts (tokens) */
  int32_t score_source;  /* CONFKV_SCORE_EMA, CONFKV_SCORE_ACCUM or CONFKV_SCORE_RANDOM (confidence mode) */
  uint32_t seed;         /* CONFKV_SCORE_RANDOM: seed of the per-token draws */
  int32_t single_stream; /* nonzero: every kernel of a call runs inside that call, on the caller's
                            stream (the EMA pass runs in confkv_decode_attn instead of being deferred
                            to the next eviction, and no event joins calls), so that a caller can
                            capture a whole decode step in a CUDA graph. Launch configurations are
                            then fixed at capture time, and the handle's host-side length bounds are
                            not advanced by replays */
} confkv_params;

typedef struct {
  int64_t tokens_int8;        /* tokens stored INT8, all segments */
  int64_t tokens_fp16;        /* tokens stored FP16, all segments */
  int64_t bytes_payload;      /* K/V payload bytes + INT8 scales resident (all segments) */
  int64_t bytes_meta;         /* position + EMA/priority bytes resident */
  int64_t bytes_capacity;     /* device bytes the handle allocated */
  int32_t min_len, max_len;   /* over the active segments */
  int64_t attn_tokens_int8;   /* cumulative INT8 token-rows read by attention (per KV head) */
  int64_t attn_tokens_fp16;   /* cumulative FP16 token-rows read by attention (per KV head) */
  int64_t evict_tokens;       /* cumulative tokens scanned by eviction */
  int64_t moved_rows;         /* cumulative rows moved by compaction */
  int64_t requant_rows;       /* cumulative tokens converted FP16 -> INT8 */
  int64_t kernel_launches;    /* cumulative kernels launched by this handle */
  int64_t evict_block_segments; /* cumulative segments evicted by the whole-CTA path (many victims) */
  int64_t moved_window_rows;  /* cumulative FP16 window rows moved (the linear layout's window shifts) */
} confkv_stats;

/* Fill *p with the defaults: CONF mode, N_low 256, N_high 512, tau 0.6,
 * alpha 0.5, beta 0.9, P 64, W 128, s 0, prose gate, INT8 on, hole-fill
 * compaction, max_batch 1, max_prefill 4096. Returns CONFKV_ERR_ARG if p is
 * NULL. */
CONFKV_API confkv_status confkv_default_params(confkv_params* p);

/* Allocate a cache for `layers` layers of `kv_heads` KV heads of head_dim
 * (64 or 128) each, for up to params->max_batch sequences, with q_heads query
 * heads (a multiple of kv_heads, at most 8 per KV head). All device memory is
 * allocated here, on the current device; nothing allocates later. *out
 * receives the handle. Errors: ARG (invalid shape or parameter), OOM, CUDA. */
CONFKV_API confkv_status confkv_create(int32_t layers, int32_t kv_heads, int32_t q_heads, int32_t head_dim,
                            const confkv_params* params, confkv_handle** out);

/* Free everything the handle owns (synchronises the device first). A NULL
 * handle is a no-op returning OK. The handle must not be used afterwards. */
CONFKV_API confkv_status confkv_destroy(confkv_handle* h);

/* Ingest prompts and reset the cache of `layer` (or every layer with
 * CONFKV_ALL_LAYERS) for `batch` sequences (1..max_batch).
 *   lens_host[batch]  prompt length per sequence, 0..max_prefill (host)
 *   k, v   fp16 [batch][kv_heads][t_stride][head_dim] for one layer, or with a
 *          leading [layers] dimension for CONFKV_ALL_LAYERS; rows >= len unused
 *   priority  fp32 [batch][kv_heads][t_stride] (leading [layers] likewise);
 *          required in fixed mode, must be NULL otherwise
 * Confidence mode evicts nothing here. Fixed mode keeps the s sinks, the last
 * w and the top k by (priority, position) as it ingests (KVpop summary 2.1).
 * With INT8 on, positions <= len - W are quantised (per token, per KV head,
 * K and V separately, round-half-even). Positions restart at 0. The batch
 * size given here is the active batch of later calls. */
CONFKV_API confkv_status confkv_prefill(confkv_handle* h, int32_t layer, int32_t batch, const int32_t* lens_host,
                             int32_t t_stride, const void* k, const void* v, const float* priority,
                             void* stream);

/* Confidence of each sequence's next-token distribution and its budget
 * (CONF-KV post, pseudo-code and method paragraphs):
 *   c = 0.4(1 - H(p)/ln V) + 0.3 sigmoid(l_(1) - l_(2)) + 0.3 max p,
 *   p = softmax(logits), H in nats, l_(1) >= l_(2) the two largest logits
 *   counted with multiplicity.
 * logits fp32 [batch][vocab] (batch = the active batch, vocab >= 2). The
 * budget N per sequence follows the gate polarity, then the pyramid; the
 * handle keeps budget[batch][layers] for confkv_evict_compact. c_out fp32
 * [batch] and budget_out int32 [batch][layers] are optional (NULL skips). A
 * row with a NaN/Inf logit gets c = NaN and the larger budget, and sets the
 * device word CONFKV_ERR_NONFINITE. Not used in fixed mode (returns STATE). */
CONFKV_API confkv_status confkv_confidence(confkv_handle* h, const float* logits, int32_t batch, int32_t vocab,
                                float* c_out, int32_t* budget_out, void* stream);

/* One decode step's attention for `layer` (or CONFKV_ALL_LAYERS):
 * append the new token at the next position of every segment (FP16), then
 * softmax attention of the G = q_heads/kv_heads query heads of each KV head
 * over its whole cache (scale 1/sqrt(head_dim), INT8 rows dequantised
 * in-kernel), then, in confidence mode, the attention-mass EMA update of every
 * cached token: ema <- beta*ema + (1-beta)*mean over the G heads of its
 * normalised attention probability (new tokens start at 0).
 *   q      fp16 [batch][q_heads][head_dim]   (leading [layers] for ALL)
 *   k_new, v_new  fp16 [batch][kv_heads][head_dim]  (likewise)
 *   prio_new  fp32 [batch][kv_heads] (likewise); fixed mode only, else NULL
 *   out    fp32 [batch][q_heads][head_dim]   (likewise)
 *   lse_out  fp32 [batch][q_heads] (likewise) natural-log log-sum-exp of the
 *          scaled scores; optional
 * Query head h reads KV head h / G. Errors: STATE before prefill, CAPACITY if
 * the cache could overflow (calls without eviction grow it).
 * Unless single_stream is set, the EMA update is deferred: the next
 * confkv_evict_compact over the same layers runs it inside the eviction kernel
 * (one launch for both). Whatever reads the cache first -- another decode call
 * over those layers, confkv_query, confkv_export_segment -- sees it applied;
 * a prefill of those layers discards it. */
CONFKV_API confkv_status confkv_decode_attn(confkv_handle* h, int32_t layer, const void* q, const void* k_new,
                                 const void* v_new, const float* prio_new, float* out, float* lse_out,
                                 void* stream);

/* Evict and compact `layer` (or CONFKV_ALL_LAYERS): for every segment over its
 * effective budget max(budget_l, P + s) (fixed mode: B), evict the
 * lowest-ranked unprotected tokens by the key (score, position), score =
 * fp32(fp32(alpha*ema) + fp32((1-alpha)*recency)), recency =
 * (pos+1)/(t+1) (fixed mode: the priority), equal scores keeping the newer
 * token; tokens with age < P and positions < s are never evicted. Survivors
 * are compacted so the INT8 region stays a hole-free prefix, and the token
 * the next append would push out of the FP16 window is quantised to INT8
 * (CONF-KV post, pseudo-code). Called on the stream of the handle's last
 * confkv_confidence, right after it, the deferred EMA pass runs beside that
 * confidence reduction and only the eviction waits for its budgets. */
CONFKV_API confkv_status confkv_evict_compact(confkv_handle* h, int32_t layer, void* stream);

/* Synchronising: counts of the active segments and cumulative counters. */
CONFKV_API confkv_status confkv_query(confkv_handle* h, confkv_stats* out);

/* Synchronising: copy the raw state of one segment (layer, seq, kv_head) to
 * host memory. With host_buf NULL, *bytes receives the size needed. Layout
 * (all little-endian, packed in this order):
 *   int32 header[8] = { n_cold, ring_slots, next_pos, cold_int8, head_dim,
 *                       mode, 0, 0 }
 *   cold region, n_cold rows in physical order:
 *     int32 pos[n_cold]; float score_src[n_cold]; float ks[n_cold]; float vs[n_cold];
 *     K rows [n_cold][head_dim] (int8 if cold_int8 else fp16); V rows likewise
 *   ring, ring_slots rows (slot order; pos < 0 marks an empty slot):
 *     int32 pos[W]; float score_src[W]; fp16 K[W][head_dim]; fp16 V[W][head_dim]
 * score_src is the EMA (confidence mode) or the priority (fixed mode). */
CONFKV_API confkv_status confkv_export_segment(confkv_handle* h, int32_t layer, int32_t seq, int32_t kv_head,
                                    void* host_buf, size_t* bytes);

/* Synchronising: the sticky device error word (CONFKV_OK if none); with
 * clear nonzero it is reset. */
CONFKV_API confkv_status confkv_last_error(confkv_handle* h, int32_t clear);

/* Synchronising: like confkv_last_error (not clearing), and when a device-side
 * check failed, detail[3] receives (check site, segment id, offending value)
 * of the first failure. Sites: 1xx append, 2xx attention, 3xx EMA, 4xx
 * eviction, 5xx prefill, 6xx combine; the work guarded by a failed check is
 * skipped, never performed out of bounds. */
CONFKV_API confkv_status confkv_last_error_detail(confkv_handle* h, int32_t* detail);

/* Per-kernel timing. While enabled, every kernel launch of the handle is
 * bracketed by CUDA events on its stream (a few microseconds of host work per
 * launch, nothing on the device). confkv_profile_read synchronises on the
 * recorded events and returns, per kernel kind, the launches and the summed
 * milliseconds since the last reset. */
enum {
  CONFKV_K_CONFIDENCE = 0, CONFKV_K_APPEND = 1, CONFKV_K_ATTENTION = 2, CONFKV_K_COMBINE = 3,
  CONFKV_K_EMA = 4, CONFKV_K_EVICT = 5, CONFKV_K_PREFILL = 6,
  CONFKV_K_EMA_EVICT = 7,   /* the eviction kernel with the step's EMA pass fused in */
  CONFKV_K_KINDS = 8
};
typedef struct {
  int64_t launches[CONFKV_K_KINDS];
  double ms[CONFKV_K_KINDS];
} confkv_profile;
CONFKV_API confkv_status confkv_profile_enable(confkv_handle* h, int32_t enable);
CONFKV_API confkv_status confkv_profile_read(confkv_handle* h, confkv_profile* out, int32_t reset);

/* Confidence and per-layer budgets without a handle and without allocating.
 * The pages describe no counterpart: this entry point exists for callers that
 * cannot allocate device memory, such as code running under an allocator
 * that owns the whole device or a runtime that hands the library a fixed
 * memory budget. It computes what confkv_confidence computes, for the gate,
 * threshold, budgets and pyramid in *params (its other fields are ignored),
 * for `layers` layers:
 *   logits fp32 [batch][vocab], c_out fp32 [batch], budget_out int32
 *   [batch][layers], all device memory owned by the caller (required).
 * Its scratch is a fixed array inside the library (about 197 KB per device,
 * held by every GPU that loads the library until the process exits), so:
 *  - batch may be at most 256 and vocab at most 262144; larger sizes return
 *    CONFKV_ERR_CAPACITY before anything runs;
 *  - the first call on a device looks up the array's device address (a
 *    host-side step, no allocation) and keeps it for the life of the process;
 *    make that first call before any stream capture. A device reset
 *    (cudaDeviceReset, or a reset of the primary context) reloads the library
 *    on that device and leaves the kept address stale: do not call this entry
 *    point on a device after resetting it;
 *  - every call shares the one array: calls that overlap on the GPU (on two
 *    streams, or from two threads) race and give wrong results. Serialise them.
 * It calls no cudaMalloc, cudaFree or allocating routine. A row with a NaN or
 * Inf logit gets c = NaN and the larger budget; no error word is kept. */
CONFKV_API confkv_status confkv_confidence_noalloc(const confkv_params* params, int32_t layers, const float* logits,
                                                   int32_t batch, int32_t vocab, float* c_out, int32_t* budget_out,
                                                   void* stream);

/* Static description of a status code. */
CONFKV_API const char* confkv_status_string(confkv_status s);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
CONFKV_API int32_t confkv_version(void);

#ifdef __cplusplus
}
#endif
#endif /* CONFKV_H */
