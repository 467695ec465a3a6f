// C ABI of libconfkv: handle, argument validation, device allocation, host-side
// capacity bookkeeping and stream-ordered launches. See include/confkv.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_set>
#include <vector>

#include "../../include/confkv.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr uint32_t kMagic = 0xC0F1C0DEu;
constexpr uint32_t kDead = 0xDEADC0DEu;
constexpr int kMaxCpr = 128;   // CTAs per logit row (one per ~4096 logits)

struct Buffers {
  std::vector<void*> ptrs;
  size_t bytes = 0;
  template <class T>
  cudaError_t alloc(T** p, size_t count) {
    *p = nullptr;
    if (count == 0) return cudaSuccess;
    void* q = nullptr;
    cudaError_t e = cudaMalloc(&q, count * sizeof(T));
    if (e != cudaSuccess) return e;
    ptrs.push_back(q);
    bytes += count * sizeof(T);
    *p = static_cast<T*>(q);
    return cudaSuccess;
  }
  void release() {
    for (void* p : ptrs) cudaFree(p);
    ptrs.clear();
  }
};

int round_up(long long x, int m) { return (int)(((x + m - 1) / m) * m); }

int layer_budget(int N, int l, int L, bool pyramidal) {
  if (!pyramidal || L == 1) return N;
  const long long L1 = L - 1;
  return (int)(((long long)N * (4 * L1 - 3 * (long long)l)) / (2 * L1));
}

}  // namespace

struct confkv_handle {
  uint32_t magic;
  int device;
  int num_sms;
  int L, Hkv, Hq, G, D;
  confkv_params p;
  confkv::Cache c;
  confkv::Policy pol;
  int score_stride;
  int batch;                     // active batch (0 = nothing ingested yet)
  std::vector<int> prefilled;    // per layer
  std::vector<long long> ub_len; // per layer, upper bound of any segment length
  std::vector<int> max_eff;      // per layer, largest effective budget
  Buffers buf;
  int32_t* lens_dev;
  int32_t* budget;               // [Bmax][L]
  float* c_ws;
  confkv::ConfPartial* cpart;    // [Bmax][kMaxCpr]
  unsigned* tickets;             // [Bmax]
  float* lse_ws;
  float* scores;
  float* part;
  int part_units;
  uint32_t* vmask;
  int mask_words;
  unsigned char* qfrag;          // [S][qf_stride] query operands of the attention kernel
  int qf_stride;
  confkv::EvictCand* cand;       // [S] eviction candidates from the EMA pass
  uint32_t* kscratch;            // evict scratch, per CTA of the largest evict grid (scratch_ctas)
  int* sched;                    // attention unit counters (zero between launches)
  int* bulk_sched;               // bulk eviction segment counters (zero between launches)
  // The EMA pass of a decode call is deferred (unless single_stream): the
  // next eviction of the same layers runs it fused into the eviction kernel
  // (one launch, no candidate records). Anything else that needs the EMA
  // values first -- another decode call over those layers, export, query --
  // runs the pass on its own; prefill drops it (the segment starts over).
  std::vector<char> ema_pending;   // per layer
  cudaEvent_t attn_done;           // recorded after each deferred decode call's attention
  cudaStream_t attn_stream;        // the stream it was recorded on
  // The handle's last launch was its confidence reduction, on conf_stream: an
  // eviction call right after it on the same stream lets the fused kernel run
  // its EMA pass beside that reduction (EvictLaunch::ema_early).
  bool conf_last = false;
  cudaStream_t conf_stream = nullptr;
  int scratch_stride;
  int scratch_ctas;               // CTAs kscratch covers
  int32_t* keep_list;
  int32_t* keep_count;
  long long launches;
  confkv::Prof prof;
  confkv::Prof* prof_ptr() { return prof.on ? &prof : nullptr; }
};

// Handles currently alive; lets a destroyed or foreign pointer be rejected
// without reading freed memory.
static std::mutex g_live_mu;
static std::unordered_set<const confkv_handle*> g_live;

static bool alive(const confkv_handle* h) {
  if (!h) return false;
  std::lock_guard<std::mutex> lk(g_live_mu);
  return g_live.count(h) != 0 && h->magic == kMagic;
}

static confkv_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return CONFKV_OK;
  if (e == cudaErrorMemoryAllocation) return CONFKV_ERR_OOM;
  return CONFKV_ERR_CUDA;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool layer_range(const confkv_handle* h, int32_t layer, confkv::Range* r) {
  if (layer == CONFKV_ALL_LAYERS) {
    r->l0 = 0;
    r->nl = h->L;
  } else if (layer >= 0 && layer < h->L) {
    r->l0 = layer;
    r->nl = 1;
  } else {
    return false;
  }
  r->B = h->batch;
  return true;
}

extern "C" {

int32_t confkv_version(void) { return 101; }

const char* confkv_status_string(confkv_status s) {
  switch (s) {
    case CONFKV_OK: return "ok";
    case CONFKV_ERR_ARG: return "invalid argument";
    case CONFKV_ERR_CAPACITY: return "cache capacity would be exceeded";
    case CONFKV_ERR_STATE: return "call not valid in the current state";
    case CONFKV_ERR_NONFINITE: return "non-finite logits were seen (the larger budget was used)";
    case CONFKV_ERR_CUDA: return "CUDA runtime error";
    case CONFKV_ERR_OOM: return "device allocation failed";
    case CONFKV_ERR_DEVICE: return "a device-side check failed (work skipped)";
  }
  return "unknown status";
}

confkv_status confkv_default_params(confkv_params* p) {
  if (!p) return CONFKV_ERR_ARG;
  std::memset(p, 0, sizeof(*p));
  p->mode = CONFKV_MODE_CONF;
  p->n_low = 256;
  p->n_high = 512;
  p->tau = 0.6f;
  p->alpha = 0.5f;
  p->ema_decay = 0.9f;
  p->protect_last = 64;
  p->fp16_window = 128;
  p->n_sink = 0;
  p->fixed_budget = 0;
  p->pyramidal = 0;
  p->gate = CONFKV_GATE_PROSE;
  p->int8_enable = 1;
  p->compact = CONFKV_COMPACT_HOLEFILL;
  p->max_batch = 1;
  p->max_prefill = 4096;
  p->score_source = CONFKV_SCORE_EMA;
  p->seed = 0u;
  return CONFKV_OK;
}

confkv_status confkv_create(int32_t layers, int32_t kv_heads, int32_t q_heads, int32_t head_dim,
                            const confkv_params* params, confkv_handle** out) {
  if (!out || !params) return CONFKV_ERR_ARG;
  *out = nullptr;
  const confkv_params& p = *params;
  if (layers < 1 || kv_heads < 1 || q_heads < 1 || q_heads % kv_heads) return CONFKV_ERR_ARG;
  if (head_dim != 64 && head_dim != 128) return CONFKV_ERR_ARG;
  const int G = q_heads / kv_heads;
  if (G < 1 || G > 8) return CONFKV_ERR_ARG;
  if (p.mode != CONFKV_MODE_CONF && p.mode != CONFKV_MODE_FIXED) return CONFKV_ERR_ARG;
  if (p.gate != CONFKV_GATE_PROSE && p.gate != CONFKV_GATE_LITERAL) return CONFKV_ERR_ARG;
  if (p.compact != CONFKV_COMPACT_HOLEFILL && p.compact != CONFKV_COMPACT_STABLE &&
      p.compact != CONFKV_COMPACT_LINEAR)
    return CONFKV_ERR_ARG;
  if (p.compact == CONFKV_COMPACT_LINEAR && (p.mode != CONFKV_MODE_CONF || !p.int8_enable)) return CONFKV_ERR_ARG;
  if (p.score_source != CONFKV_SCORE_EMA && p.score_source != CONFKV_SCORE_ACCUM &&
      p.score_source != CONFKV_SCORE_RANDOM)
    return CONFKV_ERR_ARG;
  if (p.max_batch < 1 || p.max_prefill < 0 || p.protect_last < 0 || p.n_sink < 0) return CONFKV_ERR_ARG;
  if (!(p.alpha >= 0.0f && p.alpha <= 1.0f) || !(p.ema_decay >= 0.0f && p.ema_decay <= 1.0f)) return CONFKV_ERR_ARG;
  if (!std::isfinite(p.tau)) return CONFKV_ERR_ARG;
  if (p.int8_enable && p.fp16_window < 1) return CONFKV_ERR_ARG;
  if (p.mode == CONFKV_MODE_CONF && (p.n_low < 1 || p.n_high < 1)) return CONFKV_ERR_ARG;
  if (p.mode == CONFKV_MODE_FIXED &&
      (p.fixed_budget < 1 || (long long)p.fixed_budget < (long long)p.n_sink + p.protect_last))
    return CONFKV_ERR_ARG;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return CONFKV_ERR_CUDA;
  confkv_handle* h = new (std::nothrow) confkv_handle();
  if (!h) return CONFKV_ERR_OOM;
  h->magic = kMagic;
  h->device = dev;
  cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev);
  h->L = layers;
  h->Hkv = kv_heads;
  h->Hq = q_heads;
  h->G = G;
  h->D = head_dim;
  h->p = p;
  h->batch = 0;
  h->prefilled.assign(layers, 0);
  h->ub_len.assign(layers, 0);
  h->max_eff.assign(layers, 0);
  h->launches = 0;

  // effective-budget ceiling per layer and the cold-region capacity
  long long need = p.max_prefill;
  for (int l = 0; l < layers; ++l) {
    int eff;
    if (p.mode == CONFKV_MODE_FIXED) {
      eff = p.fixed_budget;
    } else {
      const int big = std::max(p.n_low, p.n_high);
      eff = std::max(layer_budget(big, l, layers, p.pyramidal != 0), p.protect_last + p.n_sink);
    }
    h->max_eff[l] = eff;
    need = std::max<long long>(need, eff);
  }
  if (p.mode == CONFKV_MODE_FIXED) need = p.fixed_budget;
  const long long cap_ll = round_up(need + 2, 64);
  if (cap_ll > (1ll << 28)) {
    delete h;
    return CONFKV_ERR_ARG;
  }
  const int W = p.int8_enable ? p.fp16_window : 0;
  confkv::Cache& c = h->c;
  std::memset(&c, 0, sizeof(c));
  c.L = layers;
  c.Bmax = p.max_batch;
  c.Hkv = kv_heads;
  c.Hq = q_heads;
  c.G = G;
  c.D = head_dim;
  c.W = W;
  c.Wst = round_up(W, 64);   // whole 64-slot tiles for the attention copies
  c.cap = (int)cap_ll;
  c.cold_int8 = p.int8_enable ? 1 : 0;
  c.linear = p.compact == CONFKV_COMPACT_LINEAR ? 1 : 0;

  confkv::Policy& pol = h->pol;
  pol.mode = p.mode;
  pol.n_low = p.n_low;
  pol.n_high = p.n_high;
  pol.tau = p.tau;
  pol.alpha = p.alpha;
  pol.one_minus_alpha = 1.0f - p.alpha;
  // The EMA pass computes fl(beta*x + w*m) with m the step's mean attention:
  // EMA w = 1 - beta; accumulated attention beta = w = 1 (x + m); a static
  // draw beta = 1, w = 0 (x unchanged).
  pol.score_source = p.mode == CONFKV_MODE_CONF ? p.score_source : CONFKV_SCORE_EMA;
  pol.seed = p.seed;
  pol.beta = pol.score_source == CONFKV_SCORE_EMA ? p.ema_decay : 1.0f;
  pol.one_minus_beta = pol.score_source == CONFKV_SCORE_EMA    ? 1.0f - p.ema_decay
                       : pol.score_source == CONFKV_SCORE_ACCUM ? 1.0f
                                                                : 0.0f;
  pol.P = p.protect_last;
  pol.n_sink = p.n_sink;
  pol.fixed_budget = p.fixed_budget;
  pol.gate = p.gate;
  pol.pyramidal = p.pyramidal ? 1 : 0;

  const size_t S = (size_t)layers * p.max_batch * kv_heads;
  const size_t rows = S * (size_t)c.cap;
  const size_t rrows = S * (size_t)c.Wst;
  Buffers& B = h->buf;
  e = cudaSuccess;
  auto chk = [&](cudaError_t x) { if (e == cudaSuccess) e = x; };
  if (c.cold_int8) {
    chk(B.alloc(&c.k8, rows * head_dim));
    chk(B.alloc(&c.v8, rows * head_dim));
    chk(B.alloc(&c.ks, rows));
    chk(B.alloc(&c.vs, rows));
  } else {
    chk(B.alloc(&c.kc, rows * head_dim));
    chk(B.alloc(&c.vc, rows * head_dim));
  }
  chk(B.alloc(&c.pos_c, rows));
  chk(B.alloc(&c.sc_c, rows));
  chk(B.alloc(&c.kr, rrows * head_dim));
  chk(B.alloc(&c.vr, rrows * head_dim));
  chk(B.alloc(&c.pos_r, rrows));
  chk(B.alloc(&c.sc_r, rrows));
  chk(B.alloc(&c.n_cold, S));
  chk(B.alloc(&c.next_pos, S));
  chk(B.alloc(&c.err, 4));
  chk(B.alloc(&c.counters, (size_t)confkv::kNumCounters));
  chk(B.alloc(&h->lens_dev, (size_t)p.max_batch));
  chk(B.alloc(&h->budget, (size_t)p.max_batch * layers));
  chk(B.alloc(&h->c_ws, (size_t)p.max_batch));
  chk(B.alloc(&h->cpart, (size_t)p.max_batch * kMaxCpr));
  chk(B.alloc(&h->tickets, (size_t)p.max_batch));
  chk(B.alloc(&h->lse_ws, S * G));
  h->score_stride = c.cap + c.Wst;
  chk(B.alloc(&h->scores, S * G * (size_t)h->score_stride));
  h->part_units = (int)std::max<size_t>(std::min<size_t>(S * 8, 65536), 4096);
  chk(B.alloc(&h->part, (size_t)h->part_units * G * (head_dim + 2)));
  h->mask_words = (c.cap + 31) / 32;
  chk(B.alloc(&h->vmask, S * (size_t)h->mask_words));
  h->qf_stride = confkv::qfrag_bytes(head_dim, G);
  chk(B.alloc(&h->qfrag, S * (size_t)h->qf_stride));
  chk(B.alloc(&h->cand, S));
  chk(B.alloc(&h->sched, 2));
  chk(B.alloc(&h->bulk_sched, 2));
  h->scratch_stride = 3 * c.cap + c.Wst;
  h->scratch_ctas = std::max(confkv::evict_grid((int)S), std::min((int)S, confkv::few_segment_limit(h->num_sms)));
  chk(B.alloc(&h->kscratch, (size_t)h->scratch_ctas * h->scratch_stride));
  if (p.mode == CONFKV_MODE_FIXED) {
    chk(B.alloc(&h->keep_list, S * (size_t)p.fixed_budget));
    chk(B.alloc(&h->keep_count, S));
  }
  if (e == cudaSuccess) {
    // zero everything once so that no kernel ever reads uninitialised bytes
    if (c.k8) chk(cudaMemset(c.k8, 0, rows * head_dim));
    if (c.v8) chk(cudaMemset(c.v8, 0, rows * head_dim));
    if (c.ks) chk(cudaMemset(c.ks, 0, rows * 4));
    if (c.vs) chk(cudaMemset(c.vs, 0, rows * 4));
    if (c.kc) chk(cudaMemset(c.kc, 0, rows * head_dim * 2));
    if (c.vc) chk(cudaMemset(c.vc, 0, rows * head_dim * 2));
    chk(cudaMemset(c.pos_c, 0xff, rows * 4));
    chk(cudaMemset(c.sc_c, 0, rows * 4));
    if (rrows) {
      chk(cudaMemset(c.kr, 0, rrows * head_dim * 2));
      chk(cudaMemset(c.vr, 0, rrows * head_dim * 2));
      chk(cudaMemset(c.pos_r, 0xff, rrows * 4));
      chk(cudaMemset(c.sc_r, 0, rrows * 4));
    }
    chk(cudaMemset(c.n_cold, 0, S * 4));
    chk(cudaMemset(c.next_pos, 0, S * 4));
    chk(cudaMemset(c.err, 0, 16));
    chk(cudaMemset(c.counters, 0, confkv::kNumCounters * 8));
    chk(cudaMemset(h->tickets, 0, (size_t)p.max_batch * 4));
    chk(cudaMemset(h->scores, 0, S * G * (size_t)h->score_stride * 4));
    chk(cudaMemset(h->qfrag, 0, S * (size_t)h->qf_stride));
    chk(cudaMemset(h->cand, 0xff, S * sizeof(confkv::EvictCand)));   // stamp -1: no record
    chk(cudaMemset(h->sched, 0, 2 * sizeof(int)));
    chk(cudaMemset(h->bulk_sched, 0, 2 * sizeof(int)));
    chk(cudaDeviceSynchronize());
  }
  if (e != cudaSuccess) {
    B.release();
    h->magic = kDead;
    delete h;
    return cuda_status(e);
  }
  h->attn_done = nullptr;
  h->attn_stream = nullptr;
  h->ema_pending.assign(layers, 0);
  if (!p.single_stream && cudaEventCreateWithFlags(&h->attn_done, cudaEventDisableTiming) != cudaSuccess) {
    B.release();
    h->magic = kDead;
    delete h;
    return CONFKV_ERR_CUDA;
  }
  {
    std::lock_guard<std::mutex> lk(g_live_mu);
    g_live.insert(h);
  }
  *out = h;
  return CONFKV_OK;
}

static confkv::AttnLaunch ema_launch(const confkv_handle* h, int l0, int nl) {
  confkv::AttnLaunch a;
  std::memset(&a, 0, sizeof(a));
  a.r.l0 = l0;
  a.r.nl = nl;
  a.r.B = h->batch;
  a.lse_ws = h->lse_ws;
  a.scores = h->scores;
  a.score_stride = h->score_stride;
  a.num_sms = h->num_sms;
  a.cand = h->cand;
  return a;
}

// Order st after the attention whose EMA pass was deferred (a no-op on the
// stream that ran it).
static cudaError_t join_attention(confkv_handle* h, cudaStream_t st) {
  if (h->attn_done == nullptr || st == h->attn_stream) return cudaSuccess;
  return cudaStreamWaitEvent(st, h->attn_done, 0);
}

// Run the deferred EMA passes of the layers in [l0, l0 + nl) on st, one
// launch per run of consecutive pending layers. st first waits for the
// attention that produced them (it may have run on another stream).
static cudaError_t flush_ema(confkv_handle* h, int l0, int nl, cudaStream_t st) {
  bool any = false;
  for (int l = l0; l < l0 + nl; ++l) any = any || h->ema_pending[l];
  if (!any) return cudaSuccess;
  cudaError_t e = join_attention(h, st);
  for (int l = l0; l < l0 + nl && e == cudaSuccess;) {
    if (!h->ema_pending[l]) {
      ++l;
      continue;
    }
    int l1 = l;
    while (l1 < l0 + nl && h->ema_pending[l1]) ++l1;
    const confkv::AttnLaunch a = ema_launch(h, l, l1 - l);
    {
      confkv::ProfScope ps(h->prof_ptr(), confkv::kKEma, st);
      e = confkv::run_ema(h->c, h->pol, a, st);
    }
    ++h->launches;
    for (int k = l; k < l1; ++k) h->ema_pending[k] = 0;
    l = l1;
  }
  return e;
}

// Every deferred pass, for the synchronising queries: after the device is
// idle, on the legacy stream, then idle again.
static cudaError_t flush_all_ema(confkv_handle* h) {
  h->conf_last = false;
  bool any = false;
  for (char f : h->ema_pending) any = any || f;
  if (!any) return cudaSuccess;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = flush_ema(h, 0, h->L, nullptr);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  return e;
}

confkv_status confkv_destroy(confkv_handle* h) {
  if (!h) return CONFKV_OK;
  {
    std::lock_guard<std::mutex> lk(g_live_mu);
    if (g_live.erase(h) == 0) return CONFKV_ERR_STATE;
  }
  cudaDeviceSynchronize();
  if (h->attn_done) cudaEventDestroy(h->attn_done);
  h->buf.release();
  h->magic = kDead;
  delete h;
  return CONFKV_OK;
}

confkv_status confkv_prefill(confkv_handle* h, int32_t layer, int32_t batch, const int32_t* lens_host,
                             int32_t t_stride, const void* k, const void* v, const float* priority,
                             void* stream) {
  if (!alive(h)) return CONFKV_ERR_STATE;
  if (batch < 1 || batch > h->p.max_batch || !lens_host || t_stride < 1 || !k || !v) return CONFKV_ERR_ARG;
  if (!aligned16(k) || !aligned16(v) || (priority && !aligned16(priority))) return CONFKV_ERR_ARG;
  const bool fixed = h->p.mode == CONFKV_MODE_FIXED;
  if (fixed != (priority != nullptr)) return CONFKV_ERR_ARG;
  h->conf_last = false;
  int maxlen = 0;
  for (int b = 0; b < batch; ++b) {
    if (lens_host[b] < 0 || lens_host[b] > h->p.max_prefill || lens_host[b] > t_stride) return CONFKV_ERR_ARG;
    maxlen = std::max(maxlen, lens_host[b]);
  }
  if (layer != CONFKV_ALL_LAYERS && (layer < 0 || layer >= h->L)) return CONFKV_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (batch != h->batch) {
    // a new batch: every layer must be ingested again, budgets start at the larger one
    std::fill(h->prefilled.begin(), h->prefilled.end(), 0);
    std::fill(h->ema_pending.begin(), h->ema_pending.end(), 0);
    h->batch = batch;
    std::vector<int32_t> init((size_t)batch * h->L);
    for (int b = 0; b < batch; ++b)
      for (int l = 0; l < h->L; ++l)
        init[(size_t)b * h->L + l] =
            fixed ? h->p.fixed_budget
                  : layer_budget(std::max(h->p.n_low, h->p.n_high), l, h->L, h->p.pyramidal != 0);
    cudaError_t e = cudaMemcpyAsync(h->budget, init.data(), init.size() * 4, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return CONFKV_ERR_CUDA;
  }
  confkv::Range r;
  layer_range(h, layer, &r);
  cudaError_t e = cudaMemcpyAsync(h->lens_dev, lens_host, (size_t)batch * 4, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return CONFKV_ERR_CUDA;
  // a deferred EMA pass of these layers is moot: their segments start over
  for (int l = r.l0; l < r.l0 + r.nl; ++l) h->ema_pending[l] = 0;
  confkv::PrefillLaunch a;
  a.r = r;
  a.lens = h->lens_dev;
  a.t_stride = t_stride;
  a.k = static_cast<const __half*>(k);
  a.v = static_cast<const __half*>(v);
  a.prio = priority;
  a.keep_list = h->keep_list;
  a.keep_count = h->keep_count;
  a.cand = h->cand;
  e = confkv::launch_prefill(h->c, h->pol, a, st, &h->launches, h->prof_ptr());
  if (e != cudaSuccess) return CONFKV_ERR_CUDA;
  // the host copy of lens must stay valid until the copy has been consumed
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return CONFKV_ERR_CUDA;
  for (int l = r.l0; l < r.l0 + r.nl; ++l) {
    h->prefilled[l] = 1;
    h->ub_len[l] = fixed ? std::min(maxlen, h->p.fixed_budget) : maxlen;
  }
  return CONFKV_OK;
}

confkv_status confkv_confidence(confkv_handle* h, const float* logits, int32_t batch, int32_t vocab, float* c_out,
                                int32_t* budget_out, void* stream) {
  if (!alive(h)) return CONFKV_ERR_STATE;
  if (h->p.mode == CONFKV_MODE_FIXED || h->batch == 0) return CONFKV_ERR_STATE;
  if (!logits || batch != h->batch || vocab < 2) return CONFKV_ERR_ARG;
  confkv::ConfLaunch a;
  a.logits = logits;
  a.B = batch;
  a.V = vocab;
  a.L = h->L;
  a.part = h->cpart;
  a.tickets = h->tickets;
  a.cpr = std::max(1, std::min(kMaxCpr, (vocab + 4095) / 4096));
  a.c_ws = h->c_ws;
  a.budget_ws = h->budget;
  a.c_out = c_out;
  a.budget_out = budget_out;
  a.err = h->c.err;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = confkv::launch_confidence(a, h->pol, st, &h->launches, h->prof_ptr());
  h->conf_last = e == cudaSuccess;
  h->conf_stream = st;
  return cuda_status(e);
}

confkv_status confkv_decode_attn(confkv_handle* h, int32_t layer, const void* q, const void* k_new,
                                 const void* v_new, const float* prio_new, float* out, float* lse_out,
                                 void* stream) {
  if (!alive(h)) return CONFKV_ERR_STATE;
  if (!q || !k_new || !v_new || !out) return CONFKV_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out)) return CONFKV_ERR_ARG;
  const bool fixed = h->p.mode == CONFKV_MODE_FIXED;
  if (fixed != (prio_new != nullptr)) return CONFKV_ERR_ARG;
  confkv::Range r;
  if (!layer_range(h, layer, &r)) return CONFKV_ERR_ARG;
  if (h->batch == 0) return CONFKV_ERR_STATE;
  long long ub = 0;
  for (int l = r.l0; l < r.l0 + r.nl; ++l) {
    if (!h->prefilled[l]) return CONFKV_ERR_STATE;
    if (h->ub_len[l] + 1 > h->c.cap) return CONFKV_ERR_CAPACITY;
    ub = std::max(ub, h->ub_len[l] + 1);
  }
  confkv::AttnLaunch a;
  a.r = r;
  a.q = static_cast<const __half*>(q);
  a.k_new = static_cast<const __half*>(k_new);
  a.v_new = static_cast<const __half*>(v_new);
  a.prio_new = prio_new;
  a.out = out;
  a.lse_out = lse_out;
  a.lse_ws = h->lse_ws;
  a.scores = h->scores;
  a.score_stride = h->score_stride;
  a.part = h->part;
  a.part_units = h->part_units;
  a.max_cold_tokens = (int)std::min<long long>(ub, h->c.cap);
  a.num_sms = h->num_sms;
  a.qfrag = h->qfrag;
  a.qf_stride = h->qf_stride;
  a.cand = h->cand;
  a.sched = h->sched;
  const bool defer = h->pol.mode == 0 && !h->p.single_stream;
  a.run_ema = (h->pol.mode == 0 && !defer) ? 1 : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->conf_last = false;
  // a pass still deferred from the previous call over these layers reads the
  // scores this call is about to overwrite: run it first
  cudaError_t e = flush_ema(h, r.l0, r.nl, st);
  if (e != cudaSuccess) return cuda_status(e);
  e = confkv::launch_decode_attn(h->c, h->pol, a, st, &h->launches, h->prof_ptr());
  if (e != cudaSuccess) return cuda_status(e);
  if (defer) {
    e = cudaEventRecord(h->attn_done, st);
    if (e != cudaSuccess) return cuda_status(e);
    h->attn_stream = st;
    for (int l = r.l0; l < r.l0 + r.nl; ++l) h->ema_pending[l] = 1;
  }
  for (int l = r.l0; l < r.l0 + r.nl; ++l) h->ub_len[l] += 1;
  return CONFKV_OK;
}

confkv_status confkv_evict_compact(confkv_handle* h, int32_t layer, void* stream) {
  if (!alive(h)) return CONFKV_ERR_STATE;
  confkv::Range r;
  if (!layer_range(h, layer, &r)) return CONFKV_ERR_ARG;
  if (h->batch == 0) return CONFKV_ERR_STATE;
  for (int l = r.l0; l < r.l0 + r.nl; ++l)
    if (!h->prefilled[l]) return CONFKV_ERR_STATE;
  confkv::EvictLaunch a;
  a.r = r;
  a.budget = h->budget;
  a.vmask = h->vmask;
  a.mask_words = h->mask_words;
  a.stable = h->p.compact != CONFKV_COMPACT_HOLEFILL;   // the linear layout compacts in order too
  a.cand = h->cand;
  a.kscratch = h->kscratch;
  a.scratch_stride = h->scratch_stride;
  a.scratch_ctas = h->scratch_ctas;
  a.scratch_keys = h->c.cap + h->c.Wst;
  a.bulk_sched = h->bulk_sched;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  a.ema_early = h->conf_last && h->conf_stream == st ? 1 : 0;
  h->conf_last = false;
  // Every layer of the call has its EMA pass deferred (the steady decode
  // step): the eviction kernel runs it fused. Otherwise the deferred passes
  // run on their own first and eviction reads their candidate records.
  bool all_pending = h->pol.mode == 0;
  for (int l = r.l0; l < r.l0 + r.nl; ++l) all_pending = all_pending && h->ema_pending[l];
  cudaError_t e = cudaSuccess;
  confkv::EmaIn ein{h->lse_ws, h->scores, h->score_stride};
  if (all_pending) {
    // a segment may hold more than even the largest budget allows by more
    // than the warp path takes (the first step after a long prompt, or after
    // skipped evictions): the bulk-shaped variant
    bool bulk = false;
    for (int l = r.l0; l < r.l0 + r.nl; ++l) bulk = bulk || h->ub_len[l] > h->max_eff[l] + confkv::kWarpMaxVictims;
    e = join_attention(h, st);
    if (e == cudaSuccess)
      e = confkv::launch_evict_compact(h->c, h->pol, a, &ein, bulk, h->num_sms, st, &h->launches, h->prof_ptr());
    if (e == cudaSuccess)
      for (int l = r.l0; l < r.l0 + r.nl; ++l) h->ema_pending[l] = 0;
  } else {
    e = flush_ema(h, r.l0, r.nl, st);
    if (e == cudaSuccess)
      e = confkv::launch_evict_compact(h->c, h->pol, a, nullptr, false, h->num_sms, st, &h->launches, h->prof_ptr());
  }
  if (e != cudaSuccess) return cuda_status(e);
  for (int l = r.l0; l < r.l0 + r.nl; ++l) h->ub_len[l] = std::min<long long>(h->ub_len[l], h->max_eff[l]);
  return CONFKV_OK;
}

confkv_status confkv_query(confkv_handle* h, confkv_stats* out) {
  if (!alive(h)) return CONFKV_ERR_STATE;
  if (!out) return CONFKV_ERR_ARG;
  std::memset(out, 0, sizeof(*out));
  cudaError_t e = flush_all_ema(h);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return CONFKV_ERR_CUDA;
  const confkv::Cache& c = h->c;
  unsigned long long cnt[confkv::kNumCounters];
  e = cudaMemcpy(cnt, c.counters, sizeof(cnt), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return CONFKV_ERR_CUDA;
  out->attn_tokens_int8 = (int64_t)cnt[confkv::kCntAttnInt8];
  out->attn_tokens_fp16 = (int64_t)cnt[confkv::kCntAttnFp16];
  out->evict_tokens = (int64_t)cnt[confkv::kCntEvictScanned];
  out->moved_rows = (int64_t)cnt[confkv::kCntMovedRows];
  out->requant_rows = (int64_t)cnt[confkv::kCntRequant];
  out->kernel_launches = h->launches;
  out->evict_block_segments = (int64_t)cnt[confkv::kCntEvictBlock];
  out->moved_window_rows = (int64_t)cnt[confkv::kCntMovedWin];
  out->bytes_capacity = (int64_t)h->buf.bytes;
  out->min_len = 0;
  out->max_len = 0;
  if (h->batch == 0) return CONFKV_OK;
  const size_t S = (size_t)h->L * c.Bmax * c.Hkv;
  std::vector<int32_t> ncold(S), posr(S * (size_t)c.Wst);
  e = cudaMemcpy(ncold.data(), c.n_cold, S * 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && c.Wst) e = cudaMemcpy(posr.data(), c.pos_r, posr.size() * 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return CONFKV_ERR_CUDA;
  int mn = 1 << 30, mx = 0;
  const int cold_row = c.cold_int8 ? 2 * c.D + 8 : 4 * c.D;
  for (int l = 0; l < h->L; ++l) {
    if (!h->prefilled[l]) continue;
    for (int b = 0; b < h->batch; ++b)
      for (int k = 0; k < c.Hkv; ++k) {
        const size_t s = ((size_t)l * c.Bmax + b) * c.Hkv + k;
        int nr = 0;
        for (int slot = 0; slot < c.W; ++slot) nr += posr[s * c.Wst + slot] >= 0;
        const int n = ncold[s] + nr;
        mn = std::min(mn, n);
        mx = std::max(mx, n);
        if (c.cold_int8) out->tokens_int8 += ncold[s];
        else out->tokens_fp16 += ncold[s];
        out->tokens_fp16 += nr;
        out->bytes_payload += (int64_t)ncold[s] * cold_row + (int64_t)nr * 4 * c.D;
        out->bytes_meta += (int64_t)n * 8;
      }
  }
  out->min_len = mx ? mn : 0;
  out->max_len = mx;
  return CONFKV_OK;
}

confkv_status confkv_export_segment(confkv_handle* h, int32_t layer, int32_t seq, int32_t kv_head, void* host_buf,
                                    size_t* bytes) {
  if (!alive(h)) return CONFKV_ERR_STATE;
  if (!bytes || layer < 0 || layer >= h->L || seq < 0 || seq >= h->p.max_batch || kv_head < 0 || kv_head >= h->Hkv)
    return CONFKV_ERR_ARG;
  const confkv::Cache& c = h->c;
  const size_t s = ((size_t)layer * c.Bmax + seq) * c.Hkv + kv_head;
  cudaError_t e = flush_all_ema(h);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return CONFKV_ERR_CUDA;
  int32_t hdr[8] = {0, c.W, 0, c.cold_int8, c.D, h->p.mode, 0, 0};
  e = cudaMemcpy(&hdr[0], c.n_cold + s, 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(&hdr[2], c.next_pos + s, 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return CONFKV_ERR_CUDA;
  const size_t n = (size_t)hdr[0];
  const size_t row = c.cold_int8 ? (size_t)c.D : (size_t)c.D * 2;
  const size_t W = (size_t)c.W;
  const size_t need = 32 + n * 16 + 2 * n * row + W * 8 + 2 * W * c.D * 2;
  if (!host_buf) {
    *bytes = need;
    return CONFKV_OK;
  }
  if (*bytes < need) {
    *bytes = need;
    return CONFKV_ERR_ARG;
  }
  unsigned char* o = static_cast<unsigned char*>(host_buf);
  std::memcpy(o, hdr, 32);
  o += 32;
  const size_t cs = s * c.cap;
  auto d2h = [&](void* dst, const void* src, size_t nb) {
    if (e == cudaSuccess && nb) e = cudaMemcpy(dst, src, nb, cudaMemcpyDeviceToHost);
  };
  d2h(o, c.pos_c + cs, n * 4);
  o += n * 4;
  d2h(o, c.sc_c + cs, n * 4);
  o += n * 4;
  if (c.cold_int8) {
    d2h(o, c.ks + cs, n * 4);
    d2h(o + n * 4, c.vs + cs, n * 4);
  } else {
    std::memset(o, 0, n * 8);
  }
  o += n * 8;
  // K and V rows leave the device permuted (see layout.cuh); they are copied
  // raw and put back in logical row order here
  const int D = c.D;
  const size_t nr = (size_t)round_up((long long)n, 32);   // whole 128-byte lines and 32-token blocks
  std::vector<unsigned char> raw(nr * row);
  auto unpermute_cold = [&](const void* src, bool v_codes) {
    d2h(raw.data(), src, nr * row);
    for (size_t i = 0; i < n; ++i)
      for (size_t b = 0; b < row; ++b) {
        size_t off;
        if (!c.cold_int8) off = confkv::h_off((int)i, (int)b, D);
        else if (v_codes) off = confkv::v8_off((int)i, (int)b, D);
        else off = confkv::k8_off((int)i, (int)b, D);
        o[i * row + b] = raw[off];
      }
    o += n * row;
  };
  unpermute_cold(c.cold_int8 ? (const void*)(c.k8 + cs * c.D) : (const void*)(c.kc + cs * c.D), false);
  unpermute_cold(c.cold_int8 ? (const void*)(c.v8 + cs * c.D) : (const void*)(c.vc + cs * c.D), true);
  const size_t rs = s * c.Wst;
  d2h(o, c.pos_r + rs, W * 4);
  o += W * 4;
  d2h(o, c.sc_r + rs, W * 4);
  o += W * 4;
  std::vector<unsigned char> rraw((size_t)c.Wst * c.D * 2);
  for (int which = 0; which < 2; ++which) {
    d2h(rraw.data(), which ? (const void*)(c.vr + rs * c.D) : (const void*)(c.kr + rs * c.D), rraw.size());
    for (size_t i = 0; i < W; ++i)
      for (size_t b = 0; b < (size_t)c.D * 2; ++b) o[i * c.D * 2 + b] = rraw[confkv::h_off((int)i, (int)b, D)];
    o += W * c.D * 2;
  }
  *bytes = need;
  return e == cudaSuccess ? CONFKV_OK : CONFKV_ERR_CUDA;
}

confkv_status confkv_last_error_detail(confkv_handle* h, int32_t* detail) {
  if (!alive(h)) return CONFKV_ERR_STATE;
  if (!detail) return CONFKV_ERR_ARG;
  int32_t v[4] = {0, 0, 0, 0};
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(v, h->c.err, 16, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return CONFKV_ERR_CUDA;
  detail[0] = v[1];
  detail[1] = v[2];
  detail[2] = v[3];
  return static_cast<confkv_status>(v[0]);
}

confkv_status confkv_profile_enable(confkv_handle* h, int32_t enable) {
  if (!alive(h)) return CONFKV_ERR_STATE;
  h->prof.collect();
  h->prof.on = enable != 0;
  return CONFKV_OK;
}

confkv_status confkv_profile_read(confkv_handle* h, confkv_profile* out, int32_t reset) {
  if (!alive(h)) return CONFKV_ERR_STATE;
  if (!out) return CONFKV_ERR_ARG;
  h->prof.collect();
  for (int i = 0; i < CONFKV_K_KINDS; ++i) {
    out->launches[i] = h->prof.launches[i];
    out->ms[i] = h->prof.ms[i];
  }
  if (reset) h->prof.reset();
  return CONFKV_OK;
}

confkv_status confkv_last_error(confkv_handle* h, int32_t clear) {
  if (!alive(h)) return CONFKV_ERR_STATE;
  int32_t v = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&v, h->c.err, 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && clear) e = cudaMemset(h->c.err, 0, 16);
  if (e == cudaSuccess && clear) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return CONFKV_ERR_CUDA;
  return static_cast<confkv_status>(v);
}

}  // extern "C"
