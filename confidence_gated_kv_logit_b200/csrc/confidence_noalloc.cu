// confkv_confidence_noalloc: the confidence-and-budget reduction for callers
// that must not allocate device memory. Some callers cannot allocate: code
// running inside a memory pool or allocator that owns the whole device,
// embedded runtimes that give the library a fixed memory budget up front,
// and paths that must stay valid while a CUDA graph is being built. This
// entry point needs no handle and calls no allocating routine. Its scratch
// (per-row partial reductions and per-row tickets) lives in a fixed array in
// this file, which every GPU that loads the library keeps until the process
// exits.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/confkv.h"
#include "kernels.h"

namespace {

constexpr int kNoAllocMaxRows = 256;   // sequences per call
constexpr int kNoAllocMaxCpr = 32;     // CTAs per row (vocab up to 32 * 8192 = 262144)
constexpr size_t kPartialBytes = sizeof(confkv::ConfPartial) * kNoAllocMaxRows * kNoAllocMaxCpr;
constexpr size_t kTicketBytes = sizeof(unsigned) * kNoAllocMaxRows;
constexpr size_t kScratchBytes = kPartialBytes + kTicketBytes + 256;   // + the error word, padded

// The scratch: about 197 KB per device. Its name is only a host-side stand-in
// in host code; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_conf_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Resolves (once per device, with that device current) the device address of
// g_conf_scratch. Returns null on failure.
unsigned char* scratch_for_current_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  *dev_out = dev;
  std::lock_guard<std::mutex> lk(g_setup_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_conf_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return static_cast<unsigned char*>(g_scratch_addr[dev]);
}

}  // namespace

extern "C" {

confkv_status confkv_confidence_noalloc(const confkv_params* params, int32_t layers, const float* logits,
                                        int32_t batch, int32_t vocab, float* c_out, int32_t* budget_out,
                                        void* stream) {
  if (!params || !logits || !c_out || !budget_out || layers < 1 || vocab < 2 || batch < 1) return CONFKV_ERR_ARG;
  const confkv_params& p = *params;
  if (p.gate != CONFKV_GATE_PROSE && p.gate != CONFKV_GATE_LITERAL) return CONFKV_ERR_ARG;
  if (p.n_low < 1 || p.n_high < 1) return CONFKV_ERR_ARG;
  const int cpr = (vocab + 8191) / 8192;
  if (batch > kNoAllocMaxRows || cpr > kNoAllocMaxCpr) return CONFKV_ERR_CAPACITY;
  int dev = 0;
  unsigned char* base = scratch_for_current_device(&dev);
  if (!base) return CONFKV_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the tickets and the error word must start at zero on every call; the array
  // keeps whatever the previous call (possibly a failed one) left in it
  unsigned* tickets = reinterpret_cast<unsigned*>(base + kPartialBytes);
  int32_t* err = reinterpret_cast<int32_t*>(base + kPartialBytes + kTicketBytes);
  if (cudaMemsetAsync(tickets, 0, kTicketBytes + sizeof(int32_t), st) != cudaSuccess) return CONFKV_ERR_CUDA;

  confkv::Policy pol{};
  pol.mode = 0;
  pol.n_low = p.n_low;
  pol.n_high = p.n_high;
  pol.tau = p.tau;
  pol.gate = p.gate;
  pol.pyramidal = p.pyramidal ? 1 : 0;
  confkv::ConfLaunch a;
  a.logits = logits;
  a.B = batch;
  a.V = vocab;
  a.L = layers;
  a.part = reinterpret_cast<confkv::ConfPartial*>(base);
  a.tickets = tickets;
  a.cpr = cpr;
  a.c_ws = c_out;          // the workspace copies of c and budgets are the caller's outputs
  a.budget_ws = budget_out;
  a.c_out = nullptr;
  a.budget_out = nullptr;
  a.err = err;
  long long launches = 0;
  return confkv::launch_confidence(a, pol, st, &launches, nullptr, false) == cudaSuccess ? CONFKV_OK : CONFKV_ERR_CUDA;
}

}  // extern "C"
