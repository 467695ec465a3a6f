// Optional per-kernel timing: CUDA events recorded around every launch on the
// launching stream, accumulated per kernel kind when read back.
#pragma once

#include <cuda_runtime.h>

#include <vector>

namespace confkv {

enum KernelKind { kKConfidence = 0, kKAppend = 1, kKAttention = 2, kKCombine = 3, kKEma = 4, kKEvict = 5,
                  kKPrefill = 6, kKEmaEvict = 7, kNumKinds = 8 };

struct Prof {
  bool on = false;
  struct Rec {
    int kind;
    cudaEvent_t a, b;
  };
  std::vector<Rec> pending;
  std::vector<cudaEvent_t> pool;
  long long launches[kNumKinds] = {};
  double ms[kNumKinds] = {};

  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e;
    cudaEventCreate(&e);
    return e;
  }
  void begin(int kind, cudaStream_t st) {
    if (!on) return;
    Rec r{kind, get(), get()};
    cudaEventRecord(r.a, st);
    pending.push_back(r);
  }
  void end(cudaStream_t st) {
    if (!on || pending.empty()) return;
    cudaEventRecord(pending.back().b, st);
  }
  // Synchronises on the recorded events and folds them into the totals.
  void collect() {
    for (Rec& r : pending) {
      cudaEventSynchronize(r.b);
      float t = 0.0f;
      cudaEventElapsedTime(&t, r.a, r.b);
      ms[r.kind] += t;
      launches[r.kind] += 1;
      pool.push_back(r.a);
      pool.push_back(r.b);
    }
    pending.clear();
  }
  void reset() {
    collect();
    for (int i = 0; i < kNumKinds; ++i) {
      ms[i] = 0.0;
      launches[i] = 0;
    }
  }
  ~Prof() {
    for (Rec& r : pending) {
      cudaEventDestroy(r.a);
      cudaEventDestroy(r.b);
    }
    for (cudaEvent_t e : pool) cudaEventDestroy(e);
  }
};

// RAII bracket around one launch.
struct ProfScope {
  Prof* p;
  cudaStream_t st;
  ProfScope(Prof* p_, int kind, cudaStream_t s) : p(p_), st(s) {
    if (p) p->begin(kind, st);
  }
  ~ProfScope() {
    if (p) p->end(st);
  }
};

}  // namespace confkv
