// Warp-level tensor-core instructions used by the attention kernel.
//
// Fragment shapes (g = lane / 4, t = lane % 4), from the PTX ISA's
// description of mma.m16n8k16 (.f16) and mma.m16n8k32 (.s8/.u8); in bytes the
// two are the same:
//   A (16 rows x 32 bytes): r0 = row g, bytes 4t..4t+3; r1 = row g+8, same
//       bytes; r2 = row g, bytes 16+4t..; r3 = row g+8, bytes 16+4t..
//   B (32 bytes x 8 columns): r0 = column g, bytes 4t..4t+3; r1 = column g,
//       bytes 16+4t..
//   C (16 x 8, 32-bit): c0, c1 = row g, columns 2t, 2t+1; c2, c3 = row g+8.
// ldmatrix .x4 loads four 8x(16-byte) matrices; lanes 8j..8j+7 give the row
// addresses of matrix j and register j receives matrix j, lane i holding row
// i/4, bytes 4(i%4)..+3 (with .trans: 16-bit elements (2(i%4), i/4) and
// (2(i%4)+1, i/4)).
#pragma once

#include <stdint.h>

namespace confkv {

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// d += a (16x32 s8) * b (32x8 s8), exact int32 accumulation
__device__ __forceinline__ void mma_s8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// d += a (16x32 u8) * b (32x8 s8), exact int32 accumulation
__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// d += a (16x16 f16) * b (16x8 f16), fp32 accumulation
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Barrier over `threads` threads of named barrier `id` that also returns the
// OR of `pred` over them (every participant gets the same answer).
__device__ __forceinline__ bool named_barrier_or(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

}  // namespace confkv
