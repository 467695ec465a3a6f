// Placement of cache rows in HBM, chosen for the tensor-core fragment loads
// of the attention kernel.
//
// The attention kernel copies tiles of consecutive rows into shared memory
// with plain 1-D bulk copies and then reads them with ldmatrix, which fetches
// eight rows of 16 bytes at the same column at once. Stored straight, those
// eight 16-byte pieces would sit in the same shared-memory bank group; the
// rows are therefore stored with their 16-byte chunks permuted (an XOR of the
// chunk index within a 128-byte line), so that a straight copy of a whole
// tile lands conflict-free. Every offset below is relative to the start of
// the segment's region, which is a multiple of 1 KB, and every tile starts at
// a multiple of the permutation's period, so tile-relative offsets in shared
// memory follow the same formulas.
//
//   K codes (INT8):  token-major rows of D bytes; chunk bits [4:6] of the
//                    byte offset XOR bits [7:9].
//   V codes (INT8):  dimension-major blocks of 32 tokens, [i/32][d][i%32], so
//                    that four consecutive tokens of one dimension form one
//                    32-bit word (the shape of an int8 MMA operand whose
//                    reduction axis is the token axis); same XOR.
//   fp16 rows:       token-major rows of 2D bytes (window ring, or the cold
//                    region when INT8 is off); chunk bits [4:6] XOR (row & 7).
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace confkv {

__host__ __device__ __forceinline__ size_t swz128(size_t o) { return o ^ (((o >> 7) & 7u) << 4); }

// byte b (0 <= b < D) of token i's K codes
__host__ __device__ __forceinline__ size_t k8_off(int i, int b, int D) { return swz128((size_t)i * D + b); }

// the code of token i, dimension d, in the V codes
__host__ __device__ __forceinline__ size_t v8_off(int i, int d, int D) {
  return swz128(((size_t)(i >> 5) * D + d) * 32 + (i & 31));
}

// byte b (0 <= b < 2D) of fp16 row i
__host__ __device__ __forceinline__ size_t h_off(int i, int b, int D) {
  return ((size_t)i * 2 * D + b) ^ ((size_t)(i & 7) << 4);
}

}  // namespace confkv
