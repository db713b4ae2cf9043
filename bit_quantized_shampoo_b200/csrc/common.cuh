// Shared helpers of the shampoo4 CUDA library (product code only).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>
#include "shampoo4.h"

#define S4_TRY(expr)                                        \
  do {                                                      \
    shampoo4_status s4_st_ = (expr);                        \
    if (s4_st_ != SHAMPOO4_OK) return s4_st_;               \
  } while (0)

#define S4_CUDA(expr)                                       \
  do {                                                      \
    cudaError_t s4_ce_ = (expr);                            \
    if (s4_ce_ != cudaSuccess) return SHAMPOO4_ERR_CUDA;    \
  } while (0)

namespace s4 {

// ---- 4-bit codebooks -------------------------------------------------------
// kCodebookLinearSquare ("4-bit Shampoo ...", abstract: linear square
// quantization): level j is sgn(y) y^2 for y = (2j - 15)/15, evaluated in
// double as ((2j-15)|2j-15|) / 225.
// kCodebookDynamicTree (the abstract's alternative, read as Dettmers' 2016
// dynamic tree data type restricted to 4 bits): a sign, then in the three
// remaining bits a run of E zeros (the decimal exponent), an indicator 1 and
// k = 2 - E fraction bits i, magnitude 10^-E (0.1 + 0.9 (i + 1) / 2^k); the
// pattern 000 is zero.  In the 16-level order (ascending) the three bits p
// of level 8 + p hold +magnitude(p) and level 7 - p holds -magnitude(p), so
// levels 7 and 8 are both zero.  Evaluated in double as the integer ratio
// (2^k + 9 (i + 1)) / (10^(E+1) 2^k).
// Threshold k of either codebook is the fp32 rounding of the double
// midpoint of levels k and k+1.
enum { kCodebookLinearSquare = 0, kCodebookDynamicTree = 1, kCodebookCount = 2 };

__host__ __device__ constexpr double dyn_tree_magnitude(int p) {
  if (p == 0) return 0.0;
  const int e = p >= 4 ? 0 : (p >= 2 ? 1 : 2);       // zeros before the indicator bit
  const int k = 2 - e;                                // fraction bits after it
  const int i = p & ((1 << k) - 1);
  double den = double(1 << k) * 10.0;
  for (int q = 0; q < e; ++q) den *= 10.0;
  return double((1 << k) + 9 * (i + 1)) / den;
}
__host__ __device__ constexpr double level_f64(int cb, int j) {
  return cb == kCodebookDynamicTree
             ? (j >= 8 ? dyn_tree_magnitude(j - 8) : -dyn_tree_magnitude(7 - j))
             : double((2 * j - 15) * ((2 * j - 15) < 0 ? -(2 * j - 15) : (2 * j - 15))) / 225.0;
}
__host__ __device__ constexpr float level_f32(int cb, int j) { return float(level_f64(cb, j)); }
__host__ __device__ constexpr float threshold_f32(int cb, int k) {
  return float((level_f64(cb, k) + level_f64(cb, k + 1)) / 2.0);
}

constexpr int kQuantBlock = 64;

// Round to the nearest TF32 number (ties away from zero).
__device__ __forceinline__ float tf32_rn(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// Store the TF32 split of v: h[i] = RN(v) and, if l, l[i] = RN(v - h[i]).
__device__ __forceinline__ void put_split(float v, float* h, float* l, int64_t i) {
  if (!h) return;
  const float hv = tf32_rn(v);
  h[i] = hv;
  if (l) l[i] = tf32_rn(v - hv);
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace s4
