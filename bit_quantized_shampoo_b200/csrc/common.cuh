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

// ---- linear square codebook ("4-bit Shampoo ...", abstract) -------------
// Level j is sgn(y) y^2 for y = (2j - 15)/15, evaluated in double as
// ((2j-15)|2j-15|) / 225; threshold k is the fp32 rounding of the double
// midpoint of levels k and k+1.  Everything is a compile-time constant.
__host__ __device__ constexpr double level_f64(int j) {
  return double((2 * j - 15) * ((2 * j - 15) < 0 ? -(2 * j - 15) : (2 * j - 15))) / 225.0;
}
__host__ __device__ constexpr float level_f32(int j) { return float(level_f64(j)); }
__host__ __device__ constexpr float threshold_f32(int k) {
  return float((level_f64(k) + level_f64(k + 1)) / 2.0);
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
