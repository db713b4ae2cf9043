// Device-side pieces of the block-wise 4-bit codec ("4-bit Shampoo for
// Memory-Efficient Network Training", abstract: linear square quantization,
// block-wise, of the eigenvector matrix; the dynamic tree map is the
// alternative it compares against).
//
// Layout: a block is 64 consecutive elements; 8 consecutive lanes of a warp
// own one block, 8 elements each, so the block's absmax is a 3-step
// xor-shuffle inside each 8-lane segment.
#pragma once
#include <string.h>
#include "common.cuh"

namespace s4 {

// The code decision by buckets.  Both codebooks are symmetric (t_7 = 0,
// t_14-k = -t_k), so with a = |v| the count of thresholds below v is
//   v > 0:  8 + #{j >= 8 : a > t_j}          v <= 0 (or NaN):  7 - #{j >= 8 : a >= t_j}
// and for a in [0, 1] the positive thresholds are found by bucket: the
// bits of a above bit 20 (exponent and three mantissa bits) index 64
// buckets over [2^-8, 1), each holding at most one positive threshold of
// either codebook.  Bucket i stores (t, n): that threshold (NaN if none)
// and the number of positive thresholds below the bucket, so
//   #{a > t_j} = n + (a > t),   #{a >= t_j} = n + (a >= t).
// Entry 0 takes everything below 2^-8 (no threshold there: n = 0), entry 65
// everything from 1 up, infinities and NaN (n = 7, t = NaN), which gives
// 15 for +Inf, 0 for -Inf and NaN, as the count rule does.  Checked against
// the count rule on every fp32 value in [-1, 1] of both codebooks.
constexpr uint32_t kBucketBase = 0x3B8u;        // bits(2^-8) >> 20
constexpr int kBuckets = 66;

// The tables of one codebook: its 16 levels, the bucket table above, and
// the 15 thresholds (t_15 = +Inf).  Built once on the host
// (codec_tables), passed in the launch parameters and copied to shared
// memory by each CTA.
struct CodecTables {
  float level[16];
  float thr[16];
  float2 bucket[kBuckets];                      // (t, the bits of the integer n)
};

__host__ __device__ inline CodecTables make_codec_tables(int codebook) {
  CodecTables c{};
  for (int j = 0; j < 16; ++j) {
    c.level[j] = level_f32(codebook, j);
    c.thr[j] = j < 15 ? threshold_f32(codebook, j) : __builtin_huge_valf();
  }
  for (int j = 0; j < kBuckets; ++j) {
    float t = __builtin_nanf("");
    int n = 7;
    if (j == 0) {
      n = 0;
    } else if (j < kBuckets - 1) {
      const uint32_t lo_bits = (kBucketBase + j - 1) << 20, hi_bits = (kBucketBase + j) << 20;
      float lo, hi;
      memcpy(&lo, &lo_bits, 4);
      memcpy(&hi, &hi_bits, 4);
      n = 0;
      for (int k = 8; k < 15; ++k) {
        const float tk = threshold_f32(codebook, k);
        if (tk < lo) ++n;
        else if (tk < hi) t = tk;
      }
    }
    float nb;
    memcpy(&nb, &n, 4);
    c.bucket[j] = make_float2(t, nb);
  }
  return c;
}

// The code decision of the common case, by signed buckets.  For q in
// [-1, 1], qb = RN(q + 3) lies in [2, 4]; its bits above bit SHIFT index
// uniform buckets of width 2^(SHIFT - 22) (129 for SHIFT = 16, 513 for 14),
// monotone in q, each holding at most one threshold of the codebook.  With
// c0 = the number of thresholds in lower buckets (one byte per bucket), the
// thresholds are sorted, so the only one that can lie in q's bucket is
// t_c0, and
//   code = #{k : q > t_k} = c0 + (q > t_c0),   t_15 = +Inf,
// exactly, whatever the rounding of q + 3 (only its monotonicity is used).
// The width must stay below the smallest gap between thresholds: 0.022 for
// linear square (SHIFT 16: 2^-6), 0.005 for the dynamic tree (SHIFT 14:
// 2^-8).  make_signed_buckets reports a bucket with two thresholds.
__host__ __device__ constexpr int signed_bucket_shift(int codebook) {
  return codebook == kCodebookDynamicTree ? 14 : 16;
}
__host__ __device__ constexpr int signed_bucket_count(int shift) {
  return int((0x40800000u >> shift) - (0x40000000u >> shift)) + 1;
}
constexpr int kSignedBucketBytes = 516;         // signed_bucket_count(14), padded to words
struct SignedBuckets {
  uint8_t below[kSignedBucketBytes];            // c0 of each bucket
  int32_t shift;
  int32_t ok;                                   // 0 if some bucket holds two thresholds
};

__host__ __device__ inline uint32_t signed_bucket_of(float q, int shift) {
  const float qb = q + 3.0f;
  uint32_t b;
  memcpy(&b, &qb, 4);
  return (b >> shift) - (0x40000000u >> shift);
}

__host__ __device__ inline SignedBuckets make_signed_buckets(int codebook) {
  SignedBuckets sb{};
  sb.shift = signed_bucket_shift(codebook);
  sb.ok = 1;
  uint32_t kb[15];
  for (int j = 0; j < 15; ++j) kb[j] = signed_bucket_of(threshold_f32(codebook, j), sb.shift);
  for (int j = 1; j < 15; ++j)
    if (kb[j] == kb[j - 1]) sb.ok = 0;
  for (int k = 0; k < signed_bucket_count(sb.shift); ++k) {
    int c0 = 0;
    for (int j = 0; j < 15; ++j) c0 += kb[j] < uint32_t(k) ? 1 : 0;
    sb.below[k] = uint8_t(c0);
  }
  return sb;
}

using CodecSmem = CodecTables;

// Copy the tables (a CodecTables in the launch parameters) to shared
// memory; the caller synchronizes.
__device__ __forceinline__ void codec_smem_init(CodecSmem& sm, const CodecTables& src) {
  const uint32_t* a = reinterpret_cast<const uint32_t*>(&src);
  uint32_t* b = reinterpret_cast<uint32_t*>(&sm);
  for (int i = threadIdx.x; i < int(sizeof(CodecTables) / 4); i += blockDim.x) b[i] = a[i];
}

// code = number of thresholds t_k strictly below v, by the buckets above.
__device__ __forceinline__ uint32_t code_bucket(float v, const float2* bucket) {
  const uint32_t ab = __float_as_uint(v) & 0x7fffffffu;
  const uint32_t i = min(max(ab >> 20, kBucketBase - 1u), kBucketBase + 64u) - (kBucketBase - 1u);
  const float2 e = bucket[i];
  const float a = __uint_as_float(ab);
  const int n = __float_as_int(e.y);
  return v > 0.0f ? uint32_t(8 + n + (a > e.x ? 1 : 0)) : uint32_t(7 - n - (a >= e.x ? 1 : 0));
}

// IEEE round-to-nearest x / s for a block that shares one divisor s.
// Markstein's correction (P. Markstein, "Computation of elementary functions
// on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990):
// with r = RN(1/s) and q0 = RN(x r) within an ulp of x/s, the residual
// e = x - s q0 is exact under an FMA and RN(q0 + e r) is the correctly
// rounded quotient, provided nothing underflows.  Callers pass a normal,
// finite s; operands or quotients below 2^-100 (where the residual could
// underflow) take the plain IEEE division instead.
__device__ __forceinline__ float div_rn_shared(float x, float s, float r) {
  float q0 = x * r;
  if (fabsf(x) < 0x1p-100f || fabsf(q0) < 0x1p-100f) return __fdiv_rn(x, s);
  float e = fmaf(-q0, s, x);
  return fmaf(e, r, q0);
}

// Absmax of the 8 values a lane owns, as the bits of |x| with the sign
// cleared: as unsigned integers these order NaN above +Inf above every
// finite magnitude, so one integer max tracks the absmax and whether the
// block holds a NaN (bits > 0x7f800000) or an infinity (== 0x7f800000).
__device__ __forceinline__ uint32_t absmax_bits8(const float (&v)[8]) {
  uint32_t m = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) m = max(m, __float_as_uint(v[e]) & 0x7fffffffu);
  return m;
}

// Quantize 8 values owned by this lane; the 8 lanes of the block are the
// aligned 8-lane segment of the warp that contains this lane.  All 32 lanes
// of the warp must call it together.  Returns the 8 codes packed as 4 bytes
// (element 0 in the low nibble of byte 0) and the block scale in *scale:
// the absmax, NaN (canonical) if the block holds a NaN, +Inf if it holds an
// infinity and no NaN.  Lanes whose elements lie past the end pass zeros and
// a valid mask of 0 for those elements; their codes are forced to 0.
__device__ __forceinline__ uint32_t quantize8(const float (&v)[8], uint32_t valid_mask,
                                              const float2* bucket, float* scale) {
  uint32_t m = absmax_bits8(v);
#pragma unroll
  for (int off = 4; off >= 1; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
  const float s = m > 0x7f800000u ? __int_as_float(0x7fc00000) : __uint_as_float(m);
  *scale = s;
  uint32_t packed = 0;
  if (s == 0.0f) {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      packed |= ((valid_mask >> e) & 1u ? 7u : 0u) << (4 * e);
    return packed;
  }
  // s normal and finite: shared-reciprocal division; otherwise (NaN, Inf,
  // subnormal) the plain IEEE division.
  bool fast = (s >= 1.17549435e-38f) && (s <= 3.0e38f);
  float r = fast ? __frcp_rn(s) : 0.0f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    float q = fast ? div_rn_shared(v[e], s, r) : __fdiv_rn(v[e], s);
    uint32_t c = code_bucket(q, bucket);
    c = ((valid_mask >> e) & 1u) ? c : 0u;
    packed |= c << (4 * e);
  }
  return packed;
}

// max(|a|, |b|, |c|), NaN if any operand is NaN.
__device__ __forceinline__ float absmax3_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(fabsf(a)), "f"(fabsf(b)), "f"(fabsf(c)));
  return d;
}
__device__ __forceinline__ float max2_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// The absmax of the block (the aligned 8-lane segment's 64 values) as a
// float: NaN if the block holds a NaN.  All 32 lanes call it together.
__device__ __forceinline__ float block_absmax_nan(const float (&v)[8]) {
  float m = max2_nan(absmax3_nan(v[0], v[1], v[2]), absmax3_nan(v[3], v[4], v[5]));
  m = max2_nan(m, max2_nan(fabsf(v[6]), fabsf(v[7])));
#pragma unroll
  for (int off = 4; off >= 1; off >>= 1) m = max2_nan(m, __shfl_xor_sync(0xffffffffu, m, off));
  return m;
}

// Quantize 8 values of a block with scale s in [2^-60, 1] (so |q| <= 1 and
// no NaN), all elements valid.  below: the signed-bucket bytes in shared
// memory; t_lane: threshold t_(lane mod 16) of the codebook (t_15 = +Inf)
// held by each lane, fetched by a shuffle.  All 32 lanes call it together.
// The quotient is Markstein's sequence without the small-operand test: for
// |x| >= 2^-100 it is the IEEE quotient, below that a quotient under 2^-30
// with the IEEE quotient's sign (+0 and -0 both counting as not positive),
// and the code of such a quotient depends on its sign alone.
template <int SHIFT>
__device__ __forceinline__ uint32_t quantize8_signed(const float (&v)[8], float s, const uint8_t* below,
                                                     float t_lane) {
  constexpr uint32_t off = 0x40000000u >> SHIFT;
  const float r = __frcp_rn(s);
  uint32_t packed = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float q0 = v[e] * r;
    const float q = fmaf(fmaf(-q0, s, v[e]), r, q0);
    const float qb = q + 3.0f;
    const uint32_t c0 = below[(__float_as_uint(qb) >> SHIFT) - off];
    const float t = __shfl_sync(0xffffffffu, t_lane, int(c0));
    packed += (c0 + (q > t ? 1u : 0u)) << (4 * e);
  }
  return packed;
}

__device__ __forceinline__ void dequantize8(uint32_t packed, float s, const float* level,
                                            float (&out)[8]) {
#pragma unroll
  for (int e = 0; e < 8; ++e) out[e] = level[(packed >> (4 * e)) & 0xFu] * s;
}

}  // namespace s4
