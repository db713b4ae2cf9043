// Stand-alone 4-bit codec: quant4_pack / quant4_unpack over batches of fp32
// tensors ("4-bit Shampoo for Memory-Efficient Network Training", abstract:
// block-wise linear square quantization; the dynamic tree map is the
// alternative codebook).
//
// Memory-bound.  One CTA of 256 threads covers 4096 consecutive elements of
// one tensor (64 quantization blocks); each thread owns two groups of 8
// elements and issues both groups' loads before it computes either.  8
// consecutive lanes own one block.  A warp whose blocks all have a scale in
// [2^-60, 1] and no missing elements takes the code decision by signed
// buckets: one byte per bucket in shared memory (broadcast-friendly, almost
// free of bank conflicts) and the threshold by a shuffle from the lane that
// holds it; any other warp takes the general decision (quantize8).
// (Measured on a 1 GiB tensor: four groups per thread and persistent
// grid-stride loops were slower; a float2 table of 129 to 513 entries lost
// to bank conflicts.)
#include "quant4.cuh"
#include "plan.h"

namespace s4 {

constexpr int kCodecThreads = 256;
constexpr int kCodecGroupsPerThread = 2;
constexpr int kCodecEltsPerCta = kCodecThreads * 8 * kCodecGroupsPerThread;   // 4096
constexpr int kCodecMaxBatch = 64;

struct PackTensor {
  const float* x;
  uint8_t* codes;
  float* scales;
  int64_t n;
  int64_t cta_begin;
  const uint32_t* skip;   // optional: tensor left untouched when *skip != 0
  int32_t vec_x;          // x is 16-byte aligned: 128-bit loads
  int32_t vec_codes;      // codes is 4-byte aligned: 32-bit stores
};
struct PackBatch {
  int32_t count;
  int32_t codebook;
  CodecTables tables;
  SignedBuckets sb;
  PackTensor t[kCodecMaxBatch];
};

struct UnpackTensor {
  const uint8_t* codes;
  const float* scales;
  float* x;
  int64_t n;
  int64_t cta_begin;
  int32_t vec_x;
  int32_t vec_codes;
};
struct UnpackBatch {
  int32_t count;
  int32_t codebook;
  CodecTables tables;
  UnpackTensor t[kCodecMaxBatch];
};

// The tables of each codebook, built once on the host.
const CodecTables& host_tables(int codebook) {
  static const CodecTables t[kCodebookCount] = {make_codec_tables(kCodebookLinearSquare),
                                               make_codec_tables(kCodebookDynamicTree)};
  return t[codebook];
}
const SignedBuckets& host_signed_buckets(int codebook) {
  static const SignedBuckets t[kCodebookCount] = {make_signed_buckets(kCodebookLinearSquare),
                                                 make_signed_buckets(kCodebookDynamicTree)};
  return t[codebook];
}

template <class B>
__device__ __forceinline__ int find_tensor(const B& b, int64_t cta) {
  int lo = 0, hi = b.count - 1;
  while (lo < hi) {                    // last tensor with cta_begin <= cta
    int mid = (lo + hi + 1) >> 1;
    if (b.t[mid].cta_begin <= cta) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The 8 elements starting at element e0 of tensor t into v (zeros past the
// end; valid marks the elements that exist).
__device__ __forceinline__ void load_group(const PackTensor& t, int64_t e0, float (&v)[8], uint32_t& valid) {
  valid = 0;
  if (t.vec_x && e0 + 8 <= t.n) {
    const float4* p = reinterpret_cast<const float4*>(t.x + e0);
    float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    valid = 0xffu;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      bool ok = e0 + e < t.n;
      v[e] = ok ? __ldg(t.x + e0 + e) : 0.0f;
      valid |= ok ? (1u << e) : 0u;
    }
  }
}

// Quantize one loaded group (all lanes of the warp call this together) and
// store its codes and, from the block's first lane, its scale.  FULL: the
// group lies inside the tensor, x is 16-byte and codes 4-byte aligned.
template <int SHIFT, bool FULL>
__device__ __forceinline__ void pack_group(const PackTensor& t, int64_t e0, const float (&v)[8], uint32_t valid,
                                           const uint8_t* below, float t_lane, const float2* bucket) {
  float s = block_absmax_nan(v);
  uint32_t packed;
  if (__all_sync(0xffffffffu, (FULL || valid == 0xffu) && s >= 0x1p-60f && s <= 1.0f))   // warp-uniform
    packed = quantize8_signed<SHIFT>(v, s, below, t_lane);
  else
    packed = quantize8(v, FULL ? 0xffu : valid, bucket, &s);
  if ((threadIdx.x & 7) == 0 && (FULL || e0 < t.n)) t.scales[e0 / kQuantBlock] = s;
  if (FULL) {
    *reinterpret_cast<uint32_t*>(t.codes + (e0 >> 1)) = packed;
    return;
  }
  if (valid == 0) return;
  int64_t byte0 = e0 >> 1;
  if (t.vec_codes && valid == 0xffu) {
    *reinterpret_cast<uint32_t*>(t.codes + byte0) = packed;
  } else {
    int64_t nbytes = (t.n + 1) >> 1;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (byte0 + k < nbytes) t.codes[byte0 + k] = uint8_t(packed >> (8 * k));
  }
}

template <int SHIFT, bool FULL>
__device__ __forceinline__ void pack_cta(const PackTensor& t, int64_t e_base, bool skip, const uint8_t* below,
                                         float t_lane, const float2* bucket) {
  float v[kCodecGroupsPerThread][8];
  uint32_t valid[kCodecGroupsPerThread];
#pragma unroll
  for (int g = 0; g < kCodecGroupsPerThread; ++g) {
    const int64_t e0 = e_base + (int64_t(g) * kCodecThreads + threadIdx.x) * 8;
    if (FULL) {
      const float4* p = reinterpret_cast<const float4*>(t.x + e0);
      const float4 a = __ldg(p), c = __ldg(p + 1);
      v[g][0] = a.x; v[g][1] = a.y; v[g][2] = a.z; v[g][3] = a.w;
      v[g][4] = c.x; v[g][5] = c.y; v[g][6] = c.z; v[g][7] = c.w;
      valid[g] = 0xffu;
    } else {
      load_group(t, skip ? t.n : e0, v[g], valid[g]);
    }
  }
  __syncthreads();                                      // the bucket bytes
  if (skip) return;                                     // CTA-uniform
#pragma unroll
  for (int g = 0; g < kCodecGroupsPerThread; ++g) {
    const int64_t e0 = e_base + (int64_t(g) * kCodecThreads + threadIdx.x) * 8;
    pack_group<SHIFT, FULL>(t, e0, v[g], valid[g], below, t_lane, bucket);
  }
}

// SHIFT = signed_bucket_shift(b.codebook).  The general decision reads its
// bucket table from the launch parameters (rare: ragged ends, scales
// outside [2^-60, 1], NaN and infinities).  A CTA whose 4096 elements all
// lie inside an aligned tensor takes the unchecked loads and stores.
template <int SHIFT>
__global__ void __launch_bounds__(kCodecThreads)
k_quant4_pack(const __grid_constant__ PackBatch b) {
  constexpr int kWords = (signed_bucket_count(SHIFT) + 3) / 4;
  __shared__ uint32_t below[kWords];
  const uint32_t* src = reinterpret_cast<const uint32_t*>(b.sb.below);
  for (int i = threadIdx.x; i < kWords; i += kCodecThreads) below[i] = src[i];
  const float t_lane = b.tables.thr[threadIdx.x & 15];
  const PackTensor t = b.t[find_tensor(b, blockIdx.x)];
  const int64_t e_base = (int64_t(blockIdx.x) - t.cta_begin) * kCodecEltsPerCta;
  const bool skip = t.skip && *t.skip;
  const uint8_t* bl = reinterpret_cast<const uint8_t*>(below);
  if (!skip && t.vec_x && t.vec_codes && e_base + kCodecEltsPerCta <= t.n)
    pack_cta<SHIFT, true>(t, e_base, false, bl, t_lane, b.tables.bucket);
  else
    pack_cta<SHIFT, false>(t, e_base, skip, bl, t_lane, b.tables.bucket);
}

__device__ __forceinline__ void unpack_group(const UnpackTensor& t, int64_t e0, const float* level) {
  if (e0 >= t.n) return;
  float s = __ldg(t.scales + e0 / kQuantBlock);
  int64_t byte0 = e0 >> 1;
  uint32_t packed;
  bool full = e0 + 8 <= t.n;
  if (t.vec_codes && full) {
    packed = __ldg(reinterpret_cast<const uint32_t*>(t.codes + byte0));
  } else {
    packed = 0;
    int64_t nbytes = (t.n + 1) >> 1;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (byte0 + k < nbytes) packed |= uint32_t(__ldg(t.codes + byte0 + k)) << (8 * k);
  }
  float v[8];
  dequantize8(packed, s, level, v);
  if (t.vec_x && full) {
    float4* p = reinterpret_cast<float4*>(t.x + e0);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (e0 + e < t.n) t.x[e0 + e] = v[e];
  }
}

__global__ void __launch_bounds__(kCodecThreads)
k_quant4_unpack(const __grid_constant__ UnpackBatch b) {
  __shared__ CodecSmem sm;
  codec_smem_init(sm, b.tables);
  __syncthreads();
  const UnpackTensor& t = b.t[find_tensor(b, blockIdx.x)];
  int64_t e_base = (int64_t(blockIdx.x) - t.cta_begin) * kCodecEltsPerCta;
#pragma unroll
  for (int g = 0; g < kCodecGroupsPerThread; ++g) {
    int64_t e0 = e_base + (int64_t(g) * kCodecThreads + threadIdx.x) * 8;
    unpack_group(t, e0, sm.level);
  }
}

// Host launchers, shared with the optimizer's own requantization.
shampoo4_status launch_pack(const float* const* x, const int64_t* n, int32_t count,
                            uint8_t* const* codes, float* const* scales, cudaStream_t st,
                            const uint32_t* const* skip, int* launched, int codebook) {
  if (launched) *launched = 0;
  if (codebook < 0 || codebook >= kCodebookCount) return SHAMPOO4_ERR_INVALID_ARG;
  for (int32_t base = 0; base < count; base += kCodecMaxBatch) {
    PackBatch b;
    b.count = 0;
    b.codebook = codebook;
    b.tables = host_tables(codebook);
    b.sb = host_signed_buckets(codebook);
    if (!b.sb.ok) return SHAMPOO4_ERR_INVALID_ARG;           // no codebook in use has such a bucket
    int64_t ctas = 0;
    for (int32_t i = base; i < count && i < base + kCodecMaxBatch; ++i) {
      if (n[i] == 0) continue;
      PackTensor& t = b.t[b.count++];
      t.x = x[i]; t.codes = codes[i]; t.scales = scales[i]; t.n = n[i];
      t.cta_begin = ctas;
      t.skip = skip ? skip[i] : nullptr;
      t.vec_x = aligned(x[i], 16);
      t.vec_codes = aligned(codes[i], 4);
      ctas += (n[i] + kCodecEltsPerCta - 1) / kCodecEltsPerCta;
    }
    if (b.count == 0) continue;
    if (ctas > 0x7fffffffLL) return SHAMPOO4_ERR_INVALID_ARG;
    if (b.sb.shift == 14) k_quant4_pack<14><<<unsigned(ctas), kCodecThreads, 0, st>>>(b);
    else k_quant4_pack<16><<<unsigned(ctas), kCodecThreads, 0, st>>>(b);
    S4_CUDA(cudaGetLastError());
    if (launched) ++*launched;
  }
  return SHAMPOO4_OK;
}

shampoo4_status launch_unpack(const uint8_t* const* codes, const float* const* scales,
                              const int64_t* n, int32_t count, float* const* x, cudaStream_t st, int codebook) {
  if (codebook < 0 || codebook >= kCodebookCount) return SHAMPOO4_ERR_INVALID_ARG;
  for (int32_t base = 0; base < count; base += kCodecMaxBatch) {
    UnpackBatch b;
    b.count = 0;
    b.codebook = codebook;
    b.tables = host_tables(codebook);
    int64_t ctas = 0;
    for (int32_t i = base; i < count && i < base + kCodecMaxBatch; ++i) {
      if (n[i] == 0) continue;
      UnpackTensor& t = b.t[b.count++];
      t.codes = codes[i]; t.scales = scales[i]; t.x = x[i]; t.n = n[i];
      t.cta_begin = ctas;
      t.vec_x = aligned(x[i], 16);
      t.vec_codes = aligned(codes[i], 4);
      ctas += (n[i] + kCodecEltsPerCta - 1) / kCodecEltsPerCta;
    }
    if (b.count == 0) continue;
    if (ctas > 0x7fffffffLL) return SHAMPOO4_ERR_INVALID_ARG;
    k_quant4_unpack<<<unsigned(ctas), kCodecThreads, 0, st>>>(b);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

}  // namespace s4

// ------------------------------------------------------------------ C ABI

static shampoo4_status check_codec_args(const void* const* a, const void* const* b,
                                        const void* const* c, const int64_t* n, int32_t count) {
  if (count < 0) return SHAMPOO4_ERR_INVALID_ARG;
  if (count == 0) return SHAMPOO4_OK;
  if (!a || !b || !c || !n) return SHAMPOO4_ERR_INVALID_ARG;
  for (int32_t i = 0; i < count; ++i) {
    if (n[i] < 0) return SHAMPOO4_ERR_INVALID_ARG;
    if (n[i] == 0) continue;
    if (!a[i] || !b[i] || !c[i]) return SHAMPOO4_ERR_INVALID_ARG;
  }
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status quant4_pack_ex(const float* const* d_x, const int64_t* n, int32_t count,
                                          uint8_t* const* d_codes, float* const* d_scales, int32_t codebook,
                                          shampoo4_stream_t stream) {
  if (codebook < 0 || codebook >= s4::kCodebookCount) return SHAMPOO4_ERR_INVALID_ARG;
  S4_TRY(check_codec_args(reinterpret_cast<const void* const*>(d_x),
                          reinterpret_cast<const void* const*>(d_codes),
                          reinterpret_cast<const void* const*>(d_scales), n, count));
  for (int32_t i = 0; i < count; ++i)
    if (n[i] > 0 && (!s4::aligned(d_x[i], 4) || !s4::aligned(d_scales[i], 4)))
      return SHAMPOO4_ERR_INVALID_ARG;
  if (count == 0) return SHAMPOO4_OK;
  return s4::launch_pack(d_x, n, count, d_codes, d_scales, reinterpret_cast<cudaStream_t>(stream), nullptr,
                         nullptr, codebook);
}

extern "C" shampoo4_status quant4_unpack_ex(const uint8_t* const* d_codes, const float* const* d_scales,
                                            const int64_t* n, int32_t count, float* const* d_x, int32_t codebook,
                                            shampoo4_stream_t stream) {
  if (codebook < 0 || codebook >= s4::kCodebookCount) return SHAMPOO4_ERR_INVALID_ARG;
  S4_TRY(check_codec_args(reinterpret_cast<const void* const*>(d_codes),
                          reinterpret_cast<const void* const*>(d_scales),
                          reinterpret_cast<const void* const*>(d_x), n, count));
  for (int32_t i = 0; i < count; ++i)
    if (n[i] > 0 && (!s4::aligned(d_x[i], 4) || !s4::aligned(d_scales[i], 4)))
      return SHAMPOO4_ERR_INVALID_ARG;
  if (count == 0) return SHAMPOO4_OK;
  return s4::launch_unpack(d_codes, d_scales, n, count, d_x, reinterpret_cast<cudaStream_t>(stream), codebook);
}

extern "C" shampoo4_status quant4_pack(const float* const* d_x, const int64_t* n, int32_t count,
                                       uint8_t* const* d_codes, float* const* d_scales,
                                       shampoo4_stream_t stream) {
  return quant4_pack_ex(d_x, n, count, d_codes, d_scales, s4::kCodebookLinearSquare, stream);
}

extern "C" shampoo4_status quant4_unpack(const uint8_t* const* d_codes, const float* const* d_scales,
                                         const int64_t* n, int32_t count, float* const* d_x,
                                         shampoo4_stream_t stream) {
  return quant4_unpack_ex(d_codes, d_scales, n, count, d_x, s4::kCodebookLinearSquare, stream);
}

extern "C" shampoo4_status quant4_tables_ex(int32_t codebook, float levels[16], float thresholds[15]) {
  if (!levels || !thresholds || codebook < 0 || codebook >= s4::kCodebookCount) return SHAMPOO4_ERR_INVALID_ARG;
  for (int j = 0; j < 16; ++j) levels[j] = s4::level_f32(codebook, j);
  for (int k = 0; k < 15; ++k) thresholds[k] = s4::threshold_f32(codebook, k);
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status quant4_tables(float codebook[16], float thresholds[15]) {
  return quant4_tables_ex(s4::kCodebookLinearSquare, codebook, thresholds);
}
