// CUDA-core batched GEMMs.
//
//  * k_gemm_f32: fp32-output products of the preconditioner step, for the
//    shapes the tensor-core kernel does not take (ragged edges, unaligned
//    leading dimensions).  TF32 mode rounds both operands to TF32 (round to
//    nearest) before an exact-product fp32 FMA, the arithmetic of a TF32
//    tensor-core MMA; FP32 mode multiplies in plain fp32.
//  * k_gemm_f64: fp64-accumulating products of the Cholesky-QR used by the
//    subspace step (Gram matrix, trailing Cholesky updates, triangular-solve
//    updates), with fp32 or fp64 operands.
//
// Both: one CTA per (tile, problem), grid.x = tiles of the largest problem,
// grid.y = problem; CTAs past a problem's tile count exit at once.
#include "plan.h"

namespace s4 {

__device__ __forceinline__ float to_tf32_rn(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

__device__ __forceinline__ const float* resolve(const float* p, int64_t& ld, const OperandRef& r,
                                                const PtrEntry* tabs, int nparams_tab) {
  if (r.tab < 0) return p;
  const PtrEntry& e = tabs[r.tab * nparams_tab + r.param];
  ld = e.ld;
  return e.ptr + r.r0 * e.ld + r.c0;
}

// ------------------------------------------------------------------ fp32
constexpr int kF32Tile = 128;
constexpr int kF32BK = 8;
constexpr int kF32Threads = 256;

__global__ void __launch_bounds__(kF32Threads)
k_gemm_f32(const GemmF32Desc* __restrict__ descs, const PtrEntry* __restrict__ tabs, int nparams_tab) {
  const GemmF32Desc& g = descs[blockIdx.y];
  const int tiles_m = (g.M + kF32Tile - 1) / kF32Tile;
  const int tiles_n = (g.N + kF32Tile - 1) / kF32Tile;
  if (int(blockIdx.x) >= tiles_m * tiles_n) return;
  const int tm = blockIdx.x / tiles_n, tn = blockIdx.x % tiles_n;
  if (g.symmetric && tn > tm) return;
  if (g.skip && *g.skip) return;
  int64_t lda = g.lda, ldb = g.ldb, ldc = g.ldc;
  const float* A = resolve(g.A, lda, g.a_ref, tabs, nparams_tab);
  const float* B = resolve(g.B, ldb, g.b_ref, tabs, nparams_tab);
  float* C = const_cast<float*>(resolve(g.C, ldc, g.c_ref, tabs, nparams_tab));
  const int m0 = tm * kF32Tile, n0 = tn * kF32Tile;
  const bool tf32 = g.mode == kModeTF32;

  __shared__ float As[kF32BK][kF32Tile + 4];
  __shared__ float Bs[kF32BK][kF32Tile + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

  for (int k0 = 0; k0 < g.K; k0 += kF32BK) {
    // op(A)[m0+i, k0+kk] -> As[kk][i]
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      int i, kk;
      if (!g.ta) { i = tid / 2; kk = (tid % 2) * 4 + r; }
      else       { kk = tid / 32; i = (tid % 32) * 4 + r; }
      int gi = m0 + i, gk = k0 + kk;
      float v = 0.0f;
      if (gi < g.M && gk < g.K) {
        v = g.ta ? A[int64_t(gk) * lda + gi] : A[int64_t(gi) * lda + gk];
        if (g.kscale) v *= g.kscale[gk];
      }
      As[kk][i] = tf32 ? to_tf32_rn(v) : v;
    }
    // op(B)[k0+kk, n0+j] -> Bs[kk][j]
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      int j, kk;
      if (!g.tb) { kk = tid / 32; j = (tid % 32) * 4 + r; }
      else       { j = tid / 2; kk = (tid % 2) * 4 + r; }
      int gj = n0 + j, gk = k0 + kk;
      float v = 0.0f;
      if (gj < g.N && gk < g.K) v = g.tb ? B[int64_t(gj) * ldb + gk] : B[int64_t(gk) * ldb + gj];
      Bs[kk][j] = tf32 ? to_tf32_rn(v) : v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kF32BK; ++kk) {
      float a[8], b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 8; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  // symmetric output: every element below the diagonal is written twice,
  // at (i, j) and (j, i), from one accumulator -- also inside diagonal tiles,
  // where a product whose operands are scaled on one side only (kscale)
  // would otherwise round differently at (i, j) and (j, i)
  const bool diag_tile = g.symmetric && tm == tn;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int gi = m0 + ty + 16 * i;
    if (gi >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      int gj = n0 + tx + 16 * j;
      if (gj >= g.N) continue;
      if (diag_tile && gj > gi) continue;     // written by its mirror
      const bool mirror = g.symmetric && gj != gi;
      float v = g.alpha * acc[i][j];
      if (g.beta != 0.0f) v = fmaf(g.beta, g.Cin[int64_t(gi) * g.ldcin + gj], v);
      C[int64_t(gi) * ldc + gj] = v;
      if (mirror) {
        float w = g.alpha * acc[i][j];
        if (g.beta != 0.0f) w = fmaf(g.beta, g.Cin[int64_t(gj) * g.ldcin + gi], w);
        C[int64_t(gj) * ldc + gi] = w;
      }
    }
  }
}

shampoo4_status launch_gemm_f32(const GemmF32Desc* d_desc, int count, int max_tiles,
                                const PtrEntry* tabs, int nparams, cudaStream_t st) {
  for (int base = 0; base < count; base += 65535) {
    int c = count - base < 65535 ? count - base : 65535;
    if (max_tiles <= 0) break;
    k_gemm_f32<<<dim3(unsigned(max_tiles), unsigned(c)), kF32Threads, 0, st>>>(d_desc + base, tabs, nparams);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

// ------------------------------------------------------------------ fp64
constexpr int kF64Tile = 64;
constexpr int kF64BK = 16;
constexpr int kF64Threads = 256;

__device__ __forceinline__ double ld_any(const void* p, bool f64, int64_t idx) {
  return f64 ? static_cast<const double*>(p)[idx] : double(static_cast<const float*>(p)[idx]);
}

// Work items (tile, problem) looped over by a fixed grid, so that a launch
// whose problems are all skipped (the fp64 fallback of the QR) costs only
// its flag reads.
__global__ void __launch_bounds__(kF64Threads)
k_gemm_f64(const GemmF64Desc* __restrict__ descs, int count, int max_tiles,
           const uint32_t* __restrict__ guard) {
  if (guard && *guard == 0u) return;                      // no factor needs this launch
  __shared__ double As[kF64BK][kF64Tile + 1];
  __shared__ double Bs[kF64BK][kF64Tile + 1];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  for (int w = blockIdx.x; w < count * max_tiles; w += gridDim.x) {
    const GemmF64Desc& g = descs[w / max_tiles];
    const int t = w % max_tiles;
    if (g.M <= 0 || g.N <= 0) continue;
    const int tiles_m = (g.M + kF64Tile - 1) / kF64Tile;
    const int tiles_n = (g.N + kF64Tile - 1) / kF64Tile;
    if (t >= tiles_m * tiles_n) continue;
    const int tm = t / tiles_n, tn = t % tiles_n;
    if (g.lower_only && tn > tm) continue;
    if (g.skip && *g.skip) continue;
    const int m0 = tm * kF64Tile, n0 = tn * kF64Tile;
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    const bool af = g.a_f64, bf = g.b_f64;
    for (int k0 = 0; k0 < g.K; k0 += kF64BK) {
      __syncthreads();
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        int e = tid + r * kF64Threads;          // 0..1023 over a 64 x 16 tile
        int i, kk;
        if (!g.ta) { i = e / kF64BK; kk = e % kF64BK; }
        else       { kk = e / kF64Tile; i = e % kF64Tile; }
        int gi = m0 + i, gk = k0 + kk;
        double v = 0.0;
        if (gi < g.M && gk < g.K)
          v = g.ta ? ld_any(g.A, af, int64_t(gk) * g.lda + gi) : ld_any(g.A, af, int64_t(gi) * g.lda + gk);
        As[kk][i] = v;
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        int e = tid + r * kF64Threads;
        int j, kk;
        if (!g.tb) { kk = e / kF64Tile; j = e % kF64Tile; }
        else       { j = e / kF64BK; kk = e % kF64BK; }
        int gj = n0 + j, gk = k0 + kk;
        double v = 0.0;
        if (gj < g.N && gk < g.K)
          v = g.tb ? ld_any(g.B, bf, int64_t(gj) * g.ldb + gk) : ld_any(g.B, bf, int64_t(gk) * g.ldb + gj);
        Bs[kk][j] = v;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kF64BK; ++kk) {
        double a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int gi = m0 + ty + 16 * i;
      if (gi >= g.M) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int gj = n0 + tx + 16 * j;
        if (gj >= g.N) continue;
        double v = g.alpha * acc[i][j];
        if (g.beta != 0.0) v = fma(g.beta, ld_any(g.Cin, g.cin_f64, int64_t(gi) * g.ldcin + gj), v);
        int64_t o = int64_t(gi) * g.ldc + gj;
        if (g.c_f64) static_cast<double*>(g.C)[o] = v;
        else static_cast<float*>(g.C)[o] = float(v);
      }
    }
  }
}

shampoo4_status launch_gemm_f64(const GemmF64Desc* d_desc, int count, int max_tiles, cudaStream_t st,
                                const uint32_t* guard) {
  if (count <= 0 || max_tiles <= 0) return SHAMPOO4_OK;
  const int64_t items = int64_t(count) * max_tiles;
  const unsigned ctas = unsigned(items < 148 * 8 ? items : 148 * 8);
  k_gemm_f64<<<ctas, kF64Threads, 0, st>>>(d_desc, count, max_tiles, guard);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

}  // namespace s4
