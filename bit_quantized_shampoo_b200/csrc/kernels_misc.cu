// Small batched kernels of the refresh and precondition programs: blocked
// Cholesky panels and triangular solves (fp64), basis initialization,
// Rayleigh quotients, root weights, non-finite scans and conversions.
#include "quant4.cuh"
#include "plan.h"

namespace s4 {

constexpr int kPanel = 64;     // Cholesky / triangular-solve panel width

// ---- Cholesky of a jb x jb diagonal block, lower, in place ---------------
__global__ void __launch_bounds__(256) k_potrf(const PotrfDesc* __restrict__ descs, const uint32_t* __restrict__ guard) {
  if (guard && *guard == 0u) return;                      // no factor needs this launch
  const PotrfDesc& g = descs[blockIdx.x];
  const int jb = g.jb;
  if (jb <= 0 || (g.skip && *g.skip)) return;
  __shared__ double L[kPanel][kPanel + 1];
  __shared__ int bad;
  for (int e = threadIdx.x; e < jb * jb; e += blockDim.x) {
    int r = e / jb, c = e % jb;
    L[r][c] = (c <= r) ? g.A[int64_t(r) * g.ld + c] : 0.0;
  }
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int c = 0; c < jb; ++c) {
    if (threadIdx.x == 0) {
      double p = L[c][c];
      if (!(p > 0.0) || !isfinite(p)) { bad = 1; p = 1.0; }
      L[c][c] = sqrt(p);
    }
    __syncthreads();
    double piv = L[c][c];
    for (int r = c + 1 + threadIdx.x; r < jb; r += blockDim.x) L[r][c] /= piv;
    __syncthreads();
    const int w = jb - c - 1;                 // trailing (w x w) lower triangle
    for (int e = threadIdx.x; e < w * w; e += blockDim.x) {
      int r = c + 1 + e / w, s = c + 1 + e % w;
      if (s <= r) L[r][s] -= L[r][c] * L[s][c];
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < jb * jb; e += blockDim.x) {
    int r = e / jb, c = e % jb;
    if (c <= r) g.A[int64_t(r) * g.ld + c] = L[r][c];
  }
  if (threadIdx.x == 0 && bad) {
    *g.fail = 1u;
    atomicOr(g.gflags, SHAMPOO4_FLAG_REFRESH_FAILED);
  }
}

shampoo4_status launch_potrf(const PotrfDesc* d_desc, int count, cudaStream_t st, const uint32_t* guard) {
  if (count <= 0) return SHAMPOO4_OK;
  k_potrf<<<count, 256, 0, st>>>(d_desc, guard);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

// ---- X[r, 0:jb] <- X[r, 0:jb] L^-T, one warp per row --------------------
constexpr int kTrsmRowsPerCta = 64;
constexpr unsigned kWorkCtas = 148 * 8;     // grid of the work-item loops

// Work items (row chunk, problem), looped over by a fixed grid so that a
// launch whose problems are all skipped costs only its flag reads.
__global__ void __launch_bounds__(256) k_trsm(const TrsmDesc* __restrict__ descs, int count, int chunks,
                                              const uint32_t* __restrict__ guard) {
  if (guard && *guard == 0u) return;                      // no factor needs this launch
  __shared__ double L[kPanel][kPanel + 1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int w = blockIdx.x; w < count * chunks; w += gridDim.x) {
    const TrsmDesc& g = descs[w / chunks];
    const int jb = g.jb;
    const int row0 = (w % chunks) * kTrsmRowsPerCta;
    if (jb <= 0 || row0 >= g.rows || (g.skip && *g.skip)) continue;
    __syncthreads();                           // previous item done with L
    for (int e = threadIdx.x; e < jb * jb; e += blockDim.x) {
      int r = e / jb, c = e % jb;
      L[r][c] = (c <= r) ? g.L[int64_t(r) * g.ldl + c] : 0.0;
    }
    __syncthreads();
    const int row_end = min(g.rows, row0 + kTrsmRowsPerCta);
    for (int r = row0 + warp; r < row_end; r += 8) {
      double* x = g.X + int64_t(r) * g.ldx;
      double x0 = lane < jb ? x[lane] : 0.0;
      double x1 = lane + 32 < jb ? x[lane + 32] : 0.0;
      for (int c = 0; c < jb; ++c) {
        double xc = __shfl_sync(0xffffffffu, c < 32 ? x0 : x1, c & 31);
        xc /= L[c][c];
        if (c < 32) { if (lane == c) x0 = xc; } else { if (lane + 32 == c) x1 = xc; }
        if (lane > c && lane < jb) x0 -= xc * L[lane][c];
        if (lane + 32 > c && lane + 32 < jb) x1 -= xc * L[lane + 32][c];
      }
      if (lane < jb) x[lane] = x0;
      if (lane + 32 < jb) x[lane + 32] = x1;
    }
  }
}

shampoo4_status launch_trsm(const TrsmDesc* d_desc, int count, int max_rows, cudaStream_t st,
                            const uint32_t* guard) {
  if (count <= 0 || max_rows <= 0) return SHAMPOO4_OK;
  const int chunks = (max_rows + kTrsmRowsPerCta - 1) / kTrsmRowsPerCta;
  const int64_t items = int64_t(count) * chunks;
  k_trsm<<<unsigned(items < kWorkCtas ? items : kWorkCtas), 256, 0, st>>>(d_desc, count, chunks, guard);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

// ---- U = dequant(codes, scales) or I ------------------------------------
// The matrix is walked as a flat array: each thread takes groups of 8
// consecutive elements (4 code bytes, one scale, two 16-byte stores per
// output), kBasisGroups groups per thread with all loads issued first.
// A group that a row boundary splits (d not a multiple of 8) takes the
// per-element path.
constexpr int kBasisGroups = 2;
constexpr int kBasisEltsPerCta = 256 * 8 * kBasisGroups;

__device__ __forceinline__ void basis_put8(const BasisDesc& g, int64_t e0, int c0, const float (&v)[8]) {
  if (g.U) {
    float4* p = reinterpret_cast<float4*>(g.U + e0);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
  if (g.Uh) {
    float h[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) h[k] = tf32_rn(v[k]);
    float4* ph = reinterpret_cast<float4*>(g.Uh + e0);
    ph[0] = make_float4(h[0], h[1], h[2], h[3]);
    ph[1] = make_float4(h[4], h[5], h[6], h[7]);
    if (g.Ul) {
      float4* pl = reinterpret_cast<float4*>(g.Ul + e0);
      pl[0] = make_float4(tf32_rn(v[0] - h[0]), tf32_rn(v[1] - h[1]), tf32_rn(v[2] - h[2]), tf32_rn(v[3] - h[3]));
      pl[1] = make_float4(tf32_rn(v[4] - h[4]), tf32_rn(v[5] - h[5]), tf32_rn(v[6] - h[6]), tf32_rn(v[7] - h[7]));
    }
  }
  if (g.Vh) {
    const float4 m0 = *reinterpret_cast<const float4*>(g.mu + c0);
    const float4 m1 = *reinterpret_cast<const float4*>(g.mu + c0 + 4);
    const float mm[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
    float w[8], h[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) { w[k] = v[k] * mm[k]; h[k] = tf32_rn(w[k]); }
    float4* ph = reinterpret_cast<float4*>(g.Vh + e0);
    ph[0] = make_float4(h[0], h[1], h[2], h[3]);
    ph[1] = make_float4(h[4], h[5], h[6], h[7]);
    if (g.Vl) {
      float4* pl = reinterpret_cast<float4*>(g.Vl + e0);
      pl[0] = make_float4(tf32_rn(w[0] - h[0]), tf32_rn(w[1] - h[1]), tf32_rn(w[2] - h[2]), tf32_rn(w[3] - h[3]));
      pl[1] = make_float4(tf32_rn(w[4] - h[4]), tf32_rn(w[5] - h[5]), tf32_rn(w[6] - h[6]), tf32_rn(w[7] - h[7]));
    }
  }
}

__global__ void __launch_bounds__(256) k_basis(const BasisDesc* __restrict__ descs) {
  const BasisDesc& g = descs[blockIdx.y];
  const int d = g.d;
  const int64_t n = int64_t(d) * d;
  const int64_t base = int64_t(blockIdx.x) * kBasisEltsPerCta;
  if (base >= n) return;                                   // CTA-uniform
  __shared__ float level[16];
  if (threadIdx.x < 16) level[threadIdx.x] = level_f32(g.codebook, threadIdx.x);
  const bool vec = (d & 7) == 0;
  uint32_t packed[kBasisGroups];
  float sc[kBasisGroups];
#pragma unroll
  for (int q = 0; q < kBasisGroups; ++q) {                 // loads first
    const int64_t e0 = base + (int64_t(q) * 256 + threadIdx.x) * 8;
    packed[q] = 0;
    sc[q] = 0.0f;
    if (vec && !g.identity && e0 < n) {
      packed[q] = *reinterpret_cast<const uint32_t*>(g.codes + (e0 >> 1));
      sc[q] = g.scales[e0 / kQuantBlock];
    }
  }
  __syncthreads();                                          // the level table
#pragma unroll
  for (int q = 0; q < kBasisGroups; ++q) {
    const int64_t e0 = base + (int64_t(q) * 256 + threadIdx.x) * 8;
    if (e0 >= n) continue;
    const int r = int(e0 / d), c0 = int(e0 - int64_t(r) * d);
    if (vec) {
      float v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        v[k] = g.identity ? ((r == c0 + k) ? 1.0f : 0.0f) : level[(packed[q] >> (4 * k)) & 15u] * sc[q];
      basis_put8(g, e0, c0, v);
      continue;
    }
    for (int k = 0; k < 8 && e0 + k < n; ++k) {            // d not a multiple of 8
      const int64_t e = e0 + k;
      const int rr = int(e / d), c = int(e - int64_t(rr) * d);
      float x;
      if (g.identity) {
        x = (rr == c) ? 1.0f : 0.0f;
      } else {
        const uint32_t byte = g.codes[e >> 1];
        x = level[(e & 1) ? (byte >> 4) : (byte & 15u)] * g.scales[e / kQuantBlock];
      }
      if (g.U) g.U[e] = x;
      put_split(x, g.Uh, g.Ul, e);
      if (g.Vh) put_split(x * g.mu[c], g.Vh, g.Vl, e);
    }
  }
}

shampoo4_status launch_basis(const BasisDesc* d_desc, int count, int64_t max_elems, cudaStream_t st) {
  if (count <= 0 || max_elems <= 0) return SHAMPOO4_OK;
  const int64_t ctas = (max_elems + kBasisEltsPerCta - 1) / kBasisEltsPerCta;
  if (ctas > 0x7fffffffLL) return SHAMPOO4_ERR_INVALID_ARG;
  for (int base = 0; base < count; base += 65535) {
    int c = count - base < 65535 ? count - base : 65535;
    k_basis<<<dim3(unsigned(ctas), c), 256, 0, st>>>(d_desc + base);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

// ---- lambda_i = max(q_i . (S q)_i, 0) -----------------------------------
// One CTA per strip of 32 columns: warp w sums rows w, w + 8, ... of its
// lane's column in fp64 (coalesced 128-byte rows of Q and T), and the
// eight partial sums are added in warp order, so the result does not
// depend on scheduling.
__global__ void __launch_bounds__(256) k_rayleigh(const RayleighDesc* __restrict__ descs) {
  const RayleighDesc& g = descs[blockIdx.y];
  const int c0 = blockIdx.x * 32;
  if (c0 >= g.d) return;                                   // CTA-uniform
  if (g.skip && *g.skip) return;
  __shared__ double part[8][32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, i = c0 + lane;
  double acc = 0.0;
  if (i < g.d) {
#pragma unroll 4
    for (int r = w; r < g.d; r += 8)
      acc = fma(double(g.Q[int64_t(r) * g.d + i]), double(g.T[int64_t(r) * g.d + i]), acc);
  }
  part[w][lane] = acc;
  __syncthreads();
  if (w == 0 && i < g.d) {
    double s = 0.0;
#pragma unroll
    for (int k = 0; k < 8; ++k) s += part[k][lane];
    g.lam[i] = float(s > 0.0 ? s : 0.0);
  }
}

shampoo4_status launch_rayleigh(const RayleighDesc* d_desc, int count, int max_d, cudaStream_t st) {
  if (count <= 0 || max_d <= 0) return SHAMPOO4_OK;
  for (int base = 0; base < count; base += 65535) {
    int c = count - base < 65535 ? count - base : 65535;
    k_rayleigh<<<dim3((max_d + 31) / 32, c), 256, 0, st>>>(d_desc + base);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

// ---- mu_i = (lambda_i + eps)^(-1/4), evaluated in fp64 -------------------
__global__ void __launch_bounds__(256) k_mu(const MuDesc* __restrict__ descs, float eps) {
  const MuDesc& g = descs[blockIdx.y];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= g.d) return;
  if (g.sqrt_mode) {
    g.mu[i] = float(sqrt(fmax(double(g.lam[i]), 0.0)));
    return;
  }
  double x = double(g.lam[i]) + double(eps);
  g.mu[i] = float(1.0 / sqrt(sqrt(x)));
}

shampoo4_status launch_mu(const MuDesc* d_desc, int count, int max_d, float eps, cudaStream_t st) {
  if (count <= 0 || max_d <= 0) return SHAMPOO4_OK;
  for (int base = 0; base < count; base += 65535) {
    int c = count - base < 65535 ? count - base : 65535;
    k_mu<<<dim3((max_d + 255) / 256, c), 256, 0, st>>>(d_desc + base, eps);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

// ---- per-call pointer table --------------------------------------------------
struct TableArgs {
  PtrEntry e[kMaxTableEntries];
  PtrEntry* dst;
  int32_t n;
};

__global__ void __launch_bounds__(32) k_set_table(const __grid_constant__ TableArgs a) {
  for (int i = threadIdx.x; i < a.n; i += 32) a.dst[i] = a.e[i];
}

shampoo4_status launch_set_table(const PtrEntry* entries, int n, PtrEntry* dst, cudaStream_t st) {
  if (n < 0 || n > kMaxTableEntries) return SHAMPOO4_ERR_UNSUPPORTED;
  if (n == 0) return SHAMPOO4_OK;
  static thread_local TableArgs a;                 // 16 KB: off the host stack
  for (int i = 0; i < n; ++i) a.e[i] = entries[i];
  a.dst = dst;
  a.n = n;
  k_set_table<<<1, 32, 0, st>>>(a);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

// ---- non-finite scan -------------------------------------------------------
__global__ void __launch_bounds__(256)
k_scan(const ScanDesc* __restrict__ descs, const PtrEntry* __restrict__ tabs, int nparams,
       uint32_t* __restrict__ gflags) {
  const ScanDesc& g = descs[blockIdx.y];
  int64_t ld = g.ld;
  const float* X = g.X;
  if (g.ref.tab >= 0) {
    const PtrEntry& e = tabs[g.ref.tab * nparams + g.ref.param];
    ld = e.ld;
    X = e.ptr + g.ref.r0 * e.ld + g.ref.c0;
  }
  bool bad = false;
  const bool vec = ((reinterpret_cast<uintptr_t>(X) | uintptr_t(ld * 4) | reinterpret_cast<uintptr_t>(g.oh) |
                     reinterpret_cast<uintptr_t>(g.ol)) & 15) == 0 && (g.cols & 3) == 0;
  if (vec) {
    // 16-byte pieces over the whole matrix, four independent pieces in
    // flight per thread
    // rows x cols / 4 pieces fit in 32 bits (a tile is at most 1024 x 1024,
    // a statistic 1024 x 1024): 32-bit index arithmetic
    const int c4n = g.cols >> 2;
    const int n4 = g.rows * c4n;
    const int step = int(gridDim.x) * int(blockDim.x);
#pragma unroll 4
    for (int e = int(blockIdx.x) * int(blockDim.x) + int(threadIdx.x); e < n4; e += step) {
      const int r = e / c4n, c = (e - r * c4n) * 4;
      const float4 v = *reinterpret_cast<const float4*>(X + int64_t(r) * ld + c);
      bad |= !isfinite(v.x) || !isfinite(v.y) || !isfinite(v.z) || !isfinite(v.w);
      if (g.oh) {
        const float4 h = make_float4(tf32_rn(v.x), tf32_rn(v.y), tf32_rn(v.z), tf32_rn(v.w));
        const int64_t o = int64_t(r) * g.cols + c;
        *reinterpret_cast<float4*>(g.oh + o) = h;
        if (g.ol)
          *reinterpret_cast<float4*>(g.ol + o) =
              make_float4(tf32_rn(v.x - h.x), tf32_rn(v.y - h.y), tf32_rn(v.z - h.z), tf32_rn(v.w - h.w));
      }
    }
  } else {
    for (int r = blockIdx.x; r < g.rows; r += gridDim.x) {    // rows, coalesced columns
      const float* xr = X + int64_t(r) * ld;
      const int64_t o = int64_t(r) * g.cols;
      for (int c = threadIdx.x; c < g.cols; c += blockDim.x) {
        const float v = xr[c];
        bad |= !isfinite(v);
        put_split(v, g.oh, g.ol, o + c);
      }
    }
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) {
    *g.flag = 1u;
    atomicOr(gflags, g.bit);
  }
}

shampoo4_status launch_scan(const ScanDesc* d_desc, int count, int64_t max_rows,
                            const PtrEntry* tabs, int nparams, uint32_t* flags, cudaStream_t st) {
  if (count <= 0 || max_rows <= 0) return SHAMPOO4_OK;
  const unsigned ctas = unsigned(max_rows < 128 ? max_rows : 128);
  for (int base = 0; base < count; base += 65535) {
    int c = count - base < 65535 ? count - base : 65535;
    k_scan<<<dim3(ctas, c), 256, 0, st>>>(d_desc + base, tabs, nparams, flags);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

// ---- shifted Gram diagonal (fp64) -----------------------------------------
__global__ void __launch_bounds__(256) k_shift(const ShiftDesc* __restrict__ descs, const uint32_t* __restrict__ guard) {
  if (guard && *guard == 0u) return;                      // no factor needs this launch
  const ShiftDesc& g = descs[blockIdx.x];
  if (g.skip && *g.skip) return;
  __shared__ double part[256];
  double t = 0.0;
  for (int i = threadIdx.x; i < g.d; i += blockDim.x) t += g.W[int64_t(i) * g.ld + i];
  part[threadIdx.x] = t;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  const double d = double(g.d);
  const double s = 11.0 * (2.0 * d * d + d) * 0x1p-53 * part[0];
  for (int i = threadIdx.x; i < g.d; i += blockDim.x) g.W[int64_t(i) * g.ld + i] += s;
}

shampoo4_status launch_shift(const ShiftDesc* d_desc, int count, cudaStream_t st, const uint32_t* guard) {
  if (count <= 0) return SHAMPOO4_OK;
  k_shift<<<count, 256, 0, st>>>(d_desc, guard);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

// ---- fp32-storage Cholesky panel (fp64 inside) ------------------------------
// Factor the jb x jb diagonal block, then (if requested) invert the factor.
// Shared memory: the factor and the inverse as fp64 64 x 65 arrays (for the
// coalesced write-out and the inverse's column reads) and two
// double-buffered 64-vectors.
constexpr int kPotrfFSmem = (2 * kPanel * (kPanel + 1) + 4 * kPanel) * 8;

// One 64 x 64 block per CTA, fp64, 256 threads as a 16 x 16 grid: thread
// (ty, tx) holds rows ty + 16 i and columns tx + 16 j (i, j < 4) of the
// factor and of the inverse in registers.  The factorization keeps columns
// unscaled while they are read -- the LDL^T form: A[r][s] -= A[r][c]
// A[s][c] / A[c][c] -- and the inverse X = U^-1 of the unit-lower factor
// (U[r][k] = A[r][k] / A[k][k]) runs by rows, right-looking, in the same
// sweep: step c needs column c of A and row c of X, both final by then.
// Their owners publish them to double-buffered shared vectors, so one
// barrier per step suffices, and the two sequential chains are one.  The
// square roots and divisions are applied once at the end: L = U D^1/2,
// L^-1 = D^-1/2 U^-1.  Padding beyond jb is the identity in the
// factorization and zero in the written inverse.
template <int N>
__device__ __forceinline__ double pick4(const double (&v)[N], int j) {
  return j == 0 ? v[0] : (j == 1 ? v[1] : (j == 2 ? v[2] : v[3]));
}

__global__ void __launch_bounds__(256) k_potrf_f(const PotrfDescF* __restrict__ descs,
                                                 const uint32_t* __restrict__ guard) {
  if (guard && *guard == 0u) return;                      // no factor needs this launch
  const PotrfDescF& g = descs[blockIdx.x];
  const int jb = g.jb;
  if (jb <= 0 || *g.fail || (g.skip && *g.skip)) return;
  extern __shared__ double sm_potrf[];
  double (*A)[kPanel + 1] = reinterpret_cast<double (*)[kPanel + 1]>(sm_potrf);
  double (*X)[kPanel + 1] = reinterpret_cast<double (*)[kPanel + 1]>(sm_potrf + kPanel * (kPanel + 1));
  double (*vec)[kPanel] = reinterpret_cast<double (*)[kPanel]>(sm_potrf + 2 * kPanel * (kPanel + 1));
  __shared__ int bad;
  const int t = threadIdx.x, ty = t >> 4, tx = t & 15;
  double a[4][4], x[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty + 16 * i;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = tx + 16 * j;
      a[i][j] = (r < jb && c <= r) ? double(g.A[int64_t(r) * g.ld + c]) : (r == c ? 1.0 : 0.0);
      x[i][j] = r == c ? 1.0 : 0.0;
    }
  }
  if (t == 0) bad = 0;
  // step c: after it, A[c][c] is the pivot d_c, column c below it holds
  // L[:, c] sqrt(d_c), and rows > c of X have taken column c of U
  for (int c = 0; c < jb; ++c) {
    double* col = vec[c & 1];
    double* row = vec[2 + (c & 1)];
    if (tx == (c & 15)) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        double v[4] = {a[i][0], a[i][1], a[i][2], a[i][3]};
        col[ty + 16 * i] = pick4(v, c >> 4);
      }
    }
    if (ty == (c & 15)) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        double v[4] = {x[0][j], x[1][j], x[2][j], x[3][j]};
        row[tx + 16 * j] = pick4(v, c >> 4);
      }
    }
    __syncthreads();
    double p = col[c];
    if (!(p > double(g.min_pivot)) || !isfinite(p)) {      // breakdown: a pivot of 1 keeps
      if (t == 0) bad = 1;                                  // everything below finite
      p = 1.0;
    }
    const double ip = 1.0 / p;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty + 16 * i;
      if (r <= c || r >= jb) continue;
      const double arc = col[r] * ip;                       // also U[r][c]
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int s2 = tx + 16 * jj;
        if (s2 > c && s2 <= r) a[i][jj] = fma(-arc, col[s2], a[i][jj]);
        if (s2 <= c) x[i][jj] = fma(-arc, row[s2], x[i][jj]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      A[ty + 16 * i][tx + 16 * j] = a[i][j];
      X[ty + 16 * i][tx + 16 * j] = x[i][j];
    }
  __syncthreads();
  // pivots of the write-out: a breakdown's 1, as in the sweep
  for (int c = t; c < kPanel; c += blockDim.x) {
    const double p = A[c][c];
    if (c < jb && (!(p > double(g.min_pivot)) || !isfinite(p))) A[c][c] = 1.0;
  }
  __syncthreads();
  // write L = U D^1/2 (fp32 + split) and L^-1 = D^-1/2 U^-1 (split, zero
  // outside jb x jb)
  for (int r = t >> 6; r < kPanel; r += 4) {
    const int c = t & 63;
    const double sr = sqrt(A[r][r]);
    if (r < jb && c <= r) {
      const double l = (c == r) ? sr : A[r][c] / sqrt(A[c][c]);
      const float v = float(l);
      g.A[int64_t(r) * g.ld + c] = v;
      put_split(v, g.oh, g.ol, int64_t(r) * g.ld + c);
    }
    if (g.ih) {
      const float xi = (r < jb && c <= r) ? float(X[r][c] / sr) : 0.0f;
      put_split(xi, g.ih, g.il, int64_t(r) * kPanel + c);
    }
  }
  if (t == 0 && bad) {
    *g.fail = 1u;
    if (g.clear) {                        // fp32 attempt: fall back to fp64
      *g.clear = 0u;
      if (g.any_fallback) *g.any_fallback = 1u;
      if (g.gflags) atomicOr(g.gflags, SHAMPOO4_FLAG_QR_FALLBACK);
    } else if (g.gflags) {
      atomicOr(g.gflags, SHAMPOO4_FLAG_REFRESH_FAILED);
    }
  }
}

shampoo4_status launch_potrf_f(const PotrfDescF* d_desc, int count, cudaStream_t st, const uint32_t* guard) {
  if (count <= 0) return SHAMPOO4_OK;
  static bool configured = false;
  if (!configured) {
    S4_CUDA(cudaFuncSetAttribute(k_potrf_f, cudaFuncAttributeMaxDynamicSharedMemorySize, kPotrfFSmem));
    configured = true;
  }
  k_potrf_f<<<count, 256, kPotrfFSmem, st>>>(d_desc, guard);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

__global__ void __launch_bounds__(256) k_shift_f(const ShiftDescF* __restrict__ descs) {
  const ShiftDescF& g = descs[blockIdx.x];
  if (g.skip && *g.skip) return;
  for (int i = threadIdx.x; i < g.d; i += blockDim.x) {
    float* w = g.W + int64_t(i) * g.ld + i;
    *w = fmaf(g.coef, *w, *w);
  }
}

// ---- exact Gram diagonal ------------------------------------------------------
__global__ void __launch_bounds__(256) k_diag(const DiagDesc* __restrict__ descs, const uint32_t* __restrict__ guard) {
  if (guard && *guard == 0u) return;
  const DiagDesc& g = descs[blockIdx.y];
  if (g.skip && *g.skip) return;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < g.d) {
    double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
    const float* x = g.X + i;
    int k = 0;
    for (; k + 4 <= g.d; k += 4) {
      const double a = x[int64_t(k) * g.d], b = x[int64_t(k + 1) * g.d];
      const double c = x[int64_t(k + 2) * g.d], e = x[int64_t(k + 3) * g.d];
      s0 = fma(a, a, s0); s1 = fma(b, b, s1); s2 = fma(c, c, s2); s3 = fma(e, e, s3);
    }
    for (; k < g.d; ++k) { const double a = x[int64_t(k) * g.d]; s0 = fma(a, a, s0); }
    g.W[int64_t(i) * g.ldw + i] = float((s0 + s1) + (s2 + s3));
  }
}

shampoo4_status launch_diag(const DiagDesc* d_desc, int count, int max_d, cudaStream_t st, const uint32_t* guard) {
  if (count <= 0 || max_d <= 0) return SHAMPOO4_OK;
  for (int base = 0; base < count; base += 65535) {
    const int c = count - base < 65535 ? count - base : 65535;
    k_diag<<<dim3(unsigned((max_d + 255) / 256), unsigned(c)), 256, 0, st>>>(d_desc + base, guard);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

// ---- exact diagonal of a product of split operands --------------------------
__global__ void __launch_bounds__(256) k_rowdiag(const RowDiagDesc* __restrict__ descs) {
  const RowDiagDesc& g = descs[blockIdx.y];
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (i >= g.d) return;                                    // warp-uniform
  const int64_t r = int64_t(i) * g.ld;
  double s = 0.0;
  for (int k = lane; k < g.d; k += 32) {
    const double a = double(g.ah[r + k]) + (g.al ? double(g.al[r + k]) : 0.0);
    const double b = double(g.bh[r + k]) + (g.bl ? double(g.bl[r + k]) : 0.0);
    s = fma(a, b, s);
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    const float v = float(s);
    if (g.C) g.C[r + i] = v;
    if (g.Chi) {
      const float hv = tf32_rn(v);
      g.Chi[r + i] = hv;
      if (g.Clo) g.Clo[r + i] = tf32_rn(v - hv);
    }
  }
}

shampoo4_status launch_rowdiag(const RowDiagDesc* d_desc, int count, int max_d, cudaStream_t st) {
  if (count <= 0 || max_d <= 0) return SHAMPOO4_OK;
  for (int base = 0; base < count; base += 65535) {
    const int c = count - base < 65535 ? count - base : 65535;
    k_rowdiag<<<dim3(unsigned((max_d + 7) / 8), unsigned(c)), 256, 0, st>>>(d_desc + base);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

// ---- 128 x 128 inverse blocks from 64 x 64 ones -------------------------------
// Three 64 x 64 fp64 arrays (100 KB: two CTAs per SM): T = C A^-1 first,
// then A^-1's space takes B^-1 and C's space takes -B^-1 T.
constexpr int kInvSmem = 3 * 64 * 65 * 8;

__global__ void __launch_bounds__(256) k_inv128(const Inv128Desc* __restrict__ descs,
                                                const uint32_t* __restrict__ guard) {
  if (guard && *guard == 0u) return;
  const Inv128Desc& g = descs[blockIdx.x];
  if (g.skip && *g.skip) return;
  extern __shared__ double sm_inv[];
  double (*Xi)[65] = reinterpret_cast<double (*)[65]>(sm_inv);              // A^-1, then B^-1
  double (*Cm)[65] = reinterpret_cast<double (*)[65]>(sm_inv + 64 * 65);    // C, then M
  double (*Tm)[65] = reinterpret_cast<double (*)[65]>(sm_inv + 2 * 64 * 65);
  const int t = threadIdx.x, ty = t >> 4, tx = t & 15;
  const int n1 = min(64, g.d - g.j), n2 = max(0, min(64, g.d - g.j - 64));
  auto out = [&](int r, int c, double v) { put_split(float(v), g.jh, g.jl, int64_t(g.j + r) * 128 + c); };
  {
    // every load in flight before the stores (16 rows per thread)
    float xh[16], xl[16], ch[16], cl[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int r = (t >> 6) + 4 * q, c = t & 63;
      const int64_t a = int64_t(g.j + r) * 64 + c;
      xh[q] = g.ih[a];
      xl[q] = g.il[a];
      const bool in = r < n2 && c < n1;
      const int64_t o = int64_t(g.j + 64 + r) * g.d + g.j + c;
      ch[q] = in ? g.oh[o] : 0.0f;
      cl[q] = in ? g.ol[o] : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int r = (t >> 6) + 4 * q, c = t & 63;
      Xi[r][c] = double(xh[q]) + double(xl[q]);
      Cm[r][c] = double(ch[q]) + double(cl[q]);
    }
  }
  __syncthreads();
  // T = C A^-1 (thread (ty, tx): rows ty + 16 i, columns tx + 16 k)
  {
    double acc[4][4] = {};
    for (int kk = 0; kk < 64; ++kk) {
      double lft[4], rgt[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) lft[i] = Cm[ty + 16 * i][kk];
#pragma unroll
      for (int k = 0; k < 4; ++k) rgt[k] = Xi[kk][tx + 16 * k];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[i][k] = fma(lft[i], rgt[k], acc[i][k]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) Tm[ty + 16 * i][tx + 16 * k] = acc[i][k];
  }
  // top half of the output: [A^-1 0]
  for (int e = t; e < 64 * 128; e += blockDim.x) {
    const int r = e >> 7, c = e & 127;
    out(r, c, (c < 64 && r < n1 && c < n1) ? Xi[r][c] : 0.0);
  }
  __syncthreads();
  {
    float bh[16], bl[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int r = (t >> 6) + 4 * q, c = t & 63;
      const int64_t b = int64_t(g.j + 64 + r) * 64 + c;
      bh[q] = n2 > 0 ? g.ih[b] : 0.0f;
      bl[q] = n2 > 0 ? g.il[b] : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < 16; ++q) Xi[(t >> 6) + 4 * q][t & 63] = double(bh[q]) + double(bl[q]);
  }
  __syncthreads();
  // M = -B^-1 T into Cm
  {
    double acc[4][4] = {};
    for (int kk = 0; kk < 64; ++kk) {
      double lft[4], rgt[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) lft[i] = Xi[ty + 16 * i][kk];
#pragma unroll
      for (int k = 0; k < 4; ++k) rgt[k] = Tm[kk][tx + 16 * k];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[i][k] = fma(lft[i], rgt[k], acc[i][k]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) Cm[ty + 16 * i][tx + 16 * k] = -acc[i][k];
  }
  __syncthreads();
  // bottom half: [M B^-1]
  for (int e = t; e < 64 * 128; e += blockDim.x) {
    const int r = e >> 7, c = e & 127;
    double v = 0.0;
    if (r < n2) v = c < 64 ? (c < n1 ? Cm[r][c] : 0.0) : (c - 64 < n2 ? Xi[r][c - 64] : 0.0);
    out(64 + r, c, v);
  }
}

shampoo4_status launch_inv128(const Inv128Desc* d_desc, int count, cudaStream_t st, const uint32_t* guard) {
  if (count <= 0) return SHAMPOO4_OK;
  static bool configured = false;
  if (!configured) {
    S4_CUDA(cudaFuncSetAttribute(k_inv128, cudaFuncAttributeMaxDynamicSharedMemorySize, kInvSmem));
    configured = true;
  }
  k_inv128<<<count, 256, kInvSmem, st>>>(d_desc, guard);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

// ---- orthogonality sketch ------------------------------------------------------
// Sign bits of columns 16 m .. 16 m + 15: the lowbias32 integer mixer
// (C. Wellons, "Prospecting for Hash Functions", 2018) of m.
__device__ __forceinline__ uint32_t sketch_signs(uint32_t m) {
  uint32_t x = m + 0x9e3779b9u;
  x ^= x >> 16;
  x *= 0x7feb352du;
  x ^= x >> 15;
  x *= 0x846ca68bu;
  x ^= x >> 16;
  return x;
}

__device__ __forceinline__ double signed_by(float v, uint32_t bit) {
  return double(__uint_as_float(__float_as_uint(v) ^ (bit << 31)));
}

// Pass one: row r of Z = Q Omega, z_j = sum over columns c = j (mod 16) of
// +-Q[r][c] (exact fp32 values, fp64 sums).
__global__ void __launch_bounds__(128) k_sketch_z(const SketchDesc* __restrict__ descs) {
  const SketchDesc& g = descs[blockIdx.y];
  const int d = g.d;
  const int r = blockIdx.x * 128 + threadIdx.x;
  if (r >= d || (g.skip && *g.skip)) return;
  const float* q = g.Q + int64_t(r) * d;
  double z[kSketchCols];
#pragma unroll
  for (int j = 0; j < kSketchCols; ++j) z[j] = 0.0;
  for (int c0 = 0; c0 < d; c0 += 16) {
    const uint32_t s = sketch_signs(uint32_t(c0 >> 4));
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (c0 + 4 * u < d) {                                 // d % 4 == 0
        const float4 v = *reinterpret_cast<const float4*>(q + c0 + 4 * u);
        z[4 * u + 0] += signed_by(v.x, (s >> (4 * u + 0)) & 1u);
        z[4 * u + 1] += signed_by(v.y, (s >> (4 * u + 1)) & 1u);
        z[4 * u + 2] += signed_by(v.z, (s >> (4 * u + 2)) & 1u);
        z[4 * u + 3] += signed_by(v.w, (s >> (4 * u + 3)) & 1u);
      }
    }
  }
  double* zr = g.Z + int64_t(r) * kSketchCols;
#pragma unroll
  for (int j = 0; j < kSketchCols; ++j) zr[j] = z[j];
}

// Pass two: column c of Q^T Z - Omega, its squares clamped and summed as
// integers (order-independent), one atomic per warp.
__global__ void __launch_bounds__(128) k_sketch_r(const SketchDesc* __restrict__ descs) {
  const SketchDesc& g = descs[blockIdx.y];
  const int d = g.d;
  if (int(blockIdx.x) * 128 >= d || (g.skip && *g.skip)) return;   // CTA-uniform
  __shared__ double zs[32][kSketchCols];
  const int c = blockIdx.x * 128 + threadIdx.x;
  const bool ok = c < d;
  double y[kSketchCols];
#pragma unroll
  for (int j = 0; j < kSketchCols; ++j) y[j] = 0.0;
  for (int r0 = 0; r0 < d; r0 += 32) {
    const int nr = min(32, d - r0);
    __syncthreads();                                        // previous rows consumed
    for (int e = threadIdx.x; e < nr * kSketchCols; e += 128)
      zs[e / kSketchCols][e % kSketchCols] = g.Z[int64_t(r0) * kSketchCols + e];
    __syncthreads();
    if (ok) {
      // eight rows' loads in flight before their products (the pass is
      // bound by the latency of these column reads otherwise)
      const float* qc = g.Q + int64_t(r0) * d + c;
      for (int rr = 0; rr < nr; rr += 8) {
        float qv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) qv[u] = rr + u < nr ? qc[int64_t(rr + u) * d] : 0.0f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (rr + u >= nr) break;                          // rows past nr hold no staged Z
          const double qd = double(qv[u]);
#pragma unroll
          for (int j = 0; j < kSketchCols; ++j) y[j] = fma(qd, zs[rr + u][j], y[j]);
        }
      }
    }
  }
  unsigned long long t = 0;
  if (ok) {
    const uint32_t bit = (sketch_signs(uint32_t(c >> 4)) >> (c & 15)) & 1u;
#pragma unroll
    for (int j = 0; j < kSketchCols; ++j) {
      const double w = j == (c & 15) ? (bit ? -1.0 : 1.0) : 0.0;
      const double e = y[j] - w;
      const double sq = fmin(e * e, double(kDevFineClamp));
      t += static_cast<unsigned long long>(sq * double(kDevFineUnit));
    }
  }
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  if ((threadIdx.x & 31) == 0 && t) atomicAdd(g.devsq, t);
}

shampoo4_status launch_sketch(const SketchDesc* d_desc, int count, int max_d, int pass, cudaStream_t st) {
  if (count <= 0 || max_d <= 0) return SHAMPOO4_OK;
  for (int base = 0; base < count; base += 65535) {
    const int c = count - base < 65535 ? count - base : 65535;
    const dim3 grid(unsigned((max_d + 127) / 128), unsigned(c));
    if (pass == 0)
      k_sketch_z<<<grid, 128, 0, st>>>(d_desc + base);
    else
      k_sketch_r<<<grid, 128, 0, st>>>(d_desc + base);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

// ---- last-pass gate -----------------------------------------------------------
__global__ void __launch_bounds__(256) k_gate(const GateDesc* __restrict__ descs, int count) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= count) return;
  const GateDesc& g = descs[i];
  const uint32_t skip = (*g.bad != 0u || *g.devsq <= g.thr) ? 1u : 0u;
  *g.out = skip;
  if (!skip && g.any) *g.any = 1u;
}

shampoo4_status launch_gate(const GateDesc* d_desc, int count, cudaStream_t st) {
  if (count <= 0) return SHAMPOO4_OK;
  k_gate<<<unsigned((count + 255) / 256), 256, 0, st>>>(d_desc, count);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

shampoo4_status launch_shift_f(const ShiftDescF* d_desc, int count, cudaStream_t st) {
  if (count <= 0) return SHAMPOO4_OK;
  k_shift_f<<<count, 256, 0, st>>>(d_desc);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}


// ---- fp64 -> fp32 ----------------------------------------------------------
constexpr int64_t kConvertChunk = 1 << 16;
__global__ void __launch_bounds__(256) k_convert(const ConvertDesc* __restrict__ descs, int count, int chunks,
                                                 const uint32_t* __restrict__ guard) {
  if (guard && *guard == 0u) return;                      // no factor needs this launch
  for (int w = blockIdx.x; w < count * chunks; w += gridDim.x) {
    const ConvertDesc& g = descs[w / chunks];
    const int64_t lo = int64_t(w % chunks) * kConvertChunk;
    if (lo >= g.n || (g.skip && *g.skip)) continue;
    const int64_t hi = lo + kConvertChunk < g.n ? lo + kConvertChunk : g.n;
    for (int64_t e = lo + threadIdx.x; e < hi; e += blockDim.x) {
      const float v = float(g.src[e]);
      g.dst[e] = v;
      put_split(v, g.dh, g.dl, e);
    }
  }
}

shampoo4_status launch_convert(const ConvertDesc* d_desc, int count, int64_t max_elems, cudaStream_t st,
                               const uint32_t* guard) {
  if (count <= 0 || max_elems <= 0) return SHAMPOO4_OK;
  const int chunks = int((max_elems + kConvertChunk - 1) / kConvertChunk);
  const int64_t items = int64_t(count) * chunks;
  k_convert<<<unsigned(items < kWorkCtas ? items : kWorkCtas), 256, 0, st>>>(d_desc, count, chunks, guard);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

__global__ void __launch_bounds__(256) k_copy(const CopyDesc* __restrict__ descs, int count, int chunks) {
  for (int w = blockIdx.x; w < count * chunks; w += gridDim.x) {
    const CopyDesc& g = descs[w / chunks];
    const int64_t lo = int64_t(w % chunks) * kConvertChunk;
    if (lo >= g.n || !g.dst) continue;
    const int64_t hi = lo + kConvertChunk < g.n ? lo + kConvertChunk : g.n;
    for (int64_t e = lo + threadIdx.x; e < hi; e += blockDim.x) g.dst[e] = g.src[e];
  }
}

shampoo4_status launch_copy(const CopyDesc* d_desc, int count, int64_t max_elems, cudaStream_t st) {
  if (count <= 0 || max_elems <= 0) return SHAMPOO4_OK;
  const int chunks = int((max_elems + kConvertChunk - 1) / kConvertChunk);
  const int64_t items = int64_t(count) * chunks;
  k_copy<<<unsigned(items < kWorkCtas ? items : kWorkCtas), 256, 0, st>>>(d_desc, count, chunks);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

// ---- coupled Newton inverse fourth root: norm and elementwise steps ---------
__global__ void __launch_bounds__(512) k_newton_norm(const NewtonNormDesc* __restrict__ descs) {
  const NewtonNormDesc& g = descs[blockIdx.x];
  if (g.skip && *g.skip) return;
  const int d = g.d;
  const int64_t n = int64_t(d) * d;
  double t = 0.0;
  for (int64_t e = threadIdx.x; e < n; e += blockDim.x) {
    const int64_t r = e / d, c = e - r * d;
    const double a = double(g.S[e]) + (r == c ? double(g.eps) : 0.0);
    t = fma(a, a, t);
  }
  __shared__ double part[512];
  part[threadIdx.x] = t;
  __syncthreads();
  for (int w = 256; w > 0; w >>= 1) {
    if (int(threadIdx.x) < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double c = sqrt(part[0]);
    g.sc[0] = float(1.0 / c);
    g.sc[1] = float(1.0 / sqrt(sqrt(c)));
  }
}

shampoo4_status launch_newton_norm(const NewtonNormDesc* d_desc, int count, cudaStream_t st) {
  if (count <= 0) return SHAMPOO4_OK;
  k_newton_norm<<<count, 512, 0, st>>>(d_desc);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

__global__ void __launch_bounds__(256) k_newton_elt(const NewtonEltDesc* __restrict__ descs, int count, int chunks) {
  for (int w = blockIdx.x; w < count * chunks; w += gridDim.x) {
    const NewtonEltDesc& g = descs[w / chunks];
    const int d = g.d;
    const int64_t n = int64_t(d) * d;
    const int64_t lo = int64_t(w % chunks) * kConvertChunk;
    if (lo >= n || (g.skip && *g.skip)) continue;
    const int64_t hi = lo + kConvertChunk < n ? lo + kConvertChunk : n;
    const double inv_c = double(g.sc[0]);
    const float root_c = g.sc[1];
    for (int64_t e = lo + threadIdx.x; e < hi; e += blockDim.x) {
      const int64_t r = e / d, c = e - r * d;
      const bool diag = r == c;
      if (g.mode == kNewtonFinal) {
        g.m[e] = g.in[e] * root_c;
        continue;
      }
      float mv;
      if (g.mode == kNewtonInit) {
        mv = float((double(g.in[e]) + (diag ? double(g.eps) : 0.0)) * inv_c);
        g.m[e] = mv;
        put_split(mv, g.mh, g.ml, e);
      } else {
        mv = g.in[e];
      }
      const float fv = (diag ? 1.25f : 0.0f) - 0.25f * mv;
      if (g.f) g.f[e] = fv;
      put_split(fv, g.fh, g.fl, e);
      if (g.x) {
        g.x[e] = fv;
        put_split(fv, g.xh, g.xl, e);
      }
    }
  }
}

shampoo4_status launch_newton_elt(const NewtonEltDesc* d_desc, int count, int64_t max_elems, cudaStream_t st) {
  if (count <= 0 || max_elems <= 0) return SHAMPOO4_OK;
  const int chunks = int((max_elems + kConvertChunk - 1) / kConvertChunk);
  const int64_t items = int64_t(count) * chunks;
  k_newton_elt<<<unsigned(items < kWorkCtas ? items : kWorkCtas), 256, 0, st>>>(d_desc, count, chunks);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

}  // namespace s4
