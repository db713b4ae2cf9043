// Small batched kernels of the refresh and precondition programs: blocked
// Cholesky panels and triangular solves (fp64), basis initialization,
// Rayleigh quotients, root weights, non-finite scans and conversions.
#include "quant4.cuh"
#include "plan.h"

namespace s4 {

constexpr int kPanel = 64;     // Cholesky / triangular-solve panel width

// ---- Cholesky of a jb x jb diagonal block, lower, in place ---------------
__global__ void __launch_bounds__(256) k_potrf(const PotrfDesc* __restrict__ descs) {
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

shampoo4_status launch_potrf(const PotrfDesc* d_desc, int count, cudaStream_t st) {
  if (count <= 0) return SHAMPOO4_OK;
  k_potrf<<<count, 256, 0, st>>>(d_desc);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

// ---- X[r, 0:jb] <- X[r, 0:jb] L^-T, one warp per row --------------------
constexpr int kTrsmRowsPerCta = 64;
__global__ void __launch_bounds__(256) k_trsm(const TrsmDesc* __restrict__ descs) {
  const TrsmDesc& g = descs[blockIdx.y];
  const int jb = g.jb;
  const int row0 = blockIdx.x * kTrsmRowsPerCta;
  if (jb <= 0 || row0 >= g.rows || (g.skip && *g.skip)) return;
  __shared__ double L[kPanel][kPanel + 1];
  for (int e = threadIdx.x; e < jb * jb; e += blockDim.x) {
    int r = e / jb, c = e % jb;
    L[r][c] = (c <= r) ? g.L[int64_t(r) * g.ldl + c] : 0.0;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row_end = min(g.rows, row0 + kTrsmRowsPerCta);
  for (int r = row0 + warp; r < row_end; r += 8) {
    double* x = g.X + int64_t(r) * g.ldx;
    double x0 = lane < jb ? x[lane] : 0.0;
    double x1 = lane + 32 < jb ? x[lane + 32] : 0.0;
    for (int c = 0; c < jb; ++c) {
      // x_c is final once columns < c are applied; divide by L[c][c]
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

shampoo4_status launch_trsm(const TrsmDesc* d_desc, int count, int max_rows, cudaStream_t st) {
  if (count <= 0 || max_rows <= 0) return SHAMPOO4_OK;
  for (int base = 0; base < count; base += 65535) {
    int c = count - base < 65535 ? count - base : 65535;
    dim3 grid((max_rows + kTrsmRowsPerCta - 1) / kTrsmRowsPerCta, c);
    k_trsm<<<grid, 256, 0, st>>>(d_desc + base);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

// ---- U = dequant(codes, scales) or I ------------------------------------
__global__ void __launch_bounds__(256) k_basis(const BasisDesc* __restrict__ descs) {
  const BasisDesc& g = descs[blockIdx.y];
  __shared__ float level[16];
  if (threadIdx.x < 16) level[threadIdx.x] = level_f32(threadIdx.x);
  __syncthreads();
  const int64_t n = int64_t(g.d) * g.d;
  const int64_t e0 = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (e0 >= n) return;
  float v[8];
  if (g.identity) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      int64_t i = e0 + e;
      v[e] = (i / g.d == i % g.d) ? 1.0f : 0.0f;
    }
  } else {
    uint32_t packed = 0;
    const int64_t nbytes = (n + 1) >> 1;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if ((e0 >> 1) + k < nbytes) packed |= uint32_t(g.codes[(e0 >> 1) + k]) << (8 * k);
    dequantize8(packed, g.scales[e0 / kQuantBlock], level, v);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int64_t i = e0 + e;
    if (i >= n) break;
    if (g.U) g.U[i] = v[e];
    put_split(v[e], g.Uh, g.Ul, i);
    if (g.Vh) put_split(v[e] * g.mu[i % g.d], g.Vh, g.Vl, i);
  }
}

shampoo4_status launch_basis(const BasisDesc* d_desc, int count, int64_t max_elems, cudaStream_t st) {
  if (count <= 0 || max_elems <= 0) return SHAMPOO4_OK;
  int64_t ctas = (max_elems + 256 * 8 - 1) / (256 * 8);
  for (int base = 0; base < count; base += 65535) {
    int c = count - base < 65535 ? count - base : 65535;
    k_basis<<<dim3(unsigned(ctas), c), 256, 0, st>>>(d_desc + base);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

// ---- lambda_i = max(q_i . (S q)_i, 0) -----------------------------------
__global__ void __launch_bounds__(256) k_rayleigh(const RayleighDesc* __restrict__ descs) {
  const RayleighDesc& g = descs[blockIdx.y];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= g.d) return;
  if (g.skip && *g.skip) return;
  double acc = 0.0;
  for (int r = 0; r < g.d; ++r)
    acc += double(g.Q[int64_t(r) * g.d + i]) * double(g.T[int64_t(r) * g.d + i]);
  g.lam[i] = float(acc > 0.0 ? acc : 0.0);
}

shampoo4_status launch_rayleigh(const RayleighDesc* d_desc, int count, int max_d, cudaStream_t st) {
  if (count <= 0 || max_d <= 0) return SHAMPOO4_OK;
  for (int base = 0; base < count; base += 65535) {
    int c = count - base < 65535 ? count - base : 65535;
    k_rayleigh<<<dim3((max_d + 255) / 256, c), 256, 0, st>>>(d_desc + base);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

// ---- mu_i = (lambda_i + eps)^(-1/4), evaluated in fp64 -------------------
__global__ void __launch_bounds__(256) k_mu(const MuDesc* __restrict__ descs, float eps) {
  const MuDesc& g = descs[blockIdx.y];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= g.d) return;
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

// ---- non-finite scan -------------------------------------------------------
__global__ void __launch_bounds__(256)
k_scan(const ScanDesc* __restrict__ descs, const PtrEntry* __restrict__ tabs, int nparams,
       uint32_t* __restrict__ gflags) {
  const ScanDesc& g = descs[blockIdx.y];
  const int64_t n = int64_t(g.rows) * g.cols;
  int64_t ld = g.ld;
  const float* X = g.X;
  if (g.ref.tab >= 0) {
    const PtrEntry& e = tabs[g.ref.tab * nparams + g.ref.param];
    ld = e.ld;
    X = e.ptr + g.ref.r0 * e.ld + g.ref.c0;
  }
  bool bad = false;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += int64_t(gridDim.x) * blockDim.x) {
    int64_t r = e / g.cols, c = e % g.cols;
    float v = X[r * ld + c];
    bad |= !isfinite(v);
    put_split(v, g.oh, g.ol, e);
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) {
    *g.flag = 1u;
    atomicOr(gflags, g.bit);
  }
}

shampoo4_status launch_scan(const ScanDesc* d_desc, int count, int64_t max_elems,
                            const PtrEntry* tabs, int nparams, uint32_t* flags, cudaStream_t st) {
  if (count <= 0 || max_elems <= 0) return SHAMPOO4_OK;
  int64_t ctas = (max_elems + 256 * 8 - 1) / (256 * 8);
  if (ctas > 1024) ctas = 1024;
  for (int base = 0; base < count; base += 65535) {
    int c = count - base < 65535 ? count - base : 65535;
    k_scan<<<dim3(unsigned(ctas), c), 256, 0, st>>>(d_desc + base, tabs, nparams, flags);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

// ---- shifted Gram diagonal ------------------------------------------------
__global__ void __launch_bounds__(256) k_shift(const ShiftDesc* __restrict__ descs) {
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

shampoo4_status launch_shift(const ShiftDesc* d_desc, int count, cudaStream_t st) {
  if (count <= 0) return SHAMPOO4_OK;
  k_shift<<<count, 256, 0, st>>>(d_desc);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

// ---- fp32-storage Cholesky panel (fp64 inside) ------------------------------
__global__ void __launch_bounds__(256) k_potrf_f(const PotrfDescF* __restrict__ descs) {
  const PotrfDescF& g = descs[blockIdx.x];
  const int jb = g.jb;
  if (jb <= 0 || *g.fail) return;
  __shared__ double L[kPanel][kPanel + 1];
  __shared__ int bad;
  for (int e = threadIdx.x; e < jb * jb; e += blockDim.x) {
    int r = e / jb, c = e % jb;
    L[r][c] = (c <= r) ? double(g.A[int64_t(r) * g.ld + c]) : 0.0;
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
    const int w = jb - c - 1;
    for (int e = threadIdx.x; e < w * w; e += blockDim.x) {
      int r = c + 1 + e / w, s = c + 1 + e % w;
      if (s <= r) L[r][s] -= L[r][c] * L[s][c];
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < jb * jb; e += blockDim.x) {
    int r = e / jb, c = e % jb;
    if (c <= r) {
      const float v = float(L[r][c]);
      g.A[int64_t(r) * g.ld + c] = v;
      put_split(v, g.oh, g.ol, int64_t(r) * g.ld + c);
    }
  }
  if (threadIdx.x == 0 && bad) {
    *g.fail = 1u;
    if (g.clear) {                        // fp32 attempt: fall back to fp64
      *g.clear = 0u;
      if (g.gflags) atomicOr(g.gflags, SHAMPOO4_FLAG_QR_FALLBACK);
    } else if (g.gflags) {
      atomicOr(g.gflags, SHAMPOO4_FLAG_REFRESH_FAILED);
    }
  }
}

shampoo4_status launch_potrf_f(const PotrfDescF* d_desc, int count, cudaStream_t st) {
  if (count <= 0) return SHAMPOO4_OK;
  k_potrf_f<<<count, 256, 0, st>>>(d_desc);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

__global__ void __launch_bounds__(256) k_trsm_f(const TrsmDescF* __restrict__ descs) {
  const TrsmDescF& g = descs[blockIdx.y];
  const int jb = g.jb;
  const int row0 = blockIdx.x * kTrsmRowsPerCta;
  if (jb <= 0 || row0 >= g.rows) return;
  if (g.skip && *g.skip) return;
  __shared__ double L[kPanel][kPanel + 1];
  __shared__ double rdiag[kPanel];
  for (int e = threadIdx.x; e < jb * jb; e += blockDim.x) {
    int r = e / jb, c = e % jb;
    L[r][c] = (c <= r) ? double(g.L[int64_t(r) * g.ldl + c]) : 0.0;
  }
  __syncthreads();
  if (threadIdx.x < jb) rdiag[threadIdx.x] = 1.0 / L[threadIdx.x][threadIdx.x];
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row_end = min(g.rows, row0 + kTrsmRowsPerCta);
  const float* in = g.Xin ? g.Xin : g.X;
  // two rows per warp at a time: their dependency chains interleave
  for (int ra = row0 + 2 * warp; ra < row_end; ra += 16) {
    const int rb = ra + 1;
    const bool hb = rb < row_end;
    const float* xa = in + int64_t(ra) * g.ldx;
    const float* xb = in + int64_t(hb ? rb : ra) * g.ldx;
    double a0 = lane < jb ? double(xa[lane]) : 0.0;
    double a1 = lane + 32 < jb ? double(xa[lane + 32]) : 0.0;
    double b0 = lane < jb ? double(xb[lane]) : 0.0;
    double b1 = lane + 32 < jb ? double(xb[lane + 32]) : 0.0;
    for (int c = 0; c < jb; ++c) {
      const bool lo = c < 32;
      double ac = __shfl_sync(0xffffffffu, lo ? a0 : a1, c & 31) * rdiag[c];
      double bc = __shfl_sync(0xffffffffu, lo ? b0 : b1, c & 31) * rdiag[c];
      if (lo) { if (lane == c) { a0 = ac; b0 = bc; } } else { if (lane + 32 == c) { a1 = ac; b1 = bc; } }
      if (lane > c && lane < jb) { const double l = L[lane][c]; a0 -= ac * l; b0 -= bc * l; }
      if (lane + 32 > c && lane + 32 < jb) { const double l = L[lane + 32][c]; a1 -= ac * l; b1 -= bc * l; }
    }
    for (int k = 0; k < 2; ++k) {
      const int r = k == 0 ? ra : rb;
      if (k == 1 && !hb) break;
      const float f0 = float(k == 0 ? a0 : b0), f1 = float(k == 0 ? a1 : b1);
      float* xo = g.X + int64_t(r) * g.ldx;
      if (lane < jb) xo[lane] = f0;
      if (lane + 32 < jb) xo[lane + 32] = f1;
      if (g.oh) {
        const int64_t o = int64_t(r) * g.ldo;
        if (lane < jb) put_split(f0, g.oh, g.ol, o + lane);
        else if (g.zero_pad) put_split(0.0f, g.oh, g.ol, o + lane);
        if (lane + 32 < jb) put_split(f1, g.oh, g.ol, o + lane + 32);
        else if (g.zero_pad) put_split(0.0f, g.oh, g.ol, o + lane + 32);
      }
    }
  }
}

shampoo4_status launch_trsm_f(const TrsmDescF* d_desc, int count, int max_rows, cudaStream_t st) {
  if (count <= 0 || max_rows <= 0) return SHAMPOO4_OK;
  for (int base = 0; base < count; base += 65535) {
    int c = count - base < 65535 ? count - base : 65535;
    dim3 grid((max_rows + kTrsmRowsPerCta - 1) / kTrsmRowsPerCta, c);
    k_trsm_f<<<grid, 256, 0, st>>>(d_desc + base);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

__global__ void __launch_bounds__(256) k_shift_f(const ShiftDescF* __restrict__ descs) {
  const ShiftDescF& g = descs[blockIdx.x];
  if (g.skip && *g.skip) return;
  __shared__ double part[256];
  double t = 0.0;
  for (int i = threadIdx.x; i < g.d; i += blockDim.x) t += double(g.W[int64_t(i) * g.ld + i]);
  part[threadIdx.x] = t;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  const float s = float(double(g.coef) * part[0]);
  for (int i = threadIdx.x; i < g.d; i += blockDim.x) g.W[int64_t(i) * g.ld + i] += s;
}

shampoo4_status launch_shift_f(const ShiftDescF* d_desc, int count, cudaStream_t st) {
  if (count <= 0) return SHAMPOO4_OK;
  k_shift_f<<<count, 256, 0, st>>>(d_desc);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

__global__ void __launch_bounds__(256) k_split(const SplitDesc* __restrict__ descs) {
  const SplitDesc& g = descs[blockIdx.y];
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < g.n;
       e += int64_t(gridDim.x) * blockDim.x)
    put_split(g.x[e], g.h, g.l, e);
}

shampoo4_status launch_split(const SplitDesc* d_desc, int count, int64_t max_elems, cudaStream_t st) {
  if (count <= 0 || max_elems <= 0) return SHAMPOO4_OK;
  int64_t ctas = (max_elems + 1023) / 1024;
  if (ctas > 1024) ctas = 1024;
  for (int base = 0; base < count; base += 65535) {
    int c = count - base < 65535 ? count - base : 65535;
    k_split<<<dim3(unsigned(ctas), c), 256, 0, st>>>(d_desc + base);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

// ---- fp64 -> fp32 ----------------------------------------------------------
__global__ void __launch_bounds__(256) k_convert(const ConvertDesc* __restrict__ descs) {
  const ConvertDesc& g = descs[blockIdx.y];
  if (g.skip && *g.skip) return;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < g.n;
       e += int64_t(gridDim.x) * blockDim.x) {
    const float v = float(g.src[e]);
    g.dst[e] = v;
    put_split(v, g.dh, g.dl, e);
  }
}

shampoo4_status launch_convert(const ConvertDesc* d_desc, int count, int64_t max_elems, cudaStream_t st) {
  if (count <= 0 || max_elems <= 0) return SHAMPOO4_OK;
  int64_t ctas = (max_elems + 1023) / 1024;
  if (ctas > 1024) ctas = 1024;
  for (int base = 0; base < count; base += 65535) {
    int c = count - base < 65535 ? count - base : 65535;
    k_convert<<<dim3(unsigned(ctas), c), 256, 0, st>>>(d_desc + base);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

}  // namespace s4
