// Grafted weight update ("Shampoo -- Second-Order Optimizer", section
// "Grafting: borrow a step size that already works").
//
// Per tile b of the blocked partition:
//   d_graft = G (SGD) or, for Adam (Kingma and Ba, ICLR 2015, Algorithm 1),
//             m <- b1 m + (1-b1) G,  v <- b2 v + (1-b2) G^2,
//             d_graft = (m / (1-b1^t)) / (sqrt(v / (1-b2^t)) + adam_eps);
//   W_b    <- W_b - lr * ||d_graft_b||_F / (||D_b||_F + graft_eps) * D_b.
//
// Both passes are HBM-bound elementwise sweeps:
//   k_graft_norms  reads G, D (and m, v), writes m, v, and one fp64 pair of
//                  partial sums (sum d_graft^2, sum D^2) per band of rows;
//                  with recorded norms (dir_norms) a tensor-core tile's sum
//                  D^2 comes from the apply's epilogue and D is not read;
//   k_graft_apply  sums its tile's partials in a fixed order (the result is
//                  independent of scheduling), then W <- W - r D with one
//                  fused multiply-add per element, r rounded to fp32 once.
// A tile whose gradient the statistics update flagged as non-finite is
// skipped whole (moments and weights unchanged).  A tile whose norms or
// fp32 ratio are not finite keeps its weights and raises
// SHAMPOO4_FLAG_GRAFT_SKIPPED.
#include "plan.h"

namespace s4 {
namespace {

constexpr int kGraftThreads = 256;

template <bool kAdam>
__device__ __forceinline__ float graft_dir(const GraftArgs& a, float g, float& m, float& v) {
  if (!kAdam) return g;
  m = fmaf(a.beta1, m, a.omb1 * g);
  v = fmaf(a.beta2, v, a.omb2 * (g * g));
  return (m * a.c1) / (sqrtf(v * a.c2) + a.adam_eps);
}

__device__ __forceinline__ void block_sum2(double& x, double& y) {
  __shared__ double sx[kGraftThreads / 32], sy[kGraftThreads / 32];
  for (int o = 16; o > 0; o >>= 1) {
    x += __shfl_xor_sync(0xffffffffu, x, o);
    y += __shfl_xor_sync(0xffffffffu, y, o);
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { sx[w] = x; sy[w] = y; }
  __syncthreads();
  if (threadIdx.x == 0) {
    x = 0.0; y = 0.0;
    for (int i = 0; i < kGraftThreads / 32; ++i) { x += sx[i]; y += sy[i]; }
  }
}

// Moments and the item's partial sums; kReadD: D's sum of squares from D
// itself (else it was recorded by the apply and is added in k_graft_apply).
template <bool kAdam, bool kReadD>
__device__ __forceinline__ void graft_norms_item(const GraftArgs& a, const GraftItem& it, double& sg, double& sd) {
  {
    const PtrEntry eg = a.tabs[it.param], ed = a.tabs[a.nparams + it.param];
    const float* G = eg.ptr + it.r0 * eg.ld + it.c0;
    const float* D = ed.ptr + it.r0 * ed.ld + it.c0;
    float* M = kAdam ? a.state + it.m_off : nullptr;
    float* V = kAdam ? a.state + it.v_off : nullptr;
    const bool vec = ((reinterpret_cast<uintptr_t>(G) | reinterpret_cast<uintptr_t>(D) |
                       reinterpret_cast<uintptr_t>(M) | reinterpret_cast<uintptr_t>(V) |
                       uintptr_t(eg.ld * 4) | uintptr_t(ed.ld * 4) | uintptr_t(it.state_ld * 4)) & 15) == 0 &&
                     (it.cols & 3) == 0;
    if (vec) {
      const int c4n = it.cols >> 2;
      const int n4 = it.rows * c4n;
#pragma unroll 2
      for (int e = threadIdx.x; e < n4; e += kGraftThreads) {
        const int r = e / c4n, c = (e - r * c4n) * 4;
        const float4 g = *reinterpret_cast<const float4*>(G + r * eg.ld + c);
        const float4 d = kReadD ? *reinterpret_cast<const float4*>(D + r * ed.ld + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        float4 m = make_float4(0.f, 0.f, 0.f, 0.f), v = m;
        if (kAdam) {
          m = *reinterpret_cast<const float4*>(M + r * it.state_ld + c);
          v = *reinterpret_cast<const float4*>(V + r * it.state_ld + c);
        }
        const float q0 = graft_dir<kAdam>(a, g.x, m.x, v.x);
        const float q1 = graft_dir<kAdam>(a, g.y, m.y, v.y);
        const float q2 = graft_dir<kAdam>(a, g.z, m.z, v.z);
        const float q3 = graft_dir<kAdam>(a, g.w, m.w, v.w);
        if (kAdam) {
          *reinterpret_cast<float4*>(M + r * it.state_ld + c) = m;
          *reinterpret_cast<float4*>(V + r * it.state_ld + c) = v;
        }
        sg += double(q0) * q0 + double(q1) * q1 + double(q2) * q2 + double(q3) * q3;
        sd += double(d.x) * d.x + double(d.y) * d.y + double(d.z) * d.z + double(d.w) * d.w;
      }
    } else {
      for (int r = 0; r < it.rows; ++r)
        for (int c = threadIdx.x; c < it.cols; c += kGraftThreads) {
          const float g = G[r * eg.ld + c], d = kReadD ? D[r * ed.ld + c] : 0.0f;
          float m = 0.f, v = 0.f;
          if (kAdam) { m = M[r * it.state_ld + c]; v = V[r * it.state_ld + c]; }
          const float q = graft_dir<kAdam>(a, g, m, v);
          if (kAdam) { M[r * it.state_ld + c] = m; V[r * it.state_ld + c] = v; }
          sg += double(q) * q;
          sd += double(d) * d;
        }
    }
  }
}

template <bool kAdam>
__global__ void __launch_bounds__(kGraftThreads) k_graft_norms(const GraftArgs a) {
  const GraftItem it = a.items[blockIdx.x];
  double sg = 0.0, sd = 0.0;
  if (a.bflag[it.block] == 0u) {
    if (a.use_dsq && it.dsq_n > 0) graft_norms_item<kAdam, false>(a, it, sg, sd);
    else graft_norms_item<kAdam, true>(a, it, sg, sd);
  }
  block_sum2(sg, sd);
  if (threadIdx.x == 0) {
    a.parts[2 * int64_t(blockIdx.x)] = sg;
    a.parts[2 * int64_t(blockIdx.x) + 1] = sd;
  }
}

__global__ void __launch_bounds__(kGraftThreads) k_graft_apply(const GraftArgs a) {
  const GraftItem it = a.items[blockIdx.x];
  if (a.bflag[it.block] != 0u) return;
  __shared__ float s_r;
  __shared__ int s_ok;
  if (threadIdx.x == 0) {
    double sg = 0.0, sd = 0.0;
    for (int i = 0; i < it.nparts; ++i) {
      sg += a.parts[2 * int64_t(it.part0 + i)];
      sd += a.parts[2 * int64_t(it.part0 + i) + 1];
    }
    if (a.use_dsq && it.dsq_n > 0)                          // D's norm as the apply recorded it
      for (int i = 0; i < it.dsq_n; ++i) sd += a.dsq[it.dsq_off + i];
    const double den = sqrt(sd) + a.graft_eps;
    const double r = den > 0.0 ? a.lr * (sqrt(sg) / den) : 0.0;
    const float rf = float(r);
    const bool ok = isfinite(sg) && isfinite(sd) && isfinite(rf);
    if (!ok && int(blockIdx.x) == it.part0) atomicOr(a.flags, SHAMPOO4_FLAG_GRAFT_SKIPPED);
    s_r = rf;
    s_ok = ok && rf != 0.0f;
  }
  __syncthreads();
  if (!s_ok) return;
  const float nr = -s_r;
  const PtrEntry ed = a.tabs[a.nparams + it.param], ew = a.tabs[2 * a.nparams + it.param];
  const float* D = ed.ptr + it.r0 * ed.ld + it.c0;
  float* W = const_cast<float*>(ew.ptr) + it.r0 * ew.ld + it.c0;
  const bool vec = ((reinterpret_cast<uintptr_t>(D) | reinterpret_cast<uintptr_t>(W) | uintptr_t(ed.ld * 4) |
                     uintptr_t(ew.ld * 4)) & 15) == 0 && (it.cols & 3) == 0;
  if (vec) {
    const int c4n = it.cols >> 2;
    const int n4 = it.rows * c4n;
#pragma unroll 4
    for (int e = threadIdx.x; e < n4; e += kGraftThreads) {
      const int r = e / c4n, c = (e - r * c4n) * 4;
      const float4 d = *reinterpret_cast<const float4*>(D + r * ed.ld + c);
      float4* wp = reinterpret_cast<float4*>(W + r * ew.ld + c);
      float4 w = *wp;
      w.x = fmaf(nr, d.x, w.x);
      w.y = fmaf(nr, d.y, w.y);
      w.z = fmaf(nr, d.z, w.z);
      w.w = fmaf(nr, d.w, w.w);
      *wp = w;
    }
  } else {
    for (int r = 0; r < it.rows; ++r)
      for (int c = threadIdx.x; c < it.cols; c += kGraftThreads)
        W[r * ew.ld + c] = fmaf(nr, D[r * ed.ld + c], W[r * ew.ld + c]);
  }
}

}  // namespace

shampoo4_status launch_graft(const GraftArgs& a, cudaStream_t st) {
  if (a.nitems <= 0) return SHAMPOO4_OK;
  if (a.kind == kGraftAdam)
    k_graft_norms<true><<<a.nitems, kGraftThreads, 0, st>>>(a);
  else
    k_graft_norms<false><<<a.nitems, kGraftThreads, 0, st>>>(a);
  S4_CUDA(cudaGetLastError());
  k_graft_apply<<<a.nitems, kGraftThreads, 0, st>>>(a);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

}  // namespace s4
