// Allocation-free statistics update of one tile.
//
// shampoo4_update_stats_noalloc runs the EMA update of the two Kronecker
// statistics of a single gradient tile (the statistics stage of the
// "4-bit Shampoo for Memory-Efficient Network Training" algorithm, the
// L/R accumulation of Shampoo) without a handle, a workspace or any device
// allocation.  It is meant for callers that cannot allocate device memory
// at the point of the call: code that runs while a caching allocator holds
// its lock (a hook inside the allocator, a memory-pressure callback), or a
// process whose device memory is entirely reserved by another allocator, so
// that cudaMalloc -- directly or through a library -- would fail or deadlock.
//
// Scratch: one file-scope __device__ array (kNoallocScratchBytes, 1 MiB +
// 4 KiB, one instance per device), whose device address every call looks up
// with cudaGetSymbolAddress while the caller's device is current.  The
// lookup allocates nothing and is cheap once the module is loaded; doing it
// on every call (rather than caching it per device ordinal) keeps the
// address right when a context is torn down and created again, which can
// move the module.  It holds
//   - the launch descriptors and the gradient's pointer table, written on
//     the stream by a one-warp setup kernel at the start of every call;
//   - two flag words that must start every call at zero (the tile's
//     non-finite flag, which gates both products, and a status word used
//     when the caller passes no flag pointer); the setup kernel zeroes them;
//   - the TF32-rounded copy of the gradient (at most 2^18 elements), written
//     by the scan kernel and read by both products.
// Overlapping calls (on different streams, or from different host threads
// without ordering) share that scratch and race; calls must be ordered.
// The first call on a device may load the module, so it should come before
// any stream capture.
//
// The kernels are the library's own: the gradient scan that also writes the
// TF32 copy, and the CUDA-core fp32-output GEMM in TF32 mode (operands
// rounded to TF32, exact products, fp32 sums) with a symmetric output.
#include "plan.h"

namespace s4 {
namespace {

constexpr int kNoallocMaxEdge = 1024;                     // m, n
constexpr int64_t kNoallocMaxElems = int64_t(1) << 18;   // m * n (staged gradient copy)
constexpr size_t kNoallocHeaderBytes = 4096;
constexpr size_t kNoallocScratchBytes = kNoallocHeaderBytes + size_t(kNoallocMaxElems) * sizeof(float);

struct alignas(256) NoallocHeader {
  uint32_t flag;                // non-finite gradient: gates both products
  uint32_t status;              // status bits when the caller passes no flag word
  uint32_t pad_[2];
  PtrEntry tab;                 // pointer table: the gradient
  ScanDesc scan;
  GemmF32Desc gemm[2];          // L, R
};
static_assert(sizeof(NoallocHeader) <= kNoallocHeaderBytes, "header fits its slot");

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

// Copy the descriptors into scratch (zeroing the flag words with them).
__global__ void __launch_bounds__(32) k_noalloc_setup(const __grid_constant__ NoallocHeader h,
                                                      NoallocHeader* __restrict__ dst) {
  const uint32_t* src = reinterpret_cast<const uint32_t*>(&h);
  uint32_t* out = reinterpret_cast<uint32_t*>(dst);
  for (int i = threadIdx.x; i < int(sizeof(NoallocHeader) / 4); i += 32) out[i] = src[i];
}

// The scratch array's device address in the current device's context.  In
// host code g_noalloc_scratch names a host-side stand-in, never a device
// address: only this lookup gives one.
shampoo4_status noalloc_scratch(uint8_t** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p) return SHAMPOO4_ERR_CUDA;
  *out = static_cast<uint8_t*>(p);
  return SHAMPOO4_OK;
}

int tiles128_of(int M, int N) { return ((M + 127) / 128) * ((N + 127) / 128); }

}  // namespace
}  // namespace s4

using namespace s4;

extern "C" shampoo4_status shampoo4_update_stats_noalloc(float* d_L, float* d_R, const float* d_G, int32_t m,
                                                         int32_t n, int64_t ldg, float beta, uint32_t* d_flags,
                                                         shampoo4_stream_t stream) {
  if (!d_L || !d_R || !d_G || m < 1 || n < 1 || ldg < n) return SHAMPOO4_ERR_INVALID_ARG;
  if (!(beta >= 0.0f && beta < 1.0f)) return SHAMPOO4_ERR_INVALID_ARG;
  if (!aligned(d_L, 4) || !aligned(d_R, 4) || !aligned(d_G, 4) || (d_flags && !aligned(d_flags, 4)))
    return SHAMPOO4_ERR_INVALID_ARG;
  if (m > kNoallocMaxEdge || n > kNoallocMaxEdge || int64_t(m) * n > kNoallocMaxElems)
    return SHAMPOO4_ERR_WORKSPACE;                        // beyond the static scratch
  uint8_t* scratch = nullptr;
  S4_TRY(noalloc_scratch(&scratch));
  NoallocHeader* dh = reinterpret_cast<NoallocHeader*>(scratch);
  float* copy = reinterpret_cast<float*>(scratch + kNoallocHeaderBytes);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  NoallocHeader h{};
  h.flag = 0;
  h.status = 0;
  h.tab = {d_G, ldg};
  ScanDesc& s = h.scan;
  s.rows = m;
  s.cols = n;
  s.ref = {0, 0, 0, 0};
  s.flag = &dh->flag;
  s.bit = SHAMPOO4_FLAG_NONFINITE_GRAD;
  s.oh = copy;                                            // TF32 copy, dense, ld = n
  s.ol = nullptr;
  const float omb = 1.0f - beta;
  for (int side = 0; side < 2; ++side) {
    GemmF32Desc& x = h.gemm[side];
    const int d = side == 0 ? m : n;
    x.M = d; x.N = d; x.K = side == 0 ? n : m;
    x.ta = side == 0 ? 0 : 1;                             // L = G G^T, R = G^T G
    x.tb = side == 0 ? 1 : 0;
    x.mode = kModeTF32;
    x.symmetric = 1;
    x.alpha = omb;
    x.beta = beta;
    x.A = copy; x.lda = n;
    x.B = copy; x.ldb = n;
    x.C = side == 0 ? d_L : d_R; x.ldc = d;
    x.Cin = x.C; x.ldcin = d;
    x.kscale = nullptr;
    x.skip = &dh->flag;
    x.a_ref.tab = x.b_ref.tab = x.c_ref.tab = -1;
  }
  k_noalloc_setup<<<1, 32, 0, st>>>(h, dh);
  S4_CUDA(cudaGetLastError());
  S4_TRY(launch_scan(&dh->scan, 1, m, &dh->tab, 1, d_flags ? d_flags : &dh->status, st));
  S4_TRY(launch_gemm_f32(dh->gemm, 2, std::max(tiles128_of(m, m), tiles128_of(n, n)), &dh->tab, 1, st));
  return SHAMPOO4_OK;
}
