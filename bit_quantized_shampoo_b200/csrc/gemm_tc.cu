// Tensor-core batched GEMM for sm_100a: tcgen05.mma (kind::tf32) with the
// accumulator in tensor memory, operands staged in shared memory by TMA.
//
//   C = alpha * op(A) op(B) + beta * Cin        (one CTA per 128 x BN tile)
//
// Operands are fp32 matrices in global memory whose values are already
// TF32 numbers (the kernels that write them round to nearest), so the
// tensor core's use of the top 19 bits loses nothing.  In split mode each
// operand comes as a high and a low TF32 part and three products per K step
// (hi*hi + hi*lo + lo*hi) give fp32-accurate results.
//
// Shared memory tiles use the 128-byte swizzle.  An operand whose contraction
// index is contiguous in memory ("K-major") is loaded as one TMA box of
// 32 x rows; one whose row index is contiguous ("MN-major") as boxes of
// 32 x 32, one per 32 rows.  The MMA reads both forms through its matrix
// descriptors, so no operand is ever transposed.
//
// Warp roles (192 threads): warp 0 issues the TMA loads, warp 1 owns the
// tensor memory and issues the MMAs, warps 2..5 drain the accumulator
// (warp w reads TMEM lanes 32*(w%4) .. +31, one output row per thread).
// Every wait on an mbarrier is bounded in time.  The three waits of the
// pipeline (the producer's for a free stage, the MMA issuer's for a loaded
// one, the epilogue's for the finished accumulator) give up after a limit
// the host passes (2 s unless a diagnostic sets another); on expiry the CTA
// raises SHAMPOO4_FLAG_TIMEOUT and stops issuing.  Before it exits it still
// waits, with the 2 s limit, for everything it issued: the producer for its
// TMA loads, the MMA warp for its MMAs (before it frees tensor memory).
#include <cuda.h>
#include <cudaTypedefs.h>
#include "tc.h"

namespace s4 {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 32;                  // fp32 elements per row of a 128-byte swizzle atom
constexpr uint64_t kWaitNs = 2000000000ull;   // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// try_wait with an explicit bound on how long the hardware may suspend the
// thread inside the instruction (its suspendTimeHint, in ns).
__device__ __forceinline__ bool mbar_try_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
// Bounded wait: false after about limit_ns without the phase completing.
// try_wait may suspend the thread until the phase completes, so a limit
// below the 2 s default (a diagnostic) is also passed as the suspend hint:
// otherwise a short wait would simply be absorbed inside the instruction.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitNs) {
  if (limit_ns < kWaitNs) {
    const uint32_t hint = limit_ns < 1000000ull ? uint32_t(limit_ns) : 1000000u;
    const uint64_t t0 = now_ns();
    for (;;) {
      if (mbar_try_hint(bar, parity, hint)) return true;
      if (now_ns() - t0 > limit_ns) return false;
    }
  }
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  for (;;) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try(bar, parity)) return true;
    if (now_ns() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor, sm_100 version field.  layout: 2 =
// 128-byte swizzle (16-byte atoms), 1 = 128-byte swizzle with 32-byte atoms
// (the only swizzled form the MMA accepts for MN-major 32-bit operands).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= uint64_t((addr >> 4) & 0x3FFF);
  d |= uint64_t((lbo >> 4) & 0x3FFF) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFF) << 32;
  d |= uint64_t(1) << 46;                 // descriptor version for tcgen05
  d |= uint64_t(layout & 7) << 61;
  return d;
}

// Instruction descriptor: dense, fp32 accumulator, TF32 A and B.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 16-byte asynchronous copies global -> shared (cp.async groups).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ float rn_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

template <int BN, bool SPLIT, int STAGES>
struct TcCfg {
  static constexpr int kATile = kBM * kBK * 4;                  // bytes
  static constexpr int kBTile = BN * kBK * 4;
  static constexpr int kStage = (kATile + kBTile) * (SPLIT ? 2 : 1);
  static constexpr int kStages = STAGES;
  static constexpr int kSmem = kStage * kStages + 1024;         // + alignment slack
  // Epilogue staging, carved out of the pipeline buffers once the main loop
  // is over: per warp two Cin buffers and one transposing output buffer of
  // 32 rows, row pitch 36 floats (16-byte aligned rows, conflict-free
  // 16-byte accesses both by lane = row and by 8 lanes along a row).
  static constexpr int kPitch = 36;
  static constexpr int kRowBuf = 32 * kPitch * 4;
  static constexpr int kEpiWarp = 3 * kRowBuf;
  static_assert(4 * kEpiWarp <= kStage * kStages, "epilogue staging fits the pipeline buffers");
  // The tensor cores' fp32 accumulation truncates: a long sum drifts low
  // (about 1e-8 K relative when its terms share a sign) and its rounding
  // noise grows with the accumulator's magnitude.  The fp32-accurate
  // instances therefore keep kAcc accumulators, k-block kb going to
  // accumulator kb mod kAcc, and add them in the epilogue with
  // round-to-nearest: the drift drops kAcc-fold, the noise about
  // sqrt(kAcc)-fold.
  static constexpr int kAcc = SPLIT ? 4 : 1;
  static constexpr int kTmemCols = BN * kAcc;                   // 256 or 512: a power of two
};

// Issue the loads of one operand tile (rows mn0.. of the problem, K block k0).
__device__ __forceinline__ void load_operand(const CUtensorMap* map, const TcOperand& op, int rows, int mn0,
                                             int k0, uint32_t dst, uint64_t* bar) {
  if (!op.mn_major) {
    tma_load_2d(dst, map, op.col0 + k0, op.row0 + mn0, bar);          // box {32 (K), rows}
  } else {
    for (int g = 0; g < rows / 32; ++g)                                // boxes {32 (MN), 32 (K)}
      tma_load_2d(dst + g * 4096, map, op.col0 + mn0 + 32 * g, op.row0 + k0, bar);
  }
}

// The B operand of K block k0 of an output tile at column n0: as given, or,
// past the stored tiles of a symmetric operand (bt maps), its transpose
// read MN-major.
__device__ __forceinline__ bool b_transposed(const CUtensorMap* bt_hi, int k0, int n0, int bn) {
  return bt_hi != nullptr && k0 >= n0 + bn;
}
// The same for the A operand of an output tile at row m0: the stored tiles
// of the symmetric operand (width bn) cover K block k0 of rows m0.. when
// its bn-wide block starts below m0 + 128.
__device__ __forceinline__ bool a_transposed(const CUtensorMap* at_hi, int k0, int m0, int bn) {
  return at_hi != nullptr && (k0 / bn) * bn >= m0 + kBM;
}
// First K index read through the second operand pair (a2, b2), or one past
// any K when the product has none.
__device__ __forceinline__ int second_pair_k(const TcGemmDesc& g) { return g.a2.hi ? g.ksplit : 0x7fffffff; }

__device__ __forceinline__ uint64_t operand_desc(int mn_major, uint32_t base, int kk) {
  // K-major (128 B swizzle): rows of 128 B, 8-row groups 1024 B apart; a K
  // step of 8 is 32 B along the row.
  // MN-major (128 B swizzle, 32 B atoms): 32-wide MN groups 4096 B apart,
  // 4-row K groups 512 B apart; a K step of 8 rows is 1024 B.
  return mn_major ? smem_desc(base + kk * 1024, 4096, 512, 1) : smem_desc(base + kk * 32, 16, 1024, 2);
}

// Output fields of one problem, held in registers by the epilogue warps.
struct EpiArgs {
  int M, N, symmetric, out_round;
  float alpha, beta;
  float* C; int64_t ldc;
  float* Chi; float* Clo; int64_t ldh;
  const float* Cin; int64_t ldcin;
  double* sumsq;

  __device__ __forceinline__ void load(const TcGemmDesc& g, const PtrEntry* tabs, int nparams) {
    M = g.M; N = g.N; out_round = g.out_round;
    symmetric = g.symmetric == 3 ? 0 : g.symmetric;      // mode 3 writes its tiles in full
    alpha = g.alpha; beta = g.beta;
    C = g.C; ldc = g.ldc;
    if (g.c_ref.tab >= 0) {
      const PtrEntry& t = tabs[g.c_ref.tab * nparams + g.c_ref.param];
      ldc = t.ld;
      C = const_cast<float*>(t.ptr) + g.c_ref.r0 * t.ld + g.c_ref.c0;
    }
    Chi = g.Chi; Clo = g.Clo; ldh = g.ldh;
    Cin = g.Cin; ldcin = g.ldcin;
    sumsq = C ? g.sumsq : nullptr;
  }
  // Sum of squares of the C values of one lane's row segment (columns
  // cb .. cb + 31 below N; the symmetric triangle as written).  A full
  // segment of a plain product sums in fp32 (eight chains of four fused
  // multiply-adds, then pairwise: within 7 units of fp32 rounding of the
  // segment's sum), the rest in fp64.
  __device__ __forceinline__ double seg_sumsq(const float (&v)[32], int64_t row, int cb) const {
    if (cb + 32 <= N && !symmetric && !out_round) {
      float s[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) s[k] = v[k] * v[k];
#pragma unroll
      for (int j = 8; j < 32; j += 8)
#pragma unroll
        for (int k = 0; k < 8; ++k) s[k] = fmaf(v[j + k], v[j + k], s[k]);
      return double(((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7])));
    }
    double acc = 0.0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int c = cb + j;
      if (c < N && (!symmetric || c <= row)) {
        const double x = double(out_round ? rn_tf32(v[j]) : v[j]);
        acc = fma(x, x, acc);
      }
    }
    return acc;
  }
  // The warp's share of the tile's sum of squares into its slot.
  __device__ __forceinline__ void put_sumsq(double acc, int m0, int n0, int bn, int q, int lane) const {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    const int tiles_n = (N + bn - 1) / bn;
    if (lane == 0) sumsq[4 * ((m0 / 128) * tiles_n + n0 / bn) + q] = acc;
  }
  // One element to every requested output: C (optionally TF32-rounded) and
  // the TF32 split (Chi, Clo).
  __device__ __forceinline__ void put(int64_t r, int c, float v) const {
    if (C) C[r * ldc + c] = out_round ? rn_tf32(v) : v;
    if (Chi) {
      const float h = rn_tf32(v);
      Chi[r * ldh + c] = h;
      if (Clo) Clo[r * ldh + c] = rn_tf32(v - h);
    }
  }
  __device__ __forceinline__ void put4(int64_t r, int c, float a, float b, float x, float y) const {
    if (C) {
      const float4 o = out_round ? make_float4(rn_tf32(a), rn_tf32(b), rn_tf32(x), rn_tf32(y))
                                 : make_float4(a, b, x, y);
      *reinterpret_cast<float4*>(C + r * ldc + c) = o;
    }
    if (Chi) {
      const float4 h = make_float4(rn_tf32(a), rn_tf32(b), rn_tf32(x), rn_tf32(y));
      *reinterpret_cast<float4*>(Chi + r * ldh + c) = h;
      if (Clo)
        *reinterpret_cast<float4*>(Clo + r * ldh + c) =
            make_float4(rn_tf32(a - h.x), rn_tf32(b - h.y), rn_tf32(x - h.z), rn_tf32(y - h.w));
    }
  }
};

// Epilogue of one output tile (rows m0.., columns n0..) by an epilogue warp
// of TMEM lane quarter q, for the tile's 32-column chunks [i_lo, i_hi):
// reads the tile's accumulator(s) at TMEM column tacc, stages through this
// warp's staging rows wbuf (Cfg::kEpiWarp bytes), writes every requested
// output.
template <int BN, bool SPLIT, int STAGES>
__device__ __forceinline__ void epilogue_tile(const TcGemmDesc& g, const PtrEntry* __restrict__ tabs, int nparams,
                                              int m0, int n0, int kblocks, uint32_t tacc, int q, int lane,
                                              uint8_t* wbuf, int i_lo = 0, int i_hi = BN / 32) {
  using Cfg = TcCfg<BN, SPLIT, STAGES>;
  EpiArgs e;
  e.load(g, tabs, nparams);
  // Lane l of warp q holds accumulator row 32 q + l (TMEM lane), 32
  // columns per load.  When bases and leading dimensions are 16-byte
  // aligned, Cin comes in by 16-byte cp.async pieces (four full rows per
  // warp instruction, double-buffered in the staging rows) and the outputs
  // go out through a transposing staging row block, four full 128-byte
  // lines per store instruction; otherwise each lane loads and stores its
  // row directly.  The mirror of a symmetric product writes column
  // segments, contiguous across the lanes.
  const int rbase = m0 + 32 * q;
  const int row = rbase + lane;
  const int nacc = kblocks < Cfg::kAcc ? kblocks : Cfg::kAcc;   // accumulators written
  const bool row_ok = row < e.M;
  const int nrows = min(32, e.M - rbase);
  const int ncols = min(BN, e.N - n0);
  const int nchunks = ncols > 0 ? (ncols + 31) / 32 : 0;
  const int i_end = i_hi < nchunks ? i_hi : nchunks;
  const bool cin_bulk = e.beta != 0.0f &&
                        ((reinterpret_cast<uintptr_t>(e.Cin) | uintptr_t(e.ldcin * 4)) & 15) == 0 &&
                        (e.N & 3) == 0;
  const bool out_bulk = ((reinterpret_cast<uintptr_t>(e.C) | uintptr_t(e.ldc * 4) |
                          reinterpret_cast<uintptr_t>(e.Chi) | reinterpret_cast<uintptr_t>(e.Clo) |
                          uintptr_t(e.ldh * 4)) & 15) == 0 &&
                        (e.N & 3) == 0;
  const bool out_vec = out_bulk;                        // same alignment conditions
  const uint32_t wsm = smem_u32(wbuf);
  const uint32_t my_row = uint32_t(lane * Cfg::kPitch * 4);
  double ss_acc = 0.0;                                  // sum of squares of C (sumsq)
  // Cin chunk i into buffer i & 1 with 16-byte cp.async pieces, four
  // full 128-byte rows per warp instruction: lane l copies rows
  // 4 t + l / 8 (t < 8), columns 4 (l % 8).  One group per chunk.
  auto issue_cin = [&](int i) {
    const int cb = n0 + 32 * i, sr = lane >> 3, sc = 4 * (lane & 7);
    if (cb + sc < e.N) {
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int rr = 4 * t + sr;
        if (rbase + rr < e.M)
          cp_async16(wsm + (i & 1) * Cfg::kRowBuf + uint32_t((rr * Cfg::kPitch + sc) * 4),
                     e.Cin + int64_t(rbase + rr) * e.ldcin + cb + sc);
      }
    }
    cp_async_commit();
  };
  if (nrows > 0 && i_lo < i_end) {
    if (cin_bulk) issue_cin(i_lo);
#pragma unroll 1
    for (int i = i_lo; i < i_end; ++i) {
      const int c0 = 32 * i, cb = n0 + c0;
      if (cin_bulk && i + 1 < i_end) {
        __syncwarp();                                   // buffer (i + 1) & 1: chunk i - 1's reads done
        issue_cin(i + 1);
      }
      uint32_t r[32];
      tmem_ld32(tacc + (uint32_t(32 * q) << 16) + uint32_t(c0), r);
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
      for (int a = 1; a < nacc; ++a) {                  // the other accumulators, added with RN
        tmem_ld32(tacc + (uint32_t(32 * q) << 16) + uint32_t(a * BN + c0), r);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += __uint_as_float(r[j]);
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= e.alpha;
      if (e.beta != 0.0f) {
        if (cin_bulk) {
          if (i + 1 < i_end) cp_async_wait<1>(); else cp_async_wait<0>();
          __syncwarp();                                 // every lane's pieces of chunk i visible
          if (row_ok) {
            const float4* src = reinterpret_cast<const float4*>(wbuf + (i & 1) * Cfg::kRowBuf + my_row);
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              if (cb + 4 * t >= e.N) break;
              const float4 x = src[t];
              v[4 * t + 0] = fmaf(e.beta, x.x, v[4 * t + 0]);
              v[4 * t + 1] = fmaf(e.beta, x.y, v[4 * t + 1]);
              v[4 * t + 2] = fmaf(e.beta, x.z, v[4 * t + 2]);
              v[4 * t + 3] = fmaf(e.beta, x.w, v[4 * t + 3]);
            }
          }
        } else if (row_ok) {
          const float* src = e.Cin + int64_t(row) * e.ldcin + cb;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (cb + j < e.N) v[j] = fmaf(e.beta, __ldg(src + j), v[j]);
        }
      }
      if (e.sumsq && row_ok) ss_acc += e.seg_sumsq(v, row, cb);
      // row segment: columns cb.. of this lane's row (only col <= row
      // when the product is symmetric)
      const bool below = !e.symmetric || cb + 31 < rbase;   // whole chunk left of every row
      if (out_bulk && below) {
        // Through this warp's staging rows: each lane writes its row
        // segment as 16-byte pieces, then every store instruction takes
        // 4 rows x 128 bytes (lane l: row 4 i + l / 8, columns 4 (l % 8)).
        float* stage = reinterpret_cast<float*>(wbuf + 2 * Cfg::kRowBuf);
        const int sr = lane >> 3, sc = 4 * (lane & 7);
        const bool col_ok = cb + sc < e.N;
#pragma unroll 1
        for (int o = 0; o < 3; ++o) {
          float* out = o == 0 ? e.C : (o == 1 ? e.Chi : e.Clo);
          if (!out) continue;                             // warp-uniform
          const int64_t ld = o == 0 ? e.ldc : e.ldh;
          __syncwarp();                                   // previous output's reads done
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            float4 x = make_float4(v[4 * t], v[4 * t + 1], v[4 * t + 2], v[4 * t + 3]);
            if (o == 1 || (o == 0 && e.out_round)) {
              x = make_float4(rn_tf32(x.x), rn_tf32(x.y), rn_tf32(x.z), rn_tf32(x.w));
            } else if (o == 2) {
              x = make_float4(rn_tf32(x.x - rn_tf32(x.x)), rn_tf32(x.y - rn_tf32(x.y)),
                              rn_tf32(x.z - rn_tf32(x.z)), rn_tf32(x.w - rn_tf32(x.w)));
            }
            *reinterpret_cast<float4*>(stage + lane * Cfg::kPitch + 4 * t) = x;
          }
          __syncwarp();
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int rr = 4 * t + sr;
            if (rbase + rr < e.M && col_ok)
              *reinterpret_cast<float4*>(out + int64_t(rbase + rr) * ld + cb + sc) =
                  *reinterpret_cast<const float4*>(stage + rr * Cfg::kPitch + sc);
          }
        }
        __syncwarp();
      } else if (row_ok) {
        if (out_vec) {
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int c = cb + 4 * t;
            if (c >= e.N) break;
            if (!e.symmetric || c + 3 <= row) {
              e.put4(int64_t(row), c, v[4 * t + 0], v[4 * t + 1], v[4 * t + 2], v[4 * t + 3]);
            } else {
#pragma unroll
              for (int u = 0; u < 4; ++u)
                if (c + u <= row) e.put(int64_t(row), c + u, v[4 * t + u]);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int c = cb + j;
            if (c < e.N && (!e.symmetric || c <= row)) e.put(int64_t(row), c, v[j]);
          }
        }
      }
      // mirror of the strictly-lower part: element (row, c) also at (c, row)
      if (e.symmetric == 1 && cb < rbase + 32) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int c = cb + j;
          if (row_ok && c < e.N && c < row) e.put(int64_t(c), row, v[j]);
        }
      }
    }
    cp_async_wait<0>();                                 // nothing in flight into the buffers
  }
  if (e.sumsq && i_lo == 0) e.put_sumsq(ss_acc, m0, n0, BN, q, lane);   // every warp of the tile, once
}

template <int BN, bool SPLIT, int STAGES>
__global__ void __launch_bounds__(192, STAGES <= 2 ? 2 : 1)
k_gemm_tc(const TcGemmDesc* __restrict__ descs, const PtrEntry* __restrict__ tabs, int nparams,
          uint32_t* __restrict__ gflags, uint64_t wait_ns, const uint32_t* __restrict__ guard) {
  using Cfg = TcCfg<BN, SPLIT, STAGES>;
  if (guard && *guard == 0u) return;                      // no problem of the launch runs
  const TcGemmDesc& g = descs[blockIdx.y];
  const int tiles_n = (g.N + BN - 1) / BN;
  const int tiles_m = (g.M + kBM - 1) / kBM;
  if (int(blockIdx.x) >= tiles_m * tiles_n) return;
  const int tm = blockIdx.x / tiles_n, tn = blockIdx.x % tiles_n;
  const int m0 = tm * kBM, n0 = tn * BN;
  if (g.symmetric && n0 >= m0 + kBM) return;             // wholly above the diagonal
  if (g.skip && *g.skip) return;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full_bar[Cfg::kStages], empty_bar[Cfg::kStages], done_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&done_bar, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                 "r"(Cfg::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = tmem_slot;
  const int kblocks = (g.K + kBK - 1) / kBK;

  if (warp == 0) {
    if (lane == 0) {                                        // ---- TMA producer
      // Register copies: after every asm statement with a "memory" clobber a
      // field read through `g` would be fetched from global memory again,
      // several hundred cycles on the path of each issue.
      const TcOperand ga = g.a, gb = g.b;
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(ga.hi)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(gb.hi)) : "memory");
      if (SPLIT) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(ga.lo)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(gb.lo)) : "memory");
      }
      const CUtensorMap* bt_hi = g.bt_hi;
      const CUtensorMap* bt_lo = g.bt_lo;
      TcOperand gt = gb;                                    // transposed reads of B
      gt.hi = bt_hi; gt.lo = bt_lo; gt.mn_major = 1;
      const CUtensorMap* at_hi = g.at_hi;
      TcOperand gat = ga;                                   // transposed reads of A
      gat.hi = at_hi; gat.lo = g.at_lo; gat.mn_major = 1;
      const int ks = second_pair_k(g);
      const TcOperand ga2 = g.a2, gb2 = g.b2;
      int issued = 0;
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % Cfg::kStages;
        if (kb >= Cfg::kStages && !mbar_wait(&empty_bar[s], ((kb / Cfg::kStages) - 1) & 1, wait_ns)) {
          atomicOr(gflags, SHAMPOO4_FLAG_TIMEOUT);
          abort_flag = 1;
          break;
        }
        if (*(volatile int*)&abort_flag) break;
        const uint32_t st = smem_u32(smem + s * Cfg::kStage);
        mbar_expect_tx(&full_bar[s], Cfg::kStage);
        const int k0 = kb * kBK;
        const bool sec = k0 >= ks;
        const int kc = sec ? k0 - ks : k0;
        TcOperand oa = a_transposed(at_hi, k0, m0, BN) ? gat : ga;   // by value: stays in registers
        TcOperand ob = b_transposed(bt_hi, k0, n0, BN) ? gt : gb;
        if (sec) { oa = ga2; ob = gb2; }
        load_operand(oa.hi, oa, kBM, m0, kc, st, &full_bar[s]);
        load_operand(ob.hi, ob, BN, n0, kc, st + Cfg::kATile, &full_bar[s]);
        if (SPLIT) {
          load_operand(oa.lo, oa, kBM, m0, kc, st + Cfg::kATile + Cfg::kBTile, &full_bar[s]);
          load_operand(ob.lo, ob, BN, n0, kc, st + 2 * Cfg::kATile + Cfg::kBTile, &full_bar[s]);
        }
        issued = kb + 1;
      }
      // Whatever happened, the loads issued last must land before the CTA
      // exits: wait for the final phases of the live stages (the 2 s limit,
      // whatever limit the pipeline waits had).  Every earlier load was
      // consumed by an MMA before its stage was refilled.
      for (int kb = issued - Cfg::kStages < 0 ? 0 : issued - Cfg::kStages; kb < issued; ++kb)
        if (!mbar_wait(&full_bar[kb % Cfg::kStages], (kb / Cfg::kStages) & 1, kWaitNs))
          atomicOr(gflags, SHAMPOO4_FLAG_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {                                        // ---- MMA issuer
      // register copies, as in the producer; the MMA needs only each K
      // block's operand layouts
      const CUtensorMap* bt_hi = g.bt_hi;
      const CUtensorMap* at_hi = g.at_hi;
      const int ks = second_pair_k(g);
      const TcOperand ga = g.a, gb = g.b, ga2 = g.a2, gb2 = g.b2;
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % Cfg::kStages;
        if (!mbar_wait(&full_bar[s], (kb / Cfg::kStages) & 1, wait_ns)) {
          atomicOr(gflags, SHAMPOO4_FLAG_TIMEOUT);
          abort_flag = 1;
          break;
        }
        if (*(volatile int*)&abort_flag) break;
        fence_after_sync();
        const uint32_t st = smem_u32(smem + s * Cfg::kStage);
        const uint32_t a_hi = st, b_hi = st + Cfg::kATile;
        const uint32_t a_lo = st + Cfg::kATile + Cfg::kBTile, b_lo = a_lo + Cfg::kATile;
        const bool sec = kb * kBK >= ks;
        const int amn = sec ? ga2.mn_major : (a_transposed(at_hi, kb * kBK, m0, BN) ? 1 : ga.mn_major);
        const int bmn = sec ? gb2.mn_major : (b_transposed(bt_hi, kb * kBK, n0, BN) ? 1 : gb.mn_major);
        const uint32_t idesc = idesc_tf32(kBM, BN, amn, bmn);
#pragma unroll
        for (int kk = 0; kk < kBK / 8; ++kk) {
          // first MMA into accumulator kb mod kAcc overwrites it
          const uint32_t acc = (kb >= Cfg::kAcc || kk != 0) ? 1u : 0u;
          const uint32_t dt = tmem + uint32_t((kb % Cfg::kAcc) * BN);
          mma_tf32(dt, operand_desc(amn, a_hi, kk), operand_desc(bmn, b_hi, kk), idesc, acc);
          if (SPLIT) {
            mma_tf32(dt, operand_desc(amn, a_hi, kk), operand_desc(bmn, b_lo, kk), idesc, 1);
            mma_tf32(dt, operand_desc(amn, a_lo, kk), operand_desc(bmn, b_hi, kk), idesc, 1);
          }
        }
        mma_commit(&empty_bar[s]);                          // stage free once these MMAs finish
      }
      mma_commit(&done_bar);                                // accumulator complete
      // every MMA this thread issued completes before tensor memory is
      // freed below, even when the epilogue gave up waiting for them
      if (!mbar_wait(&done_bar, 0, kWaitNs)) atomicOr(gflags, SHAMPOO4_FLAG_TIMEOUT);
    }
  } else {                                                  // ---- epilogue, warps 2..5
    const int q = warp & 3;                                 // TMEM lane quarter = 32-row slab
    const bool ok = mbar_wait(&done_bar, 0, wait_ns);
    if (!ok) atomicOr(gflags, SHAMPOO4_FLAG_TIMEOUT);
    fence_after_sync();
    if (ok && !*(volatile int*)&abort_flag) {
      epilogue_tile<BN, SPLIT, STAGES>(g, tabs, nparams, m0, n0, kblocks, tmem, q, lane, smem + q * Cfg::kEpiWarp);
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(Cfg::kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// Persistent form (the fp32-accurate 128-wide instance).  One CTA per SM
// walks the batch's running tiles (tile t, t + gridDim.x, ...).  The
// operand ring runs on across tiles, so the next tile's loads start while
// this one's MMAs finish.  The epilogue reads a finished tile's four
// accumulators into registers (each lane one row of 128 columns, the
// partial sums added with round-to-nearest), hands tensor memory back to
// the MMA warp at once, and writes the outputs from registers while the
// next tile's main loop runs.  Each epilogue warp has one staging block of
// 32 rows, used in turn for the Cin chunk and for the transposed output
// rows.
template <int BN, bool SPLIT, int STAGES>
struct PersCfg {
  using Base = TcCfg<BN, SPLIT, STAGES>;
  static constexpr int kPitch = 36;
  static constexpr int kRowBuf = 32 * kPitch * 4;       // one staging block per epilogue warp
  static constexpr int kSmem = Base::kStage * STAGES + 4 * kRowBuf + 1024;
  static_assert(kSmem <= 227 * 1024, "persistent GEMM fits in shared memory");
};

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__host__ __device__ __forceinline__ int tiles_in_row(int symmetric, int N, int bn, int tm) {
  const int tiles_n = (N + bn - 1) / bn;
  if (!symmetric) return tiles_n;
  const int c = ((tm + 1) * kBM + bn - 1) / bn;            // tn * bn < (tm + 1) * kBM
  return c < tiles_n ? c : tiles_n;
}

// Running tile t of the batch (tc_assign_tiles numbered them): problem p
// (a cursor that only moves forward, as t does), tile origin (m0, n0);
// false when the problem is skipped.  Every role walks the same tiles.
// With the batch's tile list the lookup is one load; without it the cursor
// walks the problems, one dependent load per problem passed, which on a
// batch of many small problems costs microseconds per tile.
template <int BN>
__device__ __forceinline__ bool pers_tile(const TcGemmDesc* __restrict__ descs, int count,
                                          const uint64_t* __restrict__ list, int64_t t, int& p, int& m0, int& n0) {
  if (list) {
    const uint64_t e = list[t];
    p = int(uint32_t(e));
    m0 = int((e >> 32) & 0xffffu) * kBM;
    n0 = int(e >> 48) * BN;
    const uint32_t* skip = descs[p].skip;
    return !(skip && *skip);
  }
  while (p + 1 < count && descs[p + 1].tile_begin <= t) ++p;
  const TcGemmDesc& g = descs[p];
  int x = int(t - g.tile_begin);
  const int tiles_m = (g.M + kBM - 1) / kBM;
  int tm = 0;
  for (; tm < tiles_m; ++tm) {
    const int c = tiles_in_row(g.symmetric, g.N, BN, tm);
    if (x < c) break;
    x -= c;
  }
  m0 = tm * kBM;
  n0 = x * BN;
  return !(g.skip && *g.skip);
}

// Outputs of one tile from the accumulator values in registers (lane l of
// epilogue warp q holds row m0 + 32 q + l, columns n0 + 32 i + j in
// v[i][j]).  Same outputs and rounding as epilogue_tile, except the sum of
// squares (sumsq), which only the one-tile-per-CTA kernels record: in this
// epilogue, at the register limit, it cost the QR solve products 8%.
template <int BN>
__device__ __forceinline__ void epilogue_regs(const TcGemmDesc& g, const PtrEntry* __restrict__ tabs, int nparams,
                                              int m0, int n0, float (&v)[BN / 32][32], int q, int lane,
                                              uint8_t* wbuf) {
  constexpr int kPitch = 36, kChunks = BN / 32;
  EpiArgs e;
  e.load(g, tabs, nparams);
  const int rbase = m0 + 32 * q;
  const int row = rbase + lane;
  const bool row_ok = row < e.M;
  const int nrows = min(32, e.M - rbase);
  const int ncols = min(BN, e.N - n0);
  const int nchunks = ncols > 0 ? (ncols + 31) / 32 : 0;
  if (nrows <= 0) return;
  const bool cin_bulk = e.beta != 0.0f &&
                        ((reinterpret_cast<uintptr_t>(e.Cin) | uintptr_t(e.ldcin * 4)) & 15) == 0 &&
                        (e.N & 3) == 0;
  const bool out_bulk = ((reinterpret_cast<uintptr_t>(e.C) | uintptr_t(e.ldc * 4) |
                          reinterpret_cast<uintptr_t>(e.Chi) | reinterpret_cast<uintptr_t>(e.Clo) |
                          uintptr_t(e.ldh * 4)) & 15) == 0 &&
                        (e.N & 3) == 0;
  const uint32_t wsm = smem_u32(wbuf);
  float* stage = reinterpret_cast<float*>(wbuf);
  const int sr = lane >> 3, sc = 4 * (lane & 7);
#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    if (i >= nchunks) break;
    const int cb = n0 + 32 * i;
#pragma unroll
    for (int j = 0; j < 32; ++j) v[i][j] *= e.alpha;
    if (e.beta != 0.0f) {
      if (cin_bulk) {
        // Cin chunk into the staging block, 4 full 128-byte rows per warp
        // instruction (lane l: rows 4 t + l / 8, columns 4 (l % 8))
        __syncwarp();                                   // previous reads of the block done
        if (cb + sc < e.N) {
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int rr = 4 * t + sr;
            if (rbase + rr < e.M)
              cp_async16(wsm + uint32_t((rr * kPitch + sc) * 4), e.Cin + int64_t(rbase + rr) * e.ldcin + cb + sc);
          }
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncwarp();
        if (row_ok) {
          const float4* src = reinterpret_cast<const float4*>(stage + lane * kPitch);
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            if (cb + 4 * t < e.N) {
              const float4 x = src[t];
              v[i][4 * t + 0] = fmaf(e.beta, x.x, v[i][4 * t + 0]);
              v[i][4 * t + 1] = fmaf(e.beta, x.y, v[i][4 * t + 1]);
              v[i][4 * t + 2] = fmaf(e.beta, x.z, v[i][4 * t + 2]);
              v[i][4 * t + 3] = fmaf(e.beta, x.w, v[i][4 * t + 3]);
            }
          }
        }
      } else if (row_ok) {
        const float* src = e.Cin + int64_t(row) * e.ldcin + cb;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (cb + j < e.N) v[i][j] = fmaf(e.beta, __ldg(src + j), v[i][j]);
      }
    }
    const bool below = !e.symmetric || cb + 31 < rbase;   // whole chunk left of every row
    if (out_bulk && below) {
      const bool col_ok = cb + sc < e.N;
#pragma unroll 1
      for (int o = 0; o < 3; ++o) {
        float* out = o == 0 ? e.C : (o == 1 ? e.Chi : e.Clo);
        if (!out) continue;                             // warp-uniform
        const int64_t ld = o == 0 ? e.ldc : e.ldh;
        __syncwarp();                                   // previous reads of the block done
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          float4 x = make_float4(v[i][4 * t], v[i][4 * t + 1], v[i][4 * t + 2], v[i][4 * t + 3]);
          if (o == 1 || (o == 0 && e.out_round)) {
            x = make_float4(rn_tf32(x.x), rn_tf32(x.y), rn_tf32(x.z), rn_tf32(x.w));
          } else if (o == 2) {
            x = make_float4(rn_tf32(x.x - rn_tf32(x.x)), rn_tf32(x.y - rn_tf32(x.y)),
                            rn_tf32(x.z - rn_tf32(x.z)), rn_tf32(x.w - rn_tf32(x.w)));
          }
          *reinterpret_cast<float4*>(stage + lane * kPitch + 4 * t) = x;
        }
        __syncwarp();
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int rr = 4 * t + sr;
          if (rbase + rr < e.M && col_ok)
            *reinterpret_cast<float4*>(out + int64_t(rbase + rr) * ld + cb + sc) =
                *reinterpret_cast<const float4*>(stage + rr * kPitch + sc);
        }
      }
    } else if (row_ok) {
      if (out_bulk) {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int c = cb + 4 * t;
          if (c >= e.N) break;
          if (!e.symmetric || c + 3 <= row) {
            e.put4(int64_t(row), c, v[i][4 * t + 0], v[i][4 * t + 1], v[i][4 * t + 2], v[i][4 * t + 3]);
          } else {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (c + u <= row) e.put(int64_t(row), c + u, v[i][4 * t + u]);
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int c = cb + j;
          if (c < e.N && (!e.symmetric || c <= row)) e.put(int64_t(row), c, v[i][j]);
        }
      }
    }
    if (e.symmetric == 1 && cb < rbase + 32) {          // mirror of the strictly-lower part
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int c = cb + j;
        if (row_ok && c < e.N && c < row) e.put(int64_t(c), row, v[i][j]);
      }
    }
  }
  __syncwarp();                                         // the block is free for the next tile
}

template <int BN, bool SPLIT, int STAGES>
__global__ void __launch_bounds__(192, 1)
k_gemm_tc_pers(const TcGemmDesc* __restrict__ descs, int count, int64_t total, const PtrEntry* __restrict__ tabs,
               int nparams, uint32_t* __restrict__ gflags, uint64_t wait_ns, const uint32_t* __restrict__ guard,
               const uint64_t* __restrict__ tile_list) {
  using Cfg = TcCfg<BN, SPLIT, STAGES>;
  if (guard && *guard == 0u) return;                      // no problem of the launch runs
  using PCfg = PersCfg<BN, SPLIT, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + Cfg::kStage * STAGES;
  __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES], acc_full, acc_empty;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_full, 1);
    mbar_init(&acc_empty, 4);                           // one arrival per epilogue warp
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                 "r"(Cfg::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = tmem_slot;
  int p = 0;                                                // each role's problem cursor

  if (warp == 0) {
    if (lane == 0) {                                        // ---- TMA producer
      uint32_t it = 0;                                      // k-blocks issued, over all tiles
      int last_p = -1;
      for (int64_t t = blockIdx.x; t < total && !*(volatile int*)&abort_flag; t += gridDim.x) {
        int m0, n0;
        if (!pers_tile<BN>(descs, count, tile_list, t, p, m0, n0)) continue;
        const TcOperand ga = descs[p].a, gb = descs[p].b;   // registers (see k_gemm_tc)
        const CUtensorMap* bt_hi = descs[p].bt_hi;
        TcOperand gt = gb;                                  // transposed reads of B
        gt.hi = bt_hi; gt.lo = descs[p].bt_lo; gt.mn_major = 1;
        const CUtensorMap* at_hi = descs[p].at_hi;
        TcOperand gat = ga;                                 // transposed reads of A
        gat.hi = at_hi; gat.lo = descs[p].at_lo; gat.mn_major = 1;
        const int ks = second_pair_k(descs[p]);
        const TcOperand ga2 = descs[p].a2, gb2 = descs[p].b2;
        const int kblocks = (descs[p].K + kBK - 1) / kBK;
        if (p != last_p) {
          asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(ga.hi)) : "memory");
          asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(gb.hi)) : "memory");
          if (SPLIT) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(ga.lo)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(gb.lo)) : "memory");
          }
          last_p = p;
        }
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % STAGES;
          if (it >= STAGES && !mbar_wait(&empty_bar[s], ((it / STAGES) - 1) & 1, wait_ns)) {
            atomicOr(gflags, SHAMPOO4_FLAG_TIMEOUT);
            abort_flag = 1;
            break;
          }
          if (*(volatile int*)&abort_flag) break;
          const uint32_t st = smem_u32(smem + s * Cfg::kStage);
          mbar_expect_tx(&full_bar[s], Cfg::kStage);
          const int k0 = kb * kBK;
          const bool sec = k0 >= ks;
          const int kc = sec ? k0 - ks : k0;
          TcOperand oa = a_transposed(at_hi, k0, m0, BN) ? gat : ga;   // by value: stays in registers
          TcOperand ob = b_transposed(bt_hi, k0, n0, BN) ? gt : gb;
          if (sec) { oa = ga2; ob = gb2; }
          load_operand(oa.hi, oa, kBM, m0, kc, st, &full_bar[s]);
          load_operand(ob.hi, ob, BN, n0, kc, st + Cfg::kATile, &full_bar[s]);
          if (SPLIT) {
            load_operand(oa.lo, oa, kBM, m0, kc, st + Cfg::kATile + Cfg::kBTile, &full_bar[s]);
            load_operand(ob.lo, ob, BN, n0, kc, st + 2 * Cfg::kATile + Cfg::kBTile, &full_bar[s]);
          }
        }
      }
      // the loads issued last land before the CTA exits (earlier ones were
      // consumed by MMAs before their stages were refilled)
      for (uint32_t k = it > uint32_t(STAGES) ? it - STAGES : 0; k < it; ++k)
        if (!mbar_wait(&full_bar[k % STAGES], (k / STAGES) & 1, kWaitNs)) atomicOr(gflags, SHAMPOO4_FLAG_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {                                        // ---- MMA issuer
      uint32_t it = 0, ntiles = 0;
      for (int64_t t = blockIdx.x; t < total && !*(volatile int*)&abort_flag; t += gridDim.x) {
        int m0, n0;
        if (!pers_tile<BN>(descs, count, tile_list, t, p, m0, n0)) continue;
        const CUtensorMap* bt_hi = descs[p].bt_hi;
        const CUtensorMap* at_hi = descs[p].at_hi;
        const int ks = second_pair_k(descs[p]);
        const TcOperand ga = descs[p].a, gb = descs[p].b, ga2 = descs[p].a2, gb2 = descs[p].b2;
        const int kblocks = (descs[p].K + kBK - 1) / kBK;
        // the epilogue has read the previous tile's accumulators
        if (ntiles > 0 && !mbar_wait(&acc_empty, (ntiles - 1) & 1, wait_ns)) {
          atomicOr(gflags, SHAMPOO4_FLAG_TIMEOUT);
          abort_flag = 1;
          break;
        }
        fence_after_sync();
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&full_bar[s], (it / STAGES) & 1, wait_ns)) {
            atomicOr(gflags, SHAMPOO4_FLAG_TIMEOUT);
            abort_flag = 1;
            ok = false;
            break;
          }
          if (*(volatile int*)&abort_flag) { ok = false; break; }
          fence_after_sync();
          const uint32_t st = smem_u32(smem + s * Cfg::kStage);
          const uint32_t a_hi = st, b_hi = st + Cfg::kATile;
          const uint32_t a_lo = st + Cfg::kATile + Cfg::kBTile, b_lo = a_lo + Cfg::kATile;
          const bool sec = kb * kBK >= ks;
          const int amn = sec ? ga2.mn_major : (a_transposed(at_hi, kb * kBK, m0, BN) ? 1 : ga.mn_major);
          const int bmn = sec ? gb2.mn_major : (b_transposed(bt_hi, kb * kBK, n0, BN) ? 1 : gb.mn_major);
          const uint32_t idesc = idesc_tf32(kBM, BN, amn, bmn);
#pragma unroll
          for (int kk = 0; kk < kBK / 8; ++kk) {
            const uint32_t acc = (kb >= Cfg::kAcc || kk != 0) ? 1u : 0u;
            const uint32_t dt = tmem + uint32_t((kb % Cfg::kAcc) * BN);
            mma_tf32(dt, operand_desc(amn, a_hi, kk), operand_desc(bmn, b_hi, kk), idesc, acc);
            if (SPLIT) {
              mma_tf32(dt, operand_desc(amn, a_hi, kk), operand_desc(bmn, b_lo, kk), idesc, 1);
              mma_tf32(dt, operand_desc(amn, a_lo, kk), operand_desc(bmn, b_hi, kk), idesc, 1);
            }
          }
          mma_commit(&empty_bar[s]);
        }
        mma_commit(&acc_full);                              // this tile's accumulators complete
        ++ntiles;
        if (!ok) break;
      }
      // every MMA issued completes before tensor memory is freed
      if (ntiles > 0 && !mbar_wait(&acc_full, (ntiles - 1) & 1, kWaitNs)) atomicOr(gflags, SHAMPOO4_FLAG_TIMEOUT);
    }
  } else {                                                  // ---- epilogue, warps 2..5
    const int q = warp & 3;
    uint8_t* wbuf = staging + q * PCfg::kRowBuf;
    uint32_t ntiles = 0;
    for (int64_t t = blockIdx.x; t < total; t += gridDim.x) {
      int m0, n0;
      if (!pers_tile<BN>(descs, count, tile_list, t, p, m0, n0)) continue;
      const bool ok = mbar_wait(&acc_full, ntiles & 1, wait_ns);
      if (!ok) atomicOr(gflags, SHAMPOO4_FLAG_TIMEOUT);
      if (!ok || *(volatile int*)&abort_flag) break;
      fence_after_sync();
      const int kblocks = (descs[p].K + kBK - 1) / kBK;
      const int nacc = kblocks < Cfg::kAcc ? kblocks : Cfg::kAcc;
      float v[BN / 32][32];
#pragma unroll
      for (int i = 0; i < BN / 32; ++i) {
        uint32_t r[32];
        tmem_ld32(tmem + (uint32_t(32 * q) << 16) + uint32_t(32 * i), r);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[i][j] = __uint_as_float(r[j]);
        for (int a = 1; a < nacc; ++a) {                    // the other accumulators, added with RN
          tmem_ld32(tmem + (uint32_t(32 * q) << 16) + uint32_t(a * BN + 32 * i), r);
#pragma unroll
          for (int j = 0; j < 32; ++j) v[i][j] += __uint_as_float(r[j]);
        }
      }
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty);               // tensor memory free for the next tile
      ++ntiles;
      epilogue_regs<BN>(descs[p], tabs, nparams, m0, n0, v, q, lane, wbuf);
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(Cfg::kTmemCols)
                 : "memory");
  }
}

template <int BN, bool SPLIT, int STAGES>
shampoo4_status launch_tc_pers(const TcGemmDesc* d_desc, int count, int64_t total, const PtrEntry* tabs,
                               int nparams, uint32_t* gflags, uint64_t wait_ns, cudaStream_t st,
                               const uint32_t* guard, const uint64_t* tile_list) {
  using PCfg = PersCfg<BN, SPLIT, STAGES>;
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    S4_CUDA(cudaGetDevice(&dev));
    S4_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    S4_CUDA(cudaFuncSetAttribute(k_gemm_tc_pers<BN, SPLIT, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 PCfg::kSmem));
  }
  if (total <= 0) return SHAMPOO4_OK;
  const int grid = int(total < sms ? total : sms);
  k_gemm_tc_pers<BN, SPLIT, STAGES><<<grid, 192, PCfg::kSmem, st>>>(d_desc, count, total, tabs, nparams, gflags,
                                                                     wait_ns, guard, tile_list);
  S4_CUDA(cudaGetLastError());
  return SHAMPOO4_OK;
}

template <int BN, bool SPLIT, int STAGES>
shampoo4_status launch_tc_impl(const TcGemmDesc* d_desc, int count, int max_tiles, const PtrEntry* tabs,
                               int nparams, uint32_t* gflags, uint64_t wait_ns, cudaStream_t st,
                               const uint32_t* guard) {
  using Cfg = TcCfg<BN, SPLIT, STAGES>;
  static bool configured = false;
  if (!configured) {
    S4_CUDA(cudaFuncSetAttribute(k_gemm_tc<BN, SPLIT, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg::kSmem));
    configured = true;
  }
  for (int base = 0; base < count; base += 65535) {
    const int c = count - base < 65535 ? count - base : 65535;
    k_gemm_tc<BN, SPLIT, STAGES><<<dim3(unsigned(max_tiles), unsigned(c)), 192, Cfg::kSmem, st>>>(
        d_desc + base, tabs, nparams, gflags, wait_ns, guard);
    S4_CUDA(cudaGetLastError());
  }
  return SHAMPOO4_OK;
}

}  // namespace

int tc_block_n(int split) { return split ? 128 : 256; }

// The 128-wide fp32-accurate instance runs in its persistent form (0: one
// tile per CTA, for comparisons).
int tc_persistent = 1;

int tc_tiles_in_row(const TcGemmDesc& g, int bn, int tm) { return tiles_in_row(g.symmetric, g.N, bn, tm); }

int64_t tc_assign_tiles(TcGemmDesc* v, int count, int bn, std::vector<uint64_t>* list) {
  int64_t total = 0;
  for (int i = 0; i < count; ++i) {
    v[i].tile_begin = int32_t(total);
    const int tiles_m = (v[i].M + kBM - 1) / kBM;
    for (int tm = 0; tm < tiles_m; ++tm) {
      const int c = tiles_in_row(v[i].symmetric, v[i].N, bn, tm);
      if (list)
        for (int tn = 0; tn < c; ++tn)
          list->push_back(uint64_t(uint32_t(i)) | (uint64_t(uint32_t(tm)) << 32) | (uint64_t(uint32_t(tn)) << 48));
      total += c;
    }
  }
  return total;
}

shampoo4_status launch_gemm_tc(const TcGemmDesc* d_desc, int count, int max_tiles, int split, int bn,
                               const PtrEntry* tabs, int nparams, uint32_t* gflags, cudaStream_t st,
                               uint64_t wait_ns, int64_t total_tiles, const uint32_t* guard,
                               const uint64_t* tile_list) {
  if (count <= 0 || max_tiles <= 0) return SHAMPOO4_OK;
  if (wait_ns == 0 || wait_ns > kWaitNs) wait_ns = kWaitNs;
  // TF32: one tile per CTA, two 2-stage CTAs per SM, so one tile's
  // epilogue overlaps the other's main loop.  (Persistent forms were
  // measured against it on 960 products of 1024 x 1024 x 1024 and lost: two
  // 256-column accumulators drained by four epilogue warps, 1.3x slower with
  // three outputs and 2.2x on mirrored symmetric products; 128-wide tiles
  // with the register epilogue, 1.2x to 5.9x slower.  A TF32 tile's main
  // loop is too short to hide four warps' epilogue.)  Split mode, 128 wide:
  // the persistent register form (1.35x to 1.47x faster than one tile per
  // CTA: the main loop of three products per K step hides the epilogue),
  // or one tile per CTA when no tile numbering is given; 64 wide (the
  // narrow panel updates): two 2-stage CTAs per SM, where the MMA issue rate
  // of a 64-wide instruction makes a second issuing CTA per SM worth more
  // than overlap (its persistent register form was 1.4x to 2.1x slower on
  // the panel shapes, K = 64 to 512).
  const bool pers = total_tiles >= 0 && total_tiles < 0x7fffffffLL;
  if (!split)
    return launch_tc_impl<256, false, 2>(d_desc, count, max_tiles, tabs, nparams, gflags, wait_ns, st, guard);
  if (bn == 64)
    return launch_tc_impl<64, true, 2>(d_desc, count, max_tiles, tabs, nparams, gflags, wait_ns, st, guard);
  if (pers && tc_persistent)
    return launch_tc_pers<128, true, 3>(d_desc, count, total_tiles, tabs, nparams, gflags, wait_ns, st, guard,
                                        tile_list);
  return launch_tc_impl<128, true, 3>(d_desc, count, max_tiles, tabs, nparams, gflags, wait_ns, st, guard);
}

// ---------------------------------------------------------------- host side

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
}

shampoo4_status tc_encode_map(CUtensorMap* out, const float* base, int64_t rows, int64_t cols, int64_t ld,
                              int box_rows, int mn_major) {
  if (!g_encode) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return SHAMPOO4_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  if ((ld * 4) % 16 != 0 || (reinterpret_cast<uintptr_t>(base) % 16) != 0) return SHAMPOO4_ERR_INVALID_ARG;
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(ld) * 4};
  cuuint32_t box[2] = {32u, cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        mn_major ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SHAMPOO4_OK : SHAMPOO4_ERR_CUDA;
}

}  // namespace s4
