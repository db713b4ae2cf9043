// Descriptors of the tensor-core GEMM (gemm_tc.cu).
#pragma once
#include <cuda.h>
#include <vector>
#include "plan.h"

namespace s4 {

// One operand of a tensor-core product: TMA tensor maps of its TF32 value
// (hi) and, in split mode, of its TF32 residual (lo).  mn_major = 0 when the
// contraction index is contiguous in memory (map box 32 x rows), 1 when the
// row index of op(X) is (map box 32 x 32).  (row0, col0) offset the tile
// coordinates inside the mapped matrix.
struct TcOperand {
  const CUtensorMap* hi;
  const CUtensorMap* lo;
  int32_t mn_major;
  int32_t row0, col0;
  int32_t pad_;
};

// C = alpha * op(A) op(B) + beta * Cin for one problem.  Outputs, each
// optional: C (fp32, rounded to TF32 when out_round), and the TF32 split
// Chi = RN(v), Clo = RN(v - Chi) with leading dimension ldh.  symmetric:
// only tiles touching the lower triangle run; 1: every element below the
// diagonal is also written to its mirror position; 2: only the lower
// triangle (diagonal included) is written; 3: the running tiles are
// written in full (a symmetric matrix stored by those tiles, read back
// through bt_hi/bt_lo).  skip: problem skipped when *skip != 0.  c_ref: C
// taken from the per-call pointer tables.
//
// bt_hi/bt_lo (optional): op(B) is a symmetric matrix stored only in the
// tiles of a symmetric-mode-3 product of this tile width, and b reads it
// K-major (op(B)[k, n] = X[n, k]).  K blocks at or beyond n0 + BN, outside
// the stored tiles, read X[k, n] instead through these MN-major maps of X.
// at_hi/at_lo (optional): the same for op(A) = X read K-major: K blocks
// whose BN-wide block starts at or beyond m0 + 128 read X[k, m] through
// these MN-major maps.
struct TcGemmDesc {
  int32_t M, N, K;
  int32_t symmetric;
  int32_t out_round;
  // index of the problem's first tile in the batch's list of tiles that
  // run (tc_assign_tiles); read by the persistent kernel only
  int32_t tile_begin;
  float alpha, beta;
  TcOperand a, b;
  float* C; int64_t ldc;
  float* Chi; float* Clo; int64_t ldh;
  const float* Cin; int64_t ldcin;
  const uint32_t* skip;
  OperandRef c_ref;
  const CUtensorMap* bt_hi;
  const CUtensorMap* bt_lo;
  const CUtensorMap* at_hi;
  const CUtensorMap* at_lo;
  // optional (TF32 and 64-wide instances; the persistent 128-wide one
  // ignores it): the sum of squares (fp64) of the values each epilogue warp
  // writes to C, at sumsq[4 * (tile_row * tiles_n + tile_col) + warp]
  // (tiles_n = ceil(N / tile width)); every running tile writes its four
  // slots, so the sum over them, in any fixed order, is ||C||_F^2
  double* sumsq;
  // optional second operand pair (split mode, 128-wide tiles): K blocks at
  // or beyond ksplit (a multiple of 32) read op(A) through a2 and op(B)
  // through b2, at K coordinate k - ksplit, so that C = [A1 A2] [B1; B2]
  // for pieces stored apart.  Unused when a2.hi is null; when set, a and b
  // must hold valid maps too (ksplit > 0).
  TcOperand a2, b2;
  int32_t ksplit;
  int32_t pad2_;
};

// Tile width N of the kernel instance: 256 (TF32), 128 (split), or 64
// (split, narrow products).
int tc_block_n(int split);
// wait_ns: how long each pipeline wait may take before the CTA gives up
// (SHAMPOO4_FLAG_TIMEOUT); 0 means the default of 2 s, which is also the cap.
// total_tiles: the batch's number of running tiles from tc_assign_tiles on
// the same descriptors; without it (-1) every instance runs one tile per CTA.
// guard (optional): the whole launch is skipped when *guard == 0.
// tile_list (optional, persistent instance): entry t names running tile t
// of the batch, packed as problem | tile row << 32 | tile column << 48
// (tc_assign_tiles writes it), so that a CTA finds its tile with one load
// instead of walking the problem list.
shampoo4_status launch_gemm_tc(const TcGemmDesc* d_desc, int count, int max_tiles, int split, int bn,
                               const PtrEntry* tabs, int nparams, uint32_t* gflags, cudaStream_t st,
                               uint64_t wait_ns = 0, int64_t total_tiles = -1, const uint32_t* guard = nullptr,
                               const uint64_t* tile_list = nullptr);
// Tiles of one problem that run for tile width bn: all, or for a symmetric
// product those touching the lower triangle (row block tm runs column
// blocks tn with tn * bn < (tm + 1) * 128).
int tc_tiles_in_row(const TcGemmDesc& g, int bn, int tm);
// Number the running tiles of a batch: sets tile_begin of each descriptor,
// returns the total; with list, also appends each running tile's packed
// entry (problem | tile row << 32 | tile column << 48) in that order.
int64_t tc_assign_tiles(TcGemmDesc* v, int count, int bn, std::vector<uint64_t>* list = nullptr);
// Encode a 2-D fp32 tensor map (rows x cols, leading dimension ld elements),
// box 32 (contiguous) x box_rows, zero fill out of bounds; 128-byte swizzle,
// with 32-byte atoms for an operand read MN-major.
shampoo4_status tc_encode_map(CUtensorMap* out, const float* base, int64_t rows, int64_t cols, int64_t ld,
                              int box_rows, int mn_major);

}  // namespace s4
