// Device descriptors and launchers of the shampoo4 library.
//
// The host planner turns a handle's tile partition into a fixed list of
// launches per API call (a "program"); every launch processes a whole batch
// of problems -- one per tile or per factor -- described by an array of
// descriptors that lives in the workspace.  The descriptors are written once
// at bind time; only the per-call gradient and output addresses change, and
// those sit in two small pointer tables that descriptors refer to by index.
#pragma once
#include "common.cuh"

namespace s4 {

// A per-call operand: either an absolute address (tab < 0) or parameter
// `param` of pointer table `tab` (0 = gradients, 1 = outputs), offset by
// (r0, c0) with that table's leading dimension.
struct PtrEntry {
  const float* ptr;
  int64_t ld;
};

struct OperandRef {
  int32_t tab;
  int32_t param;
  int64_t r0, c0;
};

// ---- fp32-output batched GEMM --------------------------------------------
// C = alpha * op(A) op(B) + beta * Cin, op(X) = X or X^T (row-major storage).
// kscale (optional) multiplies op(A)[i,k] by kscale[k]; skip (optional)
// suppresses the whole problem when *skip != 0.  mode selects arithmetic.
enum GemmMode : int32_t { kModeTF32 = 0, kModeFP32 = 1 };

struct GemmF32Desc {
  int32_t M, N, K;
  int32_t ta, tb;
  int32_t mode;
  int32_t symmetric;          // output known symmetric: only tiles on or below
                              // the diagonal are computed, then mirrored
  int32_t pad_;
  float alpha, beta;
  const float* A; int64_t lda;
  const float* B; int64_t ldb;
  float* C; int64_t ldc;
  const float* Cin; int64_t ldcin;
  const float* kscale;
  const uint32_t* skip;
  OperandRef a_ref, b_ref, c_ref;
};

// ---- fp64-accumulating batched GEMM (QR of the subspace step) --------------
struct GemmF64Desc {
  int32_t M, N, K;
  int32_t ta, tb;
  int32_t lower_only;         // skip tiles strictly above the diagonal
  int32_t a_f64, b_f64, c_f64, cin_f64;
  double alpha, beta;
  const void* A; int64_t lda;
  const void* B; int64_t ldb;
  void* C; int64_t ldc;
  const void* Cin; int64_t ldcin;
  const uint32_t* skip;
};

// Cholesky of one jb x jb diagonal block (lower, in place).
struct PotrfDesc {
  double* A; int64_t ld;
  int32_t jb; int32_t pad_;
  uint32_t* fail;             // set to 1 on a non-positive or non-finite pivot
  uint32_t* gflags;           // ... and SHAMPOO4_FLAG_REFRESH_FAILED ORed here
  const uint32_t* skip;       // optional: block skipped when *skip != 0
};

// X[r, 0:jb] <- X[r, 0:jb] * L^-T for r < rows, L the jb x jb lower block.
struct TrsmDesc {
  const double* L; int64_t ldl;
  double* X; int64_t ldx;
  int32_t jb, rows;
  const uint32_t* skip;       // optional
};

// A basis from the state: U = dequant(codes, scales), or the identity.
// Outputs, each optional: U (fp32), its TF32 split (Uh, Ul), and the TF32
// split of U diag(mu) (Vh, Vl; column j scaled by mu[j]).
struct BasisDesc {
  const uint8_t* codes;
  const float* scales;
  float* U;
  float* Uh; float* Ul;
  const float* mu;
  float* Vh; float* Vl;
  int32_t d;
  int32_t identity;
  int32_t codebook;
};

// lambda_i = max(sum_r Q[r,i] T[r,i], 0), T = S Q; written only if *skip==0.
struct RayleighDesc {
  const float* Q;
  const float* T;
  float* lam;
  int32_t d; int32_t pad_;
  const uint32_t* skip;
};

// mu_i = (lambda_i + eps)^(-1/4)
// mu_i = (lambda_i + eps)^(-1/4) (the root's scale), or, with sqrt_mode,
// sqrt(max(lambda_i, 0)) (the half scale of a rebuilt U diag(lambda) U^T).
struct MuDesc {
  const float* lam;
  float* mu;
  int32_t d; int32_t sqrt_mode;
};

// Scan a matrix (absolute or per-call) for NaN/Inf; on one, set *flag = 1
// and OR `bit` into the global flag word.
struct ScanDesc {
  const float* X; int64_t ld;
  int32_t rows, cols;
  OperandRef ref;
  uint32_t* flag;
  uint32_t bit; int32_t pad_;
  float* oh; float* ol;       // optional dense TF32 split of the matrix
};

// W <- W + s I with s = 11 (2 d^2 + d) 2^-53 trace(W): the shift of the
// first pass of shifted Cholesky-QR (Fukaya, Kannan, Nakatsukasa, Zhang,
// Yamamoto, "Shifted Cholesky QR for computing the QR factorization of
// ill-conditioned matrices", SIAM J. Sci. Comput. 42(1), 2020), with the
// Frobenius norm standing in for the spectral norm (a larger, still valid
// shift).
struct ShiftDesc {
  double* W; int64_t ld;
  int32_t d; int32_t pad_;
  const uint32_t* skip;
};

// ---- fp32-storage pieces of the tensor-core Cholesky-QR ------------------
// Cholesky of the jb x jb diagonal block of an fp32 matrix, lower, in place,
// carried out in fp64.
// On a breakdown: *fail = 1, *clear = 0 (if set), gflags |= REFRESH_FAILED
// (if set).  Skipped when *fail is already set.
struct PotrfDescF {
  float* A; int64_t ld;
  int32_t jb; int32_t pad_;
  uint32_t* fail;
  uint32_t* gflags;
  uint32_t* clear;
  float* oh; float* ol;       // optional TF32 split of the factor (same ld)
  float* ih; float* il;       // optional TF32 split of the inverse factor,
                              // 64 x 64 with leading dimension 64, zero-padded
  const uint32_t* skip;       // optional: block skipped when *skip != 0
  float min_pivot;            // a pivot (Schur-complement diagonal) at or
                              // below this counts as a breakdown; 0 = only
                              // non-positive or non-finite pivots do
  int32_t pad2_;
  uint32_t* any_fallback;     // optional: set to 1 when the block sends its
                              // factor to the fp64 redo (guard of those launches)
};

// W_ii <- W_ii (1 + coef) for i < d: the shift of the first Cholesky-QR
// pass, applied to the column-equilibrated Gram (D^-1 W D^-1 + coef I with
// D = diag(W)^1/2), i.e. a shift of coef times each column's squared norm.
struct ShiftDescF {
  float* W; int64_t ld;
  int32_t d; float coef;
  const uint32_t* skip;
};


// dst = fp32(src); optionally also the TF32 split (dh, dl).
struct ConvertDesc {
  const double* src;
  float* dst;
  float* dh; float* dl;
  int64_t n;
  const uint32_t* skip;       // optional
};


// Coupled Newton inverse fourth root ("Shampoo -- Second-Order Optimizer",
// "Computing the inverse fourth root"), A = S + eps I:
//   norm:  c = ||A||_F in fp64; sc[0] = 1/c, sc[1] = c^(-1/4) (fp32)
//   INIT:  M = A / c (fp32 master + TF32 split), F = 1.25 I - 0.25 M
//          (split), X = F (fp32 + split): the first iteration's X = I F
//   STEP:  F = 1.25 I - 0.25 M from the fp32 M (split)
//   FINAL: P = sc[1] X (fp32)
// Splits are written when the pointers are set; everything is skipped for
// a factor with *skip != 0.
struct NewtonNormDesc {
  const float* S;
  float* sc;
  int32_t d; float eps;
  const uint32_t* skip;
};
enum { kNewtonInit = 0, kNewtonStep = 1, kNewtonFinal = 2 };
struct NewtonEltDesc {
  const float* in;
  const float* sc;
  float* m; float* mh; float* ml;      // INIT: M; FINAL: P (m only)
  float* f;                            // INIT, STEP: F in fp32 (CUDA-core factors)
  float* fh; float* fl;                // INIT, STEP: F as a TF32 split (tensor-core factors)
  float* x; float* xh; float* xl;      // INIT: X = F
  int32_t d; int32_t mode;
  float eps; int32_t pad_;
  const uint32_t* skip;
};

// dst[0, n) = src[0, n): the debug capture of a refresh's intermediate
// matrices into a caller buffer.
struct CopyDesc {
  const float* src;
  float* dst;
  int64_t n;
};


// W_ii <- sum_k X[k, i]^2 (fp64 sums, one thread per column, rounded once
// to fp32) for i < d, X row-major d x d.  The tensor cores' accumulation
// truncates, so a Gram's diagonal -- a sum of positive terms -- comes out
// low by about 1e-8 K relative; this restores it.
struct DiagDesc {
  const float* X;
  float* W; int64_t ldw;
  int32_t d; int32_t pad_;
  const uint32_t* skip;
};

// Diagonal of a product C = A B^T of two split operands with the same rows:
// C_ii = sum_k (ah + al)_ik (bh + bl)_ik in fp64 over the d columns, rounded
// once to fp32 into C, and its TF32 split into (Chi, Clo) (each optional).
// A sum of positive terms -- the diagonal of U diag(mu) U^T -- comes out of
// the tensor cores' truncating accumulation low by about 1e-8 K relative;
// this rewrites it.  One warp per row.
struct RowDiagDesc {
  const float* ah; const float* al;
  const float* bh; const float* bl;
  int64_t ld;                 // of the operands and of C / Chi / Clo
  int32_t d; int32_t pad_;
  float* C; float* Chi; float* Clo;
};

// Deviation sums (the orthogonality sketch below) clamp each square at
// 2^-20 and add in units of 2^-60: an exact integer sum, independent of the
// order of additions.
constexpr float kDevFineClamp = 0x1p-20f, kDevFineUnit = 0x1p60f;

// Inverse of a 128 x 128 lower-triangular diagonal block of L from the
// inverses of its two 64 x 64 diagonal blocks:
//   [A 0; C B]^-1 = [A^-1 0; -B^-1 C A^-1  B^-1],
// with A^-1, B^-1 the split 64 x 64 blocks (ld 64, zero-padded) at ih/il
// rows j and j + 64, C = L[j+64 :, j : j+64] from the split factor (oh/ol,
// ld d).  fp64 inside; out: the TF32 split of the 128 x 128 inverse
// (ld 128), zero outside the d - j valid rows and columns.  One CTA per
// block.
struct Inv128Desc {
  const float* ih; const float* il;    // 64 x 64 inverse blocks, rows j..
  const float* oh; const float* ol;    // split of L, ld d
  float* jh; float* jl;                // 128 x 128 output, rows j..
  int32_t d, j;
  const uint32_t* skip;
};

// Orthogonality sketch of a factor's Q (d x d fp32, row-major, d % 4 == 0),
// two fp64 passes.  Omega (d x 16) holds one sign per row: Omega[c][c mod
// 16] = -1 or +1 from bit c mod 16 of the lowbias32 integer mixer of c / 16,
// zero elsewhere.  Pass one: Z = Q Omega (Z row-major d x 16, fp64).  Pass
// two: devsq += sum_cj min((Q^T Z - Omega)_cj^2, 2^-20), in units of 2^-60.
// (Q^T Z - Omega) = E Omega with E = Q^T Q - I, and for independent signs
// E ||E Omega||_F^2 = ||E||_F^2: the sum estimates the Gram deviation that
// the gate compares, without the Gram.  One thread per row (pass one) or
// column (pass two), 128 per CTA.
constexpr int kSketchCols = 16;
struct SketchDesc {
  const float* Q;
  double* Z;                    // d x 16 scratch
  unsigned long long* devsq;
  int32_t d; int32_t pad_;
  const uint32_t* skip;
};

// Decision before the last Cholesky-QR pass of a factor, from the deviation
// of its input Q from orthonormal (the sketch above): out = 1 (skip the
// pass) when *bad != 0 or *devsq <= thr (Q already orthonormal to the
// arithmetic's floor), else 0.
struct GateDesc {
  const unsigned long long* devsq;
  const uint32_t* bad;
  uint32_t* out;
  unsigned long long thr;
  uint32_t* any;       // optional: set to 1 when this factor goes through the pass
};


// ---- grafted weight update ("Shampoo -- Second-Order Optimizer", section
// "Grafting: borrow a step size that already works") ------------------------
// step_b = lr * ||d_graft_b||_F / (||D_b||_F + graft_eps) * D_b per tile b,
// W_b <- W_b - step_b; d_graft = G (SGD) or the bias-corrected Adam
// direction m_hat / (sqrt(v_hat) + adam_eps).  A work item is a band of rows
// of one tile; the items of a tile are consecutive, and the partial sums of
// item i sit in parts[2i] (sum d_graft^2) and parts[2i + 1] (sum D^2).
enum GraftKind : int32_t { kGraftSgd = 0, kGraftAdam = 1 };

struct GraftItem {
  int32_t param, block;        // parameter, and tile (statistics flag index)
  int64_t r0, c0;              // band origin within the parameter
  int32_t rows, cols;
  int32_t part0, nparts;       // the tile's first item and its item count
  int64_t m_off, v_off;        // element offsets of the band origin's moments
  int64_t state_ld;            // moments are dense per parameter: ld = cols
  int64_t dsq_off;             // the tile's recorded sums of squares of D
  int32_t dsq_n, pad_;         // (0: none; a CUDA-core tile)
};

struct GraftArgs {
  const GraftItem* items;
  int32_t nitems, nparams;
  const PtrEntry* tabs;        // [0, np): gradients, [np, 2np): directions,
                               // [2np, 3np): weights
  float* state;                // Adam moments (unused for SGD)
  const uint32_t* bflag;       // per tile: non-finite gradient seen by the
                               // statistics update of this step
  double* parts;               // 2 * nitems
  uint32_t* flags;             // status word
  int32_t kind;
  const double* dsq;           // recorded sums of squares of D (use_dsq)
  int32_t use_dsq;
  float beta1, beta2, omb1, omb2;       // omb = 1 - beta, in fp32
  float c1, c2;                         // 1 / (1 - beta^t)
  float adam_eps;
  double lr, graft_eps;
};

// Two launches: moments and per-item norms, then the weight update.
shampoo4_status launch_graft(const GraftArgs& a, cudaStream_t st);

// ---- per-call pointer tables, written on the stream ---------------------------
// The table travels as a kernel parameter and one warp stores it, so setting
// it is an ordinary stream operation: nothing waits on the host, and a CUDA
// graph captured around an API call replays the table of that call.
constexpr int kMaxTableEntries = 1024;     // 16 KB of kernel parameter

shampoo4_status launch_set_table(const PtrEntry* entries, int n, PtrEntry* dst, cudaStream_t st);

// ---- launchers (each enqueues one launch over `count` descriptors) -------
shampoo4_status launch_gemm_f32(const GemmF32Desc* d_desc, int count, int max_tiles,
                                const PtrEntry* tabs, int nparams, cudaStream_t st);
// guard (optional, one word for the whole launch): the launch does nothing
// while *guard == 0 -- the fp64 QR passes run only when some factor needs
// them.
shampoo4_status launch_gemm_f64(const GemmF64Desc* d_desc, int count, int max_tiles,
                                cudaStream_t st, const uint32_t* guard = nullptr);
shampoo4_status launch_potrf(const PotrfDesc* d_desc, int count, cudaStream_t st,
                             const uint32_t* guard = nullptr);
shampoo4_status launch_trsm(const TrsmDesc* d_desc, int count, int max_rows, cudaStream_t st,
                            const uint32_t* guard = nullptr);
shampoo4_status launch_basis(const BasisDesc* d_desc, int count, int64_t max_elems, cudaStream_t st);
shampoo4_status launch_rayleigh(const RayleighDesc* d_desc, int count, int max_d, cudaStream_t st);
shampoo4_status launch_mu(const MuDesc* d_desc, int count, int max_d, float eps, cudaStream_t st);
shampoo4_status launch_scan(const ScanDesc* d_desc, int count, int64_t max_rows,
                            const PtrEntry* tabs, int nparams, uint32_t* flags, cudaStream_t st);
shampoo4_status launch_shift(const ShiftDesc* d_desc, int count, cudaStream_t st,
                             const uint32_t* guard = nullptr);
// guard (optional, as for the fp64 launches): the whole launch is skipped
// when *guard == 0.
shampoo4_status launch_potrf_f(const PotrfDescF* d_desc, int count, cudaStream_t st, const uint32_t* guard = nullptr);
shampoo4_status launch_shift_f(const ShiftDescF* d_desc, int count, cudaStream_t st);
shampoo4_status launch_convert(const ConvertDesc* d_desc, int count, int64_t max_elems, cudaStream_t st,
                               const uint32_t* guard = nullptr);
shampoo4_status launch_gate(const GateDesc* d_desc, int count, cudaStream_t st);
shampoo4_status launch_sketch(const SketchDesc* d_desc, int count, int max_d, int pass, cudaStream_t st);
shampoo4_status launch_copy(const CopyDesc* d_desc, int count, int64_t max_elems, cudaStream_t st);
shampoo4_status launch_newton_norm(const NewtonNormDesc* d_desc, int count, cudaStream_t st);
shampoo4_status launch_newton_elt(const NewtonEltDesc* d_desc, int count, int64_t max_elems, cudaStream_t st);
shampoo4_status launch_inv128(const Inv128Desc* d_desc, int count, cudaStream_t st, const uint32_t* guard = nullptr);
shampoo4_status launch_diag(const DiagDesc* d_desc, int count, int max_d, cudaStream_t st,
                            const uint32_t* guard = nullptr);
shampoo4_status launch_rowdiag(const RowDiagDesc* d_desc, int count, int max_d, cudaStream_t st);

// Codec launchers (quant4.cu).  `skip` (optional, per tensor) suppresses a
// tensor when *skip[i] != 0.  `launched` (optional) receives the number of
// kernels issued (one per batch of up to 64 non-empty tensors).
shampoo4_status launch_pack(const float* const* x, const int64_t* n, int32_t count,
                            uint8_t* const* codes, float* const* scales, cudaStream_t st,
                            const uint32_t* const* skip = nullptr, int* launched = nullptr,
                            int codebook = kCodebookLinearSquare);
shampoo4_status launch_unpack(const uint8_t* const* codes, const float* const* scales,
                              const int64_t* n, int32_t count, float* const* x, cudaStream_t st,
                              int codebook = kCodebookLinearSquare);

}  // namespace s4
