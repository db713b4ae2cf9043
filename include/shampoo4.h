/*
 * shampoo4.h -- C ABI of the B200 4-bit Shampoo preconditioner library.
 *
 * The library runs the per-layer preconditioner step of 4-bit Shampoo
 * ("4-bit Shampoo for Memory-Efficient Network Training", Wang, Zhou, Li,
 * Huang -- abstract) on one GPU:
 *
 *   update_stats    L <- beta L + (1-beta) G G^T,  R <- beta R + (1-beta) G^T G
 *                   ("Shampoo -- Second-Order Optimizer", sections "Kronecker
 *                   factorization" and "Pitfalls": EMA with decay beta)
 *   refresh_roots   per factor: dequantize the 4-bit eigenvector matrix U,
 *                   Bjorck-rectify it (U <- 1.5 U - 0.5 U U^T U, t times),
 *                   one subspace-iteration step Y = (S + eps I) U, Y = QR,
 *                   Rayleigh eigenvalues lambda_i = max(q_i^T S q_i, 0), and
 *                   requantize Q to 4-bit codes with per-64 scales
 *   precondition    P = U diag((lambda + eps)^(-1/4)) U^T per factor
 *                   ("Computing the inverse fourth root") and
 *                   D = P_L G P_R per block ("Kronecker factorization")
 *
 * Weights are cut into tiles of at most max_block x max_block, each with its
 * own pair of factors ("Blocked and distributed variants").
 *
 * Beside the step:
 *   graft_update    W <- W - lr ||d_graft|| / (||D|| + eps) D per tile, with
 *                   d_graft the SGD or Adam step ("Grafting: borrow a step
 *                   size that already works")
 *   compressed_stats (config) keeps each statistic only as its 4-bit
 *                   eigenbasis and eigenvalues and rebuilds it per update
 *   refresh_rank / refresh_world (config) deal the refresh of the factors to
 *                   several ranks, whose state spans the caller exchanges
 *   a CUDA graph captured around the step calls replays them: a call
 *                   enqueues only kernels and memsets on its stream
 *
 * Conventions shared by every entry point
 *  - All device buffers are allocated and owned by the caller; the library
 *    never allocates device memory.  It owns only host-side planning data
 *    (and small pinned host staging buffers per handle, used only for
 *    pointer tables of more than 1024 entries and for the status flags).
 *  - Calls that take a stream are asynchronous on it; none synchronizes
 *    except shampoo4_get_status_flags.  All calls on one handle must be
 *    ordered on the same stream (or by the caller's own events).
 *  - Matrices are fp32, row-major, with a leading dimension in elements.
 *  - Argument errors are returned synchronously before anything is enqueued.
 *    Errors found on the device (non-finite input, a failed factorization)
 *    are latched in a flag word inside the workspace and read back with
 *    shampoo4_get_status_flags.
 *  - Arrays of device pointers ("d_grads", "d_x", ...) are HOST arrays whose
 *    elements are device addresses.
 *  - A handle is not thread-safe; distinct handles are independent.
 */
#ifndef SHAMPOO4_H
#define SHAMPOO4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st* shampoo4_stream_t;

typedef enum {
  SHAMPOO4_OK = 0,
  SHAMPOO4_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or config  */
  SHAMPOO4_ERR_CUDA = 2,         /* a CUDA launch or copy failed            */
  SHAMPOO4_ERR_NOT_READY = 3,    /* precondition before the first refresh,
                                    or a compute call before shampoo4_bind  */
  SHAMPOO4_ERR_NONFINITE = 4,    /* reported through the status flags       */
  SHAMPOO4_ERR_WORKSPACE = 5,    /* workspace smaller than shampoo4_sizes   */
  SHAMPOO4_ERR_UNSUPPORTED = 6,  /* no device of compute capability 10.x    */
  SHAMPOO4_ERR_TIMEOUT = 7       /* reserved for bounded device waits       */
} shampoo4_status;

/* Arithmetic of the dense products.
 *  TF32: operands rounded to TF32 (round to nearest), fp32 accumulation.
 *  FP32: fp32-accurate products.
 * The subspace product (S + eps I) U, the Rayleigh product S Q and every
 * product of the QR are always fp32-accurate: they must resolve eigenvalues
 * near eps, far below TF32's resolution of the largest one.  The QR is a
 * shifted Cholesky-QR3 (Fukaya et al., SIAM J. Sci. Comput. 2020) whose
 * products run on the tensor cores as 3xTF32 with 64x64 Cholesky blocks in
 * fp64; a factor whose fp32 Cholesky breaks down is redone in fp64 on the
 * CUDA cores (SHAMPOO4_FLAG_QR_FALLBACK).  Factors whose edge is not a
 * multiple of 4 take the fp64 QR directly. */
typedef enum { SHAMPOO4_PREC_TF32 = 0, SHAMPOO4_PREC_FP32 = 1 } shampoo4_precision;

typedef struct {
  float beta;            /* EMA decay of the statistics, 0 <= beta < 1     */
  float eps;             /* added to eigenvalues in the root, and the shift
                            of the subspace step (S + eps I) U; > 0        */
  int32_t max_block;     /* tile edge b; 1 <= b <= 1024                    */
  int32_t quant_block;   /* elements per quantization scale; must be 64    */
  int32_t bjorck_iters;  /* Bjorck rectification steps per refresh, 0..16  */
  int32_t precision;     /* shampoo4_precision                             */
  int32_t compressed_stats; /* 0: each factor keeps its fp32 statistic S in
                            the state.  1: the statistic is kept only as its
                            4-bit eigenvector codes and eigenvalues ("4-bit
                            Shampoo ...", abstract: the preconditioner is
                            stored through its quantized eigenvector
                            matrix); update_stats rebuilds
                            S = beta U diag(lambda) U^T + (1-beta) G G^T
                            (U dequantized, no Bjorck) in the workspace, and
                            every update_stats must be followed by a
                            refresh_roots before the next one (the refresh
                            is what stores the new statistic; otherwise
                            ERR_NOT_READY).  The state shrinks by 4 d^2
                            bytes per factor.                               */
  int32_t refresh_rank;  /* refresh sharding ("Shampoo -- Second-Order
                            Optimizer", "Blocked and distributed variants":
                            the roots of different blocks are computed on
                            different workers).  With refresh_world > 1 the
                            factors are dealt to refresh_world ranks by
                            cost (longest d^3 first, each to the least
                            loaded rank); this handle keeps the statistics
                            of, and refreshes, only rank refresh_rank's
                            factors.  Every rank's codes, scales and
                            eigenvalues sit in one contiguous state span
                            (shampoo4_owner_span, the same offsets on every
                            rank); after refresh_roots the caller copies
                            each rank's span to the others (a broadcast per
                            rank) before precondition, which covers every
                            tile.  0 <= refresh_rank < refresh_world.       */
  int32_t refresh_world; /* 0 or 1: one rank refreshes every factor.        */
  int32_t codebook;      /* shampoo4_codebook of the 4-bit state            */
  int32_t root_method;   /* shampoo4_root_method                            */
  int32_t newton_iters;  /* coupled Newton iterations per refresh (root
                            methods NEWTON*), 1..100; 0 selects 32          */
  int32_t group_tiles;   /* tiles per group of the calls' scratch.  The
                            workspace holds the per-call scratch (the
                            refresh's matrices per factor, the split gradient
                            per tile) of two groups of consecutive tiles,
                            which the calls process in turn on two CUDA
                            streams of the handle, not of every tile at once.
                            0: one group while the whole scratch fits in
                            96 GiB, else as many tiles per group as keep a
                            group's scratch within 8 GiB; >= the tile count:
                            one group.  One group is the fastest (every
                            launch covers every factor; the QR chain's
                            latency-bound steps need that) and the largest.  With
                            refresh_world > 1 there is one group.  Results do
                            not depend on the grouping.                     */
} shampoo4_config;

/* The 4-bit codebook ("4-bit Shampoo for Memory-Efficient Network
 * Training", abstract: linear square quantization, compared there with
 * dynamic tree quantization).
 *  LINEAR_SQUARE: 16 levels sgn(y) y^2, y = (2j - 15)/15, no exact zero.
 *  DYNAMIC_TREE: Dettmers' (2016) dynamic tree data type restricted to 4
 *   bits: a sign, then in the other three bits a run of E zeros (a decimal
 *   exponent), an indicator 1 and k = 2 - E fraction bits i, magnitude
 *   10^-E (0.1 + 0.9 (i + 1) / 2^k); 000 is zero.  Magnitudes 0, 0.01,
 *   0.055, 0.1, 0.325, 0.55, 0.775, 1; levels 7 and 8 are both zero.
 * Either way threshold k is the fp32 rounding of the midpoint of levels k
 * and k+1 (in double), and a code is the number of thresholds strictly
 * below v = x / absmax. */
typedef enum { SHAMPOO4_CODEBOOK_LINEAR_SQUARE = 0, SHAMPOO4_CODEBOOK_DYNAMIC_TREE = 1 } shampoo4_codebook;

/* How each factor's inverse fourth root is obtained.
 *  EIGEN (the 4-bit Shampoo method): the 4-bit state is the eigenvector
 *   matrix U with eigenvalues lambda; refresh_roots refines U (dequantize,
 *   Bjorck, one subspace step) and precondition forms
 *   P = U diag((lambda + eps)^-1/4) U^T from the codes.
 *  NEWTON: refresh_roots computes P = (S + eps I)^-1/4 from the fp32
 *   statistic by the coupled Newton iteration of "Shampoo -- Second-Order
 *   Optimizer", "Computing the inverse fourth root" (c = ||S + eps I||_F,
 *   M = (S + eps I)/c, X = I; newton_iters times F = (5 I - M)/4, X <- X F,
 *   M <- F^4 M; P = X c^-1/4), with fp32-accurate tensor-core products, and
 *   stores P in fp32 in the state (4 d^2 bytes per factor, a 32-bit root
 *   cache); precondition applies it.
 *  NEWTON_Q4: the same root, stored block-wise in 4 bits with the codebook
 *   above -- quantizing the preconditioner itself, the alternative the
 *   4-bit Shampoo abstract argues against (its codes and scales take the
 *   place of U's).
 * The NEWTON methods need the fp32 statistic (compressed_stats = 0). */
typedef enum { SHAMPOO4_ROOT_EIGEN = 0, SHAMPOO4_ROOT_NEWTON = 1, SHAMPOO4_ROOT_NEWTON_Q4 = 2 } shampoo4_root_method;

typedef struct { int64_t rows, cols; } shampoo4_param;   /* 2-D weights only;
                            reshape convolutions to out x (in*kh*kw)        */

typedef struct shampoo4_ctx* shampoo4_handle;

/* Status flag bits (shampoo4_get_status_flags). */
#define SHAMPOO4_FLAG_NONFINITE_GRAD   0x1u  /* update_stats saw NaN/Inf in G;
                                               S was left unchanged         */
#define SHAMPOO4_FLAG_REFRESH_FAILED   0x2u  /* a factor's QR broke down; its
                                               previous codes and lambda were
                                               kept (stale-root fallback)   */
#define SHAMPOO4_FLAG_NONFINITE_STATE  0x4u  /* a statistic held NaN/Inf at
                                               refresh; that factor kept its
                                               previous basis               */
#define SHAMPOO4_FLAG_TIMEOUT          0x8u  /* a kernel's bounded wait on one
                                               of its own pipeline barriers
                                               expired; its output is invalid */
#define SHAMPOO4_FLAG_QR_FALLBACK      0x10u /* informational: the fp32 QR of
                                               some factor's subspace step was
                                               too ill-conditioned and was
                                               redone in fp64                */
#define SHAMPOO4_FLAG_GRAFT_SKIPPED    0x20u /* shampoo4_graft_update: a tile's
                                               norm ratio was not finite (its
                                               direction or moments overflowed);
                                               its weights were left unchanged */

/* Plan a set of parameters.  Host only: validates the config and shapes,
 * partitions every weight into greedy tiles of at most max_block (ragged
 * last tile), and lays out state and workspace.  *out receives a handle that
 * must be released with shampoo4_destroy.  Touches no device; shampoo4_bind
 * needs a device of compute capability 10.x (ERR_UNSUPPORTED otherwise). */
shampoo4_status shampoo4_init(const shampoo4_config* cfg, const shampoo4_param* params,
                              int32_t nparams, shampoo4_handle* out);

/* Bytes of device memory the caller must provide: the persistent optimizer
 * state (kept between steps, checkpointable) and the scratch workspace
 * (contents need not persist between calls, but the same buffer must be
 * passed to bind and used for the handle's lifetime). */
shampoo4_status shampoo4_sizes(shampoo4_handle h, size_t* state_bytes, size_t* workspace_bytes);

/* Attach caller-owned device buffers (256-byte aligned).  reset != 0 zeroes
 * the statistics and marks every factor as having no basis yet (the first
 * refresh then starts from U = I); reset == 0 adopts the buffer contents as
 * they are (resume from a checkpoint; the caller states with has_basis
 * whether it already holds a basis, see shampoo4_set_has_basis). */
shampoo4_status shampoo4_bind(shampoo4_handle h, void* d_state, void* d_workspace,
                              int32_t reset, shampoo4_stream_t stream);

/* Declare whether the bound state already holds eigenvector codes (after a
 * resume from a checkpoint taken after a refresh). */
shampoo4_status shampoo4_set_has_basis(shampoo4_handle h, int32_t has_basis);

/* S_L <- beta S_L + (1-beta) G_b G_b^T and S_R <- beta S_R + (1-beta) G_b^T G_b
 * for every tile G_b of every parameter.  d_grads[p] is the device address of
 * parameter p's gradient (rows x cols, row-major, leading dimension ld[p] >=
 * cols, 4-byte aligned).  A non-finite value anywhere in a tile leaves that
 * tile's two statistics unchanged and sets SHAMPOO4_FLAG_NONFINITE_GRAD. */
shampoo4_status shampoo4_update_stats(shampoo4_handle h, const float* const* d_grads,
                                      const int64_t* ld, shampoo4_stream_t stream);

/* Recompute every factor's 4-bit eigenvector codes, scales and eigenvalues
 * from its statistic (dequantize, Bjorck, subspace step, QR, Rayleigh,
 * requantize).  The first refresh after a reset starts from U = I. */
shampoo4_status shampoo4_refresh_roots(shampoo4_handle h, shampoo4_stream_t stream);

/* D = P_L G_b P_R for every tile, written into d_out[p] (same shape as the
 * gradient, leading dimension ld_out[p] >= cols).  d_out must not overlap
 * d_grads.  Returns ERR_NOT_READY before the first refresh. */
shampoo4_status shampoo4_precondition(shampoo4_handle h, const float* const* d_grads,
                                      const int64_t* ld, float* const* d_out,
                                      const int64_t* ld_out, shampoo4_stream_t stream);

/* Synchronize the stream, return the latched flag bits and clear them. */
shampoo4_status shampoo4_get_status_flags(shampoo4_handle h, uint32_t* flags,
                                          shampoo4_stream_t stream);

/* Counts of the plan. */
shampoo4_status shampoo4_counts(shampoo4_handle h, int32_t* nblocks, int32_t* nfactors);

/* Tile k of the plan: parameter index, first row and column, size m x n.
 * Tile k owns factor 2k (L, dimension m) and factor 2k+1 (R, dimension n). */
shampoo4_status shampoo4_block_info(shampoo4_handle h, int32_t block, int32_t* param,
                                    int64_t* r0, int64_t* c0, int32_t* m, int32_t* n);

/* Byte offsets inside the state buffer of one factor's statistic S (fp32
 * d x d, row-major, dense), codes (uint8, ceil(d*d/2), two per byte, element
 * 2i in the low nibble), scales (fp32, ceil(d*d/64)) and eigenvalues (fp32,
 * d); *dim receives d.  Any pointer may be NULL.  With compressed_stats, or
 * for a factor another rank refreshes, the statistic is not part of this
 * handle's state: *off_S receives SIZE_MAX (see shampoo4_debug_s_offset). */
shampoo4_status shampoo4_factor_layout(shampoo4_handle h, int32_t factor, size_t* off_S,
                                       size_t* off_codes, size_t* off_scales,
                                       size_t* off_lambda, int32_t* dim);

/* Root method NEWTON: byte offset inside the state of the factor's fp32
 * d x d root P = (S + eps I)^-1/4 from the last refresh_roots.
 * ERR_INVALID_ARG for the other root methods. */
shampoo4_status shampoo4_root_offset(shampoo4_handle h, int32_t factor, size_t* off_P);

/* Byte offset inside the workspace of the fp32 d x d orthonormal Q that the
 * last refresh quantized for this factor (valid until the next call that uses
 * the workspace).  Root method EIGEN and one tile group only (with several,
 * a later group reuses the scratch: ERR_UNSUPPORTED; shampoo4_debug_capture
 * works either way).  For tests and diagnostics. */
shampoo4_status shampoo4_debug_q_offset(shampoo4_handle h, int32_t factor, size_t* off_q);

/* With compressed_stats: byte offset inside the workspace of the fp32 d x d
 * statistic that the last update_stats rebuilt for this factor (valid until
 * the next refresh_roots).  ERR_INVALID_ARG without compressed_stats.  For
 * tests and diagnostics. */
shampoo4_status shampoo4_debug_s_offset(shampoo4_handle h, int32_t factor, size_t* off_s);

/* Debug capture, for tests and diagnostics: the boundaries between the
 * refresh's stages.  ("4-bit Shampoo for Memory-Efficient Network Training",
 * abstract: the dequantized eigenvector matrix is rectified, then refined;
 * the refinement is one subspace step, Y = (S + eps I) U, Y = QR.)
 *
 * shampoo4_debug_capture_bytes gives the size of the capture buffer: two
 * fp32 d x d matrices per factor, each 256-byte aligned.
 * shampoo4_debug_capture registers a caller-owned device buffer of that size
 * (256-byte aligned; NULL unregisters).  The handle must then be bound again
 * (shampoo4_bind, reset = 0 keeps the state), because the refresh programs
 * carry the buffer's addresses.  While one is registered, every
 * refresh_roots also copies, for each factor it refreshes, the rectified
 * basis that enters the subspace step (after dequantization and Bjorck; the
 * identity on a first refresh) and the orthonormal Q that is then
 * requantized (root methods NEWTON*: the root P in the second slot; the
 * first is not written).  The buffer must stay allocated until it is unregistered and
 * the handle bound again, or destroyed.  Without one, the copies are not
 * launched.  shampoo4_debug_capture_layout gives the byte offsets of a
 * factor's two row-major matrices in the buffer. */
shampoo4_status shampoo4_debug_capture_bytes(shampoo4_handle h, size_t* bytes);
shampoo4_status shampoo4_debug_capture(shampoo4_handle h, void* d_buf);
shampoo4_status shampoo4_debug_capture_layout(shampoo4_handle h, int32_t factor, size_t* off_u,
                                              size_t* off_q);

/* Diagnostic: how many parts the refresh of a one-group handle is split
 * into (1 or 2; default 1: on the Llama layer set two parts measured no
 * faster).  The factors are dealt to the parts by d^3 cost, and the parts' launch
 * sequences run concurrently on the handle's own CUDA streams, forked from
 * and joined back to the caller's stream (so a graph captured on the
 * caller's stream captures them too).  Each factor's arithmetic does not
 * depend on the split.  Takes effect at the next shampoo4_bind (reset = 0
 * keeps the state). */
shampoo4_status shampoo4_debug_refresh_parts(shampoo4_handle h, int32_t parts);

/* Diagnostic: the time limit of the tensor-core products' pipeline waits
 * (a CTA waiting for a free stage, for loaded operands or for its finished
 * accumulator).  On expiry a CTA raises SHAMPOO4_FLAG_TIMEOUT, issues
 * nothing more, waits (up to 2 s) for the loads and MMAs it already issued,
 * frees its tensor memory and exits; the call's outputs are then undefined,
 * the handle and the CUDA context stay usable.  ns = 0 restores the default
 * of 2 s, which is also the largest limit.  Used by the tests to exercise
 * that return path; it takes effect at the next launch. */
shampoo4_status shampoo4_debug_wait_limit(shampoo4_handle h, uint64_t ns);

/* Refresh sharding: the rank that refreshes a factor, and the state byte
 * range [*off, *off + *bytes) holding the codes, scales and eigenvalues of
 * every factor that rank refreshes (the same on every rank's handle). */
shampoo4_status shampoo4_factor_owner(shampoo4_handle h, int32_t factor, int32_t* rank);
shampoo4_status shampoo4_owner_span(shampoo4_handle h, int32_t rank, size_t* off, size_t* bytes);

/* Stages of the three programs, for the optional launch timing below. */
typedef enum {
  SHAMPOO4_STAGE_STATS_SCAN = 0, SHAMPOO4_STAGE_STATS_GEMM, SHAMPOO4_STAGE_REFRESH_SCAN,
  SHAMPOO4_STAGE_BASIS, SHAMPOO4_STAGE_BJORCK_GRAM, SHAMPOO4_STAGE_BJORCK_UPDATE,
  SHAMPOO4_STAGE_SUBSPACE, SHAMPOO4_STAGE_QR_GRAM, SHAMPOO4_STAGE_QR_POTRF,
  SHAMPOO4_STAGE_QR_TRSM_PANEL, SHAMPOO4_STAGE_QR_SYRK, SHAMPOO4_STAGE_QR_SOLVE_UPDATE,
  SHAMPOO4_STAGE_QR_SOLVE_PANEL, SHAMPOO4_STAGE_QR_CONVERT, SHAMPOO4_STAGE_RAYLEIGH_GEMM,
  SHAMPOO4_STAGE_RAYLEIGH, SHAMPOO4_STAGE_REQUANT, SHAMPOO4_STAGE_PRECOND_DEQUANT,
  SHAMPOO4_STAGE_PRECOND_MU, SHAMPOO4_STAGE_ROOTS, SHAMPOO4_STAGE_APPLY_LEFT,
  SHAMPOO4_STAGE_APPLY_RIGHT, SHAMPOO4_STAGE_QR_INVERSE, SHAMPOO4_STAGE_STATS_DEQUANT,
  SHAMPOO4_STAGE_STATS_REBUILD, SHAMPOO4_STAGE_TABLES, SHAMPOO4_STAGE_NEWTON_ELT,
  SHAMPOO4_STAGE_NEWTON_GEMM, SHAMPOO4_STAGE_COUNT
} shampoo4_stage;

/* Launch timing, for diagnostics and roofline figures.  While enabled, every
 * kernel launch of the handle is bracketed by a pair of CUDA events on the
 * call's stream.  Enabling or disabling clears the totals. */
shampoo4_status shampoo4_timing_enable(shampoo4_handle h, int32_t enable);

/* Totals for one stage since timing was enabled: device milliseconds,
 * launches, and the algorithmic flops and bytes of those launches (flops
 * 2 M N K per product, M (M+1) K when only one triangle of a symmetric
 * output is needed).  Synchronizes on the recorded events. */
shampoo4_status shampoo4_timing_read(shampoo4_handle h, int32_t stage, double* ms,
                                     int64_t* launches, double* flops, double* bytes);
const char* shampoo4_stage_name(int32_t stage);

/* Block-wise linear square 4-bit quantization of `count` fp32 tensors
 * ("4-bit Shampoo for Memory-Efficient Network Training", abstract: linear
 * square quantization, block-wise; the level and threshold definitions below
 * are this library's reading of the name).
 * For tensor i: n[i] elements at d_x[i] (4-byte aligned), ceil(n[i]/2) code
 * bytes to d_codes[i], ceil(n[i]/64) scales to d_scales[i].  Errors: a NULL
 * array or element pointer, count < 0, n[i] < 0 or a misaligned pointer
 * return ERR_INVALID_ARG before anything is enqueued; count == 0 and empty
 * tensors (n[i] == 0) do nothing.
 * Per block of 64 consecutive elements: scale = max |x| (NaN if the block
 * holds a NaN, +Inf if it holds an infinity), v = x / scale (IEEE division),
 * code = number of the 15 thresholds t_k strictly below v, where t_k is the
 * fp32-rounded midpoint of adjacent levels of the codebook
 * cb_j = sgn(y) y^2, y = (2j-15)/15; an all-zero block gets code 7.
 * Element 2i goes to the low nibble of byte i; a padded nibble is 0. */
shampoo4_status quant4_pack(const float* const* d_x, const int64_t* n, int32_t count,
                            uint8_t* const* d_codes, float* const* d_scales,
                            shampoo4_stream_t stream);

/* Inverse of quant4_pack: x = fp32(cb_code) * scale (one fp32 multiply),
 * n[i] fp32 elements to d_x[i]; same argument rules as quant4_pack. */
shampoo4_status quant4_unpack(const uint8_t* const* d_codes, const float* const* d_scales,
                              const int64_t* n, int32_t count, float* const* d_x,
                              shampoo4_stream_t stream);

/* The 16 codebook levels and 15 thresholds the codec uses (host copy). */
shampoo4_status quant4_tables(float codebook[16], float thresholds[15]);

/* quant4_pack / quant4_unpack / quant4_tables with a shampoo4_codebook
 * (the plain names use SHAMPOO4_CODEBOOK_LINEAR_SQUARE); an unknown
 * codebook returns SHAMPOO4_ERR_INVALID_ARG. */
shampoo4_status quant4_pack_ex(const float* const* d_x, const int64_t* n, int32_t count,
                               uint8_t* const* d_codes, float* const* d_scales, int32_t codebook,
                               shampoo4_stream_t stream);
shampoo4_status quant4_unpack_ex(const uint8_t* const* d_codes, const float* const* d_scales,
                                 const int64_t* n, int32_t count, float* const* d_x, int32_t codebook,
                                 shampoo4_stream_t stream);
shampoo4_status quant4_tables_ex(int32_t codebook, float levels[16], float thresholds[15]);

/* Statistics update of ONE tile with no handle, no workspace and no device
 * allocation (no counterpart in the 4-bit Shampoo paper: an interface for
 * callers that cannot allocate device memory at the point of the call, such
 * as a hook running while a caching allocator holds its lock, or a process
 * whose device memory is fully reserved by another allocator).
 *   L <- beta L + (1 - beta) G G^T     (m x m, row-major, ld m)
 *   R <- beta R + (1 - beta) G^T G     (n x n, row-major, ld n)
 * G: m x n row-major device matrix, leading dimension ldg >= n.  The products
 * are TF32 (operands rounded to TF32, round to nearest; fp32 sums), like
 * shampoo4_update_stats with SHAMPOO4_PREC_TF32; L and R come out exactly
 * symmetric.  A gradient holding a NaN or an infinity leaves L and R
 * unchanged and ORs SHAMPOO4_FLAG_NONFINITE_GRAD into *d_flags (a device
 * word the caller owns and zeroes; optional, may be NULL).
 * Limits: m, n <= 1024 and m * n <= 2^18 (262144); larger tiles return
 * SHAMPOO4_ERR_WORKSPACE before touching the device.  Pointers 4-byte aligned;
 * other bad arguments return SHAMPOO4_ERR_INVALID_ARG.
 * Scratch is a fixed 1 MiB + 4 KiB device array inside the library (one per
 * device); every call resets what must start at zero.  Calls that overlap
 * (different streams or unordered host threads) share it and race: order
 * them.  Every call looks up the array's address in the current device's
 * context (cudaGetSymbolAddress: no allocation, and right again after a
 * context is destroyed and recreated).  The first call on a device may load
 * the module; make it before any stream capture.  Everything is enqueued on
 * `stream`; nothing is allocated or freed. */
shampoo4_status shampoo4_update_stats_noalloc(float* d_L, float* d_R, const float* d_G, int32_t m,
                                              int32_t n, int64_t ldg, float beta, uint32_t* d_flags,
                                              shampoo4_stream_t stream);

/* ---- Grafting and the weight update -------------------------------------
 * "Shampoo -- Second-Order Optimizer", section "Grafting: borrow a step size
 * that already works": Shampoo gives each tile's direction D_b (the output of
 * shampoo4_precondition), a method with a tuned step size gives its norm:
 *   step_b = lr * ||d_graft_b||_F / (||D_b||_F + graft_eps) * D_b,
 *   W_b   <- W_b - step_b,
 * with the Frobenius norms taken per tile of the handle's partition.
 * d_graft is the grafted method's step without its learning rate:
 *   SHAMPOO4_GRAFT_SGD   d_graft = G;
 *   SHAMPOO4_GRAFT_ADAM  Adam (Kingma and Ba, ICLR 2015, Algorithm 1):
 *     m <- beta1 m + (1 - beta1) G,  v <- beta2 v + (1 - beta2) G^2,
 *     d_graft = (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + adam_eps).
 * Arithmetic: fp32 elementwise (moments by fused multiply-adds, IEEE square
 * root and division); the norms are summed in fp64 in a fixed order; the
 * ratio lr * ||d_graft|| / (||D|| + graft_eps) is formed in fp64, rounded to
 * fp32 once, and W <- fma(-r, D, W).  A zero denominator gives a zero step. */
typedef enum { SHAMPOO4_GRAFT_SGD = 0, SHAMPOO4_GRAFT_ADAM = 1 } shampoo4_graft_kind;

typedef struct {
  int32_t kind;          /* shampoo4_graft_kind                              */
  float beta1, beta2;    /* Adam moment decays, in [0, 1) (ignored for SGD)   */
  float adam_eps;        /* Adam's denominator epsilon, >= 0                  */
  float graft_eps;       /* epsilon of the norm ratio, >= 0                   */
  int32_t dir_norms;     /* 0: ||D_b|| from d_dirs.  1: from the last
                            shampoo4_precondition on this handle, whose
                            tensor-core apply records each tile's sum of
                            squares as it writes D (fp32 sums of 32-element
                            row segments, added in fp64, then summed here in
                            a fixed order), so D is read once; d_dirs must
                            then be that call's output, unmodified.  Tiles on
                            the CUDA-core path, and every tile in FP32
                            precision, still read D.  Before any
                            precondition: SHAMPOO4_ERR_NOT_READY.            */
} shampoo4_graft_config;

/* Bytes of grafting state the caller provides for this handle's parameters:
 * Adam's two fp32 moments (8 bytes per parameter element; 0 for SGD).  The
 * buffer is 256-byte aligned and zero-filled by the caller before the first
 * step; it persists between steps (checkpointable). */
shampoo4_status shampoo4_graft_state_bytes(shampoo4_handle h, int32_t kind, size_t* bytes);

/* Byte offsets inside the grafting state of parameter p's first and second
 * moments (fp32, rows x cols, row-major, dense). */
shampoo4_status shampoo4_graft_layout(shampoo4_handle h, int32_t kind, int32_t param,
                                      size_t* off_m, size_t* off_v);

/* One grafted weight update of every parameter, enqueued on `stream` (two
 * kernel launches; no synchronization, no allocation).
 *   d_grads[p]   the step's gradient (the one passed to this step's
 *                shampoo4_update_stats), leading dimension ld_grads[p];
 *   d_dirs[p]    the step's Shampoo direction D (shampoo4_precondition's
 *                output), leading dimension ld_dirs[p];
 *   d_weights[p] the weights, updated in place, leading dimension
 *                ld_weights[p]; they must not overlap any gradient or
 *                direction;
 *   step         Adam's 1-based step counter t (bias correction);
 *   lr           the learning rate (finite).
 * A tile whose gradient the statistics update of this step flagged as
 * non-finite (SHAMPOO4_FLAG_NONFINITE_GRAD) is skipped whole: moments and
 * weights unchanged.  A tile whose ratio is not finite keeps its weights and
 * raises SHAMPOO4_FLAG_GRAFT_SKIPPED.  Pointers 4-byte aligned (16-byte
 * aligned rows take the vector path); bad arguments return
 * SHAMPOO4_ERR_INVALID_ARG, an unbound handle SHAMPOO4_ERR_NOT_READY. */
shampoo4_status shampoo4_graft_update(shampoo4_handle h, const shampoo4_graft_config* cfg,
                                      void* d_graft_state, int64_t step, float lr,
                                      const float* const* d_grads, const int64_t* ld_grads,
                                      const float* const* d_dirs, const int64_t* ld_dirs,
                                      float* const* d_weights, const int64_t* ld_weights,
                                      shampoo4_stream_t stream);

void shampoo4_destroy(shampoo4_handle h);
const char* shampoo4_status_string(shampoo4_status s);

#ifdef __cplusplus
}
#endif
#endif /* SHAMPOO4_H */
