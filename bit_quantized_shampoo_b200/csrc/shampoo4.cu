// shampoo4 runtime: planner, launch programs and the C ABI entry points.
//
// init     partitions every weight into tiles of at most max_block x
//          max_block ("Shampoo -- Second-Order Optimizer", "Blocked and
//          distributed variants": each tile preconditioned independently,
//          greedy chunks from index 0, ragged last chunk) and lays out the
//          caller-owned state and workspace.
// bind     writes every descriptor of every program into the workspace once;
//          a program is the fixed list of batched launches of one API call.
// calls    upload the per-call gradient/output addresses if they changed,
//          then replay their program on the caller's stream.
#include <algorithm>
#include <cstring>
#include <new>
#include <vector>

#include "plan.h"

using namespace s4;

namespace {

enum class Kind { GemmF32, GemmF64, Potrf, Trsm, Basis, Rayleigh, Mu, Scan, Convert, Pack, Shift };

struct Launch {
  Kind kind;
  int tag;             // stage label (shampoo4_stage)
  size_t desc_off;     // byte offset of the descriptor array in the workspace
  int count;
  int64_t extent;      // max tiles / rows / elements, per kind
  double flops = 0, bytes = 0;   // algorithmic work of the launch
  // Pack launches carry host-side tensor lists instead of descriptors.
  std::vector<const float*> px;
  std::vector<int64_t> pn;
  std::vector<uint8_t*> pcodes;
  std::vector<float*> pscales;
  std::vector<const uint32_t*> pskip;
};

struct BlockPlan {
  int32_t param;
  int64_t r0, c0;
  int32_t m, n;
};

struct FactorPlan {
  int32_t block, side, d;
  size_t st_S, st_codes, st_scales, st_lam;          // state offsets
  size_t ws_U, ws_T, ws_Y, ws_W64, ws_Q64, ws_mu;   // workspace offsets
  size_t ws_q_first, ws_q_next;                      // where each refresh program leaves Q
};

constexpr size_t kAlign = 256;
constexpr int kPanelW = 64;

}  // namespace

struct shampoo4_ctx {
  shampoo4_config cfg;
  std::vector<shampoo4_param> params;
  std::vector<BlockPlan> blocks;
  std::vector<FactorPlan> factors;
  size_t state_bytes = 0, ws_bytes = 0;
  // workspace regions
  size_t ws_flags = 0, ws_tabs = 0, ws_fail = 0, ws_bflag = 0, ws_desc = 0, ws_desc_bytes = 0;
  // programs
  std::vector<Launch> prog_stats, prog_refresh_first, prog_refresh, prog_precond;
  std::vector<uint8_t> arena;      // host image of the descriptor region
  // bound buffers
  uint8_t* d_state = nullptr;
  uint8_t* d_ws = nullptr;
  bool bound = false;
  bool has_basis = false;
  bool last_refresh_first = true;
  // per-call pointer tables
  std::vector<PtrEntry> tab_host;  // last uploaded (2 * nparams)
  bool tab_valid = false;
  PtrEntry* tab_pinned = nullptr;
  uint32_t* flags_pinned = nullptr;
  cudaEvent_t tab_event = nullptr;
  bool tab_event_pending = false;
  // optional per-launch timing (diagnostics)
  struct Rec { int tag; cudaEvent_t e0, e1; double flops, bytes; };
  bool timing = false;
  std::vector<cudaEvent_t> ev_pool;
  std::vector<Rec> recs;
  double t_ms[SHAMPOO4_STAGE_COUNT] = {};
  double t_flops[SHAMPOO4_STAGE_COUNT] = {};
  double t_bytes[SHAMPOO4_STAGE_COUNT] = {};
  int64_t t_launches[SHAMPOO4_STAGE_COUNT] = {};
};

namespace {

// ---------------------------------------------------------------- planning

std::vector<std::pair<int64_t, int32_t>> chunks(int64_t extent, int32_t b) {
  std::vector<std::pair<int64_t, int32_t>> out;
  for (int64_t s = 0; s < extent; s += b) out.push_back({s, int32_t(std::min<int64_t>(b, extent - s))});
  return out;
}

size_t take(size_t& cursor, size_t bytes) {
  size_t at = align_up(cursor, kAlign);
  cursor = at + bytes;
  return at;
}

shampoo4_status plan(shampoo4_ctx* h) {
  for (size_t p = 0; p < h->params.size(); ++p) {
    const shampoo4_param& q = h->params[p];
    for (auto rc : chunks(q.rows, h->cfg.max_block))
      for (auto cc : chunks(q.cols, h->cfg.max_block))
        h->blocks.push_back({int32_t(p), rc.first, cc.first, rc.second, cc.second});
  }
  if (h->blocks.size() > (1u << 30)) return SHAMPOO4_ERR_INVALID_ARG;
  size_t st = 0;
  for (size_t k = 0; k < h->blocks.size(); ++k) {
    for (int side = 0; side < 2; ++side) {
      FactorPlan f{};
      f.block = int32_t(k);
      f.side = side;
      f.d = side == 0 ? h->blocks[k].m : h->blocks[k].n;
      size_t dd = size_t(f.d) * f.d;
      f.st_S = take(st, 4 * dd);
      f.st_codes = take(st, (dd + 1) / 2);
      f.st_scales = take(st, 4 * ((dd + kQuantBlock - 1) / kQuantBlock));
      f.st_lam = take(st, 4 * size_t(f.d));
      h->factors.push_back(f);
    }
  }
  h->state_bytes = align_up(st, kAlign);

  size_t ws = 0;
  h->ws_flags = take(ws, 16);
  h->ws_tabs = take(ws, sizeof(PtrEntry) * 2 * h->params.size());
  h->ws_fail = take(ws, 4 * h->factors.size());
  h->ws_bflag = take(ws, 4 * h->blocks.size());
  for (FactorPlan& f : h->factors) {
    size_t dd = size_t(f.d) * f.d;
    f.ws_U = take(ws, 4 * dd);
    f.ws_T = take(ws, 4 * dd);
    f.ws_Y = take(ws, 4 * dd);
    f.ws_W64 = take(ws, 8 * dd);
    f.ws_Q64 = take(ws, 8 * dd);
    f.ws_mu = take(ws, 4 * size_t(f.d));
  }
  h->ws_desc = align_up(ws, kAlign);
  h->ws_bytes = h->ws_desc;     // descriptor bytes are added by build_programs
  return SHAMPOO4_OK;
}

// ---------------------------------------------------------- program builder

struct Builder {
  shampoo4_ctx* h;
  std::vector<uint8_t>& arena;
  uint8_t* ws;        // device workspace base (descriptors point into it)
  uint8_t* stb;       // device state base

  template <class D>
  size_t put(const std::vector<D>& v) {
    size_t at = align_up(arena.size(), kAlign);
    arena.resize(at + sizeof(D) * v.size());
    if (!v.empty()) std::memcpy(arena.data() + at, v.data(), sizeof(D) * v.size());
    return at;
  }
  int tag = 0;          // stage label applied to the launches emitted next
  template <class D>
  void emit(std::vector<Launch>& prog, Kind k, const std::vector<D>& v, int64_t extent,
            double flops = 0, double bytes = 0) {
    if (v.empty()) return;
    Launch L{};
    L.kind = k;
    L.tag = tag;
    L.desc_off = put(v);
    L.count = int(v.size());
    L.extent = extent;
    L.flops = flops;
    L.bytes = bytes;
    prog.push_back(std::move(L));
  }
  float* wf(size_t off) const { return reinterpret_cast<float*>(ws + off); }
  double* wd(size_t off) const { return reinterpret_cast<double*>(ws + off); }
  uint32_t* wu(size_t off) const { return reinterpret_cast<uint32_t*>(ws + off); }
  float* sf(size_t off) const { return reinterpret_cast<float*>(stb + off); }
  uint8_t* sb(size_t off) const { return stb + off; }
  uint32_t* fail(size_t fi) const { return wu(h->ws_fail) + fi; }
  uint32_t* gflags() const { return wu(h->ws_flags); }
};

int tiles128(int M, int N) { return ((M + 127) / 128) * ((N + 127) / 128); }
int tiles64(int M, int N) { return ((M + 63) / 64) * ((N + 63) / 64); }

GemmF32Desc gemm32(int M, int N, int K, int ta, int tb, int mode, float alpha, float beta) {
  GemmF32Desc g{};
  g.M = M; g.N = N; g.K = K; g.ta = ta; g.tb = tb; g.mode = mode;
  g.alpha = alpha; g.beta = beta;
  g.a_ref.tab = g.b_ref.tab = g.c_ref.tab = -1;
  return g;
}

// Algorithmic flops of a product: 2 M N K, or M (M+1) K for an output known
// to be symmetric (only one triangle is needed).
void emit_gemm32(Builder& b, std::vector<Launch>& prog, const std::vector<GemmF32Desc>& v) {
  int mt = 0;
  double fl = 0;
  for (auto& g : v) {
    mt = std::max(mt, tiles128(g.M, g.N));
    fl += g.symmetric ? double(g.M) * (g.M + 1) * g.K : 2.0 * g.M * g.N * g.K;
  }
  b.emit(prog, Kind::GemmF32, v, mt, fl);
}
void emit_gemm64(Builder& b, std::vector<Launch>& prog, const std::vector<GemmF64Desc>& v) {
  int mt = 0;
  double fl = 0;
  for (auto& g : v) {
    mt = std::max(mt, tiles64(g.M, g.N));
    fl += g.lower_only ? double(g.M) * (g.M + 1) * g.K : 2.0 * g.M * g.N * g.K;
  }
  b.emit(prog, Kind::GemmF64, v, mt, fl);
}

int mode_of(const shampoo4_config& c) { return c.precision == SHAMPOO4_PREC_FP32 ? kModeFP32 : kModeTF32; }

void build_stats(Builder& b) {
  shampoo4_ctx* h = b.h;
  std::vector<ScanDesc> scan;
  std::vector<GemmF32Desc> g;
  int64_t max_elems = 0;
  double bytes_scan = 0;
  const float beta = h->cfg.beta, omb = 1.0f - h->cfg.beta;
  for (size_t k = 0; k < h->blocks.size(); ++k) {
    const BlockPlan& bp = h->blocks[k];
    ScanDesc s{};
    s.rows = bp.m; s.cols = bp.n;
    s.ref = {0, bp.param, bp.r0, bp.c0};
    s.flag = b.wu(h->ws_bflag) + k;
    s.bit = SHAMPOO4_FLAG_NONFINITE_GRAD;
    scan.push_back(s);
    max_elems = std::max<int64_t>(max_elems, int64_t(bp.m) * bp.n);
    bytes_scan += 4.0 * bp.m * bp.n;
    for (int side = 0; side < 2; ++side) {
      const FactorPlan& f = h->factors[2 * k + side];
      GemmF32Desc d = side == 0 ? gemm32(bp.m, bp.m, bp.n, 0, 1, mode_of(h->cfg), omb, beta)
                                : gemm32(bp.n, bp.n, bp.m, 1, 0, mode_of(h->cfg), omb, beta);
      d.a_ref = {0, bp.param, bp.r0, bp.c0};
      d.b_ref = d.a_ref;
      d.C = b.sf(f.st_S); d.ldc = f.d;
      d.Cin = d.C; d.ldcin = f.d;
      d.symmetric = 1;
      d.skip = s.flag;
      g.push_back(d);
    }
  }
  b.tag = SHAMPOO4_STAGE_STATS_SCAN;
  b.emit(h->prog_stats, Kind::Scan, scan, max_elems, 0, bytes_scan);
  b.tag = SHAMPOO4_STAGE_STATS_GEMM;
  emit_gemm32(b, h->prog_stats, g);
}

// Cholesky-QR pass: X (fp32, d x d) -> Q (fp32) through fp64 Gram W = X^T X,
// blocked right-looking Cholesky W = L L^T and a blocked solve Q L^T = X.
void build_cholqr_pass(Builder& b, std::vector<Launch>& prog, const std::vector<size_t>& x_off,
                       const std::vector<size_t>& q_off, bool shifted) {
  shampoo4_ctx* h = b.h;
  const size_t nf = h->factors.size();
  int dmax = 0;
  for (auto& f : h->factors) dmax = std::max(dmax, f.d);
  {
    std::vector<GemmF64Desc> g;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      GemmF64Desc d{};
      d.M = d.N = d.K = f.d; d.ta = 1; d.tb = 0; d.lower_only = 1;
      d.A = b.wf(x_off[i]); d.lda = f.d; d.B = d.A; d.ldb = f.d;
      d.C = b.wd(f.ws_W64); d.ldc = f.d; d.c_f64 = 1;
      d.alpha = 1.0; d.beta = 0.0;
      d.skip = b.fail(i);
      g.push_back(d);
    }
    b.tag = SHAMPOO4_STAGE_QR_GRAM;
    emit_gemm64(b, prog, g);
  }
  if (shifted) {
    std::vector<ShiftDesc> sd;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      sd.push_back({b.wd(f.ws_W64), f.d, f.d, 0, b.fail(i)});
    }
    b.tag = SHAMPOO4_STAGE_QR_GRAM;
    b.emit(prog, Kind::Shift, sd, 0);
  }
  for (int j = 0; j < dmax; j += kPanelW) {
    std::vector<PotrfDesc> po;
    std::vector<TrsmDesc> tr;
    std::vector<GemmF64Desc> sy;
    int max_rows = 0;
    double fl_po = 0, fl_tr = 0;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      if (j >= f.d) continue;
      const int jb = std::min(kPanelW, f.d - j);
      double* W = b.wd(f.ws_W64);
      const int64_t ld = f.d;
      po.push_back({W + j * ld + j, ld, jb, 0, b.fail(i), b.gflags()});
      fl_po += double(jb) * jb * jb / 3.0;
      const int rest = f.d - j - jb;
      if (rest > 0) {
        fl_tr += double(rest) * jb * jb;
        tr.push_back({W + j * ld + j, ld, W + (j + jb) * ld + j, ld, jb, rest});
        max_rows = std::max(max_rows, rest);
        GemmF64Desc d{};
        d.M = d.N = rest; d.K = jb; d.ta = 0; d.tb = 1; d.lower_only = 1;
        d.a_f64 = d.b_f64 = d.c_f64 = d.cin_f64 = 1;
        d.A = W + (j + jb) * ld + j; d.lda = ld; d.B = d.A; d.ldb = ld;
        d.C = W + (j + jb) * ld + (j + jb); d.ldc = ld; d.Cin = d.C; d.ldcin = ld;
        d.alpha = -1.0; d.beta = 1.0;
        sy.push_back(d);
      }
    }
    b.tag = SHAMPOO4_STAGE_QR_POTRF;
    b.emit(prog, Kind::Potrf, po, 0, fl_po);
    b.tag = SHAMPOO4_STAGE_QR_TRSM_PANEL;
    b.emit(prog, Kind::Trsm, tr, max_rows, fl_tr);
    b.tag = SHAMPOO4_STAGE_QR_SYRK;
    emit_gemm64(b, prog, sy);
  }
  // Solve Q L^T = X by column panels.
  for (int j = 0; j < dmax; j += kPanelW) {
    std::vector<GemmF64Desc> up;
    std::vector<TrsmDesc> tr;
    int max_rows = 0;
    double fl_tr = 0;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      if (j >= f.d) continue;
      const int jb = std::min(kPanelW, f.d - j);
      const int64_t ld = f.d;
      fl_tr += double(f.d) * jb * jb;
      double* W = b.wd(f.ws_W64);
      double* Q = b.wd(f.ws_Q64);
      GemmF64Desc d{};
      d.M = f.d; d.N = jb; d.K = j; d.ta = 0; d.tb = 1;
      d.a_f64 = 1; d.b_f64 = 1; d.c_f64 = 1; d.cin_f64 = 0;
      d.A = Q; d.lda = ld; d.B = W + j * ld; d.ldb = ld;
      d.C = Q + j; d.ldc = ld; d.Cin = b.wf(x_off[i]) + j; d.ldcin = ld;
      d.alpha = -1.0; d.beta = 1.0;
      d.skip = b.fail(i);
      up.push_back(d);
      tr.push_back({W + j * ld + j, ld, Q + j, ld, jb, f.d});
      max_rows = std::max(max_rows, f.d);
    }
    b.tag = SHAMPOO4_STAGE_QR_SOLVE_UPDATE;
    emit_gemm64(b, prog, up);
    b.tag = SHAMPOO4_STAGE_QR_SOLVE_PANEL;
    b.emit(prog, Kind::Trsm, tr, max_rows, fl_tr);
  }
  std::vector<ConvertDesc> cv;
  int64_t max_elems = 0;
  double bytes_cv = 0;
  for (size_t i = 0; i < nf; ++i) {
    const FactorPlan& f = h->factors[i];
    int64_t n = int64_t(f.d) * f.d;
    cv.push_back({b.wd(f.ws_Q64), b.wf(q_off[i]), n});
    bytes_cv += 12.0 * double(n);
    max_elems = std::max(max_elems, n);
  }
  b.tag = SHAMPOO4_STAGE_QR_CONVERT;
  b.emit(prog, Kind::Convert, cv, max_elems, 0, bytes_cv);
}

void build_refresh(Builder& b, std::vector<Launch>& prog, bool first) {
  shampoo4_ctx* h = b.h;
  const size_t nf = h->factors.size();
  int dmax = 0;
  int64_t emax = 0;
  double sum_dd = 0;
  for (auto& f : h->factors) {
    dmax = std::max(dmax, f.d);
    emax = std::max<int64_t>(emax, int64_t(f.d) * f.d);
    sum_dd += double(f.d) * f.d;
  }
  const double bytes_scan = 4.0 * sum_dd, fl_rq = 2.0 * sum_dd;
  const double bytes_bd = first ? 4.0 * sum_dd : 4.5625 * sum_dd;
  {  // non-finite statistic -> keep the factor's previous basis
    std::vector<ScanDesc> scan;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      ScanDesc s{};
      s.X = b.sf(f.st_S); s.ld = f.d; s.rows = s.cols = f.d;
      s.ref.tab = -1;
      s.flag = b.fail(i);
      s.bit = SHAMPOO4_FLAG_NONFINITE_STATE;
      scan.push_back(s);
    }
    b.tag = SHAMPOO4_STAGE_REFRESH_SCAN;
    b.emit(prog, Kind::Scan, scan, emax, 0, bytes_scan);
  }
  {
    std::vector<BasisDesc> bd;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      bd.push_back({b.sb(f.st_codes), b.sf(f.st_scales), b.wf(f.ws_U), f.d, first ? 1 : 0});
    }
    b.tag = SHAMPOO4_STAGE_BASIS;
    b.emit(prog, Kind::Basis, bd, emax, 0, bytes_bd);
  }
  // Bjorck rectification U <- 1.5 U - 0.5 U (U^T U), ping-ponging U and Y.
  std::vector<size_t> cur(nf), other(nf);
  for (size_t i = 0; i < nf; ++i) { cur[i] = h->factors[i].ws_U; other[i] = h->factors[i].ws_Y; }
  const int iters = first ? 0 : h->cfg.bjorck_iters;
  for (int it = 0; it < iters; ++it) {
    std::vector<GemmF32Desc> gram, upd;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      GemmF32Desc g = gemm32(f.d, f.d, f.d, 1, 0, mode_of(h->cfg), 1.0f, 0.0f);
      g.A = g.B = b.wf(cur[i]); g.lda = g.ldb = f.d;
      g.C = b.wf(f.ws_T); g.ldc = f.d;
      g.symmetric = 1;
      gram.push_back(g);
      GemmF32Desc u = gemm32(f.d, f.d, f.d, 0, 0, mode_of(h->cfg), -0.5f, 1.5f);
      u.A = b.wf(cur[i]); u.lda = f.d;
      u.B = b.wf(f.ws_T); u.ldb = f.d;
      u.C = b.wf(other[i]); u.ldc = f.d;
      u.Cin = b.wf(cur[i]); u.ldcin = f.d;
      upd.push_back(u);
    }
    b.tag = SHAMPOO4_STAGE_BJORCK_GRAM;
    emit_gemm32(b, prog, gram);
    b.tag = SHAMPOO4_STAGE_BJORCK_UPDATE;
    emit_gemm32(b, prog, upd);
    std::swap(cur, other);
  }
  // Subspace step Y = (S + eps I) U = S U + eps U, fp32-accurate.
  {
    std::vector<GemmF32Desc> g;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      GemmF32Desc y = gemm32(f.d, f.d, f.d, 0, 0, kModeFP32, 1.0f, h->cfg.eps);
      y.A = b.sf(f.st_S); y.lda = f.d;
      y.B = b.wf(cur[i]); y.ldb = f.d;
      y.C = b.wf(other[i]); y.ldc = f.d;
      y.Cin = b.wf(cur[i]); y.ldcin = f.d;
      g.push_back(y);
    }
    b.tag = SHAMPOO4_STAGE_SUBSPACE;
    emit_gemm32(b, prog, g);
  }
  // Shifted CholeskyQR3: a shifted pass on Y (in `other`) -> Q0 into `cur`,
  // then two plain passes cur -> other -> cur.  Q ends in `cur`.
  build_cholqr_pass(b, prog, other, cur, true);
  build_cholqr_pass(b, prog, cur, other, false);
  build_cholqr_pass(b, prog, other, cur, false);
  std::swap(cur, other);                    // from here on Q is `other`
  for (size_t i = 0; i < nf; ++i) (first ? h->factors[i].ws_q_first : h->factors[i].ws_q_next) = other[i];
  // Rayleigh quotients: T = S Q (fp32-accurate), lambda_i = max(q_i . t_i, 0).
  {
    std::vector<GemmF32Desc> g;
    std::vector<RayleighDesc> rq;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      GemmF32Desc t = gemm32(f.d, f.d, f.d, 0, 0, kModeFP32, 1.0f, 0.0f);
      t.A = b.sf(f.st_S); t.lda = f.d;
      t.B = b.wf(other[i]); t.ldb = f.d;
      t.C = b.wf(f.ws_T); t.ldc = f.d;
      g.push_back(t);
      rq.push_back({b.wf(other[i]), b.wf(f.ws_T), b.sf(f.st_lam), f.d, 0, b.fail(i)});
    }
    b.tag = SHAMPOO4_STAGE_RAYLEIGH_GEMM;
    emit_gemm32(b, prog, g);
    b.tag = SHAMPOO4_STAGE_RAYLEIGH;
    b.emit(prog, Kind::Rayleigh, rq, dmax, fl_rq);
  }
  // Requantize Q into the state (skipped for failed factors).
  {
    Launch L{};
    L.kind = Kind::Pack;
    L.tag = SHAMPOO4_STAGE_REQUANT;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      L.px.push_back(b.wf(other[i]));
      L.pn.push_back(int64_t(f.d) * f.d);
      L.pcodes.push_back(b.sb(f.st_codes));
      L.pscales.push_back(b.sf(f.st_scales));
      L.pskip.push_back(b.fail(i));
      L.bytes += 4.5625 * double(f.d) * f.d;
    }
    L.count = int(nf);
    prog.push_back(std::move(L));
  }
}

void build_precondition(Builder& b) {
  shampoo4_ctx* h = b.h;
  const size_t nf = h->factors.size();
  int dmax = 0;
  int64_t emax = 0;
  double sum_dd = 0;
  for (auto& f : h->factors) {
    dmax = std::max(dmax, f.d);
    emax = std::max<int64_t>(emax, int64_t(f.d) * f.d);
    sum_dd += double(f.d) * f.d;
  }
  const double bytes_bd = 4.5625 * sum_dd;
  std::vector<BasisDesc> bd;
  std::vector<MuDesc> mu;
  std::vector<GemmF32Desc> roots;
  for (size_t i = 0; i < nf; ++i) {
    const FactorPlan& f = h->factors[i];
    bd.push_back({b.sb(f.st_codes), b.sf(f.st_scales), b.wf(f.ws_Y), f.d, 0});
    mu.push_back({b.sf(f.st_lam), b.wf(f.ws_mu), f.d, 0});
    // P = (U diag(mu)) U^T
    GemmF32Desc g = gemm32(f.d, f.d, f.d, 0, 1, mode_of(h->cfg), 1.0f, 0.0f);
    g.A = b.wf(f.ws_Y); g.lda = f.d; g.kscale = b.wf(f.ws_mu);
    g.B = b.wf(f.ws_Y); g.ldb = f.d;
    g.C = b.wf(f.ws_U); g.ldc = f.d;
    g.symmetric = 1;
    roots.push_back(g);
  }
  b.tag = SHAMPOO4_STAGE_PRECOND_DEQUANT;
  b.emit(h->prog_precond, Kind::Basis, bd, emax, 0, bytes_bd);
  b.tag = SHAMPOO4_STAGE_PRECOND_MU;
  b.emit(h->prog_precond, Kind::Mu, mu, dmax);
  b.tag = SHAMPOO4_STAGE_ROOTS;
  emit_gemm32(b, h->prog_precond, roots);
  std::vector<GemmF32Desc> left, right;
  for (size_t k = 0; k < h->blocks.size(); ++k) {
    const BlockPlan& bp = h->blocks[k];
    const FactorPlan& fl = h->factors[2 * k];
    const FactorPlan& fr = h->factors[2 * k + 1];
    float* tmp = b.wf(bp.m >= bp.n ? fl.ws_T : fr.ws_T);   // m x n fits in max(m,n)^2
    GemmF32Desc l = gemm32(bp.m, bp.n, bp.m, 0, 0, mode_of(h->cfg), 1.0f, 0.0f);
    l.A = b.wf(fl.ws_U); l.lda = bp.m;
    l.b_ref = {0, bp.param, bp.r0, bp.c0};
    l.C = tmp; l.ldc = bp.n;
    left.push_back(l);
    GemmF32Desc r = gemm32(bp.m, bp.n, bp.n, 0, 0, mode_of(h->cfg), 1.0f, 0.0f);
    r.A = tmp; r.lda = bp.n;
    r.B = b.wf(fr.ws_U); r.ldb = bp.n;
    r.c_ref = {1, bp.param, bp.r0, bp.c0};
    right.push_back(r);
  }
  b.tag = SHAMPOO4_STAGE_APPLY_LEFT;
  emit_gemm32(b, h->prog_precond, left);
  b.tag = SHAMPOO4_STAGE_APPLY_RIGHT;
  emit_gemm32(b, h->prog_precond, right);
}

cudaEvent_t take_event(shampoo4_ctx* h) {
  if (!h->ev_pool.empty()) {
    cudaEvent_t e = h->ev_pool.back();
    h->ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

shampoo4_status run(shampoo4_ctx* h, const std::vector<Launch>& prog, cudaStream_t st) {
  const PtrEntry* tabs = reinterpret_cast<const PtrEntry*>(h->d_ws + h->ws_tabs);
  const int np = int(h->params.size());
  uint32_t* gflags = reinterpret_cast<uint32_t*>(h->d_ws + h->ws_flags);
  for (const Launch& L : prog) {
    const void* d = h->d_ws + h->ws_desc + L.desc_off;
    shampoo4_ctx::Rec rec{L.tag, nullptr, nullptr, L.flops, L.bytes};
    if (h->timing) {
      rec.e0 = take_event(h);
      rec.e1 = take_event(h);
      if (!rec.e0 || !rec.e1) return SHAMPOO4_ERR_CUDA;
      S4_CUDA(cudaEventRecord(rec.e0, st));
    }
    switch (L.kind) {
      case Kind::GemmF32:
        S4_TRY(launch_gemm_f32(static_cast<const GemmF32Desc*>(d), L.count, int(L.extent), tabs, np, st));
        break;
      case Kind::GemmF64:
        S4_TRY(launch_gemm_f64(static_cast<const GemmF64Desc*>(d), L.count, int(L.extent), st));
        break;
      case Kind::Potrf:
        S4_TRY(launch_potrf(static_cast<const PotrfDesc*>(d), L.count, st));
        break;
      case Kind::Trsm:
        S4_TRY(launch_trsm(static_cast<const TrsmDesc*>(d), L.count, int(L.extent), st));
        break;
      case Kind::Basis:
        S4_TRY(launch_basis(static_cast<const BasisDesc*>(d), L.count, L.extent, st));
        break;
      case Kind::Rayleigh:
        S4_TRY(launch_rayleigh(static_cast<const RayleighDesc*>(d), L.count, int(L.extent), st));
        break;
      case Kind::Mu:
        S4_TRY(launch_mu(static_cast<const MuDesc*>(d), L.count, int(L.extent), h->cfg.eps, st));
        break;
      case Kind::Scan:
        S4_TRY(launch_scan(static_cast<const ScanDesc*>(d), L.count, L.extent, tabs, np, gflags, st));
        break;
      case Kind::Shift:
        S4_TRY(launch_shift(static_cast<const ShiftDesc*>(d), L.count, st));
        break;
      case Kind::Convert:
        S4_TRY(launch_convert(static_cast<const ConvertDesc*>(d), L.count, L.extent, st));
        break;
      case Kind::Pack:
        S4_TRY(launch_pack(L.px.data(), L.pn.data(), L.count, L.pcodes.data(), L.pscales.data(), st,
                           L.pskip.data()));
        break;
    }
    if (h->timing) {
      S4_CUDA(cudaEventRecord(rec.e1, st));
      h->recs.push_back(rec);
    }
  }
  return SHAMPOO4_OK;
}

shampoo4_status collect_timing(shampoo4_ctx* h) {
  for (auto& r : h->recs) {
    S4_CUDA(cudaEventSynchronize(r.e1));
    float ms = 0;
    S4_CUDA(cudaEventElapsedTime(&ms, r.e0, r.e1));
    h->t_ms[r.tag] += ms;
    h->t_flops[r.tag] += r.flops;
    h->t_bytes[r.tag] += r.bytes;
    h->t_launches[r.tag] += 1;
    h->ev_pool.push_back(r.e0);
    h->ev_pool.push_back(r.e1);
  }
  h->recs.clear();
  return SHAMPOO4_OK;
}

// Upload the per-call pointer table when any entry changed.
shampoo4_status set_tables(shampoo4_ctx* h, const float* const* grads, const int64_t* ld,
                           float* const* outs, const int64_t* ld_out, cudaStream_t st) {
  const size_t np = h->params.size();
  std::vector<PtrEntry> want = h->tab_valid ? h->tab_host : std::vector<PtrEntry>(2 * np, PtrEntry{nullptr, 0});
  for (size_t p = 0; p < np; ++p) {
    want[p] = {grads[p], ld[p]};
    if (outs) want[np + p] = {outs[p], ld_out[p]};
  }
  if (h->tab_valid && std::memcmp(want.data(), h->tab_host.data(), sizeof(PtrEntry) * 2 * np) == 0)
    return SHAMPOO4_OK;
  if (h->tab_event_pending) S4_CUDA(cudaEventSynchronize(h->tab_event));
  std::memcpy(h->tab_pinned, want.data(), sizeof(PtrEntry) * 2 * np);
  S4_CUDA(cudaMemcpyAsync(h->d_ws + h->ws_tabs, h->tab_pinned, sizeof(PtrEntry) * 2 * np,
                          cudaMemcpyHostToDevice, st));
  S4_CUDA(cudaEventRecord(h->tab_event, st));
  h->tab_event_pending = true;
  h->tab_host = want;
  h->tab_valid = true;
  return SHAMPOO4_OK;
}

shampoo4_status check_matrices(const shampoo4_ctx* h, const float* const* p, const int64_t* ld) {
  if (!p || !ld) return SHAMPOO4_ERR_INVALID_ARG;
  for (size_t i = 0; i < h->params.size(); ++i) {
    if (!p[i] || !aligned(p[i], 4)) return SHAMPOO4_ERR_INVALID_ARG;
    if (ld[i] < h->params[i].cols) return SHAMPOO4_ERR_INVALID_ARG;
  }
  return SHAMPOO4_OK;
}

}  // namespace

// ===================================================================== ABI

extern "C" shampoo4_status shampoo4_init(const shampoo4_config* cfg, const shampoo4_param* params,
                                         int32_t nparams, shampoo4_handle* out) {
  if (!cfg || !out || nparams <= 0 || !params) return SHAMPOO4_ERR_INVALID_ARG;
  *out = nullptr;
  if (!(cfg->beta >= 0.0f && cfg->beta < 1.0f)) return SHAMPOO4_ERR_INVALID_ARG;
  if (!(cfg->eps > 0.0f) || !(cfg->eps < 3.0e38f)) return SHAMPOO4_ERR_INVALID_ARG;
  if (cfg->max_block < 1 || cfg->max_block > 1024) return SHAMPOO4_ERR_INVALID_ARG;
  if (cfg->quant_block != kQuantBlock) return SHAMPOO4_ERR_INVALID_ARG;
  if (cfg->bjorck_iters < 0 || cfg->bjorck_iters > 16) return SHAMPOO4_ERR_INVALID_ARG;
  if (cfg->precision != SHAMPOO4_PREC_TF32 && cfg->precision != SHAMPOO4_PREC_FP32)
    return SHAMPOO4_ERR_INVALID_ARG;
  for (int32_t i = 0; i < nparams; ++i)
    if (params[i].rows < 1 || params[i].cols < 1 || params[i].rows > (1LL << 31) ||
        params[i].cols > (1LL << 31))
      return SHAMPOO4_ERR_INVALID_ARG;
  shampoo4_ctx* h = new (std::nothrow) shampoo4_ctx();
  if (!h) return SHAMPOO4_ERR_INVALID_ARG;
  h->cfg = *cfg;
  h->params.assign(params, params + nparams);
  shampoo4_status s = plan(h);
  if (s != SHAMPOO4_OK) { delete h; return s; }
  // Descriptor bytes: build the programs once against a null base to size
  // the arena; bind rebuilds them with the real addresses.
  Builder b{h, h->arena, nullptr, nullptr};
  build_stats(b);
  build_refresh(b, h->prog_refresh_first, true);
  build_refresh(b, h->prog_refresh, false);
  build_precondition(b);
  h->ws_desc_bytes = align_up(h->arena.size(), kAlign);
  h->ws_bytes = h->ws_desc + h->ws_desc_bytes;
  h->prog_stats.clear(); h->prog_refresh_first.clear(); h->prog_refresh.clear(); h->prog_precond.clear();
  h->arena.clear();
  *out = h;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_sizes(shampoo4_handle h, size_t* state_bytes, size_t* workspace_bytes) {
  if (!h) return SHAMPOO4_ERR_INVALID_ARG;
  if (state_bytes) *state_bytes = h->state_bytes;
  if (workspace_bytes) *workspace_bytes = h->ws_bytes;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_bind(shampoo4_handle h, void* d_state, void* d_workspace,
                                         int32_t reset, shampoo4_stream_t stream) {
  if (!h || !d_state || !d_workspace) return SHAMPOO4_ERR_INVALID_ARG;
  if (!aligned(d_state, kAlign) || !aligned(d_workspace, kAlign)) return SHAMPOO4_ERR_INVALID_ARG;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SHAMPOO4_ERR_UNSUPPORTED;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10)
    return SHAMPOO4_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!h->tab_pinned) {
    S4_CUDA(cudaHostAlloc(&h->tab_pinned, sizeof(PtrEntry) * 2 * h->params.size() + 64, cudaHostAllocDefault));
    S4_CUDA(cudaHostAlloc(&h->flags_pinned, 64, cudaHostAllocDefault));
    S4_CUDA(cudaEventCreateWithFlags(&h->tab_event, cudaEventDisableTiming));
  }
  if (h->tab_event_pending) S4_CUDA(cudaEventSynchronize(h->tab_event));
  h->d_state = static_cast<uint8_t*>(d_state);
  h->d_ws = static_cast<uint8_t*>(d_workspace);
  h->prog_stats.clear(); h->prog_refresh_first.clear(); h->prog_refresh.clear(); h->prog_precond.clear();
  h->arena.clear();
  Builder b{h, h->arena, h->d_ws, h->d_state};
  build_stats(b);
  build_refresh(b, h->prog_refresh_first, true);
  build_refresh(b, h->prog_refresh, false);
  build_precondition(b);
  if (align_up(h->arena.size(), kAlign) != h->ws_desc_bytes) return SHAMPOO4_ERR_WORKSPACE;
  S4_CUDA(cudaMemcpyAsync(h->d_ws + h->ws_desc, h->arena.data(), h->arena.size(), cudaMemcpyHostToDevice, st));
  S4_CUDA(cudaMemsetAsync(h->d_ws, 0, h->ws_desc, st));
  if (reset) {
    S4_CUDA(cudaMemsetAsync(h->d_state, 0, h->state_bytes, st));
    h->has_basis = false;
  }
  S4_CUDA(cudaStreamSynchronize(st));   // the host arena is reused by the next bind
  h->tab_valid = false;
  h->bound = true;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_set_has_basis(shampoo4_handle h, int32_t has_basis) {
  if (!h) return SHAMPOO4_ERR_INVALID_ARG;
  h->has_basis = has_basis != 0;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_update_stats(shampoo4_handle h, const float* const* d_grads,
                                                 const int64_t* ld, shampoo4_stream_t stream) {
  if (!h) return SHAMPOO4_ERR_INVALID_ARG;
  if (!h->bound) return SHAMPOO4_ERR_NOT_READY;
  S4_TRY(check_matrices(h, d_grads, ld));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  S4_TRY(set_tables(h, d_grads, ld, nullptr, nullptr, st));
  S4_CUDA(cudaMemsetAsync(h->d_ws + h->ws_bflag, 0, 4 * h->blocks.size(), st));
  return run(h, h->prog_stats, st);
}

extern "C" shampoo4_status shampoo4_refresh_roots(shampoo4_handle h, shampoo4_stream_t stream) {
  if (!h) return SHAMPOO4_ERR_INVALID_ARG;
  if (!h->bound) return SHAMPOO4_ERR_NOT_READY;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  S4_CUDA(cudaMemsetAsync(h->d_ws + h->ws_fail, 0, 4 * h->factors.size(), st));
  const bool first = !h->has_basis;
  S4_TRY(run(h, first ? h->prog_refresh_first : h->prog_refresh, st));
  h->last_refresh_first = first;
  h->has_basis = true;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_precondition(shampoo4_handle h, const float* const* d_grads,
                                                 const int64_t* ld, float* const* d_out,
                                                 const int64_t* ld_out, shampoo4_stream_t stream) {
  if (!h) return SHAMPOO4_ERR_INVALID_ARG;
  if (!h->bound || !h->has_basis) return SHAMPOO4_ERR_NOT_READY;
  S4_TRY(check_matrices(h, d_grads, ld));
  S4_TRY(check_matrices(h, const_cast<const float* const*>(d_out), ld_out));
  // d_out must not overlap any gradient
  for (size_t i = 0; i < h->params.size(); ++i) {
    const uintptr_t o0 = uintptr_t(d_out[i]);
    const uintptr_t o1 = o0 + 4 * uintptr_t((h->params[i].rows - 1) * ld_out[i] + h->params[i].cols);
    for (size_t j = 0; j < h->params.size(); ++j) {
      const uintptr_t g0 = uintptr_t(d_grads[j]);
      const uintptr_t g1 = g0 + 4 * uintptr_t((h->params[j].rows - 1) * ld[j] + h->params[j].cols);
      if (o0 < g1 && g0 < o1) return SHAMPOO4_ERR_INVALID_ARG;
    }
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  S4_TRY(set_tables(h, d_grads, ld, d_out, ld_out, st));
  return run(h, h->prog_precond, st);
}

extern "C" shampoo4_status shampoo4_get_status_flags(shampoo4_handle h, uint32_t* flags,
                                                     shampoo4_stream_t stream) {
  if (!h || !flags) return SHAMPOO4_ERR_INVALID_ARG;
  if (!h->bound) return SHAMPOO4_ERR_NOT_READY;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  S4_CUDA(cudaMemcpyAsync(h->flags_pinned, h->d_ws + h->ws_flags, 4, cudaMemcpyDeviceToHost, st));
  S4_CUDA(cudaMemsetAsync(h->d_ws + h->ws_flags, 0, 4, st));
  S4_CUDA(cudaStreamSynchronize(st));
  *flags = h->flags_pinned[0];
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_counts(shampoo4_handle h, int32_t* nblocks, int32_t* nfactors) {
  if (!h) return SHAMPOO4_ERR_INVALID_ARG;
  if (nblocks) *nblocks = int32_t(h->blocks.size());
  if (nfactors) *nfactors = int32_t(h->factors.size());
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_block_info(shampoo4_handle h, int32_t block, int32_t* param,
                                               int64_t* r0, int64_t* c0, int32_t* m, int32_t* n) {
  if (!h || block < 0 || size_t(block) >= h->blocks.size()) return SHAMPOO4_ERR_INVALID_ARG;
  const BlockPlan& b = h->blocks[block];
  if (param) *param = b.param;
  if (r0) *r0 = b.r0;
  if (c0) *c0 = b.c0;
  if (m) *m = b.m;
  if (n) *n = b.n;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_factor_layout(shampoo4_handle h, int32_t factor, size_t* off_S,
                                                  size_t* off_codes, size_t* off_scales,
                                                  size_t* off_lambda, int32_t* dim) {
  if (!h || factor < 0 || size_t(factor) >= h->factors.size()) return SHAMPOO4_ERR_INVALID_ARG;
  const FactorPlan& f = h->factors[factor];
  if (off_S) *off_S = f.st_S;
  if (off_codes) *off_codes = f.st_codes;
  if (off_scales) *off_scales = f.st_scales;
  if (off_lambda) *off_lambda = f.st_lam;
  if (dim) *dim = f.d;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_debug_q_offset(shampoo4_handle h, int32_t factor, size_t* off_q) {
  if (!h || !off_q || factor < 0 || size_t(factor) >= h->factors.size()) return SHAMPOO4_ERR_INVALID_ARG;
  if (!h->bound) return SHAMPOO4_ERR_NOT_READY;
  *off_q = h->last_refresh_first ? h->factors[factor].ws_q_first : h->factors[factor].ws_q_next;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_timing_enable(shampoo4_handle h, int32_t enable) {
  if (!h) return SHAMPOO4_ERR_INVALID_ARG;
  S4_TRY(collect_timing(h));
  for (int i = 0; i < SHAMPOO4_STAGE_COUNT; ++i) {
    h->t_ms[i] = h->t_flops[i] = h->t_bytes[i] = 0;
    h->t_launches[i] = 0;
  }
  h->timing = enable != 0;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_timing_read(shampoo4_handle h, int32_t stage, double* ms,
                                                int64_t* launches, double* flops, double* bytes) {
  if (!h || stage < 0 || stage >= SHAMPOO4_STAGE_COUNT) return SHAMPOO4_ERR_INVALID_ARG;
  S4_TRY(collect_timing(h));
  if (ms) *ms = h->t_ms[stage];
  if (launches) *launches = h->t_launches[stage];
  if (flops) *flops = h->t_flops[stage];
  if (bytes) *bytes = h->t_bytes[stage];
  return SHAMPOO4_OK;
}

extern "C" const char* shampoo4_stage_name(int32_t stage) {
  static const char* names[SHAMPOO4_STAGE_COUNT] = {
      "stats_scan", "stats_gemm", "refresh_scan", "basis", "bjorck_gram", "bjorck_update",
      "subspace", "qr_gram", "qr_potrf", "qr_trsm_panel", "qr_syrk", "qr_solve_update",
      "qr_solve_panel", "qr_convert", "rayleigh_gemm", "rayleigh", "requant", "precond_dequant",
      "precond_mu", "roots", "apply_left", "apply_right"};
  if (stage < 0 || stage >= SHAMPOO4_STAGE_COUNT) return "unknown";
  return names[stage];
}

extern "C" void shampoo4_destroy(shampoo4_handle h) {
  if (!h) return;
  collect_timing(h);
  for (cudaEvent_t e : h->ev_pool) cudaEventDestroy(e);
  if (h->tab_event) {
    cudaEventSynchronize(h->tab_event);
    cudaEventDestroy(h->tab_event);
  }
  if (h->tab_pinned) cudaFreeHost(h->tab_pinned);
  if (h->flags_pinned) cudaFreeHost(h->flags_pinned);
  delete h;
}

extern "C" const char* shampoo4_status_string(shampoo4_status s) {
  switch (s) {
    case SHAMPOO4_OK: return "ok";
    case SHAMPOO4_ERR_INVALID_ARG: return "invalid argument";
    case SHAMPOO4_ERR_CUDA: return "CUDA error";
    case SHAMPOO4_ERR_NOT_READY: return "not ready (unbound, or no refresh yet)";
    case SHAMPOO4_ERR_NONFINITE: return "non-finite input";
    case SHAMPOO4_ERR_WORKSPACE: return "workspace too small";
    case SHAMPOO4_ERR_UNSUPPORTED: return "needs a compute capability 10.x device";
    case SHAMPOO4_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}
