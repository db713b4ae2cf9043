// shampoo4 runtime: planner, launch programs and the C ABI entry points.
//
// init     partitions every weight into tiles of at most max_block x
//          max_block ("Shampoo -- Second-Order Optimizer", "Blocked and
//          distributed variants": each tile preconditioned independently,
//          greedy chunks from index 0, ragged last chunk) and lays out the
//          caller-owned state and workspace.
// bind     writes every descriptor and TMA tensor map of every program into
//          the workspace once; a program is the fixed list of batched
//          launches of one API call.
// calls    upload the per-call gradient/output addresses if they changed,
//          then replay their program on the caller's stream.
//
// Kernel choice: a factor whose dimension is a multiple of 4 (rows 16-byte
// aligned, as TMA needs) runs its products on the tensor cores (gemm_tc.cu);
// a tile whose both sides are multiples of 4 does too.  The rest use the
// CUDA-core kernels (gemm_simt.cu).  Both produce the same state.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <new>
#include <tuple>
#include <vector>

#include "tc.h"

using namespace s4;

namespace {

enum class Kind { GemmF32, GemmF64, Potrf, Trsm, Basis, Rayleigh, Mu, Scan, Convert, Pack, Shift, GemmTC, GemmTCSplit,
                  GemmTCSplit64, PotrfF, ShiftF, Gate, Diag, RowDiag, Inv128, Copy, NewtonNorm, NewtonElt,
                  SketchZ, SketchR };

struct Launch {
  Kind kind;
  int tag;             // stage label (shampoo4_stage)
  size_t desc_off;     // byte offset of the descriptor array in the workspace
  int count;
  int64_t extent;      // max tiles / rows / elements, per kind
  double flops = 0, bytes = 0;   // algorithmic work of the launch
  size_t guard_off = SIZE_MAX;   // workspace word gating the whole launch (fp64 QR passes)
  int64_t tiles = -1;            // tensor-core products: the batch's running tiles
  size_t list_off = SIZE_MAX;    // persistent products: byte offset of the tile list
  // Pack launches carry host-side tensor lists instead of descriptors.
  std::vector<const float*> px;
  std::vector<int64_t> pn;
  std::vector<uint8_t*> pcodes;
  std::vector<float*> pscales;
  std::vector<const uint32_t*> pskip;
};

// The launches of one API call: one or more sequences, each run in order
// on a lane: -1 is the caller's stream, p >= 0 the handle's stream p
// (forked from and joined back to the caller's stream).
struct Program {
  std::vector<std::vector<Launch>> seq;
  std::vector<int> lane;
  void clear() { seq.clear(); lane.clear(); }
  std::vector<Launch>& add(int l) {
    seq.emplace_back();
    lane.push_back(l);
    return seq.back();
  }
};

struct BlockPlan {
  int32_t param;
  int64_t r0, c0;
  int32_t m, n;
  bool tc;
  size_t ws_Gh, ws_Gl, ws_Bh, ws_Bl;   // tensor-core path: G split, apply intermediate split
  size_t ws_tmp;                       // CUDA-core path: apply intermediate
  int64_t dsq_off = 0;                 // tensor-core path: the apply's recorded sums of squares
  int32_t dsq_n = 0;                   // of D (4 per output tile), in the ws_dsq array
};

// Per-factor workspace.  Tensor-core factors: fp32/TF32-split triplets
// X[0], X[1], Z (m = fp32, h/l = TF32 split), a split Gram or Cholesky
// factor Th/Tl, the split of S (Sh/Sl), the fp32 Gram/Cholesky matrix W,
// and fp64 W and Q for the QR fallback.  CUDA-core factors: U, T, Y fp32
// and fp64 W and Q for the Cholesky-QR.  Both: mu.
struct FactorPlan {
  int32_t block, side, d;
  bool tc;
  size_t st_S, st_codes, st_scales, st_lam;
  size_t st_P;                           // root method NEWTON: the fp32 root in the state
  size_t ws_S;                           // compressed statistics: S lives here
  size_t ws_mu;
  size_t ws_W64, ws_Q64, ws_U, ws_T, ws_Y;
  size_t ws_Xm[2], ws_Xh[2], ws_Xl[2], ws_Th, ws_Tl, ws_Sh, ws_Sl, ws_W;
  size_t ws_Zm, ws_Zh, ws_Zl;
  size_t ws_sketch;                      // d x 16 fp64: the last QR pass's orthogonality sketch
  size_t ws_Ih, ws_Il;                   // 64 x 64 inverse diagonal blocks of L (rows to a multiple of 64)
  size_t ws_Jh, ws_Jl;                   // 128 x 128 inverse diagonal blocks (rows to a multiple of 128)
  size_t ws_q_first, ws_q_next;
  size_t dbg_u, dbg_q;                   // debug capture: offsets of the rectified U and of Q
};

constexpr size_t kAlign = 256;
constexpr int kDefaultNewtonIters = 32;
// automatic grouping: one group while the whole call scratch fits in
// kOneGroupBytes (every launch then covers every factor, which the
// latency-bound steps of the QR chain need), else runs of consecutive tiles
// whose scratch fits in kGroupBytes (two such slots are allocated)
constexpr size_t kOneGroupBytes = size_t(96) << 30;
constexpr size_t kGroupBytes = size_t(8) << 30;
constexpr int kPanelW = 64;     // Cholesky panel width (64 x 64 diagonal blocks)
constexpr int kSolveW = 128;    // solve panel width (128 x 128 inverse blocks)

}  // namespace

struct shampoo4_ctx {
  shampoo4_config cfg;
  std::vector<shampoo4_param> params;
  std::vector<BlockPlan> blocks;
  std::vector<FactorPlan> factors;
  size_t state_bytes = 0, ws_bytes = 0;
  // workspace regions
  size_t ws_flags = 0, ws_tabs = 0, ws_fail = 0, ws_bflag = 0, ws_maps = 0, ws_nmaps = 0;
  size_t ws_tcbad = 0, ws_tcgood = 0, ws_devsq = 0, ws_skip3 = 0, ws_fbany = 0;
  size_t ws_p3any = 0;                   // some factor goes through the gated last QR pass
  bool any_simt = false;                 // some factor always takes the fp64 QR
  std::vector<int32_t> group_begin;      // tile groups: [group_begin[g], group_begin[g+1])
  // optional debug capture (shampoo4_debug_capture): every refresh copies
  // each refreshed factor's rectified basis and pre-quantization Q here
  uint8_t* d_dbg = nullptr;
  size_t dbg_bytes = 0;
  uint64_t wait_ns = 0;                  // tensor-core pipeline wait limit (0: the kernel's default)
  size_t ws_desc = 0, ws_desc_bytes = 0;
  // programs
  // With one tile group, statistics and precondition run on the caller's
  // stream and the refresh is split into parts of about equal d^3 cost that
  // run concurrently on the handle's streams; with several groups, every
  // call runs group g on the handle's stream g mod 2.
  Program prog_stats, prog_stats_first, prog_refresh_first, prog_refresh, prog_precond;
  static constexpr int kMaxParts = 2;
  int refresh_parts = 1;                   // requested (shampoo4_debug_refresh_parts)
  cudaStream_t part_stream[kMaxParts] = {};
  cudaEvent_t part_fork = nullptr, part_join[kMaxParts] = {};
  std::vector<uint8_t> arena;            // host image of the descriptor region
  std::vector<CUtensorMap> maps;         // host image of the tensor-map region
  // bound buffers
  uint8_t* d_state = nullptr;
  uint8_t* d_ws = nullptr;
  bool bound = false;
  bool has_basis = false;
  bool last_refresh_first = true;
  bool stats_pending = false;            // compressed statistics: rebuilt S not yet refreshed
  // refresh sharding: factor f is refreshed by rank owner[f] of world; this
  // handle's rank keeps statistics and refreshes only its own factors, and
  // the codes, scales and eigenvalues of rank r's factors form one
  // contiguous state span [span_off[r], span_off[r] + span_bytes[r])
  int32_t rank = 0, world = 1;
  std::vector<int32_t> owner;
  std::vector<size_t> span_off, span_bytes;
  // per-call pointer tables
  std::vector<PtrEntry> tab_host;  // last uploaded (2 * nparams)
  bool tab_valid = false;
  PtrEntry* tab_pinned = nullptr;
  uint32_t* flags_pinned = nullptr;
  cudaEvent_t tab_event = nullptr;
  bool tab_event_pending = false;
  // optional per-launch timing (diagnostics)
  struct Rec { int tag; cudaEvent_t e0, e1; double flops, bytes; int kernels; };
  bool timing = false;
  std::vector<cudaEvent_t> ev_pool;
  std::vector<Rec> recs;
  double t_ms[SHAMPOO4_STAGE_COUNT] = {};
  double t_flops[SHAMPOO4_STAGE_COUNT] = {};
  double t_bytes[SHAMPOO4_STAGE_COUNT] = {};
  int64_t t_launches[SHAMPOO4_STAGE_COUNT] = {};
  // grafted weight update: bands of tile rows, the moments' layout, and a
  // per-call pointer table of its own (gradients, directions, weights)
  std::vector<GraftItem> graft_items;
  size_t ws_dsq = 0;                     // sums of squares of D recorded by the apply
  bool dsq_valid = false;                // a precondition has recorded them
  std::vector<size_t> graft_off_m, graft_off_v;   // bytes, per parameter
  size_t graft_state_bytes = 0;
  size_t ws_gtab = 0, ws_gitems = 0, ws_gparts = 0;
  std::vector<PtrEntry> gtab_host;
  bool gtab_valid = false;
  PtrEntry* gtab_pinned = nullptr;
  cudaEvent_t gtab_event = nullptr;
  bool gtab_event_pending = false;
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

bool tc_dim(int d) { return d % 4 == 0; }

// Grafting: each tile is cut into bands of whole rows of at most
// kGraftBandElems elements (one CTA each); the moments are dense per
// parameter, m then v, each slice kAlign-aligned.
constexpr int64_t kGraftBandElems = 65536;

void plan_graft(shampoo4_ctx* h, size_t& ws) {
  const size_t np = h->params.size();
  size_t gs = 0;
  h->graft_off_m.resize(np);
  h->graft_off_v.resize(np);
  for (size_t p = 0; p < np; ++p) {
    const size_t elems = size_t(h->params[p].rows) * size_t(h->params[p].cols);
    h->graft_off_m[p] = take(gs, 4 * elems);
    h->graft_off_v[p] = take(gs, 4 * elems);
  }
  h->graft_state_bytes = align_up(gs, kAlign);
  // the apply's recorded sums of squares: 4 per output tile of a
  // tensor-core tile's D = B P_R, in TF32 mode (the fp32-accurate apply runs
  // the persistent kernel, which does not record them)
  int64_t nd = 0;
  const bool record = h->cfg.precision != SHAMPOO4_PREC_FP32;
  const int bn = tc_block_n(0);
  for (auto& b : h->blocks) {
    b.dsq_off = nd;
    b.dsq_n = (b.tc && record) ? 4 * ((b.m + 127) / 128) * ((b.n + bn - 1) / bn) : 0;
    nd += b.dsq_n;
  }
  h->ws_dsq = take(ws, 8 * size_t(std::max<int64_t>(nd, 1)));
  for (size_t k = 0; k < h->blocks.size(); ++k) {
    const BlockPlan& b = h->blocks[k];
    const int64_t cols = h->params[b.param].cols;
    const int32_t band = int32_t(std::max<int64_t>(1, std::min<int64_t>(b.m, kGraftBandElems / b.n)));
    const int32_t nparts = (b.m + band - 1) / band;
    const int32_t part0 = int32_t(h->graft_items.size());
    for (int32_t i = 0; i < nparts; ++i) {
      GraftItem it{};
      it.param = b.param;
      it.block = int32_t(k);
      it.r0 = b.r0 + int64_t(i) * band;
      it.c0 = b.c0;
      it.rows = std::min<int32_t>(band, b.m - i * band);
      it.cols = b.n;
      it.part0 = part0;
      it.nparts = nparts;
      const int64_t e = it.r0 * cols + it.c0;
      it.m_off = int64_t(h->graft_off_m[b.param] / 4) + e;
      it.v_off = int64_t(h->graft_off_v[b.param] / 4) + e;
      it.state_ld = cols;
      it.dsq_off = b.dsq_off;
      it.dsq_n = b.dsq_n;
      h->graft_items.push_back(it);
    }
  }
  h->ws_gtab = take(ws, sizeof(PtrEntry) * 3 * np);
  h->ws_gitems = take(ws, sizeof(GraftItem) * h->graft_items.size());
  h->ws_gparts = take(ws, 16 * h->graft_items.size());
}

shampoo4_status plan(shampoo4_ctx* h) {
  for (size_t p = 0; p < h->params.size(); ++p) {
    const shampoo4_param& q = h->params[p];
    for (auto rc : chunks(q.rows, h->cfg.max_block))
      for (auto cc : chunks(q.cols, h->cfg.max_block)) {
        BlockPlan b{};
        b.param = int32_t(p); b.r0 = rc.first; b.c0 = cc.first; b.m = rc.second; b.n = cc.second;
        b.tc = tc_dim(b.m) && tc_dim(b.n);
        h->blocks.push_back(b);
      }
  }
  if (h->blocks.size() > (1u << 30)) return SHAMPOO4_ERR_INVALID_ARG;
  for (size_t k = 0; k < h->blocks.size(); ++k) {
    for (int side = 0; side < 2; ++side) {
      FactorPlan f{};
      f.block = int32_t(k);
      f.side = side;
      f.d = side == 0 ? h->blocks[k].m : h->blocks[k].n;
      f.tc = tc_dim(f.d);
      h->factors.push_back(f);
    }
  }
  // owners: longest processing time first on the d^3 refresh cost (ties by
  // factor index), each factor to the least-loaded rank (ties: lowest rank)
  const size_t nf = h->factors.size();
  h->owner.assign(nf, 0);
  if (h->world > 1) {
    std::vector<size_t> order(nf);
    for (size_t i = 0; i < nf; ++i) order[i] = i;
    auto cost = [&](size_t i) { return double(h->factors[i].d) * h->factors[i].d * h->factors[i].d; };
    std::stable_sort(order.begin(), order.end(), [&](size_t a, size_t b) { return cost(a) > cost(b); });
    std::vector<double> load(h->world, 0.0);
    for (size_t i : order) {
      int32_t r = 0;
      for (int32_t q = 1; q < h->world; ++q)
        if (load[q] < load[r]) r = q;
      h->owner[i] = r;
      load[r] += cost(i);
    }
  }
  // state: the codes, scales and eigenvalues grouped by owner, then the fp32
  // statistics of this rank's factors (none with compressed statistics)
  size_t st = 0;
  h->span_off.assign(h->world, 0);
  h->span_bytes.assign(h->world, 0);
  for (int32_t r = 0; r < h->world; ++r) {
    h->span_off[r] = align_up(st, kAlign);
    st = h->span_off[r];
    for (size_t i = 0; i < nf; ++i) {
      if (h->owner[i] != r) continue;
      FactorPlan& f = h->factors[i];
      const size_t dd = size_t(f.d) * f.d;
      f.st_codes = take(st, (dd + 1) / 2);
      f.st_scales = take(st, 4 * ((dd + kQuantBlock - 1) / kQuantBlock));
      f.st_lam = take(st, 4 * size_t(f.d));
      f.st_P = h->cfg.root_method == SHAMPOO4_ROOT_NEWTON ? take(st, 4 * dd) : SIZE_MAX;
    }
    h->span_bytes[r] = st - h->span_off[r];
  }
  for (size_t i = 0; i < nf; ++i) {
    FactorPlan& f = h->factors[i];
    const size_t dd = size_t(f.d) * f.d;
    f.st_S = (h->cfg.compressed_stats || h->owner[i] != h->rank) ? SIZE_MAX : take(st, 4 * dd);
    if (!f.tc && h->owner[i] == h->rank) h->any_simt = true;
  }
  h->state_bytes = align_up(st, kAlign);
  size_t dbg = 0;
  for (FactorPlan& f : h->factors) {
    const size_t dd = size_t(f.d) * f.d;
    f.dbg_u = take(dbg, 4 * dd);
    f.dbg_q = take(dbg, 4 * dd);
  }
  h->dbg_bytes = align_up(dbg, kAlign);

  size_t ws = 0;
  h->ws_flags = take(ws, 16);
  h->ws_tabs = take(ws, sizeof(PtrEntry) * 2 * h->params.size());
  h->ws_fail = take(ws, 4 * h->factors.size());
  h->ws_tcbad = take(ws, 4 * h->factors.size());
  h->ws_tcgood = take(ws, 4 * h->factors.size());
  h->ws_devsq = take(ws, 8 * h->factors.size());
  h->ws_skip3 = take(ws, 4 * h->factors.size());
  h->ws_fbany = take(ws, 4);
  h->ws_p3any = take(ws, 4);
  h->ws_bflag = take(ws, 4 * h->blocks.size());
  // persistent per factor: the rebuilt statistic (compressed statistics,
  // valid from update_stats to refresh_roots) and the root weights
  for (size_t i = 0; i < h->factors.size(); ++i) {
    FactorPlan& f = h->factors[i];
    const size_t dd = size_t(f.d) * f.d;
    f.ws_S = (h->cfg.compressed_stats && h->owner[i] == h->rank) ? take(ws, 4 * dd) : SIZE_MAX;
    f.ws_mu = take(ws, 4 * size_t(f.d));
  }
  // Scratch of one call: the refresh's matrices per factor, the split
  // gradient and apply intermediate per tile.  The tiles are cut into
  // groups of consecutive tiles; group g's scratch lives in slot g mod 2,
  // so groups that share a slot run one after another on the same stream
  // and the workspace holds the scratch of two groups, not of every tile.
  auto factor_scratch = [&](FactorPlan& f, size_t& cur) {
    const size_t dd = size_t(f.d) * f.d;
    if (f.tc) {
      for (int i = 0; i < 2; ++i) {
        f.ws_Xm[i] = take(cur, 4 * dd);
        f.ws_Xh[i] = take(cur, 4 * dd);
        f.ws_Xl[i] = take(cur, 4 * dd);
      }
      f.ws_Th = take(cur, 4 * dd);
      f.ws_Tl = take(cur, 4 * dd);
      f.ws_Sh = take(cur, 4 * dd);
      f.ws_Sl = take(cur, 4 * dd);
      f.ws_W = take(cur, 4 * dd);
      f.ws_Zm = take(cur, 4 * dd);
      f.ws_Zh = take(cur, 4 * dd);
      f.ws_Zl = take(cur, 4 * dd);
      f.ws_sketch = take(cur, 8 * size_t(kSketchCols) * f.d);
      // the inverse blocks are written 64 x 64 (zero-padded): rows up to a
      // multiple of 64
      const size_t dpad = align_up(size_t(f.d), kPanelW);
      f.ws_Ih = take(cur, 4 * dpad * kPanelW);
      f.ws_Il = take(cur, 4 * dpad * kPanelW);
      const size_t dpad2 = align_up(size_t(f.d), kSolveW);
      f.ws_Jh = take(cur, 4 * dpad2 * kSolveW);
      f.ws_Jl = take(cur, 4 * dpad2 * kSolveW);
      f.ws_W64 = take(cur, 8 * dd);            // fp64 fallback of the QR
      f.ws_Q64 = take(cur, 8 * dd);
    } else {
      f.ws_W64 = take(cur, 8 * dd);
      f.ws_Q64 = take(cur, 8 * dd);
      f.ws_U = take(cur, 4 * dd);
      f.ws_T = take(cur, 4 * dd);
      f.ws_Y = take(cur, 4 * dd);
    }
  };
  auto tile_scratch = [&](BlockPlan& b, size_t& cur) {
    const size_t mn = size_t(b.m) * b.n;
    if (!b.tc) {
      b.ws_tmp = take(cur, 4 * mn);
      return;
    }
    b.ws_Gh = take(cur, 4 * mn);
    b.ws_Gl = take(cur, 4 * mn);
    b.ws_Bh = take(cur, 4 * mn);
    b.ws_Bl = take(cur, 4 * mn);
  };
  auto group_bytes = [&](size_t k0, size_t k1) {
    size_t cur = 0;
    for (size_t k = k0; k < k1; ++k) {
      FactorPlan a = h->factors[2 * k], c = h->factors[2 * k + 1];
      BlockPlan t = h->blocks[k];
      factor_scratch(a, cur);
      factor_scratch(c, cur);
      tile_scratch(t, cur);
    }
    return align_up(cur, kAlign);
  };
  // groups: group_tiles tiles each, or (0) as many as keep a group's scratch
  // within kGroupBytes; one group when the refresh is sharded over ranks
  const size_t nb = h->blocks.size();
  h->group_begin.assign(1, 0);
  if (h->world > 1 || h->cfg.group_tiles >= int64_t(nb)) {
    h->group_begin.push_back(int32_t(nb));
  } else if (h->cfg.group_tiles > 0) {
    for (size_t k = h->cfg.group_tiles; k < nb; k += h->cfg.group_tiles) h->group_begin.push_back(int32_t(k));
    h->group_begin.push_back(int32_t(nb));
  } else if (group_bytes(0, nb) <= kOneGroupBytes) {
    h->group_begin.push_back(int32_t(nb));
  } else {
    size_t k0 = 0;
    for (size_t k = 0; k < nb; ++k)
      if (k > k0 && group_bytes(k0, k + 1) > kGroupBytes) {
        h->group_begin.push_back(int32_t(k));
        k0 = k;
      }
    h->group_begin.push_back(int32_t(nb));
  }
  const int ngroups = int(h->group_begin.size()) - 1;
  const int nslots = ngroups > 1 ? 2 : 1;
  for (int sl = 0; sl < nslots; ++sl) {
    const size_t base = align_up(ws, kAlign);
    size_t extent = 0;
    for (int g = sl; g < ngroups; g += nslots) {
      size_t cur = base;
      for (int32_t k = h->group_begin[g]; k < h->group_begin[g + 1]; ++k) {
        factor_scratch(h->factors[2 * k], cur);
        factor_scratch(h->factors[2 * k + 1], cur);
        tile_scratch(h->blocks[k], cur);
      }
      extent = std::max(extent, cur - base);
    }
    ws = base + extent;
  }
  plan_graft(h, ws);
  h->ws_maps = align_up(ws, kAlign);
  h->ws_bytes = h->ws_maps;     // maps and descriptors are added by init
  return SHAMPOO4_OK;
}

// ---------------------------------------------------------- program builder

struct Builder {
  shampoo4_ctx* h;
  std::vector<uint8_t>& arena;
  uint8_t* ws;        // device workspace base (descriptors point into it)
  uint8_t* stb;       // device state base
  bool encode;        // false: only count tensor maps (sizing pass)
  int tag = 0;        // stage label applied to the launches emitted next
  size_t guard = SIZE_MAX;   // guard word applied to the launches emitted next
  shampoo4_status err = SHAMPOO4_OK;
  std::map<std::tuple<uintptr_t, int, int, int, int>, size_t> map_index;

  template <class D>
  size_t put(const std::vector<D>& v) {
    size_t at = align_up(arena.size(), kAlign);
    arena.resize(at + sizeof(D) * v.size());
    if (!v.empty()) std::memcpy(arena.data() + at, v.data(), sizeof(D) * v.size());
    return at;
  }
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
    L.guard_off = guard;
    prog.push_back(std::move(L));
  }
  float* wf(size_t off) const { return reinterpret_cast<float*>(ws + off); }
  double* wd(size_t off) const { return reinterpret_cast<double*>(ws + off); }
  uint32_t* wu(size_t off) const { return reinterpret_cast<uint32_t*>(ws + off); }
  float* sf(size_t off) const { return reinterpret_cast<float*>(stb + off); }
  uint8_t* sb(size_t off) const { return stb + off; }
  // the factor's statistic: in the state, or (compressed statistics) in the
  // workspace
  float* S(const FactorPlan& f) const { return f.st_S == SIZE_MAX ? wf(f.ws_S) : sf(f.st_S); }
  // Per-factor scratch words are indexed by the factor's index in the
  // handle; while a program is built over a subset of the factors (a rank's
  // share, a part of the refresh), gmap maps the subset's positions to it.
  const std::vector<size_t>* gmap = nullptr;
  const std::vector<size_t>* bmap = nullptr;    // the same for tiles
  size_t gi(size_t i) const { return gmap ? (*gmap)[i] : i; }
  uint32_t* bflag(size_t k) const { return wu(h->ws_bflag) + (bmap ? (*bmap)[k] : k); }
  uint32_t* fail(size_t fi) const { return wu(h->ws_fail) + gi(fi); }
  uint32_t* tcbad(size_t fi) const { return wu(h->ws_tcbad) + gi(fi); }
  uint32_t* tcgood(size_t fi) const { return wu(h->ws_tcgood) + gi(fi); }
  unsigned long long* devsq(size_t fi) const {
    return reinterpret_cast<unsigned long long*>(ws + h->ws_devsq) + gi(fi);
  }
  uint32_t* skip3(size_t fi) const { return wu(h->ws_skip3) + gi(fi); }
  uint32_t* gflags() const { return wu(h->ws_flags); }
  float* dbg(size_t off) const { return h->d_dbg ? reinterpret_cast<float*>(h->d_dbg + off) : nullptr; }

  // Device address of the tensor map of a dense d0 x d1 workspace matrix.
  const CUtensorMap* map(const float* base, int rows, int cols, int box_rows, int mn_major) {
    auto key = std::make_tuple(reinterpret_cast<uintptr_t>(base), rows, cols, box_rows, mn_major);
    auto it = map_index.find(key);
    size_t idx;
    if (it != map_index.end()) {
      idx = it->second;
    } else {
      idx = h->maps.size();
      h->maps.emplace_back();
      map_index[key] = idx;
      if (encode) {
        shampoo4_status s = tc_encode_map(&h->maps.back(), base, rows, cols, cols, box_rows, mn_major);
        if (s != SHAMPOO4_OK) err = s;
      }
    }
    return reinterpret_cast<const CUtensorMap*>(ws + h->ws_maps + idx * sizeof(CUtensorMap));
  }
  // Operand of a tensor-core product from a dense rows x cols matrix held as
  // a TF32 split (hi, lo).  as_a: the A operand (tile rows 128), else B.
  // trans: op(X) = X^T.  K-major iff the contraction index is contiguous.
  TcOperand operand(const float* hi, const float* lo, int rows, int cols, bool as_a, bool trans, bool split,
                    int bn = 0) {
    TcOperand o{};
    const bool k_major = as_a ? !trans : trans;
    o.mn_major = k_major ? 0 : 1;
    const int box = k_major ? (as_a ? 128 : (bn ? bn : tc_block_n(split))) : 32;
    o.hi = map(hi, rows, cols, box, o.mn_major);
    o.lo = split ? map(lo, rows, cols, box, o.mn_major) : nullptr;
    return o;
  }
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

TcGemmDesc gemmtc(int M, int N, int K, float alpha, float beta) {
  TcGemmDesc g{};
  g.M = M; g.N = N; g.K = K; g.alpha = alpha; g.beta = beta;
  g.c_ref.tab = -1;
  return g;
}

double product_flops(int M, int N, int K, bool symmetric) {
  return symmetric ? double(M) * (M + 1) * K : 2.0 * M * N * K;
}

// Algorithmic flops of a product: 2 M N K, or M (M+1) K for an output known
// to be symmetric (only one triangle is needed).
void emit_gemm32(Builder& b, std::vector<Launch>& prog, const std::vector<GemmF32Desc>& v) {
  int mt = 0;
  double fl = 0;
  for (auto& g : v) {
    mt = std::max(mt, tiles128(g.M, g.N));
    fl += product_flops(g.M, g.N, g.K, g.symmetric);
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
void emit_gemmtc(Builder& b, std::vector<Launch>& prog, const std::vector<TcGemmDesc>& v, bool split,
                 int bn_override = 0) {
  const int bn = bn_override ? bn_override : tc_block_n(split);
  int mt = 0;
  double fl = 0;
  for (auto& g : v) {
    mt = std::max(mt, ((g.M + 127) / 128) * ((g.N + bn - 1) / bn));
    fl += product_flops(g.M, g.N, g.K, g.symmetric);
  }
  if (v.empty()) return;
  std::vector<TcGemmDesc> w = v;
  // the 128-wide split instance runs persistent CTAs, which look their
  // tiles up in the list
  const bool pers = split && bn == 128;
  std::vector<uint64_t> list;
  const int64_t total = tc_assign_tiles(w.data(), int(w.size()), bn, pers ? &list : nullptr);
  b.emit(prog, !split ? Kind::GemmTC : (bn == 64 ? Kind::GemmTCSplit64 : Kind::GemmTCSplit), w, mt, fl);
  prog.back().tiles = total;
  if (pers && !list.empty()) prog.back().list_off = b.put(list);
}

int mode_of(const shampoo4_config& c) { return c.precision == SHAMPOO4_PREC_FP32 ? kModeFP32 : kModeTF32; }
bool split_of(const shampoo4_config& c) { return c.precision == SHAMPOO4_PREC_FP32; }

// Scan (and, for tensor-core tiles, split) the per-call gradients.
void build_grad_copy(Builder& b, std::vector<Launch>& prog, int tag, bool with_flags) {
  shampoo4_ctx* h = b.h;
  const bool split = split_of(h->cfg);
  std::vector<ScanDesc> scan;
  int64_t max_elems = 0;
  double bytes = 0;
  for (size_t k = 0; k < h->blocks.size(); ++k) {
    const BlockPlan& bp = h->blocks[k];
    if (!with_flags && !bp.tc) continue;
    ScanDesc s{};
    s.rows = bp.m; s.cols = bp.n;
    s.ref = {0, bp.param, bp.r0, bp.c0};
    s.flag = b.bflag(k);
    s.bit = with_flags ? SHAMPOO4_FLAG_NONFINITE_GRAD : 0u;
    if (bp.tc) {
      s.oh = b.wf(bp.ws_Gh);
      s.ol = split ? b.wf(bp.ws_Gl) : nullptr;
    }
    scan.push_back(s);
    max_elems = std::max<int64_t>(max_elems, int64_t(bp.m));     // rows
    bytes += (4.0 + (bp.tc ? (split ? 8.0 : 4.0) : 0.0)) * bp.m * bp.n;
  }
  b.tag = tag;
  b.emit(prog, Kind::Scan, scan, max_elems, 0, bytes);
}

// The statistics update into `prog`.  With compressed statistics and
// `rebuild`, the stored statistic is first rebuilt in the workspace as
// U diag(lambda) U^T from the codes (k_basis with lambda as the column
// scale, then one symmetric product), and the EMA reads it as Cin; without
// `rebuild` (before the first refresh) the EMA starts from zero.
void build_stats_into(Builder& b, std::vector<Launch>& prog, bool rebuild) {
  shampoo4_ctx* h = b.h;
  const bool split = split_of(h->cfg);
  const bool compressed = h->cfg.compressed_stats != 0;
  build_grad_copy(b, prog, SHAMPOO4_STAGE_STATS_SCAN, true);
  if (compressed && rebuild) {
    std::vector<MuDesc> half;
    std::vector<BasisDesc> bd;
    std::vector<TcGemmDesc> trec;
    std::vector<GemmF32Desc> rec;
    std::vector<RowDiagDesc> rdiag;
    int dmax = 0;
    int64_t emax = 0;
    double bytes_bd = 0, sum_dd = 0;
    for (size_t i = 0; i < h->factors.size(); ++i) {
      const FactorPlan& f = h->factors[i];
      if (h->owner[i] != h->rank) continue;
      const int d = f.d;
      dmax = std::max(dmax, d);
      emax = std::max<int64_t>(emax, int64_t(d) * d);
      sum_dd += double(d) * d;
      BasisDesc x{};
      x.codes = b.sb(f.st_codes); x.scales = b.sf(f.st_scales); x.d = d; x.identity = 0;
      x.codebook = h->cfg.codebook;
      if (f.tc) {
        // V = U diag(sqrt(lambda)) -> X[1] split; S = V V^T.  The same
        // rounded V on both sides keeps S positive semidefinite (up to the
        // fp32 accumulation), as G G^T is, whatever the operand rounding.
        half.push_back({b.sf(f.st_lam), b.wf(f.ws_mu), d, 1});
        x.mu = b.wf(f.ws_mu);
        x.Vh = b.wf(f.ws_Xh[1]); x.Vl = split ? b.wf(f.ws_Xl[1]) : nullptr;
        TcGemmDesc g = gemmtc(d, d, d, 1.0f, 0.0f);
        g.a = b.operand(b.wf(f.ws_Xh[1]), b.wf(f.ws_Xl[1]), d, d, true, false, split);
        g.b = b.operand(b.wf(f.ws_Xh[1]), b.wf(f.ws_Xl[1]), d, d, false, true, split);
        g.C = b.S(f); g.ldc = d;
        g.symmetric = 1;                  // exactly symmetric: lower tiles, mirrored
        trec.push_back(g);
        if (split)
          rdiag.push_back({b.wf(f.ws_Xh[1]), b.wf(f.ws_Xl[1]), b.wf(f.ws_Xh[1]), b.wf(f.ws_Xl[1]), d, d, 0,
                           b.S(f), nullptr, nullptr});
        bytes_bd += (0.5625 + 4.0 + (split ? 8.0 : 4.0)) * double(d) * d;
      } else {
        x.U = b.wf(f.ws_Y);
        GemmF32Desc g = gemm32(d, d, d, 0, 1, mode_of(h->cfg), 1.0f, 0.0f);
        g.A = b.wf(f.ws_Y); g.lda = d; g.kscale = b.sf(f.st_lam);
        g.B = b.wf(f.ws_Y); g.ldb = d;
        g.C = b.S(f); g.ldc = d;
        g.symmetric = 1;
        rec.push_back(g);
        bytes_bd += (0.5625 + 4.0 + 4.0) * double(d) * d;
      }
      bd.push_back(x);
    }
    b.tag = SHAMPOO4_STAGE_STATS_DEQUANT;
    b.emit(prog, Kind::Mu, half, dmax);
    b.emit(prog, Kind::Basis, bd, emax, 0, bytes_bd);
    b.tag = SHAMPOO4_STAGE_STATS_REBUILD;
    emit_gemmtc(b, prog, trec, split);
    b.emit(prog, Kind::RowDiag, rdiag, dmax, 0, 16.0 * sum_dd);
    emit_gemm32(b, prog, rec);
  }
  std::vector<GemmF32Desc> g;
  std::vector<TcGemmDesc> t;
  // EMA: S <- beta S + (1 - beta) G G^T; compressed statistics read the
  // rebuilt S with weight beta, or start from zero
  const float omb = 1.0f - h->cfg.beta;
  const float beta = (compressed && !rebuild) ? 0.0f : h->cfg.beta;
  for (size_t k = 0; k < h->blocks.size(); ++k) {
    const BlockPlan& bp = h->blocks[k];
    uint32_t* skip = b.bflag(k);
    for (int side = 0; side < 2; ++side) {
      if (h->owner[2 * k + side] != h->rank) continue;
      const FactorPlan& f = h->factors[2 * k + side];
      const int d = f.d, kk = side == 0 ? bp.n : bp.m;
      float* S = b.S(f);
      const float* Cin = beta == 0.0f ? nullptr : S;
      if (bp.tc) {
        // L: A = G (K-major), B = G^T as op(B)[k,j] = G[j,k] (K-major).
        // R: A = G^T (MN-major), B = G (MN-major).
        TcGemmDesc x = gemmtc(d, d, kk, omb, beta);
        x.a = b.operand(b.wf(bp.ws_Gh), b.wf(bp.ws_Gl), bp.m, bp.n, true, side == 1, split);
        x.b = b.operand(b.wf(bp.ws_Gh), b.wf(bp.ws_Gl), bp.m, bp.n, false, side == 0, split);
        x.C = S; x.ldc = d;
        x.Cin = Cin; x.ldcin = d;
        x.symmetric = 1;
        x.skip = skip;
        t.push_back(x);
      } else {
        GemmF32Desc x = side == 0 ? gemm32(d, d, kk, 0, 1, mode_of(h->cfg), omb, beta)
                                  : gemm32(d, d, kk, 1, 0, mode_of(h->cfg), omb, beta);
        x.a_ref = {0, bp.param, bp.r0, bp.c0};
        x.b_ref = x.a_ref;
        x.C = S; x.ldc = d;
        x.Cin = Cin; x.ldcin = d;
        x.symmetric = 1;
        x.skip = skip;
        g.push_back(x);
      }
    }
  }
  b.tag = SHAMPOO4_STAGE_STATS_GEMM;
  emit_gemmtc(b, prog, t, split);
  emit_gemm32(b, prog, g);
}

// Swaps one tile group in for the builders: tiles k0..k1-1 become local
// tiles 0.., their factors local factors 2(k - k0) + side, and gmap/bmap
// give the builders the handle-wide indices of the per-factor scratch words
// and tile flags.  The handle's lists come back on destruction, with the
// workspace offsets the builders assigned.
struct GroupScope {
  shampoo4_ctx* h;
  Builder& b;
  std::vector<BlockPlan> blocks;
  std::vector<FactorPlan> factors;
  std::vector<int32_t> owner;
  std::vector<size_t> fmap, bmap;
  GroupScope(Builder& bb, int32_t k0, int32_t k1) : h(bb.h), b(bb) {
    std::vector<BlockPlan> lb;
    std::vector<FactorPlan> lf;
    std::vector<int32_t> lo;
    for (int32_t k = k0; k < k1; ++k) {
      lb.push_back(h->blocks[k]);
      bmap.push_back(size_t(k));
      for (int side = 0; side < 2; ++side) {
        FactorPlan f = h->factors[2 * k + side];
        f.block = k - k0;
        lf.push_back(f);
        fmap.push_back(size_t(2 * k + side));
        lo.push_back(h->owner[2 * k + side]);
      }
    }
    blocks.swap(h->blocks);
    factors.swap(h->factors);
    owner.swap(h->owner);
    h->blocks.swap(lb);
    h->factors.swap(lf);
    h->owner.swap(lo);
    b.gmap = &fmap;
    b.bmap = &bmap;
  }
  ~GroupScope() {
    for (size_t j = 0; j < fmap.size(); ++j) {
      factors[fmap[j]].ws_q_first = h->factors[j].ws_q_first;
      factors[fmap[j]].ws_q_next = h->factors[j].ws_q_next;
    }
    h->blocks.swap(blocks);
    h->factors.swap(factors);
    h->owner.swap(owner);
    b.gmap = nullptr;
    b.bmap = nullptr;
  }
};

int ngroups(const shampoo4_ctx* h) { return int(h->group_begin.size()) - 1; }

void build_stats(Builder& b) {
  shampoo4_ctx* h = b.h;
  const int ng = ngroups(h);
  for (int g = 0; g < ng; ++g) {
    if (ng == 1) {
      build_stats_into(b, h->prog_stats.add(-1), true);
      if (h->cfg.compressed_stats) build_stats_into(b, h->prog_stats_first.add(-1), false);
      break;
    }
    GroupScope scope(b, h->group_begin[g], h->group_begin[g + 1]);
    build_stats_into(b, h->prog_stats.add(g % 2), true);
    if (h->cfg.compressed_stats) build_stats_into(b, h->prog_stats_first.add(g % 2), false);
  }
}

// fp64 Cholesky-QR pass over the factors with use[i]: X (fp32, d x d) -> Q
// (fp32) through the fp64 Gram W = X^T X (+ shift), blocked right-looking
// Cholesky W = L L^T and a blocked solve Q L^T = X, all on CUDA cores.
// qh/ql (optional) receive the TF32 split of Q.  skip[i]: per-factor flag
// that suppresses the pass.  Used by the CUDA-core factors, and by the
// tensor-core factors whose fp32 factorization broke down.
void build_cholqr_pass(Builder& b, std::vector<Launch>& prog, const std::vector<char>& use,
                       const std::vector<const float*>& X, const std::vector<float*>& Q,
                       const std::vector<float*>& qh, const std::vector<float*>& ql,
                       const std::vector<const uint32_t*>& skip, bool shifted) {
  shampoo4_ctx* h = b.h;
  const size_t nf = h->factors.size();
  int dmax = 0;
  for (size_t i = 0; i < nf; ++i) if (use[i]) dmax = std::max(dmax, h->factors[i].d);
  if (dmax == 0) return;
  {
    std::vector<GemmF64Desc> g;
    std::vector<ShiftDesc> sd;
    for (size_t i = 0; i < nf; ++i) {
      if (!use[i]) continue;
      const FactorPlan& f = h->factors[i];
      GemmF64Desc d{};
      d.M = d.N = d.K = f.d; d.ta = 1; d.tb = 0; d.lower_only = 1;
      d.A = X[i]; d.lda = f.d; d.B = d.A; d.ldb = f.d;
      d.C = b.wd(f.ws_W64); d.ldc = f.d; d.c_f64 = 1;
      d.alpha = 1.0; d.beta = 0.0;
      d.skip = skip[i];
      g.push_back(d);
      if (shifted) sd.push_back({b.wd(f.ws_W64), f.d, f.d, 0, skip[i]});
    }
    b.tag = SHAMPOO4_STAGE_QR_GRAM;
    emit_gemm64(b, prog, g);
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
      if (!use[i] || j >= f.d) continue;
      const int jb = std::min(kPanelW, f.d - j);
      double* W = b.wd(f.ws_W64);
      const int64_t ld = f.d;
      po.push_back({W + j * ld + j, ld, jb, 0, b.fail(i), b.gflags(), skip[i]});
      fl_po += double(jb) * jb * jb / 3.0;
      const int rest = f.d - j - jb;
      if (rest > 0) {
        fl_tr += double(rest) * jb * jb;
        tr.push_back({W + j * ld + j, ld, W + (j + jb) * ld + j, ld, jb, rest, skip[i]});
        max_rows = std::max(max_rows, rest);
        GemmF64Desc d{};
        d.M = d.N = rest; d.K = jb; d.ta = 0; d.tb = 1; d.lower_only = 1;
        d.a_f64 = d.b_f64 = d.c_f64 = d.cin_f64 = 1;
        d.A = W + (j + jb) * ld + j; d.lda = ld; d.B = d.A; d.ldb = ld;
        d.C = W + (j + jb) * ld + (j + jb); d.ldc = ld; d.Cin = d.C; d.ldcin = ld;
        d.alpha = -1.0; d.beta = 1.0;
        d.skip = skip[i];
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
  for (int j = 0; j < dmax; j += kPanelW) {          // solve Q L^T = X by column panels
    std::vector<GemmF64Desc> up;
    std::vector<TrsmDesc> tr;
    int max_rows = 0;
    double fl_tr = 0;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      if (!use[i] || j >= f.d) continue;
      const int jb = std::min(kPanelW, f.d - j);
      const int64_t ld = f.d;
      fl_tr += double(f.d) * jb * jb;
      double* W = b.wd(f.ws_W64);
      double* Qd = b.wd(f.ws_Q64);
      GemmF64Desc d{};
      d.M = f.d; d.N = jb; d.K = j; d.ta = 0; d.tb = 1;
      d.a_f64 = 1; d.b_f64 = 1; d.c_f64 = 1; d.cin_f64 = 0;
      d.A = Qd; d.lda = ld; d.B = W + j * ld; d.ldb = ld;
      d.C = Qd + j; d.ldc = ld; d.Cin = X[i] + j; d.ldcin = ld;
      d.alpha = -1.0; d.beta = 1.0;
      d.skip = skip[i];
      up.push_back(d);
      tr.push_back({W + j * ld + j, ld, Qd + j, ld, jb, f.d, skip[i]});
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
    if (!use[i]) continue;
    int64_t n = int64_t(f.d) * f.d;
    cv.push_back({b.wd(f.ws_Q64), Q[i], qh[i], ql[i], n, skip[i]});
    max_elems = std::max(max_elems, n);
    bytes_cv += (12.0 + (qh[i] ? 4.0 : 0.0) + (ql[i] ? 4.0 : 0.0)) * double(n);
  }
  b.tag = SHAMPOO4_STAGE_QR_CONVERT;
  b.emit(prog, Kind::Convert, cv, max_elems, 0, bytes_cv);
}

// Cholesky-QR pass over the tensor-core factors, fp32-accurate throughout:
// X -> Q.  Gram W = X^T X on the tensor cores (3xTF32), optional shift,
// left-looking blocked Cholesky W = L L^T (64-wide diagonal blocks in fp64
// on CUDA cores, panel products on the tensor cores), then Q L^T = X by
// column panels.  Up to three such passes, the first shifted, form shifted
// Cholesky-QR3 (Fukaya et al., SIAM J. Sci. Comput. 2020).
//
// The shift is taken in the column-equilibrated frame: Cholesky-QR of X and
// of X D^-1 (D = column norms) give the same Q and, in floating point, the
// same rounding behaviour, so the conditioning that matters is that of
// X D^-1 (unit columns, ||X D^-1||_F^2 = d).  The shift 1e-5 d there (1e-5 d
// W_ii on the diagonal of W) exceeds the error of the fp32-accurate Gram
// (about 2e-6 d in that frame); the first pass then leaves Q0 with a
// condition number near sqrt(1e-5 d) / sigma_min(X D^-1), and the second
// pass succeeds when that is below about 1e3.  Factors beyond that break
// down in a Cholesky panel and are redone in fp64 from the intact Y.
//
// The first pass only preconditions: with any triangular L1, Q0 = X L1^-T
// and the later passes' factors give Y = Q R with R = L3^T L2^T L1^T, so
// the final Q does not depend on how well L1 factors X^T X, as long as the
// solve uses that same L1 accurately.  Its Gram therefore runs in TF32
// (operands rounded once, fp32 accumulation, exact diagonal): in the
// equilibrated frame that errs by about 2^-11 sqrt(2 / 3d) per off-diagonal
// element, some 8e-4 in 2-norm at d = 1024, well under the shift; what the
// shift leaves of Q0's orthogonality dominates either way.  Its Cholesky,
// its solve and the later passes stay fp32-accurate.
//
// A warm subspace step (U from the previous refresh) has Y = (S + eps I) U
// with nearly orthogonal columns of very different lengths: X D^-1 is close
// to orthonormal, and two passes already reach the orthogonality floor of
// this arithmetic (||Q^T Q - I||_F / sqrt(d) near 1.1e-7 sqrt(d), set by
// the unbiased rounding of the off-diagonal sums).  So the third pass is
// gated per factor: a two-pass fp64 sketch estimates ||Q^T Q - I||_F of the
// second pass's output; its Cholesky and solve run only when that exceeds
// kLastPassTol sqrt(d) * sqrt(d) (a cold first refresh needs them).  In that
// pass a Cholesky pivot at or below kLastPassPivot -- a column of the
// (unit-column) input nearly in the span of the previous ones, so that the
// pass cannot be trusted -- counts as a breakdown, and the factor is redone
// in fp64.
constexpr float kTcShift = 1e-5f;
// Tile width of the fp32-accurate d x d x d products (QR Grams, subspace
// product, Rayleigh product): 128-wide tiles, one CTA per SM.  64-wide
// tiles with two CTAs per SM measured slower on the Llama layer set (Grams
// 42.2 against 40.3 ms, Rayleigh 12.7 against 11.7 ms per step).
constexpr int kSquareBN = 128;
constexpr double kLastPassTol = 2e-7;
constexpr float kLastPassPivot = 1e-2f;

struct Triplet { float* m; float* h; float* l; };

int dpad_of(int d) { return (d + kPanelW - 1) / kPanelW * kPanelW; }

void build_cholqr_tc(Builder& b, std::vector<Launch>& prog, const std::vector<Triplet>& X,
                     const std::vector<Triplet>& Q, bool shifted, bool gated = false) {
  shampoo4_ctx* h = b.h;
  const size_t nf = h->factors.size();
  int dmax = 0;
  for (auto& f : h->factors) if (f.tc) dmax = std::max(dmax, f.d);
  if (dmax == 0) return;
  const bool tf32_gram = shifted;          // the first pass only preconditions (above)
  {
    // Gram W = X^T X (lower triangle: fp32 into W, its TF32 split into
    // Th/Tl), optional shift
    // The gated pass first measures how far its input is from orthonormal
    // by a two-pass fp64 sketch of ||Q^T Q - I||_F (no Gram: on warm
    // refreshes every factor passes the gate, and a Gram's matrices would
    // never be read), then runs the Gram with outputs for the factors the
    // gate sends through the pass.
    std::vector<TcGemmDesc> g;
    std::vector<ShiftDescF> sd;
    std::vector<GateDesc> gd;
    std::vector<DiagDesc> dg;
    std::vector<SketchDesc> sk;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      if (!f.tc) continue;
      const int d = f.d;
      TcGemmDesc w = gemmtc(d, d, d, 1.0f, 0.0f);
      w.a = b.operand(X[i].h, tf32_gram ? nullptr : X[i].l, d, d, true, true, !tf32_gram);
      w.b = b.operand(X[i].h, tf32_gram ? nullptr : X[i].l, d, d, false, false, !tf32_gram,
                      tf32_gram ? 0 : kSquareBN);
      w.symmetric = 2;
      w.skip = b.tcbad(i);
      if (gated) {
        sk.push_back({X[i].m, b.wd(f.ws_sketch), b.devsq(i), d, 0, b.tcbad(i)});
        const double tol = kLastPassTol * std::sqrt(double(d));        // on ||Q^T Q - I||_F / sqrt(d)
        const double thr = std::min(tol * tol * d * double(kDevFineUnit), 0x1p62);
        gd.push_back({b.devsq(i), b.tcbad(i), b.skip3(i), static_cast<unsigned long long>(thr), b.wu(h->ws_p3any)});
        w.skip = b.skip3(i);
      }
      // only the lower triangles of W and of its TF32 split are ever read
      // (Cholesky blocks, panel updates, and the first panel's L21 product,
      // which takes W21 from the split): no mirror stores
      w.C = b.wf(f.ws_W); w.ldc = d;
      w.Chi = b.wf(f.ws_Th); w.Clo = b.wf(f.ws_Tl); w.ldh = d;
      g.push_back(w);
      dg.push_back({X[i].m, b.wf(f.ws_W), d, d, 0, gated ? b.skip3(i) : b.tcbad(i)});
      if (shifted) sd.push_back({b.wf(f.ws_W), d, d, kTcShift * float(d), b.tcbad(i)});
    }
    auto elems = [](const std::vector<DiagDesc>& v) { double s = 0; for (auto& x : v) s += double(x.d) * x.d; return s; };
    if (gated) {
      b.tag = SHAMPOO4_STAGE_QR_GRAM;
      double sk_elems = 0;
      for (auto& x : sk) sk_elems += double(x.d) * x.d;
      b.emit(prog, Kind::SketchZ, sk, dmax, 2.0 * sk_elems, 4.0 * sk_elems);
      b.emit(prog, Kind::SketchR, sk, dmax, 2.0 * kSketchCols * sk_elems, 4.0 * sk_elems);
      b.tag = SHAMPOO4_STAGE_QR_CONVERT;
      b.emit(prog, Kind::Gate, gd, 0);
      // the rest of the pass runs only if some factor goes through it
      b.guard = h->ws_p3any;
    }
    b.tag = SHAMPOO4_STAGE_QR_GRAM;
    emit_gemmtc(b, prog, g, !tf32_gram, tf32_gram ? 0 : kSquareBN);
    b.emit(prog, Kind::Diag, dg, dmax, 0, 4.0 * elems(dg));
    b.emit(prog, Kind::ShiftF, sd, 0);
  }
  // the rest of the pass: skipped for a broken-down factor, and for a
  // factor the gate passed
  auto skip_of = [&](size_t i) -> const uint32_t* { return gated ? b.skip3(i) : b.tcbad(i); };
  // Cholesky, left-looking by 64-wide panels.  For panel J:
  //   W[j:, J] -= L[j:, <J] L[J, <J]^T      tensor cores (also refreshes the
  //                                          TF32 split of that column block)
  //   L[J, J] = chol(W[J, J]), L[J, J]^-1     CUDA cores, fp64 inside
  //   L[j+jb:, J] = W[j+jb:, J] L[J, J]^-T    tensor cores
  // (Th, Tl) ends up holding the TF32 split of L; (Ih, Il) rows J hold the
  // split of L[J, J]^-1 for the solve.  A diagonal-shift pass may leave the
  // split of W's diagonal in Th/Tl only until the panel overwrites it.
  for (int j = 0; j < dmax; j += kPanelW) {
    std::vector<TcGemmDesc> up, l21;
    std::vector<PotrfDescF> po;
    double fl_po = 0;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      if (!f.tc || j >= f.d) continue;
      const int d = f.d, jb = std::min(kPanelW, d - j), rest = d - j - jb;
      float* W = b.wf(f.ws_W);
      float* Th = b.wf(f.ws_Th);
      float* Tl = b.wf(f.ws_Tl);
      if (j > 0) {
        TcGemmDesc u = gemmtc(d - j, jb, j, -1.0f, 1.0f);
        u.a = b.operand(Th, Tl, d, d, true, false, true);
        u.b = b.operand(Th, Tl, d, d, false, true, true, 64);
        u.a.row0 = u.b.row0 = j;
        u.C = W + int64_t(j) * d + j; u.ldc = d;
        u.Chi = Th + int64_t(j) * d + j; u.Clo = Tl + int64_t(j) * d + j; u.ldh = d;
        u.Cin = u.C; u.ldcin = d;
        u.skip = skip_of(i);
        up.push_back(u);
      }
      po.push_back({W + int64_t(j) * d + j, d, jb, 0, b.tcbad(i), b.gflags(), b.tcgood(i),
                    Th + int64_t(j) * d + j, Tl + int64_t(j) * d + j,
                    b.wf(f.ws_Ih) + int64_t(j) * kPanelW, b.wf(f.ws_Il) + int64_t(j) * kPanelW,
                    gated ? b.skip3(i) : nullptr, gated ? kLastPassPivot : 0.0f, 0, b.wu(h->ws_fbany)});
      fl_po += 2.0 * double(jb) * jb * jb / 3.0;
      if (rest <= 0) continue;
      TcGemmDesc t = gemmtc(rest, jb, jb, 1.0f, 0.0f);     // L21 = W21 L11^-T (in the split, in place)
      t.a = b.operand(Th, Tl, d, d, true, false, true);
      t.a.row0 = j + jb; t.a.col0 = j;
      t.b = b.operand(b.wf(f.ws_Ih), b.wf(f.ws_Il), dpad_of(d), kPanelW, false, true, true, 64);
      t.b.row0 = j;
      t.Chi = Th + int64_t(j + jb) * d + j; t.Clo = Tl + int64_t(j + jb) * d + j; t.ldh = d;
      t.skip = skip_of(i);
      l21.push_back(t);
    }
    b.tag = SHAMPOO4_STAGE_QR_SYRK;
    emit_gemmtc(b, prog, up, true, 64);
    b.tag = SHAMPOO4_STAGE_QR_POTRF;
    b.emit(prog, Kind::PotrfF, po, 0, fl_po);
    b.tag = SHAMPOO4_STAGE_QR_TRSM_PANEL;
    emit_gemmtc(b, prog, l21, true, 64);
  }
  // Solve Q L^T = X by 128-wide column panels J, one product each:
  //   Q[:, J] = (X[:, J] - Q[:, <J] L[J, <J]^T) L[J, J]^-T
  //           = Q[:, <J] H[J, <J]^T + X[:, J] L[J, J]^-T,
  // with H[J, <J] = -L[J, J]^-1 L[J, <J].  The 128 x 128 inverse diagonal
  // blocks are assembled from the 64 x 64 ones (k_inv128); the block rows
  // of H are one batched product written over L's split (each output tile
  // reads exactly the L tile it replaces, and nothing later reads L).  The
  // panel product takes K blocks below j from Q and H, and the last one
  // from X and L[J, J]^-1 (the second operand pair): no intermediate panel
  // goes through memory, and the 128-wide MMA runs at its full rate.
  {
    std::vector<Inv128Desc> iv;
    std::vector<TcGemmDesc> hv;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      if (!f.tc) continue;
      const int d = f.d, dp = int(align_up(size_t(d), kSolveW));
      for (int j = 0; j < d; j += kSolveW) {
        iv.push_back({b.wf(f.ws_Ih), b.wf(f.ws_Il), b.wf(f.ws_Th), b.wf(f.ws_Tl), b.wf(f.ws_Jh), b.wf(f.ws_Jl),
                      d, j, skip_of(i)});
        if (j == 0) continue;
        const int jb = std::min(kSolveW, d - j);
        TcGemmDesc g = gemmtc(jb, j, jb, -1.0f, 0.0f);               // H[J, <J]
        g.a = b.operand(b.wf(f.ws_Jh), b.wf(f.ws_Jl), dp, kSolveW, true, false, true);
        g.a.row0 = j;
        g.b = b.operand(b.wf(f.ws_Th), b.wf(f.ws_Tl), d, d, false, false, true);
        g.b.row0 = j;
        g.Chi = b.wf(f.ws_Th) + int64_t(j) * d; g.Clo = b.wf(f.ws_Tl) + int64_t(j) * d; g.ldh = d;
        g.skip = skip_of(i);
        hv.push_back(g);
      }
    }
    b.tag = SHAMPOO4_STAGE_QR_INVERSE;
    b.emit(prog, Kind::Inv128, iv, 0);
    emit_gemmtc(b, prog, hv, true, kSolveW);
  }
  for (int j = 0; j < dmax; j += kSolveW) {
    std::vector<TcGemmDesc> qp;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      if (!f.tc || j >= f.d) continue;
      const int d = f.d, jb = std::min(kSolveW, d - j);
      TcGemmDesc q = gemmtc(d, jb, j + jb, 1.0f, 0.0f);
      TcOperand xa = b.operand(X[i].h, X[i].l, d, d, true, false, true);          // X[:, J]
      xa.col0 = j;
      TcOperand jinv = b.operand(b.wf(f.ws_Jh), b.wf(f.ws_Jl), int(align_up(size_t(d), kSolveW)), kSolveW, false,
                                 true, true, kSolveW);                                 // L[J, J]^-T
      jinv.row0 = j;
      if (j > 0) {
        q.a = b.operand(Q[i].h, Q[i].l, d, d, true, false, true);                    // Q[:, <J]
        q.b = b.operand(b.wf(f.ws_Th), b.wf(f.ws_Tl), d, d, false, true, true, kSolveW);
        q.b.row0 = j;                                                                 // H[J, <J]^T
        q.a2 = xa; q.b2 = jinv; q.ksplit = j;
      } else {
        q.a = xa; q.b = jinv;
      }
      q.C = Q[i].m + j; q.ldc = d;
      q.Chi = Q[i].h + j; q.Clo = Q[i].l + j; q.ldh = d;
      q.skip = skip_of(i);
      qp.push_back(q);
    }
    b.tag = SHAMPOO4_STAGE_QR_SOLVE_UPDATE;
    emit_gemmtc(b, prog, qp, true, kSolveW);
  }
  if (gated) b.guard = SIZE_MAX;
}

// Refresh by the coupled Newton iteration (root methods NEWTON and
// NEWTON_Q4; "Shampoo -- Second-Order Optimizer", "Computing the inverse
// fourth root"): P = (S + eps I)^(-1/4) from the fp32 statistic with
// matrix products only.  A = S + eps I, c = ||A||_F, M = A / c, X = I; then
// newton_iters times F = (5 I - M) / 4, X <- X F, M <- F^4 M (F^4 as
// (F F)(F F)); P = X c^(-1/4).  Every product is fp32-accurate (3xTF32 on
// the tensor cores, fp32 on the CUDA cores): with TF32 products the
// iteration drifts off and diverges on condition numbers above about 1e5.
// The first iteration's X = I F is F itself (written by the INIT step).
// Buffers (per factor, from the eigen refresh's workspace): X in the two
// triplets X[0], X[1]; M in Z and (W, Th, Tl); F in (Sh, Sl); F^2 and F^4
// in the fp64 fallback regions, each as two fp32 d x d arrays.  A factor
// whose statistic holds NaN/Inf keeps its previous root.
void build_refresh_newton(Builder& b, std::vector<Launch>& prog) {
  shampoo4_ctx* h = b.h;
  const size_t nf = h->factors.size();
  const int iters = h->cfg.newton_iters;
  const bool q4 = h->cfg.root_method == SHAMPOO4_ROOT_NEWTON_Q4;
  int dmax = 0;
  int64_t emax = 0;
  double sum_dd = 0;
  for (auto& f : h->factors) {
    dmax = std::max(dmax, f.d);
    emax = std::max<int64_t>(emax, int64_t(f.d) * f.d);
    sum_dd += double(f.d) * f.d;
  }
  {  // non-finite statistic -> keep the previous root
    std::vector<ScanDesc> scan;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      ScanDesc sd{};
      sd.X = b.S(f); sd.ld = f.d; sd.rows = sd.cols = f.d;
      sd.ref.tab = -1;
      sd.flag = b.fail(i);
      sd.bit = SHAMPOO4_FLAG_NONFINITE_STATE;
      scan.push_back(sd);
    }
    b.tag = SHAMPOO4_STAGE_REFRESH_SCAN;
    b.emit(prog, Kind::Scan, scan, dmax, 0, 4.0 * sum_dd);
  }
  struct Bufs {
    float *xm[2], *xh[2], *xl[2], *mm[2], *mh[2], *ml[2];
    float *fm, *fh, *fl, *f2h, *f2l, *f4h, *f4l, *sc;
  };
  std::vector<Bufs> nb(nf);
  for (size_t i = 0; i < nf; ++i) {
    const FactorPlan& f = h->factors[i];
    const size_t dd = size_t(f.d) * f.d;
    Bufs& u = nb[i];
    std::memset(&u, 0, sizeof(u));
    u.sc = b.wf(f.ws_mu);
    float* w64 = reinterpret_cast<float*>(b.wd(f.ws_W64));
    float* q64 = reinterpret_cast<float*>(b.wd(f.ws_Q64));
    if (f.tc) {
      for (int k = 0; k < 2; ++k) {
        u.xm[k] = b.wf(f.ws_Xm[k]); u.xh[k] = b.wf(f.ws_Xh[k]); u.xl[k] = b.wf(f.ws_Xl[k]);
      }
      u.mm[0] = b.wf(f.ws_Zm); u.mh[0] = b.wf(f.ws_Zh); u.ml[0] = b.wf(f.ws_Zl);
      u.mm[1] = b.wf(f.ws_W); u.mh[1] = b.wf(f.ws_Th); u.ml[1] = b.wf(f.ws_Tl);
      u.fh = b.wf(f.ws_Sh); u.fl = b.wf(f.ws_Sl);
      u.f2h = w64; u.f2l = w64 + dd;
      u.f4h = q64; u.f4l = q64 + dd;
    } else {                                     // fp32 matrices only
      u.xm[0] = b.wf(f.ws_U); u.xm[1] = b.wf(f.ws_T);
      u.mm[0] = b.wf(f.ws_Y); u.mm[1] = w64;
      u.fm = w64 + dd;
      u.f2h = q64; u.f4h = q64 + dd;
    }
  }
  {
    std::vector<NewtonNormDesc> nd;
    std::vector<NewtonEltDesc> el;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      const Bufs& u = nb[i];
      nd.push_back({b.S(f), u.sc, f.d, h->cfg.eps, b.fail(i)});
      NewtonEltDesc e{};
      e.in = b.S(f); e.sc = u.sc; e.d = f.d; e.mode = kNewtonInit; e.eps = h->cfg.eps; e.skip = b.fail(i);
      e.m = u.mm[0]; e.mh = u.mh[0]; e.ml = u.ml[0];
      e.f = u.fm; e.fh = u.fh; e.fl = u.fl;
      e.x = u.xm[0]; e.xh = u.xh[0]; e.xl = u.xl[0];
      el.push_back(e);
    }
    b.tag = SHAMPOO4_STAGE_NEWTON_ELT;
    b.emit(prog, Kind::NewtonNorm, nd, 0, 0, 4.0 * sum_dd);
    b.emit(prog, Kind::NewtonElt, el, emax, 0, 20.0 * sum_dd);
  }
  int cx = 0, cm = 0;
  // C = A B for every factor: fp32-accurate on the tensor cores (split
  // operands) or on the CUDA cores; outputs as given (fp32, split)
  auto products = [&](auto pick) {
    std::vector<TcGemmDesc> t;
    std::vector<GemmF32Desc> g;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      const int d = f.d;
      float *ah, *al, *bh, *bl, *cm_, *ch, *cl;
      pick(nb[i], ah, al, bh, bl, cm_, ch, cl);
      if (f.tc) {
        TcGemmDesc x = gemmtc(d, d, d, 1.0f, 0.0f);
        x.a = b.operand(ah, al, d, d, true, false, true);
        x.b = b.operand(bh, bl, d, d, false, false, true, kSquareBN);
        x.C = cm_; x.ldc = d;
        x.Chi = ch; x.Clo = cl; x.ldh = d;
        x.skip = b.fail(i);
        t.push_back(x);
      } else {
        GemmF32Desc x = gemm32(d, d, d, 0, 0, kModeFP32, 1.0f, 0.0f);
        x.A = ah; x.lda = d;
        x.B = bh; x.ldb = d;
        x.C = cm_; x.ldc = d;
        x.skip = b.fail(i);
        g.push_back(x);
      }
    }
    b.tag = SHAMPOO4_STAGE_NEWTON_GEMM;
    emit_gemmtc(b, prog, t, true, kSquareBN);
    emit_gemm32(b, prog, g);
  };
  for (int it = 1; it <= iters; ++it) {
    if (it > 1) {                                            // X <- X F
      const int o = cx ^ 1;
      products([&](const Bufs& u, float*& ah, float*& al, float*& bh, float*& bl, float*& c, float*& ch,
                   float*& cl) {
        ah = u.xh[cx] ? u.xh[cx] : u.xm[cx]; al = u.xl[cx];
        bh = u.fh ? u.fh : u.fm; bl = u.fl;
        c = u.xm[o]; ch = u.xh[o]; cl = u.xl[o];
      });
      cx = o;
    }
    products([&](const Bufs& u, float*& ah, float*& al, float*& bh, float*& bl, float*& c, float*& ch,
                 float*& cl) {                                // F^2 = F F
      ah = bh = u.fh ? u.fh : u.fm; al = bl = u.fl;
      if (u.f2l) { c = nullptr; ch = u.f2h; cl = u.f2l; } else { c = u.f2h; ch = cl = nullptr; }
    });
    products([&](const Bufs& u, float*& ah, float*& al, float*& bh, float*& bl, float*& c, float*& ch,
                 float*& cl) {                                // F^4 = F^2 F^2
      ah = bh = u.f2h; al = bl = u.f2l;
      if (u.f4l) { c = nullptr; ch = u.f4h; cl = u.f4l; } else { c = u.f4h; ch = cl = nullptr; }
    });
    {
      const int o = cm ^ 1;
      products([&](const Bufs& u, float*& ah, float*& al, float*& bh, float*& bl, float*& c, float*& ch,
                   float*& cl) {                              // M <- F^4 M
        ah = u.f4h; al = u.f4l;
        bh = u.mh[cm] ? u.mh[cm] : u.mm[cm]; bl = u.ml[cm];
        c = u.mm[o]; ch = u.mh[o]; cl = u.ml[o];
      });
      cm = o;
    }
    if (it < iters) {                                         // F = 1.25 I - 0.25 M
      std::vector<NewtonEltDesc> el;
      for (size_t i = 0; i < nf; ++i) {
        const FactorPlan& f = h->factors[i];
        const Bufs& u = nb[i];
        NewtonEltDesc e{};
        e.in = u.mm[cm]; e.sc = u.sc; e.d = f.d; e.mode = kNewtonStep; e.skip = b.fail(i);
        e.f = u.fm; e.fh = u.fh; e.fl = u.fl;
        el.push_back(e);
      }
      b.tag = SHAMPOO4_STAGE_NEWTON_ELT;
      b.emit(prog, Kind::NewtonElt, el, emax, 0, 12.0 * sum_dd);
    }
  }
  // P = c^(-1/4) X: into the state (NEWTON) or a free workspace matrix to
  // be quantized (NEWTON_Q4)
  std::vector<float*> P(nf);
  {
    std::vector<NewtonEltDesc> el;
    std::vector<CopyDesc> cp;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      const Bufs& u = nb[i];
      P[i] = q4 ? u.mm[cm ^ 1] : b.sf(f.st_P);
      NewtonEltDesc e{};
      e.in = u.xm[cx]; e.sc = u.sc; e.d = f.d; e.mode = kNewtonFinal; e.skip = b.fail(i);
      e.m = P[i];
      el.push_back(e);
      cp.push_back({P[i], b.dbg(f.dbg_q), int64_t(f.d) * f.d});
    }
    b.tag = SHAMPOO4_STAGE_NEWTON_ELT;
    b.emit(prog, Kind::NewtonElt, el, emax, 0, 8.0 * sum_dd);
    b.tag = SHAMPOO4_STAGE_QR_CONVERT;
    b.emit(prog, Kind::Copy, cp, emax, 0, 8.0 * sum_dd);
  }
  if (q4) {  // quantize the root itself
    Launch L{};
    L.kind = Kind::Pack;
    L.tag = SHAMPOO4_STAGE_REQUANT;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      L.px.push_back(P[i]);
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

void build_refresh_owned(Builder& b, std::vector<Launch>& prog, bool first) {
  if (b.h->cfg.root_method != SHAMPOO4_ROOT_EIGEN) {
    build_refresh_newton(b, prog);
    return;
  }
  shampoo4_ctx* h = b.h;
  const size_t nf = h->factors.size();
  const bool split = split_of(h->cfg);
  int dmax = 0;
  int64_t emax = 0;
  double sum_dd = 0;
  for (auto& f : h->factors) {
    dmax = std::max(dmax, f.d);
    emax = std::max<int64_t>(emax, int64_t(f.d) * f.d);
    sum_dd += double(f.d) * f.d;
  }
  {  // non-finite statistic -> keep the factor's previous basis; split S
    std::vector<ScanDesc> scan;
    double bytes = 0;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      ScanDesc s{};
      s.X = b.S(f); s.ld = f.d; s.rows = s.cols = f.d;
      s.ref.tab = -1;
      s.flag = b.fail(i);
      s.bit = SHAMPOO4_FLAG_NONFINITE_STATE;
      if (f.tc) { s.oh = b.wf(f.ws_Sh); s.ol = b.wf(f.ws_Sl); }
      scan.push_back(s);
      bytes += (f.tc ? 12.0 : 4.0) * double(f.d) * f.d;
    }
    b.tag = SHAMPOO4_STAGE_REFRESH_SCAN;
    b.emit(prog, Kind::Scan, scan, dmax, 0, bytes);
  }
  // cur/oth: index of the current and the other triplet (tensor-core
  // factors) or buffer offsets (CUDA-core factors).
  std::vector<int> cur(nf, 0);
  std::vector<size_t> ucur(nf), uoth(nf);
  for (size_t i = 0; i < nf; ++i) { ucur[i] = h->factors[i].ws_U; uoth[i] = h->factors[i].ws_Y; }
  {
    std::vector<BasisDesc> bd;
    double bytes = 0;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      BasisDesc x{};
      x.codes = b.sb(f.st_codes); x.scales = b.sf(f.st_scales);
      x.d = f.d; x.identity = first ? 1 : 0;
      x.codebook = h->cfg.codebook;
      // TF32 Björck reads only U's hi part (and rewrites lo at its last
      // step); without Björck steps the fp32-accurate subspace product
      // reads both parts
      if (f.tc) {
        // with TF32 Björck steps the dequantized U is read only through its
        // TF32 value (the products' operand and the first step's 1.5 U): no
        // fp32 copy is written
        const bool tf32_bjorck = !split && !first && h->cfg.bjorck_iters > 0;
        x.U = tf32_bjorck ? nullptr : b.wf(f.ws_Xm[0]); x.Uh = b.wf(f.ws_Xh[0]);
        x.Ul = (split || first || h->cfg.bjorck_iters == 0) ? b.wf(f.ws_Xl[0]) : nullptr;
      }
      else x.U = b.wf(f.ws_U);
      bd.push_back(x);
      bytes += (first ? 0.0 : 0.5625) * double(f.d) * f.d +
               4.0 * ((x.U ? 1 : 0) + (x.Uh ? 1 : 0) + (x.Ul ? 1 : 0)) * double(f.d) * f.d;
    }
    b.tag = SHAMPOO4_STAGE_BASIS;
    b.emit(prog, Kind::Basis, bd, emax, 0, bytes);
  }
  // Bjorck rectification U <- 1.5 U - 0.5 U (U^T U).
  const int iters = first ? 0 : h->cfg.bjorck_iters;
  for (int it = 0; it < iters; ++it) {
    std::vector<GemmF32Desc> gram, upd;
    std::vector<TcGemmDesc> tgram, tupd;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      const int d = f.d;
      if (f.tc) {
        const int c = cur[i], o = 1 - c;
        TcGemmDesc g = gemmtc(d, d, d, 1.0f, 0.0f);          // T = U^T U
        g.a = b.operand(b.wf(f.ws_Xh[c]), b.wf(f.ws_Xl[c]), d, d, true, true, split);
        g.b = b.operand(b.wf(f.ws_Xh[c]), b.wf(f.ws_Xl[c]), d, d, false, false, split);
        // the update reads T's lo part only when fp32-accurate.  T is
        // symmetric: only the tiles touching the lower triangle are computed,
        // written in full (mode 3; no mirror stores), and the update reads
        // the K blocks beyond them from their transposes.
        g.symmetric = 3;
        g.Chi = b.wf(f.ws_Th); g.Clo = split ? b.wf(f.ws_Tl) : nullptr; g.ldh = d;
        tgram.push_back(g);
        TcGemmDesc u = gemmtc(d, d, d, -0.5f, 1.5f);         // U' = 1.5 U - 0.5 U T
        u.a = b.operand(b.wf(f.ws_Xh[c]), b.wf(f.ws_Xl[c]), d, d, true, false, split);
        u.b = b.operand(b.wf(f.ws_Th), b.wf(f.ws_Tl), d, d, false, true, split);   // T symmetric
        u.bt_hi = b.map(b.wf(f.ws_Th), d, d, 32, 1);
        u.bt_lo = split ? b.map(b.wf(f.ws_Tl), d, d, 32, 1) : nullptr;
        // With TF32 products the iterates are TF32 numbers between steps:
        // every step takes 1.5 U from U's TF32 value (the first from the
        // dequantized U's), and only the last step writes fp32 U (the
        // products' own TF32 rounding already limits the iteration to that
        // precision).
        const bool last = it + 1 == iters;
        u.Cin = split ? b.wf(f.ws_Xm[c]) : b.wf(f.ws_Xh[c]); u.ldcin = d;
        u.C = (split || last) ? b.wf(f.ws_Xm[o]) : nullptr; u.ldc = d;
        // U's lo part feeds the next Björck products only when fp32-accurate;
        // the last one always feeds the fp32-accurate subspace product
        u.Chi = b.wf(f.ws_Xh[o]); u.Clo = (split || last) ? b.wf(f.ws_Xl[o]) : nullptr; u.ldh = d;
        tupd.push_back(u);
        cur[i] = o;
      } else {
        GemmF32Desc g = gemm32(d, d, d, 1, 0, mode_of(h->cfg), 1.0f, 0.0f);
        g.A = g.B = b.wf(ucur[i]); g.lda = g.ldb = d;
        g.C = b.wf(f.ws_T); g.ldc = d;
        g.symmetric = 1;
        gram.push_back(g);
        GemmF32Desc u = gemm32(d, d, d, 0, 0, mode_of(h->cfg), -0.5f, 1.5f);
        u.A = b.wf(ucur[i]); u.lda = d;
        u.B = b.wf(f.ws_T); u.ldb = d;
        u.C = b.wf(uoth[i]); u.ldc = d;
        u.Cin = b.wf(ucur[i]); u.ldcin = d;
        upd.push_back(u);
        std::swap(ucur[i], uoth[i]);
      }
    }
    b.tag = SHAMPOO4_STAGE_BJORCK_GRAM;
    emit_gemmtc(b, prog, tgram, split);
    emit_gemm32(b, prog, gram);
    b.tag = SHAMPOO4_STAGE_BJORCK_UPDATE;
    emit_gemmtc(b, prog, tupd, split);
    emit_gemm32(b, prog, upd);
  }
  {  // debug capture of the rectified basis (launch skipped without a capture buffer)
    std::vector<CopyDesc> cp;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      const float* U = f.tc ? b.wf(f.ws_Xm[cur[i]]) : b.wf(ucur[i]);
      cp.push_back({U, b.dbg(f.dbg_u), int64_t(f.d) * f.d});
    }
    b.tag = SHAMPOO4_STAGE_BASIS;
    b.emit(prog, Kind::Copy, cp, emax, 0, 8.0 * sum_dd);
  }
  // Subspace step Y = (S + eps I) U = S U + eps U, always fp32-accurate.
  std::vector<const float*> Yx(nf);
  std::vector<float*> Q0(nf), Q1(nf), Qf(nf), Qh(nf, nullptr), Ql(nf, nullptr), none(nf, nullptr);
  {
    std::vector<GemmF32Desc> g;
    std::vector<TcGemmDesc> t;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      const int d = f.d;
      if (f.tc) {
        const int c = cur[i], o = 1 - c;
        TcGemmDesc y = gemmtc(d, d, d, 1.0f, h->cfg.eps);
        y.a = b.operand(b.wf(f.ws_Sh), b.wf(f.ws_Sl), d, d, true, false, true);
        y.b = b.operand(b.wf(f.ws_Xh[c]), b.wf(f.ws_Xl[c]), d, d, false, false, true, kSquareBN);
        y.Cin = b.wf(f.ws_Xm[c]); y.ldcin = d;
        y.C = b.wf(f.ws_Xm[o]); y.ldc = d;
        y.Chi = b.wf(f.ws_Xh[o]); y.Clo = b.wf(f.ws_Xl[o]); y.ldh = d;
        t.push_back(y);
        // shifted CholeskyQR3: Y (X[o]) -> Q0 (X[c]) -> Q1 (X[o]) -> Q (X[c] + split)
        Yx[i] = b.wf(f.ws_Xm[o]);
        Q0[i] = b.wf(f.ws_Xm[c]);
        Q1[i] = b.wf(f.ws_Xm[o]);
        Qf[i] = b.wf(f.ws_Xm[c]);
        Qh[i] = b.wf(f.ws_Xh[c]);
        Ql[i] = b.wf(f.ws_Xl[c]);
      } else {
        GemmF32Desc y = gemm32(d, d, d, 0, 0, kModeFP32, 1.0f, h->cfg.eps);
        y.A = b.S(f); y.lda = d;
        y.B = b.wf(ucur[i]); y.ldb = d;
        y.C = b.wf(uoth[i]); y.ldc = d;
        y.Cin = b.wf(ucur[i]); y.ldcin = d;
        g.push_back(y);
        Yx[i] = b.wf(uoth[i]);
        Q0[i] = b.wf(ucur[i]);
        Q1[i] = b.wf(uoth[i]);
        Qf[i] = b.wf(ucur[i]);
      }
    }
    b.tag = SHAMPOO4_STAGE_SUBSPACE;
    emit_gemmtc(b, prog, t, true, kSquareBN);
    emit_gemm32(b, prog, g);
  }
  {
    // Tensor-core factors: Y stays in X[o]; fp32 shifted Cholesky-QR
    // Y -> Z -> X[c], then the gated third pass in place on X[c] (its Gram
    // and diagonal read X[c] first; panel J of the solve reads only column
    // block J of the input and the already-rewritten blocks before it).  A
    // factor whose fp32 Cholesky breaks down (tcbad) redoes three passes in
    // fp64 from the intact Y; the others skip that work (tcgood).  CUDA-core
    // factors run the fp64 passes only.
    std::vector<Triplet> Xy(nf), Xc(nf), Xz(nf);
    std::vector<char> use_simt(nf, 0), use_fb(nf, 0);
    std::vector<const uint32_t*> sk(nf);
    std::vector<const float*> a1(nf), a2(nf), a3(nf);
    std::vector<float*> o1(nf), o2(nf), o3(nf), q3h(nf, nullptr), q3l(nf, nullptr);
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      if (f.tc) {
        const int c = cur[i], o = 1 - c;
        Xy[i] = {b.wf(f.ws_Xm[o]), b.wf(f.ws_Xh[o]), b.wf(f.ws_Xl[o])};
        Xc[i] = {b.wf(f.ws_Xm[c]), b.wf(f.ws_Xh[c]), b.wf(f.ws_Xl[c])};
        Xz[i] = {b.wf(f.ws_Zm), b.wf(f.ws_Zh), b.wf(f.ws_Zl)};
        use_fb[i] = 1;
        sk[i] = b.tcgood(i);
        a1[i] = Xy[i].m; o1[i] = Xc[i].m;
        a2[i] = Xc[i].m; o2[i] = Xz[i].m;
        a3[i] = Xz[i].m; o3[i] = Xc[i].m;
        q3h[i] = Xc[i].h; q3l[i] = Xc[i].l;
        Qf[i] = Xc[i].m; Qh[i] = Xc[i].h; Ql[i] = Xc[i].l;
        Q1[i] = Xz[i].m;                                  // free after the QR
      } else {
        use_simt[i] = 1;
        sk[i] = b.fail(i);
        a1[i] = Yx[i]; o1[i] = Q0[i];
        a2[i] = Q0[i]; o2[i] = Q1[i];
        a3[i] = Q1[i]; o3[i] = Qf[i];
      }
    }
    build_cholqr_tc(b, prog, Xy, Xz, true);
    build_cholqr_tc(b, prog, Xz, Xc, false);
    build_cholqr_tc(b, prog, Xc, Xc, false, true);
    std::vector<char> use_any(nf);
    for (size_t i = 0; i < nf; ++i) use_any[i] = use_simt[i] || use_fb[i];
    // fp64 passes: the whole launches are skipped unless some factor takes
    // them (a CUDA-core factor, or a tensor-core factor that broke down)
    b.guard = h->ws_fbany;
    build_cholqr_pass(b, prog, use_any, a1, o1, none, none, sk, true);
    build_cholqr_pass(b, prog, use_any, a2, o2, none, none, sk, false);
    build_cholqr_pass(b, prog, use_any, a3, o3, q3h, q3l, sk, false);
    b.guard = SIZE_MAX;
  }
  for (size_t i = 0; i < nf; ++i) {
    const size_t off = size_t(reinterpret_cast<uint8_t*>(Qf[i]) - b.ws);
    (first ? h->factors[i].ws_q_first : h->factors[i].ws_q_next) = off;
  }
  {  // debug capture of the pre-quantization Q
    std::vector<CopyDesc> cp;
    for (size_t i = 0; i < nf; ++i)
      cp.push_back({Qf[i], b.dbg(h->factors[i].dbg_q), int64_t(h->factors[i].d) * h->factors[i].d});
    b.tag = SHAMPOO4_STAGE_QR_CONVERT;
    b.emit(prog, Kind::Copy, cp, emax, 0, 8.0 * sum_dd);
  }
  // Rayleigh quotients: T = S Q (fp32-accurate), lambda_i = max(q_i . t_i, 0).
  {
    std::vector<GemmF32Desc> g;
    std::vector<TcGemmDesc> t;
    std::vector<RayleighDesc> rq;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      const int d = f.d;
      float* T;
      if (f.tc) {
        T = Q1[i];                                         // free again
        TcGemmDesc x = gemmtc(d, d, d, 1.0f, 0.0f);
        x.a = b.operand(b.wf(f.ws_Sh), b.wf(f.ws_Sl), d, d, true, false, true);
        x.b = b.operand(Qh[i], Ql[i], d, d, false, false, true, kSquareBN);
        x.C = T; x.ldc = d;
        t.push_back(x);
      } else {
        T = b.wf(f.ws_T);
        GemmF32Desc x = gemm32(d, d, d, 0, 0, kModeFP32, 1.0f, 0.0f);
        x.A = b.S(f); x.lda = d;
        x.B = Qf[i]; x.ldb = d;
        x.C = T; x.ldc = d;
        g.push_back(x);
      }
      rq.push_back({Qf[i], T, b.sf(f.st_lam), d, 0, b.fail(i)});
    }
    b.tag = SHAMPOO4_STAGE_RAYLEIGH_GEMM;
    emit_gemmtc(b, prog, t, true, kSquareBN);
    emit_gemm32(b, prog, g);
    b.tag = SHAMPOO4_STAGE_RAYLEIGH;
    b.emit(prog, Kind::Rayleigh, rq, dmax, 2.0 * sum_dd);
  }
  {  // requantize Q into the state (skipped for failed factors)
    Launch L{};
    L.kind = Kind::Pack;
    L.tag = SHAMPOO4_STAGE_REQUANT;
    for (size_t i = 0; i < nf; ++i) {
      const FactorPlan& f = h->factors[i];
      L.px.push_back(Qf[i]);
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

// The refresh programs cover this rank's factors only, split into up to
// nparts parts balanced by d^3 cost (longest first, each to the lighter
// part; each part keeps the factors' order).  Each part's program is built
// over its subset of the factors (per-factor scratch words keep the
// factors' own indices, through Builder::gmap), and the workspace offsets
// the builder assigns are copied back.
void build_refresh(Builder& b, Program& prog, bool first) {
  shampoo4_ctx* h = b.h;
  const int ng = ngroups(h);
  if (ng > 1) {
    for (int g = 0; g < ng; ++g) {
      GroupScope scope(b, h->group_begin[g], h->group_begin[g + 1]);
      build_refresh_owned(b, prog.add(g % 2), first);
    }
    return;
  }
  std::vector<size_t> owned;
  for (size_t i = 0; i < h->factors.size(); ++i)
    if (h->owner[i] == h->rank) owned.push_back(i);
  const int nparts = owned.size() >= 2 ? h->refresh_parts : 1;
  std::vector<std::vector<size_t>> parts(nparts);
  {
    std::vector<size_t> order = owned;
    auto cost = [&](size_t i) { return double(h->factors[i].d) * h->factors[i].d * h->factors[i].d; };
    std::stable_sort(order.begin(), order.end(), [&](size_t a, size_t c) { return cost(a) > cost(c); });
    std::vector<double> load(nparts, 0.0);
    for (size_t i : order) {
      int p = 0;
      for (int q = 1; q < nparts; ++q)
        if (load[q] < load[p]) p = q;
      parts[p].push_back(i);
      load[p] += cost(i);
    }
    for (auto& v : parts) std::sort(v.begin(), v.end());
  }
  for (int p = 0; p < nparts; ++p) {
    if (parts[p].empty()) continue;
    std::vector<FactorPlan> sub;
    for (size_t i : parts[p]) sub.push_back(h->factors[i]);
    std::vector<FactorPlan> all;
    all.swap(h->factors);
    h->factors = sub;
    b.gmap = &parts[p];
    build_refresh_owned(b, prog.add(nparts == 1 ? -1 : p), first);
    b.gmap = nullptr;
    for (size_t j = 0; j < parts[p].size(); ++j) {
      all[parts[p][j]].ws_q_first = h->factors[j].ws_q_first;
      all[parts[p][j]].ws_q_next = h->factors[j].ws_q_next;
    }
    h->factors.swap(all);
  }
}

void build_precondition_into(Builder& b, std::vector<Launch>& prog) {
  shampoo4_ctx* h = b.h;
  const size_t nf = h->factors.size();
  const bool split = split_of(h->cfg);
  int dmax = 0;
  int64_t emax = 0;
  double sum_dd = 0;
  for (auto& f : h->factors) {
    dmax = std::max(dmax, f.d);
    emax = std::max<int64_t>(emax, int64_t(f.d) * f.d);
    sum_dd += double(f.d) * f.d;
  }
  std::vector<BasisDesc> bd;
  std::vector<MuDesc> mu;
  std::vector<GemmF32Desc> roots;
  std::vector<TcGemmDesc> troots;
  std::vector<RowDiagDesc> rdiag;              // exact diagonal of the fp32-accurate roots
  std::vector<float*> Pm(nf);                  // fp32 root of each factor
  double bytes_bd = 0;
  const bool newton = h->cfg.root_method != SHAMPOO4_ROOT_EIGEN;
  std::vector<ScanDesc> psplit;                // NEWTON: TF32 split of the stored root
  for (size_t i = 0; i < nf; ++i) {
    const FactorPlan& f = h->factors[i];
    const int d = f.d;
    BasisDesc x{};
    x.codes = b.sb(f.st_codes); x.scales = b.sf(f.st_scales); x.d = d; x.identity = 0;
    x.codebook = h->cfg.codebook;
    if (newton) {
      // the root from the refresh: fp32 in the state (NEWTON), or its 4-bit
      // codes (NEWTON_Q4); tensor-core factors also need its TF32 split in
      // Th/Tl, and the fp32 copy feeds a tile that is not a tensor-core tile
      const bool tile_tc = h->blocks[f.block].tc;
      if (h->cfg.root_method == SHAMPOO4_ROOT_NEWTON) {
        Pm[i] = b.sf(f.st_P);
        if (f.tc) {
          ScanDesc sd{};
          sd.X = b.sf(f.st_P); sd.ld = d; sd.rows = sd.cols = d;
          sd.ref.tab = -1;
          sd.flag = b.tcbad(i);                 // scratch word; bit 0 raises nothing
          sd.oh = b.wf(f.ws_Th); sd.ol = split ? b.wf(f.ws_Tl) : nullptr;
          psplit.push_back(sd);
          bytes_bd += (4.0 + (split ? 8.0 : 4.0)) * double(d) * d;
        }
      } else {
        x.U = f.tc ? (tile_tc ? nullptr : b.wf(f.ws_Xm[1])) : b.wf(f.ws_U);
        if (f.tc) { x.Uh = b.wf(f.ws_Th); x.Ul = split ? b.wf(f.ws_Tl) : nullptr; }
        Pm[i] = f.tc ? b.wf(f.ws_Xm[1]) : b.wf(f.ws_U);
        bd.push_back(x);
        bytes_bd += (0.5625 + 4.0 + (split ? 8.0 : 4.0)) * double(d) * d;
      }
      continue;
    }
    mu.push_back({b.sf(f.st_lam), b.wf(f.ws_mu), d, 0});
    if (f.tc) {
      // U -> X[0] split, U diag(mu) -> X[1] split; P = (U mu) U^T -> Th/Tl (+ fp32 in X[1].m)
      x.Uh = b.wf(f.ws_Xh[0]); x.Ul = split ? b.wf(f.ws_Xl[0]) : nullptr;
      x.mu = b.wf(f.ws_mu);
      x.Vh = b.wf(f.ws_Xh[1]); x.Vl = split ? b.wf(f.ws_Xl[1]) : nullptr;
      TcGemmDesc g = gemmtc(d, d, d, 1.0f, 0.0f);
      g.a = b.operand(b.wf(f.ws_Xh[1]), b.wf(f.ws_Xl[1]), d, d, true, false, split);
      g.b = b.operand(b.wf(f.ws_Xh[0]), b.wf(f.ws_Xl[0]), d, d, false, true, split);
      // P is symmetric: for a tensor-core tile only the tiles touching its
      // lower triangle are computed, written in full (mode 3), and the
      // applies read the K blocks beyond them from their transposes.  Its
      // fp32 copy feeds only the CUDA-core apply of a tile that is not a
      // tensor-core tile, which reads all of it (a full product then).
      float* pm = h->blocks[f.block].tc ? nullptr : b.wf(f.ws_Xm[1]);
      if (!pm) g.symmetric = 3;
      g.C = pm; g.ldc = d;
      g.Chi = b.wf(f.ws_Th); g.Clo = split ? b.wf(f.ws_Tl) : nullptr; g.ldh = d;
      troots.push_back(g);
      if (split)
        rdiag.push_back({b.wf(f.ws_Xh[1]), b.wf(f.ws_Xl[1]), b.wf(f.ws_Xh[0]), b.wf(f.ws_Xl[0]), d, d, 0,
                         pm, b.wf(f.ws_Th), b.wf(f.ws_Tl)});
      Pm[i] = b.wf(f.ws_Xm[1]);
      bytes_bd += (0.5625 + (split ? 16.0 : 8.0)) * double(d) * d;
    } else {
      x.U = b.wf(f.ws_Y);
      GemmF32Desc g = gemm32(d, d, d, 0, 1, mode_of(h->cfg), 1.0f, 0.0f);
      g.A = b.wf(f.ws_Y); g.lda = d; g.kscale = b.wf(f.ws_mu);
      g.B = b.wf(f.ws_Y); g.ldb = d;
      g.C = b.wf(f.ws_U); g.ldc = d;
      g.symmetric = 1;
      roots.push_back(g);
      Pm[i] = b.wf(f.ws_U);
      bytes_bd += 4.5625 * double(d) * d;
    }
    bd.push_back(x);
  }
  b.tag = SHAMPOO4_STAGE_PRECOND_MU;
  b.emit(prog, Kind::Mu, mu, dmax);
  b.tag = SHAMPOO4_STAGE_PRECOND_DEQUANT;
  b.emit(prog, Kind::Basis, bd, emax, 0, bytes_bd);
  b.emit(prog, Kind::Scan, psplit, dmax, 0, bytes_bd);
  b.tag = SHAMPOO4_STAGE_ROOTS;
  emit_gemmtc(b, prog, troots, split);
  b.emit(prog, Kind::RowDiag, rdiag, dmax, 0, 16.0 * sum_dd);
  emit_gemm32(b, prog, roots);
  build_grad_copy(b, prog, SHAMPOO4_STAGE_STATS_SCAN, false);
  std::vector<GemmF32Desc> left, right;
  std::vector<TcGemmDesc> tleft, tright;
  for (size_t k = 0; k < h->blocks.size(); ++k) {
    const BlockPlan& bp = h->blocks[k];
    const FactorPlan& fl = h->factors[2 * k];
    const FactorPlan& fr = h->factors[2 * k + 1];
    if (bp.tc) {
      TcGemmDesc l = gemmtc(bp.m, bp.n, bp.m, 1.0f, 0.0f);       // B = P_L G
      l.a = b.operand(b.wf(fl.ws_Th), b.wf(fl.ws_Tl), bp.m, bp.m, true, false, split);
      if (!newton) {                                              // P_L stored by its lower tiles
        l.at_hi = b.map(b.wf(fl.ws_Th), bp.m, bp.m, 32, 1);
        l.at_lo = split ? b.map(b.wf(fl.ws_Tl), bp.m, bp.m, 32, 1) : nullptr;
      }
      l.b = b.operand(b.wf(bp.ws_Gh), b.wf(bp.ws_Gl), bp.m, bp.n, false, false, split);
      l.Chi = b.wf(bp.ws_Bh); l.Clo = split ? b.wf(bp.ws_Bl) : nullptr; l.ldh = bp.n;
      tleft.push_back(l);
      TcGemmDesc r = gemmtc(bp.m, bp.n, bp.n, 1.0f, 0.0f);       // D = B P_R
      r.a = b.operand(b.wf(bp.ws_Bh), b.wf(bp.ws_Bl), bp.m, bp.n, true, false, split);
      // P_R is symmetric for the eigen and fp32 Newton roots, read K-major as
      // P_R^T; a root quantized itself (NEWTON_Q4: blocks run along rows) is
      // not, and is read as stored
      const bool sym = h->cfg.root_method != SHAMPOO4_ROOT_NEWTON_Q4;
      r.b = b.operand(b.wf(fr.ws_Th), b.wf(fr.ws_Tl), bp.n, bp.n, false, sym, split);
      if (!newton) {                                              // P_R stored by its lower tiles
        r.bt_hi = b.map(b.wf(fr.ws_Th), bp.n, bp.n, 32, 1);
        r.bt_lo = split ? b.map(b.wf(fr.ws_Tl), bp.n, bp.n, 32, 1) : nullptr;
      }
      r.c_ref = {1, bp.param, bp.r0, bp.c0};
      r.sumsq = bp.dsq_n ? b.wd(h->ws_dsq) + bp.dsq_off : nullptr;   // ||D||^2 for the grafted update
      tright.push_back(r);
    } else {
      float* tmp = b.wf(bp.ws_tmp);
      GemmF32Desc l = gemm32(bp.m, bp.n, bp.m, 0, 0, mode_of(h->cfg), 1.0f, 0.0f);
      l.A = Pm[2 * k]; l.lda = bp.m;
      l.b_ref = {0, bp.param, bp.r0, bp.c0};
      l.C = tmp; l.ldc = bp.n;
      left.push_back(l);
      GemmF32Desc r = gemm32(bp.m, bp.n, bp.n, 0, 0, mode_of(h->cfg), 1.0f, 0.0f);
      r.A = tmp; r.lda = bp.n;
      r.B = Pm[2 * k + 1]; r.ldb = bp.n;
      r.c_ref = {1, bp.param, bp.r0, bp.c0};
      right.push_back(r);
    }
  }
  b.tag = SHAMPOO4_STAGE_APPLY_LEFT;
  emit_gemmtc(b, prog, tleft, split);
  emit_gemm32(b, prog, left);
  b.tag = SHAMPOO4_STAGE_APPLY_RIGHT;
  emit_gemmtc(b, prog, tright, split);
  emit_gemm32(b, prog, right);
}

void build_precondition(Builder& b) {
  shampoo4_ctx* h = b.h;
  const int ng = ngroups(h);
  if (ng == 1) {
    build_precondition_into(b, h->prog_precond.add(-1));
    return;
  }
  for (int g = 0; g < ng; ++g) {
    GroupScope scope(b, h->group_begin[g], h->group_begin[g + 1]);
    build_precondition_into(b, h->prog_precond.add(g % 2));
  }
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
    const uint32_t* guard =
        L.guard_off == SIZE_MAX ? nullptr : reinterpret_cast<const uint32_t*>(h->d_ws + L.guard_off);
    shampoo4_ctx::Rec rec{L.tag, nullptr, nullptr, L.flops, L.bytes, 1};
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
        S4_TRY(launch_gemm_f64(static_cast<const GemmF64Desc*>(d), L.count, int(L.extent), st, guard));
        break;
      case Kind::Potrf:
        S4_TRY(launch_potrf(static_cast<const PotrfDesc*>(d), L.count, st, guard));
        break;
      case Kind::Trsm:
        S4_TRY(launch_trsm(static_cast<const TrsmDesc*>(d), L.count, int(L.extent), st, guard));
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
      case Kind::GemmTC:
      case Kind::GemmTCSplit:
      case Kind::GemmTCSplit64:
        S4_TRY(launch_gemm_tc(static_cast<const TcGemmDesc*>(d), L.count, int(L.extent),
                              L.kind == Kind::GemmTC ? 0 : 1, L.kind == Kind::GemmTCSplit64 ? 64 : 0, tabs, np,
                              gflags, st, h->wait_ns, L.tiles, guard,
                              L.list_off == SIZE_MAX ? nullptr
                                                     : reinterpret_cast<const uint64_t*>(h->d_ws + h->ws_desc +
                                                                                         L.list_off)));
        break;
      case Kind::PotrfF:
        S4_TRY(launch_potrf_f(static_cast<const PotrfDescF*>(d), L.count, st, guard));
        break;
      case Kind::ShiftF:
        S4_TRY(launch_shift_f(static_cast<const ShiftDescF*>(d), L.count, st));
        break;
      case Kind::Gate:
        S4_TRY(launch_gate(static_cast<const GateDesc*>(d), L.count, st));
        break;
      case Kind::Diag:
        S4_TRY(launch_diag(static_cast<const DiagDesc*>(d), L.count, int(L.extent), st, guard));
        break;
      case Kind::SketchZ:
      case Kind::SketchR:
        S4_TRY(launch_sketch(static_cast<const SketchDesc*>(d), L.count, int(L.extent),
                             L.kind == Kind::SketchZ ? 0 : 1, st));
        break;
      case Kind::Inv128:
        S4_TRY(launch_inv128(static_cast<const Inv128Desc*>(d), L.count, st, guard));
        break;
      case Kind::RowDiag:
        S4_TRY(launch_rowdiag(static_cast<const RowDiagDesc*>(d), L.count, int(L.extent), st));
        break;
      case Kind::Shift:
        S4_TRY(launch_shift(static_cast<const ShiftDesc*>(d), L.count, st, guard));
        break;
      case Kind::Convert:
        S4_TRY(launch_convert(static_cast<const ConvertDesc*>(d), L.count, L.extent, st, guard));
        break;
      case Kind::NewtonNorm:
        S4_TRY(launch_newton_norm(static_cast<const NewtonNormDesc*>(d), L.count, st));
        break;
      case Kind::NewtonElt:
        S4_TRY(launch_newton_elt(static_cast<const NewtonEltDesc*>(d), L.count, L.extent, st));
        break;
      case Kind::Copy:
        if (h->d_dbg) S4_TRY(launch_copy(static_cast<const CopyDesc*>(d), L.count, L.extent, st));
        break;
      case Kind::Pack:
        S4_TRY(launch_pack(L.px.data(), L.pn.data(), L.count, L.pcodes.data(), L.pscales.data(), st,
                           L.pskip.data(), &rec.kernels, h->cfg.codebook));
        break;
    }
    if (h->timing) {
      S4_CUDA(cudaEventRecord(rec.e1, st));
      h->recs.push_back(rec);
    }
  }
  return SHAMPOO4_OK;
}

// Run one call's program: its sequences on their lanes, the handle's
// streams forked from the caller's stream and joined back to it.
shampoo4_status run_program(shampoo4_ctx* h, const Program& P, cudaStream_t st) {
  bool used[shampoo4_ctx::kMaxParts] = {};
  bool fork = false;
  for (int l : P.lane)
    if (l >= 0) used[l] = fork = true;
  if (!fork) {
    for (const auto& q : P.seq) S4_TRY(run(h, q, st));
    return SHAMPOO4_OK;
  }
  S4_CUDA(cudaEventRecord(h->part_fork, st));
  for (int p = 0; p < shampoo4_ctx::kMaxParts; ++p)
    if (used[p]) S4_CUDA(cudaStreamWaitEvent(h->part_stream[p], h->part_fork, 0));
  for (size_t i = 0; i < P.seq.size(); ++i)
    S4_TRY(run(h, P.seq[i], P.lane[i] < 0 ? st : h->part_stream[P.lane[i]]));
  for (int p = 0; p < shampoo4_ctx::kMaxParts; ++p)
    if (used[p]) {
      S4_CUDA(cudaEventRecord(h->part_join[p], h->part_stream[p]));
      S4_CUDA(cudaStreamWaitEvent(st, h->part_join[p], 0));
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
    h->t_launches[r.tag] += r.kernels;
    h->ev_pool.push_back(r.e0);
    h->ev_pool.push_back(r.e1);
  }
  h->recs.clear();
  return SHAMPOO4_OK;
}

// Write a per-call pointer table into the workspace at `region`: by a
// one-warp kernel that carries the table as its parameter (a stream
// operation, capturable), or, beyond kMaxTableEntries entries, by a copy
// from a pinned host buffer (guarded by an event; not capturable).
shampoo4_status upload_table(shampoo4_ctx* h, const std::vector<PtrEntry>& t, size_t region, PtrEntry* pinned,
                             cudaEvent_t ev, bool& ev_pending, bool capturing, cudaStream_t st) {
  PtrEntry* dst = reinterpret_cast<PtrEntry*>(h->d_ws + region);
  if (t.size() <= size_t(kMaxTableEntries)) {
    shampoo4_ctx::Rec rec{SHAMPOO4_STAGE_TABLES, nullptr, nullptr, 0.0, 16.0 * double(t.size()), 1};
    if (h->timing) {
      rec.e0 = take_event(h);
      rec.e1 = take_event(h);
      if (!rec.e0 || !rec.e1) return SHAMPOO4_ERR_CUDA;
      S4_CUDA(cudaEventRecord(rec.e0, st));
    }
    S4_TRY(launch_set_table(t.data(), int(t.size()), dst, st));
    if (h->timing) {
      S4_CUDA(cudaEventRecord(rec.e1, st));
      h->recs.push_back(rec);
    }
    return SHAMPOO4_OK;
  }
  if (capturing) return SHAMPOO4_ERR_UNSUPPORTED;
  if (ev_pending) S4_CUDA(cudaEventSynchronize(ev));
  std::memcpy(pinned, t.data(), sizeof(PtrEntry) * t.size());
  S4_CUDA(cudaMemcpyAsync(dst, pinned, sizeof(PtrEntry) * t.size(), cudaMemcpyHostToDevice, st));
  S4_CUDA(cudaEventRecord(ev, st));
  ev_pending = true;
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
  // while a graph is being captured the table is always written, so that
  // the graph carries the table of every call it replays
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  S4_CUDA(cudaStreamIsCapturing(st, &cs));
  const bool capturing = cs != cudaStreamCaptureStatusNone;
  if (!capturing && h->tab_valid &&
      std::memcmp(want.data(), h->tab_host.data(), sizeof(PtrEntry) * 2 * np) == 0)
    return SHAMPOO4_OK;
  S4_TRY(upload_table(h, want, h->ws_tabs, h->tab_pinned, h->tab_event, h->tab_event_pending, capturing, st));
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
  if (cfg->compressed_stats != 0 && cfg->compressed_stats != 1) return SHAMPOO4_ERR_INVALID_ARG;
  if (cfg->refresh_world < 0 || cfg->refresh_world > 4096) return SHAMPOO4_ERR_INVALID_ARG;
  if (cfg->codebook != SHAMPOO4_CODEBOOK_LINEAR_SQUARE && cfg->codebook != SHAMPOO4_CODEBOOK_DYNAMIC_TREE)
    return SHAMPOO4_ERR_INVALID_ARG;
  if (cfg->root_method != SHAMPOO4_ROOT_EIGEN && cfg->root_method != SHAMPOO4_ROOT_NEWTON &&
      cfg->root_method != SHAMPOO4_ROOT_NEWTON_Q4)
    return SHAMPOO4_ERR_INVALID_ARG;
  if (cfg->root_method != SHAMPOO4_ROOT_EIGEN && cfg->compressed_stats) return SHAMPOO4_ERR_INVALID_ARG;
  if (cfg->newton_iters < 0 || cfg->newton_iters > 100) return SHAMPOO4_ERR_INVALID_ARG;
  if (cfg->group_tiles < 0) return SHAMPOO4_ERR_INVALID_ARG;
  if (cfg->refresh_world > 1 && (cfg->refresh_rank < 0 || cfg->refresh_rank >= cfg->refresh_world))
    return SHAMPOO4_ERR_INVALID_ARG;
  for (int32_t i = 0; i < nparams; ++i)
    if (params[i].rows < 1 || params[i].cols < 1 || params[i].rows > (1LL << 31) ||
        params[i].cols > (1LL << 31))
      return SHAMPOO4_ERR_INVALID_ARG;
  shampoo4_ctx* h = new (std::nothrow) shampoo4_ctx();
  if (!h) return SHAMPOO4_ERR_INVALID_ARG;
  h->cfg = *cfg;
  if (h->cfg.newton_iters == 0) h->cfg.newton_iters = kDefaultNewtonIters;
  h->params.assign(params, params + nparams);
  h->world = cfg->refresh_world > 1 ? cfg->refresh_world : 1;
  h->rank = h->world > 1 ? cfg->refresh_rank : 0;
  shampoo4_status s = plan(h);
  if (s != SHAMPOO4_OK) { delete h; return s; }
  // Tensor-map and descriptor bytes: build the programs once against a null
  // base (maps counted, not encoded) to size both regions; bind rebuilds
  // them with the real addresses.
  // (sized with the most refresh parts: a split program never needs less)
  Builder b{h, h->arena, nullptr, nullptr, false};
  const int parts = h->refresh_parts;
  h->refresh_parts = shampoo4_ctx::kMaxParts;
  build_stats(b);
  build_refresh(b, h->prog_refresh_first, true);
  build_refresh(b, h->prog_refresh, false);
  build_precondition(b);
  h->refresh_parts = parts;
  h->ws_nmaps = h->maps.size();
  h->ws_desc = align_up(h->ws_maps + h->ws_nmaps * sizeof(CUtensorMap), kAlign);
  h->ws_desc_bytes = align_up(h->arena.size(), kAlign);
  h->ws_bytes = h->ws_desc + h->ws_desc_bytes;
  h->prog_stats.clear(); h->prog_stats_first.clear(); h->prog_precond.clear();
  h->prog_refresh_first.clear(); h->prog_refresh.clear();
  h->arena.clear();
  h->maps.clear();
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
    S4_CUDA(cudaHostAlloc(&h->gtab_pinned, sizeof(PtrEntry) * 3 * h->params.size() + 64, cudaHostAllocDefault));
    S4_CUDA(cudaEventCreateWithFlags(&h->gtab_event, cudaEventDisableTiming));
  }
  if (!h->part_fork) {
    S4_CUDA(cudaEventCreateWithFlags(&h->part_fork, cudaEventDisableTiming));
    for (int p = 0; p < shampoo4_ctx::kMaxParts; ++p) {
      S4_CUDA(cudaStreamCreateWithFlags(&h->part_stream[p], cudaStreamNonBlocking));
      S4_CUDA(cudaEventCreateWithFlags(&h->part_join[p], cudaEventDisableTiming));
    }
  }
  if (h->tab_event_pending) S4_CUDA(cudaEventSynchronize(h->tab_event));
  if (h->gtab_event_pending) S4_CUDA(cudaEventSynchronize(h->gtab_event));
  h->d_state = static_cast<uint8_t*>(d_state);
  h->d_ws = static_cast<uint8_t*>(d_workspace);
  h->prog_stats.clear(); h->prog_stats_first.clear(); h->prog_precond.clear();
  h->prog_refresh_first.clear(); h->prog_refresh.clear();
  h->arena.clear();
  h->maps.clear();
  Builder b{h, h->arena, h->d_ws, h->d_state, true};
  build_stats(b);
  build_refresh(b, h->prog_refresh_first, true);
  build_refresh(b, h->prog_refresh, false);
  build_precondition(b);
  if (b.err != SHAMPOO4_OK) return b.err;
  // init sized both regions with the most refresh parts; fewer parts need
  // no more room (each launch's descriptor array is 256-byte aligned, so a
  // split launch takes at least what the whole one did)
  if (align_up(h->arena.size(), kAlign) > h->ws_desc_bytes || h->maps.size() > h->ws_nmaps)
    return SHAMPOO4_ERR_WORKSPACE;
  S4_CUDA(cudaMemsetAsync(h->d_ws, 0, h->ws_maps, st));
  if (!h->maps.empty())
    S4_CUDA(cudaMemcpyAsync(h->d_ws + h->ws_maps, h->maps.data(), h->maps.size() * sizeof(CUtensorMap),
                            cudaMemcpyHostToDevice, st));
  S4_CUDA(cudaMemcpyAsync(h->d_ws + h->ws_desc, h->arena.data(), h->arena.size(), cudaMemcpyHostToDevice, st));
  if (!h->graft_items.empty())
    S4_CUDA(cudaMemcpyAsync(h->d_ws + h->ws_gitems, h->graft_items.data(),
                            sizeof(GraftItem) * h->graft_items.size(), cudaMemcpyHostToDevice, st));
  if (reset) {
    S4_CUDA(cudaMemsetAsync(h->d_state, 0, h->state_bytes, st));
    h->has_basis = false;
  }
  h->stats_pending = false;
  S4_CUDA(cudaStreamSynchronize(st));   // the host arena is reused by the next bind
  h->tab_valid = false;
  h->gtab_valid = false;
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
  if (h->cfg.compressed_stats && h->stats_pending) return SHAMPOO4_ERR_NOT_READY;
  S4_TRY(set_tables(h, d_grads, ld, nullptr, nullptr, st));
  S4_CUDA(cudaMemsetAsync(h->d_ws + h->ws_bflag, 0, 4 * h->blocks.size(), st));
  const bool rebuild = !h->cfg.compressed_stats || h->has_basis;
  S4_TRY(run_program(h, rebuild ? h->prog_stats : h->prog_stats_first, st));
  h->stats_pending = h->cfg.compressed_stats != 0;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_refresh_roots(shampoo4_handle h, shampoo4_stream_t stream) {
  if (!h) return SHAMPOO4_ERR_INVALID_ARG;
  if (!h->bound) return SHAMPOO4_ERR_NOT_READY;
  if (h->cfg.compressed_stats && !h->stats_pending) return SHAMPOO4_ERR_NOT_READY;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  S4_CUDA(cudaMemsetAsync(h->d_ws + h->ws_fail, 0, 4 * h->factors.size(), st));
  S4_CUDA(cudaMemsetAsync(h->d_ws + h->ws_tcbad, 0, 4 * h->factors.size(), st));
  S4_CUDA(cudaMemsetAsync(h->d_ws + h->ws_tcgood, 1, 4 * h->factors.size(), st));
  S4_CUDA(cudaMemsetAsync(h->d_ws + h->ws_devsq, 0, 8 * h->factors.size(), st));
  S4_CUDA(cudaMemsetAsync(h->d_ws + h->ws_fbany, h->any_simt ? 1 : 0, 4, st));
  S4_CUDA(cudaMemsetAsync(h->d_ws + h->ws_p3any, 0, 4, st));
  const bool first = !h->has_basis;
  S4_TRY(run_program(h, first ? h->prog_refresh_first : h->prog_refresh, st));
  h->last_refresh_first = first;
  h->has_basis = true;
  h->stats_pending = false;
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
  S4_TRY(run_program(h, h->prog_precond, st));
  h->dsq_valid = true;                  // the apply recorded ||D||^2 per tile
  return SHAMPOO4_OK;
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

extern "C" shampoo4_status shampoo4_root_offset(shampoo4_handle h, int32_t factor, size_t* off_P) {
  if (!h || !off_P || factor < 0 || size_t(factor) >= h->factors.size()) return SHAMPOO4_ERR_INVALID_ARG;
  if (h->cfg.root_method != SHAMPOO4_ROOT_NEWTON || h->factors[factor].st_P == SIZE_MAX)
    return SHAMPOO4_ERR_INVALID_ARG;
  *off_P = h->factors[factor].st_P;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_debug_q_offset(shampoo4_handle h, int32_t factor, size_t* off_q) {
  if (!h || !off_q || factor < 0 || size_t(factor) >= h->factors.size()) return SHAMPOO4_ERR_INVALID_ARG;
  if (h->cfg.root_method != SHAMPOO4_ROOT_EIGEN) return SHAMPOO4_ERR_INVALID_ARG;
  if (ngroups(h) > 1) return SHAMPOO4_ERR_UNSUPPORTED;    // a later group reuses the scratch
  if (!h->bound) return SHAMPOO4_ERR_NOT_READY;
  *off_q = h->last_refresh_first ? h->factors[factor].ws_q_first : h->factors[factor].ws_q_next;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_factor_owner(shampoo4_handle h, int32_t factor, int32_t* rank) {
  if (!h || !rank || factor < 0 || size_t(factor) >= h->factors.size()) return SHAMPOO4_ERR_INVALID_ARG;
  *rank = h->owner[factor];
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_owner_span(shampoo4_handle h, int32_t rank, size_t* off, size_t* bytes) {
  if (!h || rank < 0 || rank >= h->world) return SHAMPOO4_ERR_INVALID_ARG;
  if (off) *off = h->span_off[rank];
  if (bytes) *bytes = h->span_bytes[rank];
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_debug_s_offset(shampoo4_handle h, int32_t factor, size_t* off_s) {
  if (!h || !off_s || !h->cfg.compressed_stats || factor < 0 || size_t(factor) >= h->factors.size())
    return SHAMPOO4_ERR_INVALID_ARG;
  *off_s = h->factors[factor].ws_S;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_debug_capture_bytes(shampoo4_handle h, size_t* bytes) {
  if (!h || !bytes) return SHAMPOO4_ERR_INVALID_ARG;
  *bytes = h->dbg_bytes;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_debug_capture(shampoo4_handle h, void* d_buf) {
  if (!h) return SHAMPOO4_ERR_INVALID_ARG;
  if (d_buf && !aligned(d_buf, kAlign)) return SHAMPOO4_ERR_INVALID_ARG;
  h->d_dbg = static_cast<uint8_t*>(d_buf);
  h->bound = false;                       // the refresh programs carry the buffer's addresses: bind again
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_debug_capture_layout(shampoo4_handle h, int32_t factor, size_t* off_u,
                                                         size_t* off_q) {
  if (!h || factor < 0 || size_t(factor) >= h->factors.size()) return SHAMPOO4_ERR_INVALID_ARG;
  if (off_u) *off_u = h->factors[factor].dbg_u;
  if (off_q) *off_q = h->factors[factor].dbg_q;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_debug_refresh_parts(shampoo4_handle h, int32_t parts) {
  if (!h || parts < 1 || parts > shampoo4_ctx::kMaxParts) return SHAMPOO4_ERR_INVALID_ARG;
  h->refresh_parts = parts;
  h->bound = false;                       // the programs are rebuilt by the next bind
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_debug_wait_limit(shampoo4_handle h, uint64_t ns) {
  if (!h) return SHAMPOO4_ERR_INVALID_ARG;
  h->wait_ns = ns;
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
      "precond_mu", "roots", "apply_left", "apply_right", "qr_inverse", "stats_dequant", "stats_rebuild", "tables",
      "newton_elt", "newton_gemm"};
  if (stage < 0 || stage >= SHAMPOO4_STAGE_COUNT) return "unknown";
  return names[stage];
}

// ------------------------------------------------------------- grafting

namespace {

bool graft_config_ok(const shampoo4_graft_config* c) {
  if (!c) return false;
  if (c->kind != SHAMPOO4_GRAFT_SGD && c->kind != SHAMPOO4_GRAFT_ADAM) return false;
  if (c->dir_norms != 0 && c->dir_norms != 1) return false;
  if (!(c->graft_eps >= 0.0f) || !std::isfinite(c->graft_eps)) return false;
  if (c->kind == SHAMPOO4_GRAFT_ADAM) {
    if (!(c->beta1 >= 0.0f && c->beta1 < 1.0f) || !(c->beta2 >= 0.0f && c->beta2 < 1.0f)) return false;
    if (!(c->adam_eps >= 0.0f) || !std::isfinite(c->adam_eps)) return false;
  }
  return true;
}

// [p0, p1) byte range of parameter i's matrix at ptr with leading dimension ld
std::pair<uintptr_t, uintptr_t> span(const shampoo4_param& q, const float* ptr, int64_t ld) {
  const uintptr_t a = uintptr_t(ptr);
  return {a, a + 4 * uintptr_t((q.rows - 1) * ld + q.cols)};
}

}  // namespace

extern "C" shampoo4_status shampoo4_graft_state_bytes(shampoo4_handle h, int32_t kind, size_t* bytes) {
  if (!h || !bytes) return SHAMPOO4_ERR_INVALID_ARG;
  if (kind != SHAMPOO4_GRAFT_SGD && kind != SHAMPOO4_GRAFT_ADAM) return SHAMPOO4_ERR_INVALID_ARG;
  *bytes = kind == SHAMPOO4_GRAFT_ADAM ? h->graft_state_bytes : 0;
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_graft_layout(shampoo4_handle h, int32_t kind, int32_t param,
                                                 size_t* off_m, size_t* off_v) {
  if (!h || kind != SHAMPOO4_GRAFT_ADAM || param < 0 || size_t(param) >= h->params.size())
    return SHAMPOO4_ERR_INVALID_ARG;
  if (off_m) *off_m = h->graft_off_m[param];
  if (off_v) *off_v = h->graft_off_v[param];
  return SHAMPOO4_OK;
}

extern "C" shampoo4_status shampoo4_graft_update(shampoo4_handle h, const shampoo4_graft_config* cfg,
                                                 void* d_graft_state, int64_t step, float lr,
                                                 const float* const* d_grads, const int64_t* ld_grads,
                                                 const float* const* d_dirs, const int64_t* ld_dirs,
                                                 float* const* d_weights, const int64_t* ld_weights,
                                                 shampoo4_stream_t stream) {
  if (!h) return SHAMPOO4_ERR_INVALID_ARG;
  if (!h->bound) return SHAMPOO4_ERR_NOT_READY;
  if (!graft_config_ok(cfg) || !std::isfinite(lr)) return SHAMPOO4_ERR_INVALID_ARG;
  const bool adam = cfg->kind == SHAMPOO4_GRAFT_ADAM;
  if (adam && (step < 1 || !d_graft_state || !aligned(d_graft_state, kAlign))) return SHAMPOO4_ERR_INVALID_ARG;
  S4_TRY(check_matrices(h, d_grads, ld_grads));
  S4_TRY(check_matrices(h, d_dirs, ld_dirs));
  S4_TRY(check_matrices(h, const_cast<const float* const*>(d_weights), ld_weights));
  const size_t np = h->params.size();
  for (size_t i = 0; i < np; ++i) {
    const auto w = span(h->params[i], d_weights[i], ld_weights[i]);
    for (size_t j = 0; j < np; ++j) {
      const auto g = span(h->params[j], d_grads[j], ld_grads[j]);
      const auto d = span(h->params[j], d_dirs[j], ld_dirs[j]);
      if ((w.first < g.second && g.first < w.second) || (w.first < d.second && d.first < w.second))
        return SHAMPOO4_ERR_INVALID_ARG;
      if (j != i) {
        const auto w2 = span(h->params[j], d_weights[j], ld_weights[j]);
        if (w.first < w2.second && w2.first < w.second) return SHAMPOO4_ERR_INVALID_ARG;
      }
    }
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // per-call pointer table, uploaded when it changed
  std::vector<PtrEntry> want(3 * np);
  for (size_t p = 0; p < np; ++p) {
    want[p] = {d_grads[p], ld_grads[p]};
    want[np + p] = {d_dirs[p], ld_dirs[p]};
    want[2 * np + p] = {d_weights[p], ld_weights[p]};
  }
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  S4_CUDA(cudaStreamIsCapturing(st, &cs));
  const bool capturing = cs != cudaStreamCaptureStatusNone;
  if (capturing || !h->gtab_valid ||
      std::memcmp(want.data(), h->gtab_host.data(), sizeof(PtrEntry) * 3 * np) != 0) {
    S4_TRY(upload_table(h, want, h->ws_gtab, h->gtab_pinned, h->gtab_event, h->gtab_event_pending, capturing, st));
    h->gtab_host = want;
    h->gtab_valid = true;
  }
  GraftArgs a{};
  a.items = reinterpret_cast<const GraftItem*>(h->d_ws + h->ws_gitems);
  a.nitems = int32_t(h->graft_items.size());
  a.nparams = int32_t(np);
  a.tabs = reinterpret_cast<const PtrEntry*>(h->d_ws + h->ws_gtab);
  a.state = adam ? static_cast<float*>(d_graft_state) : nullptr;
  a.bflag = reinterpret_cast<const uint32_t*>(h->d_ws + h->ws_bflag);
  a.parts = reinterpret_cast<double*>(h->d_ws + h->ws_gparts);
  a.flags = reinterpret_cast<uint32_t*>(h->d_ws + h->ws_flags);
  a.kind = adam ? kGraftAdam : kGraftSgd;
  a.beta1 = cfg->beta1;
  a.beta2 = cfg->beta2;
  a.omb1 = 1.0f - cfg->beta1;
  a.omb2 = 1.0f - cfg->beta2;
  if (adam) {
    const double t = double(step);
    a.c1 = float(1.0 / (1.0 - std::pow(double(cfg->beta1), t)));
    a.c2 = float(1.0 / (1.0 - std::pow(double(cfg->beta2), t)));
    if (!std::isfinite(a.c1) || !std::isfinite(a.c2)) return SHAMPOO4_ERR_INVALID_ARG;
  }
  a.adam_eps = cfg->adam_eps;
  a.lr = double(lr);
  a.graft_eps = double(cfg->graft_eps);
  if (cfg->dir_norms) {
    if (!h->dsq_valid) return SHAMPOO4_ERR_NOT_READY;
    a.use_dsq = 1;
    a.dsq = reinterpret_cast<const double*>(h->d_ws + h->ws_dsq);
  }
  return launch_graft(a, st);
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
  if (h->gtab_event) {
    cudaEventSynchronize(h->gtab_event);
    cudaEventDestroy(h->gtab_event);
  }
  if (h->gtab_pinned) cudaFreeHost(h->gtab_pinned);
  if (h->flags_pinned) cudaFreeHost(h->flags_pinned);
  for (int p = 0; p < shampoo4_ctx::kMaxParts; ++p) {
    if (h->part_stream[p]) {
      cudaStreamSynchronize(h->part_stream[p]);
      cudaStreamDestroy(h->part_stream[p]);
    }
    if (h->part_join[p]) cudaEventDestroy(h->part_join[p]);
  }
  if (h->part_fork) cudaEventDestroy(h->part_fork);
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
