// C ABI of the tensor-product convolution: plan builder, workspace layout and the
// launch sequences of the forward, backward and double backward passes.
//
// Plan (Sobek, section 2, eqs. 3-5 and 9-10; section 4 on the generator's input):
// irreps strings are parsed into blocks, valid paths are enumerated in the fixed order
// (input block, harmonic order, output block), and every path is mapped to a
// compile-time (l_in, l_sh, l_out) kernel specialisation whose coupling
// coefficients are constants of the generated table.  Unlike the pages' generator,
// nothing is compiled at run time: all 34 order triples with l <= 3 are built ahead
// of time and selected per path.
//
// Pass structure (section 4): receiver ranges bounded by the scratch budget are
// streamed through a receiver traversal that builds the bounded state S (eq. 33),
// then channel contractions apply A (eqs. 34-36); the source-CSR traversal owns
// x_bar with the mirrored state X, and the position gradient is assembled from
// per-edge values in a fixed order.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>
#include <vector>
#include <cmath>
#include <mutex>

#include "../../include/tpconv.h"
#include "launch.h"
#include "tables.inc"

using namespace tpc;

namespace {

struct Block {
  int mul, l, parity, offset;
};

struct PathH {
  int l_in, l_sh, l_out, b_in, b_out, c_in, c_out, w_off, w_count, type, nnz;
  int in_off, out_off, st_off, xst_off;
};

constexpr size_t kDefaultBudget = size_t(128) << 20;  // the pages' 128 MiB scratch cap
constexpr int kSplits = 8;  // split-K factor of the weight-gradient contractions
constexpr int kUvuRanges = 256;  // receiver ranges of the uvu weight gradient (fixed-order partials)

int triple_index(int a, int b, int c) {
  for (int t = 0; t < tpc_tab::NTRIPLES; ++t)
    if (tpc_tab::TRIPLES[t][0] == a && tpc_tab::TRIPLES[t][1] == b && tpc_tab::TRIPLES[t][2] == c) return t;
  return -1;
}

// host access to the generated coupling tables
template <int A, int B, int C>
void cg_host(std::vector<int>& idx, std::vector<double>& val) {
  using T = tpc_tab::CG<A, B, C>;
  for (int n = 0; n < T::nnz; ++n) {
    idx.push_back(T::mi(n));
    idx.push_back(T::my(n));
    idx.push_back(T::mo(n));
    val.push_back(T::val_d(n));
  }
}

#define TPC_HCASE(n)                                                                        \
  case n:                                                                                   \
    cg_host<tpc_tab::TRIPLES[n][0], tpc_tab::TRIPLES[n][1], tpc_tab::TRIPLES[n][2]>(idx, val); \
    break;

void cg_of_type(int type, std::vector<int>& idx, std::vector<double>& val) {
  switch (type) {
    TPC_HCASE(0) TPC_HCASE(1) TPC_HCASE(2) TPC_HCASE(3) TPC_HCASE(4) TPC_HCASE(5) TPC_HCASE(6)
    TPC_HCASE(7) TPC_HCASE(8) TPC_HCASE(9) TPC_HCASE(10) TPC_HCASE(11) TPC_HCASE(12)
    TPC_HCASE(13) TPC_HCASE(14) TPC_HCASE(15) TPC_HCASE(16) TPC_HCASE(17) TPC_HCASE(18)
    TPC_HCASE(19) TPC_HCASE(20) TPC_HCASE(21) TPC_HCASE(22) TPC_HCASE(23) TPC_HCASE(24)
    TPC_HCASE(25) TPC_HCASE(26) TPC_HCASE(27) TPC_HCASE(28) TPC_HCASE(29) TPC_HCASE(30)
    TPC_HCASE(31) TPC_HCASE(32) TPC_HCASE(33)
    default: break;
  }
}

tpconv_status parse_irreps(const char* s, std::vector<Block>& out) {
  if (!s) return TPCONV_ERR_INVALID_ARG;
  out.clear();
  std::string str(s);
  size_t pos = 0;
  int off = 0;
  if (str.find_first_not_of(" \t") == std::string::npos) return TPCONV_ERR_PARSE;
  while (pos <= str.size()) {
    size_t plus = str.find('+', pos);
    std::string tok = str.substr(pos, plus == std::string::npos ? std::string::npos : plus - pos);
    std::string t;
    for (char ch : tok) if (ch != ' ' && ch != '\t') t.push_back(ch);
    if (t.empty()) return TPCONV_ERR_PARSE;
    long mul = 1;
    size_t xp = t.find('x');
    std::string lp = t;
    if (xp != std::string::npos) {
      std::string ms = t.substr(0, xp);
      if (ms.empty() || ms.find_first_not_of("0123456789") != std::string::npos || ms.size() > 6) return TPCONV_ERR_PARSE;
      mul = std::atol(ms.c_str());
      lp = t.substr(xp + 1);
    }
    if (lp.size() < 2) return TPCONV_ERR_PARSE;
    char par = lp.back();
    std::string ls = lp.substr(0, lp.size() - 1);
    if ((par != 'e' && par != 'o') || ls.empty() || ls.find_first_not_of("0123456789") != std::string::npos || ls.size() > 3)
      return TPCONV_ERR_PARSE;
    long l = std::atol(ls.c_str());
    if (mul <= 0) return TPCONV_ERR_PARSE;
    if (l > TPC_LMAX) return TPCONV_ERR_UNSUPPORTED;
    Block b{(int)mul, (int)l, par == 'e' ? 1 : -1, off};
    off += b.mul * (2 * b.l + 1);
    out.push_back(b);
    if (plus == std::string::npos) break;
    pos = plus + 1;
  }
  if ((int)out.size() > MAX_BLOCKS) return TPCONV_ERR_UNSUPPORTED;
  return TPCONV_OK;
}

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// ---------------------------------------------------------------------------
// profiling: optional CUDA-event bracketing of every kernel launch, by category
// ---------------------------------------------------------------------------

enum ProfCat {
  PC_UVW_STATE = 0, PC_UVW_STATE_TAN, PC_UVW_RECV_BWD, PC_UVW_SRC, PC_UVW_SRC_TAN, PC_GEMM,
  PC_UVU_FWD, PC_UVU_RECV_BWD, PC_UVU_GRADW, PC_UVU_SRC, PC_POS, PC_GRAPH, PC_RECV_TAN, PC_COUNT
};
static_assert(PC_COUNT == TPCONV_PROF_CATEGORIES, "category count");
const char* const kProfNames[PC_COUNT] = {
    "uvw_receiver_state", "uvw_receiver_state_tangent", "uvw_receiver_backward", "uvw_source_state",
    "uvw_source_state_tangent", "channel_gemm", "uvu_forward", "uvu_receiver_backward",
    "uvu_weight_gradient", "uvu_source_backward", "position_gradient", "graph",
    "receiver_backward_tangent"};

struct Prof {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;
  std::vector<int> cat;
  size_t used = 0;
  long long launches[PC_COUNT] = {};
};
Prof& prof() {
  static Prof p;
  return p;
}

// Kernel launches counted where their number is known only at launch time.
void prof_add_launches(int c, int n) {
  Prof& P = prof();
  std::lock_guard<std::mutex> g(P.mu);
  if (P.on) P.launches[c] += n;
}

// Brackets one library call that launches `nk` kernels on stream s.
struct ProfScope {
  int slot = -1;
  cudaStream_t s;
  ProfScope(int c, int nk, cudaStream_t st) : s(st) {
    Prof& P = prof();
    std::lock_guard<std::mutex> g(P.mu);
    if (!P.on) return;
    P.launches[c] += nk;
    if (2 * (P.used + 1) > P.pool.size()) return;
    slot = (int)P.used++;
    P.cat[slot] = c;
    cudaEventRecord(P.pool[2 * slot], s);
  }
  ~ProfScope() {
    if (slot < 0) return;
    cudaEventRecord(prof().pool[2 * slot + 1], s);
  }
};

}  // namespace

struct tpconv_plan {
  std::vector<Block> in, out;
  int lmax = 0, mode = 0;
  tpconv_radial_spec radial{};
  std::vector<PathH> paths;
  std::vector<std::vector<int>> cg_idx;
  std::vector<std::vector<double>> cg_val;
  int dim_in = 0, dim_out = 0, n_w = 0, K = 0;
  DevPlan dev{};
  Tasks t_in{};   // (path, 32-chunk of C_in)
  Tasks t_out{};  // (path, 32-chunk of C_out)
  Tasks t_bo{};   // (output block, chunk)  uvu forward
  Tasks t_bi{};   // (input block, chunk)   uvu source pass
  BlockPaths bp_out{}, bp_in{};
  size_t budget = kDefaultBudget;
  int math = TPCONV_MATH_FP32;
  int layout = TPCONV_LAYOUT_IR_MUL;
};

namespace {

struct Layout {
  int recv_chunk = 0, src_chunk = 0;
  size_t state_a = 0, state_b = 0;  // offsets of the (up to two) state arrays
  size_t gbuf = 0, part = 0;
  size_t order = 0;                 // receiver order of the pass (uvw, N ints)
  size_t total = 0;
  long long win_edges = 0;          // edges per position-gradient staging window
  size_t cursor = 0;                // per-node cursor of the window sums (N ints)
  bool has_gbuf = false, has_part = false;
};

// Position-gradient staging: g_e = dL/dr_e (16 bytes per edge) is staged for a window of
// at most win_edges edges at a time and summed into the nodes window by window.  The
// window takes an eighth of the scratch budget (at least 32 edges, at most 16 MiB = one
// million edges), so the workspace does not grow with the edge count.
constexpr size_t kMaxStagingBytes = size_t(16) << 20;
size_t staging_bytes(size_t budget) {
  return std::max<size_t>(512, std::min(budget / 8, kMaxStagingBytes)) & ~size_t(15);
}

// Upper bound on the staging windows of one receiver range (the range's edge count is
// known on the device only; windows past its end are empty and their launches return at
// once).
int windows_per_range(long long E, long long win_edges) {
  return (int)std::max<long long>(1, (E + win_edges - 1) / win_edges);
}

// Nodes per chunk: the most that fit the budget, then evened out over the chunks that
// number needs (so that no chunk is left with a small remainder).
int chunk_for(size_t budget_floats, long long fixed, long long per_node, long long N) {
  if (per_node <= 0 || N <= 0) return (int)std::max<long long>(N, 0);
  long long avail = (long long)budget_floats - fixed;
  long long c = avail > 0 ? avail / per_node : 1;
  c = std::max<long long>(1, std::min<long long>(c, N));
  const long long chunks = (N + c - 1) / c;
  return (int)((N + chunks - 1) / chunks);
}

// Workspace of one pass.  The scratch budget covers the node states of a receiver (or
// source) range, the split-K slices of the channel contractions and, in backward and
// double backward, the position-gradient staging window; nothing in it grows with E.
Layout make_layout(const tpconv_plan* P, long long N, long long E, uint32_t pass) {
  (void)E;
  Layout L;
  size_t off = 0;
  const long long st = P->dev.state_per_node, xs = P->dev.xstate_per_node;
  const bool staged = pass == TPCONV_PASS_BACKWARD || pass == TPCONV_PASS_DOUBLE_BACKWARD;
  const size_t stage = staged ? staging_bytes(P->budget) : 0;
  const size_t bf = (P->budget - std::min(P->budget, stage)) / 4;
  if (P->mode == TPCONV_UVW) {
    const int arrays = (pass == TPCONV_PASS_DOUBLE_BACKWARD) ? 2 : 1;
    const long long fixed = (pass == TPCONV_PASS_FORWARD) ? 0 : (long long)kSplits * P->K * P->n_w;
    L.recv_chunk = chunk_for(bf, fixed, arrays * st + (long long)kSplits * P->dim_out, N);
    L.src_chunk = (pass == TPCONV_PASS_FORWARD) ? 0 : chunk_for(bf, fixed, arrays * xs + (long long)kSplits * P->dim_in, N);
    const size_t one = std::max(align256(size_t(4) * L.recv_chunk * st), align256(size_t(4) * L.src_chunk * xs));
    L.state_a = off;
    off += one;
    if (arrays == 2) { L.state_b = off; off += one; }
    long long pf = std::max((long long)L.recv_chunk * P->dim_out, (long long)L.src_chunk * P->dim_in);
    if (pass != TPCONV_PASS_FORWARD) pf = std::max(pf, (long long)P->K * P->n_w);
    L.has_part = true;
    L.part = off;
    off += align256(size_t(4) * kSplits * pf);
    L.order = off;
    off += align256(size_t(4) * std::max<long long>(N, 1));
  } else {
    if (pass != TPCONV_PASS_FORWARD) {
      L.has_part = true;
      L.part = off;
      off += align256(size_t(4) * kUvuRanges * P->K * (long long)P->n_w);
    }
  }
  if (staged) {
    L.has_gbuf = true;
    L.gbuf = off;
    L.win_edges = (long long)(stage / 16);
    off += align256(stage);
    L.cursor = off;                 // per-node position in the source view (N ints)
    off += align256(size_t(4) * std::max<long long>(N, 1));
  }
  L.total = off;
  return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// mul_ir boundary: node arrays are converted to and from ir_mul in workspace buffers
// placed after the pass's own workspace (three input-width and two output-width arrays).
size_t conversion_bytes(const tpconv_plan* P, long long N) {
  if (P->layout != TPCONV_LAYOUT_MUL_IR) return 0;
  return 3 * align256(size_t(4) * N * P->dim_in) + 2 * align256(size_t(4) * N * P->dim_out) + 256;
}

LayoutMap layout_map(const std::vector<Block>& blocks) {
  LayoutMap M{};
  M.n = (int)blocks.size();
  for (int b = 0; b < M.n; ++b) {
    M.off[b] = blocks[b].offset;
    M.l[b] = blocks[b].l;
    M.mul[b] = blocks[b].mul;
  }
  return M;
}

struct ConvBufs {
  size_t inner = 0;                   // bytes left to the pass itself
  float *xin[3] = {}, *xout[2] = {};  // input-width and output-width buffers
};

tpconv_status conversion_setup(const tpconv_plan* P, int64_t N, int64_t E, uint32_t pass, void* ws,
                               size_t ws_bytes, ConvBufs& B) {
  B.inner = align256(make_layout(P, N, E, pass).total);
  const size_t need = B.inner + conversion_bytes(P, N);
  if (ws_bytes < need) return TPCONV_ERR_WORKSPACE_TOO_SMALL;
  if (!ws) return TPCONV_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 15u) != 0) return TPCONV_ERR_MISALIGNED;
  char* p = static_cast<char*>(ws) + B.inner;
  for (int i = 0; i < 3; ++i) { B.xin[i] = reinterpret_cast<float*>(p); p += align256(size_t(4) * N * P->dim_in); }
  for (int i = 0; i < 2; ++i) { B.xout[i] = reinterpret_cast<float*>(p); p += align256(size_t(4) * N * P->dim_out); }
  return TPCONV_OK;
}

// copy a node array into the ir_mul layout (NULL stays NULL)
const float* to_ir_mul(const tpconv_plan* P, bool in_side, int64_t N, const float* a, float* buf,
                       cudaStream_t s, cudaError_t& e) {
  if (!a) return nullptr;
  const LayoutMap M = layout_map(in_side ? P->in : P->out);
  if (e == cudaSuccess) e = launch_layout_convert((int)N, in_side ? P->dim_in : P->dim_out, M, 1, a, buf, s);
  return buf;
}

void from_ir_mul(const tpconv_plan* P, bool in_side, int64_t N, const float* buf, float* a, cudaStream_t s,
                 cudaError_t& e) {
  if (!a) return;
  const LayoutMap M = layout_map(in_side ? P->in : P->out);
  if (e == cudaSuccess) e = launch_layout_convert((int)N, in_side ? P->dim_in : P->dim_out, M, 0, buf, a, s);
}

}  // namespace

// ---------------------------------------------------------------------------

extern "C" {

const char* tpconv_status_string(tpconv_status s) {
  switch (s) {
    case TPCONV_OK: return "ok";
    case TPCONV_ERR_INVALID_ARG: return "invalid argument";
    case TPCONV_ERR_PARSE: return "irreps parse error";
    case TPCONV_ERR_UNSUPPORTED: return "unsupported configuration";
    case TPCONV_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case TPCONV_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case TPCONV_ERR_CUDA: return "CUDA error";
    case TPCONV_ERR_GRAPH_INVALID: return "invalid graph";
  }
  return "unknown status";
}

tpconv_status tpconv_plan_create(tpconv_plan_t* out, const char* irreps_in, int32_t sh_lmax,
                                 const char* irreps_out, int32_t mode,
                                 const tpconv_radial_spec* radial) {
  if (!out || !irreps_in || !irreps_out || !radial) return TPCONV_ERR_INVALID_ARG;
  if (mode != TPCONV_UVW && mode != TPCONV_UVU) return TPCONV_ERR_INVALID_ARG;
  if (sh_lmax < 0) return TPCONV_ERR_INVALID_ARG;
  if (sh_lmax > TPC_LMAX) return TPCONV_ERR_UNSUPPORTED;
  const tpconv_radial_spec& R = *radial;
  if (R.num_basis < 1) return TPCONV_ERR_INVALID_ARG;
  if (R.num_basis > 16) return TPCONV_ERR_UNSUPPORTED;
  if (!(R.r_cut > 0.f) || R.poly_p < 1 || R.poly_p > 32) return TPCONV_ERR_INVALID_ARG;
  if (R.kind != TPCONV_RADIAL_BESSEL && R.kind != TPCONV_RADIAL_GAUSSIAN) return TPCONV_ERR_INVALID_ARG;
  if (R.kind == TPCONV_RADIAL_GAUSSIAN && (R.num_basis < 2 || !(R.r_max > R.r_min)))
    return TPCONV_ERR_INVALID_ARG;

  tpconv_plan* P = new (std::nothrow) tpconv_plan();
  if (!P) return TPCONV_ERR_INVALID_ARG;
  tpconv_status st = parse_irreps(irreps_in, P->in);
  if (st == TPCONV_OK) st = parse_irreps(irreps_out, P->out);
  if (st != TPCONV_OK) { delete P; return st; }
  P->lmax = sh_lmax;
  P->mode = mode;
  P->radial = R;
  P->K = R.num_basis;
  for (const Block& b : P->in) P->dim_in += b.mul * (2 * b.l + 1);
  for (const Block& b : P->out) P->dim_out += b.mul * (2 * b.l + 1);

  // eq. 5 path enumeration in the fixed order
  int woff = 0, st_off = 0, xst_off = 0;
  for (int bi = 0; bi < (int)P->in.size(); ++bi)
    for (int ls = 0; ls <= sh_lmax; ++ls)
      for (int bo = 0; bo < (int)P->out.size(); ++bo) {
        const Block &a = P->in[bi], &c = P->out[bo];
        const int psh = (ls % 2 == 0) ? 1 : -1;
        if (!(std::abs(a.l - ls) <= c.l && c.l <= a.l + ls && c.parity == a.parity * psh)) continue;
        PathH p{};
        p.l_in = a.l; p.l_sh = ls; p.l_out = c.l; p.b_in = bi; p.b_out = bo;
        p.c_in = a.mul; p.c_out = c.mul;
        if (mode == TPCONV_UVU && a.mul != c.mul) { delete P; return TPCONV_ERR_INVALID_ARG; }
        p.w_off = woff;
        p.w_count = (mode == TPCONV_UVW) ? a.mul * c.mul : a.mul;
        p.type = triple_index(a.l, ls, c.l);
        p.in_off = a.offset; p.out_off = c.offset;
        p.st_off = st_off; p.xst_off = xst_off;
        woff += p.w_count;
        st_off += (2 * c.l + 1) * P->K * a.mul;
        xst_off += (2 * a.l + 1) * P->K * c.mul;
        std::vector<int> idx;
        std::vector<double> val;
        cg_of_type(p.type, idx, val);
        p.nnz = (int)val.size();
        P->paths.push_back(p);
        P->cg_idx.push_back(idx);
        P->cg_val.push_back(val);
      }
  if (P->paths.empty()) { delete P; return TPCONV_ERR_INVALID_ARG; }
  if ((int)P->paths.size() > MAX_PATHS) { delete P; return TPCONV_ERR_UNSUPPORTED; }
  P->n_w = woff;

  DevPlan& D = P->dev;
  D.n_paths = (int)P->paths.size();
  D.dim_in = P->dim_in; D.dim_out = P->dim_out; D.n_w = P->n_w; D.K = P->K; D.lmax = sh_lmax; D.mode = mode;
  D.radial_kind = R.kind; D.poly_p = R.poly_p;
  D.r_cut = R.r_cut; D.inv_r_cut = 1.0f / R.r_cut;
  D.bessel_pref = (float)std::sqrt(2.0 / R.r_cut);
  if (R.kind == TPCONV_RADIAL_GAUSSIAN) {
    const double step = (double(R.r_max) - R.r_min) / (R.num_basis - 1);
    D.g_mu0 = R.r_min; D.g_step = (float)step; D.g_inv_sigma2 = (float)(1.0 / (step * step));
  }
  const double pp = R.poly_p;
  D.env_a = (float)((pp + 1) * (pp + 2) / 2.0);
  D.env_b = (float)(pp * (pp + 2));
  D.env_c = (float)(pp * (pp + 1) / 2.0);
  D.state_per_node = st_off;
  D.xstate_per_node = xst_off;
  D.n_sh = (P->lmax + 1) * (P->lmax + 1);
  D.emb_Y = D.emb_phi = nullptr;
  D.emb_eid = nullptr;
  D.emb_gY = D.emb_gphi = nullptr;
  D.order = nullptr;
  for (int k = 0; k < D.n_paths; ++k) {
    const PathH& h = P->paths[k];
    DevPath& d = D.p[k];
    d.type = h.type; d.l_in = h.l_in; d.l_sh = h.l_sh; d.l_out = h.l_out;
    d.c_in = h.c_in; d.c_out = h.c_out; d.in_off = h.in_off; d.out_off = h.out_off;
    d.w_off = h.w_off; d.st_off = h.st_off; d.xst_off = h.xst_off; d.b_in = h.b_in; d.b_out = h.b_out;
  }
  // warp task lists
  auto push = [](Tasks& T, int a, int b) {
    if (T.n >= MAX_TASKS) return false;
    T.a[T.n] = (short)a; T.b[T.n] = (short)b; ++T.n;
    return true;
  };
  bool ok = true;
  for (int k = 0; k < D.n_paths; ++k) {
    for (int c = 0; c < (P->paths[k].c_in + 31) / 32; ++c) ok = ok && push(P->t_in, k, c);
    for (int c = 0; c < (P->paths[k].c_out + 31) / 32; ++c) ok = ok && push(P->t_out, k, c);
  }
  auto fill_bp = [&](BlockPaths& BP, Tasks& T, const std::vector<Block>& blocks, bool by_out) {
    BP.n_blocks = (int)blocks.size();
    for (int b = 0; b < BP.n_blocks; ++b) {
      BP.l[b] = blocks[b].l; BP.c[b] = blocks[b].mul; BP.off[b] = blocks[b].offset; BP.count[b] = 0;
      for (int k = 0; k < D.n_paths; ++k)
        if ((by_out ? P->paths[k].b_out : P->paths[k].b_in) == b) BP.list[b][BP.count[b]++] = (short)k;
      for (int c = 0; c < (blocks[b].mul + 31) / 32; ++c) ok = ok && push(T, b, c);
    }
  };
  fill_bp(P->bp_out, P->t_bo, P->out, true);
  fill_bp(P->bp_in, P->t_bi, P->in, false);
  if (!ok) { delete P; return TPCONV_ERR_UNSUPPORTED; }
  *out = P;
  return TPCONV_OK;
}

tpconv_status tpconv_plan_destroy(tpconv_plan_t plan) {
  delete plan;
  return TPCONV_OK;
}

tpconv_status tpconv_plan_info(tpconv_plan_t P, int64_t* num_paths, int64_t* dim_in,
                               int64_t* dim_out, int64_t* num_basis, int64_t* weight_cols) {
  if (!P) return TPCONV_ERR_INVALID_ARG;
  if (num_paths) *num_paths = (int64_t)P->paths.size();
  if (dim_in) *dim_in = P->dim_in;
  if (dim_out) *dim_out = P->dim_out;
  if (num_basis) *num_basis = P->K;
  if (weight_cols) *weight_cols = P->n_w;
  return TPCONV_OK;
}

tpconv_status tpconv_plan_path(tpconv_plan_t P, int64_t index, int32_t out[10]) {
  if (!P || !out || index < 0 || index >= (int64_t)P->paths.size()) return TPCONV_ERR_INVALID_ARG;
  const PathH& p = P->paths[index];
  const int32_t v[10] = {p.l_in, p.l_sh, p.l_out, p.b_in, p.b_out, p.c_in, p.c_out, p.w_off, p.w_count, p.nnz};
  std::memcpy(out, v, sizeof v);
  return TPCONV_OK;
}

tpconv_status tpconv_plan_path_coupling(tpconv_plan_t P, int64_t index, int32_t* idx, double* val,
                                        int64_t cap) {
  if (!P || !idx || !val || index < 0 || index >= (int64_t)P->paths.size()) return TPCONV_ERR_INVALID_ARG;
  const auto& vi = P->cg_idx[index];
  const auto& vv = P->cg_val[index];
  if ((int64_t)vv.size() > cap) return TPCONV_ERR_INVALID_ARG;
  for (size_t k = 0; k < vv.size(); ++k) {
    idx[3 * k] = vi[3 * k]; idx[3 * k + 1] = vi[3 * k + 1]; idx[3 * k + 2] = vi[3 * k + 2];
    val[k] = vv[k];
  }
  return TPCONV_OK;
}

tpconv_status tpconv_set_workspace_budget(tpconv_plan_t P, size_t bytes) {
  if (!P || bytes < 4096) return TPCONV_ERR_INVALID_ARG;
  P->budget = bytes;
  return TPCONV_OK;
}

tpconv_status tpconv_plan_set_layout(tpconv_plan_t P, int32_t layout) {
  if (!P) return TPCONV_ERR_INVALID_ARG;
  if (layout != TPCONV_LAYOUT_IR_MUL && layout != TPCONV_LAYOUT_MUL_IR) return TPCONV_ERR_UNSUPPORTED;
  P->layout = layout;
  return TPCONV_OK;
}

tpconv_status tpconv_plan_set_math(tpconv_plan_t P, int32_t math) {
  if (!P) return TPCONV_ERR_INVALID_ARG;
  if (math != TPCONV_MATH_FP32 && math != TPCONV_MATH_TF32 && math != TPCONV_MATH_BF16) return TPCONV_ERR_UNSUPPORTED;
  P->math = math;
  return TPCONV_OK;
}

tpconv_status tpconv_workspace_bytes(tpconv_plan_t P, int64_t N, int64_t E, uint32_t pass_mask,
                                     size_t* bytes) {
  if (!P || !bytes || N < 0 || E < 0) return TPCONV_ERR_INVALID_ARG;
  size_t best = 0;
  for (uint32_t b : {TPCONV_PASS_FORWARD, TPCONV_PASS_BACKWARD, TPCONV_PASS_DOUBLE_BACKWARD})
    if (pass_mask & b) best = std::max(best, make_layout(P, N, E, b).total + conversion_bytes(P, N));
  *bytes = best;
  return TPCONV_OK;
}

tpconv_status tpconv_csr_transpose_workspace_bytes(int64_t N, int64_t E, size_t* bytes) {
  if (!bytes || N < 0 || E < 0) return TPCONV_ERR_INVALID_ARG;
  *bytes = align256(size_t(4) * std::max<int64_t>(N, 1));
  return TPCONV_OK;
}

tpconv_status tpconv_csr_transpose(int64_t N, int64_t E, const int32_t* row_ptr, const int32_t* src,
                                   int32_t* t_ptr, int32_t* t_eid, int32_t* t_dst, void* ws,
                                   size_t ws_bytes, struct CUstream_st* stream) {
  if (N < 0 || E < 0 || N > 0x7ffffffe || E > 0x7ffffffe) return TPCONV_ERR_INVALID_ARG;
  if (!row_ptr || !t_ptr || (E > 0 && (!src || !t_eid || !t_dst)) || !ws) return TPCONV_ERR_INVALID_ARG;
  size_t need = 0;
  tpconv_csr_transpose_workspace_bytes(N, E, &need);
  if (ws_bytes < need) return TPCONV_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(row_ptr) || !aligned16(t_ptr) || (E > 0 && (!aligned16(src) || !aligned16(t_eid) || !aligned16(t_dst))) || !aligned16(ws))
    return TPCONV_ERR_MISALIGNED;
  cudaStream_t s = (cudaStream_t)stream;
  ProfScope ps(PC_GRAPH, 4, s);
  cudaError_t e = launch_csr_transpose((int)N, (int)E, row_ptr, src, t_ptr, t_eid, t_dst,
                                       static_cast<int*>(ws), s);
  return e == cudaSuccess ? TPCONV_OK : TPCONV_ERR_CUDA;
}

tpconv_status tpconv_validate_graph(int64_t N, int64_t E, const int32_t* row_ptr, const int32_t* src,
                                    int32_t* d_err, struct CUstream_st* stream) {
  if (N < 0 || E < 0 || N > 0x7ffffffe || E > 0x7ffffffe || !row_ptr || !d_err || (E > 0 && !src))
    return TPCONV_ERR_INVALID_ARG;
  cudaError_t e = launch_validate_graph((int)N, (int)E, row_ptr, src, d_err, (cudaStream_t)stream);
  return e == cudaSuccess ? TPCONV_OK : TPCONV_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// pass implementations
// ---------------------------------------------------------------------------

namespace {

#define TPC_TRY(expr)                                   \
  do {                                                  \
    cudaError_t e_ = (expr);                            \
    if (e_ != cudaSuccess) return TPCONV_ERR_CUDA;      \
  } while (0)

// launch under a profiling scope: category, number of kernels, call
#define TPC_RUN(cat, nk, expr)                          \
  do {                                                  \
    ProfScope ps_(cat, nk, s);                          \
    cudaError_t e_ = (expr);                            \
    if (e_ != cudaSuccess) return TPCONV_ERR_CUDA;      \
  } while (0)

tpconv_status common_checks(const tpconv_plan* P, int64_t N, int64_t E) {
  if (!P || N < 0 || E < 0 || N > 0x7ffffffe || E > 0x7ffffffe) return TPCONV_ERR_INVALID_ARG;
  return TPCONV_OK;
}

tpconv_status check_ptrs(std::initializer_list<const void*> required, std::initializer_list<const void*> optional) {
  for (const void* p : required) {
    if (!p) return TPCONV_ERR_INVALID_ARG;
    if (!aligned16(p)) return TPCONV_ERR_MISALIGNED;
  }
  for (const void* p : optional)
    if (p && !aligned16(p)) return TPCONV_ERR_MISALIGNED;
  return TPCONV_OK;
}

tpconv_status check_ws(const Layout& L, void* ws, size_t ws_bytes) {
  if (L.total == 0) return TPCONV_OK;
  if (ws_bytes < L.total) return TPCONV_ERR_WORKSPACE_TOO_SMALL;
  if (!ws) return TPCONV_ERR_INVALID_ARG;
  if (!aligned16(ws)) return TPCONV_ERR_MISALIGNED;
  return TPCONV_OK;
}

// A grouped GEMM under construction.  Problems are collected into a GemmBatch; when the
// next problem would not fit (problem or segment capacity), the batch collected so far is
// launched and a new one started, so any number of problems is accepted.
struct Batch {
  GemmBatch g{};
  cudaStream_t st;
  float* auto_part;  // split-K scratch for automatic splitting (nullptr: never split automatically)
  cudaError_t err = cudaSuccess;
  Batch(const tpconv_plan* P, cudaStream_t s, int splits, int accumulate, float* partial,
        float* auto_split_part = nullptr)
      : st(s), auto_part(auto_split_part) {
    g.math = P->math;
    g.splits = splits;
    g.accumulate = accumulate;
    g.partial = partial;
  }
  // Launch the collected problems.  With automatic splitting, split-K is used when the
  // output tiles alone would leave SMs idle: as many splits as keep the grid within one
  // wave of resident CTAs (two per SM), so that no partial second wave runs.
  void flush() {
    if (g.n_problems == 0) return;
    if (err == cudaSuccess) {
      GemmBatch h = g;
      if (h.splits == 1 && auto_part) {
        const int tiles = gemm_tiles(h);
        const int wave = 2 * 148;
        if (tiles > 0 && 2 * tiles <= wave) {
          h.splits = std::min(kSplits, wave / tiles);
          h.partial = auto_part;
        }
      }
      err = launch_gemm(h, st);
      if (h.total_tiles > 0) prof_add_launches(PC_GEMM, h.splits > 1 ? 2 : 1);
    }
    g.n_problems = 0;
    g.n_segs = 0;
  }
  cudaError_t finish() {
    flush();
    return err;
  }
  void problem(float* C, Idx2 Cm, Idx2 Cn, int M, int N, int nseg) {
    if (g.n_problems + 1 > MAX_GEMM_PROBLEMS || g.n_segs + nseg > MAX_GEMM_SEGS) flush();
    GemmProblem& p = g.pr[g.n_problems++];
    p.C = C; p.Cm = Cm; p.Cn = Cn; p.M = M; p.N = N;
    p.seg0 = g.n_segs; p.nseg = 0; p.Ktot = 0;
  }
  void seg(const float* A, Idx2 Am, Idx2 Ak, const float* B, Idx2 Bk, Idx2 Bn, int K) {
    GemmSeg& s = g.sg[g.n_segs++];
    s.A = A; s.Am = Am; s.Ak = Ak; s.B = B; s.Bk = Bk; s.Bn = Bn; s.K = K;
    // 16-byte vector loads along k: aligned base, row strides multiple of 4 floats,
    // unit stride in k and k blocks (if any) of a multiple of 32
    s.a_vec4 = ((reinterpret_cast<uintptr_t>(A) & 15u) == 0) && Am.s1 % 4 == 0 && Am.s2 % 4 == 0 &&
               Ak.s2 == 1 && (Ak.d == 0x7fffffff || (Ak.d % 32 == 0 && Ak.s1 % 4 == 0));
    s.b_vec4 = ((reinterpret_cast<uintptr_t>(B) & 15u) == 0) && Bn.s1 % 4 == 0 && Bn.s2 % 4 == 0 &&
               Bk.s2 == 1 && (Bk.d == 0x7fffffff || (Bk.d % 32 == 0 && Bk.s1 % 4 == 0));
    // 16-byte vector loads along m: unit m stride and every k offset a multiple of 4 floats
    s.a_mvec4 = ((reinterpret_cast<uintptr_t>(A) & 15u) == 0) && Am.d == 0x7fffffff && Am.s2 == 1 &&
                Ak.s1 % 4 == 0 && Ak.s2 % 4 == 0;
    GemmProblem& p = g.pr[g.n_problems - 1];
    ++p.nseg;
    p.Ktot += K;
  }
};

int paths_into(const tpconv_plan* P, int block, bool out_side) {
  int n = 0;
  for (const PathH& p : P->paths) n += (out_side ? p.b_out : p.b_in) == block;
  return n;
}

// m_g[(i,mo), w] = sum_{pi in g} sum_{q,u} S_pi[(i,mo),(q,u)] A_pi[(q,u), w]   (eqs. 34-35),
// optionally + sum_pi S2_pi A2_pi (eq. 37: dm = dS A + S dA)
cudaError_t gemm_state_times_A(const tpconv_plan* P, const float* S, const float* W, const float* S2,
                               const float* W2, float* out, int n0, int cn, float* part, cudaStream_t st) {
  Batch b(P, st, 1, 0, nullptr, part);
  for (int bo = 0; bo < (int)P->out.size(); ++bo) {
    const Block& B = P->out[bo];
    const int RO = 2 * B.l + 1;
    const int np = paths_into(P, bo, true);
    if (np == 0) continue;
    b.problem(out + (long long)n0 * P->dim_out + B.offset, idx2(RO, P->dim_out, B.mul), idx1(1), cn * RO, B.mul,
              np * ((S ? 1 : 0) + (S2 ? 1 : 0)));
    for (const PathH& p : P->paths) {
      if (p.b_out != bo) continue;
      const Idx2 Am = idx2(RO, P->dev.state_per_node, (long long)P->K * p.c_in);
      const Idx2 Bk = idx2(p.c_in, P->n_w, p.c_out);
      if (S) b.seg(S + p.st_off, Am, idx1(1), W + p.w_off, Bk, idx1(1), P->K * p.c_in);
      if (S2) b.seg(S2 + p.st_off, Am, idx1(1), W2 + p.w_off, Bk, idx1(1), P->K * p.c_in);
    }
  }
  return b.finish();
}

// S_bar_pi[(i,mo),(q,u)] = sum_w m_bar[(i,mo), w] A_pi[(q,u), w]        (eq. 36)
cudaError_t gemm_sbar(const tpconv_plan* P, const float* gout, const float* W, float* Sbar, int n0,
                      int cn, cudaStream_t st) {
  Batch b(P, st, 1, 0, nullptr);
  for (const PathH& p : P->paths) {
    const int RO = 2 * p.l_out + 1;
    b.problem(Sbar + p.st_off, idx2(RO, P->dev.state_per_node, (long long)P->K * p.c_in), idx1(1), cn * RO,
              P->K * p.c_in, 1);
    b.seg(gout + (long long)n0 * P->dim_out + p.out_off, idx2(RO, P->dim_out, p.c_out), idx1(1), W + p.w_off,
          idx1(1), idx2(p.c_in, P->n_w, p.c_out), p.c_out);
  }
  return b.finish();
}

// x_bar[(j,mi), u] = sum_{pi from block} sum_{q,w} X_pi[(j,mi),(q,w)] A_pi[(q,u), w]
// (mirrored eq. 21), optionally + X2 A2^T (eq. 30 with A_dot)
cudaError_t gemm_xbar(const tpconv_plan* P, const float* X, const float* W, const float* X2, const float* W2,
                      float* gx, int n0, int cn, float* part, cudaStream_t st) {
  Batch b(P, st, 1, 0, nullptr, part);
  for (int bi = 0; bi < (int)P->in.size(); ++bi) {
    const Block& B = P->in[bi];
    const int RI = 2 * B.l + 1;
    const int np = paths_into(P, bi, false);
    if (np == 0) continue;
    b.problem(gx + (long long)n0 * P->dim_in + B.offset, idx2(RI, P->dim_in, B.mul), idx1(1), cn * RI, B.mul,
              np * ((X ? 1 : 0) + (X2 ? 1 : 0)));
    for (const PathH& p : P->paths) {
      if (p.b_in != bi) continue;
      const Idx2 Am = idx2(RI, P->dev.xstate_per_node, (long long)P->K * p.c_out);
      const Idx2 Bk = idx2(p.c_out, P->n_w, 1);
      if (X) b.seg(X + p.xst_off, Am, idx1(1), W + p.w_off, Bk, idx1(p.c_out), P->K * p.c_out);
      if (X2) b.seg(X2 + p.xst_off, Am, idx1(1), W2 + p.w_off, Bk, idx1(p.c_out), P->K * p.c_out);
    }
  }
  return b.finish();
}

// A_bar_pi[(q,u), w] (+)= sum_{(j,mi)} x[(j,mi), u] X_pi[(j,mi),(q,w)]     (mirrored eq. 19)
// computed as its transpose, rows (q,w) and columns u, so the wide side fills the MMA rows.
// The sum over (j, mi) is one segment per mi, so that every k map is a single stride
// (the node) and operand tiles never cross a node boundary.
cudaError_t gemm_abar_src(const tpconv_plan* P, const float* x, const float* X, float* gW, int n0, int cn,
                          int accumulate, float* part, cudaStream_t st) {
  Batch b(P, st, 1, accumulate, nullptr, part);
  for (const PathH& p : P->paths) {
    const int RI = 2 * p.l_in + 1;
    b.problem(gW + p.w_off, idx2(p.c_out, P->n_w, 1), idx1(p.c_out), P->K * p.c_out, p.c_in, RI);
    for (int mi = 0; mi < RI; ++mi)
      b.seg(X + p.xst_off + (long long)mi * P->K * p.c_out, idx1(1), idx1(P->dev.xstate_per_node),
            x + (long long)n0 * P->dim_in + p.in_off + (long long)mi * p.c_in, idx1(P->dim_in), idx1(1), cn);
  }
  return b.finish();
}

// A_bar_pi[(q,u), w] (+)= sum_{(i,mo)} dS_pi[(i,mo),(q,u)] m_bar[(i,mo), w]   (eq. 39),
// one segment per mo (single-stride k maps, as above)
cudaError_t gemm_abar_recv(const tpconv_plan* P, const float* S, const float* gout, float* gW, int n0, int cn,
                           int accumulate, float* part, cudaStream_t st) {
  Batch b(P, st, 1, accumulate, nullptr, part);
  for (const PathH& p : P->paths) {
    const int RO = 2 * p.l_out + 1;
    b.problem(gW + p.w_off, idx2(p.c_in, P->n_w, p.c_out), idx1(1), P->K * p.c_in, p.c_out, RO);
    for (int mo = 0; mo < RO; ++mo)
      b.seg(S + p.st_off + (long long)mo * P->K * p.c_in, idx1(1), idx1(P->dev.state_per_node),
            gout + (long long)n0 * P->dim_out + p.out_off + (long long)mo * p.c_out, idx1(P->dim_out), idx1(1), cn);
  }
  return b.finish();
}

bool every_block_reached(const tpconv_plan* P, bool out_side) {
  const int nb = (int)(out_side ? P->out.size() : P->in.size());
  for (int b = 0; b < nb; ++b) {
    bool any = false;
    for (const PathH& p : P->paths) any = any || (out_side ? p.b_out : p.b_in) == b;
    if (!any) return false;
  }
  return true;
}

// CTAs per receiver of the lane-per-edge receiver backward (each takes every split-th
// 32-edge chunk of its receiver): twice the mean number of chunks, 1 to 8, so that
// receivers far above the mean degree are shared while at the mean every CTA has work.
int chunk_split(long long N, long long E) {
  const long long mean_chunks2 = (2 * E / std::max<long long>(N, 1) + 31) / 32;
  return (int)std::max<long long>(1, std::min<long long>(8, mean_chunks2));
}

float* fptr(void* ws, size_t off) { return reinterpret_cast<float*>(static_cast<char*>(ws) + off); }

// The receiver order of a uvw pass (chunks of L.recv_chunk nodes, heaviest first), written
// to the workspace and attached to a copy of the plan's device image.
cudaError_t attach_order(DevPlan& D, const Layout& L, void* ws, int n, const int32_t* row_ptr, cudaStream_t s) {
  int* order = reinterpret_cast<int*>(static_cast<char*>(ws) + L.order);
  D.order = order;
  return launch_degree_order(n, row_ptr, L.recv_chunk, order, s);
}

}  // namespace

extern "C" {

static tpconv_status forward_ir_mul(tpconv_plan_t P, int64_t N, int64_t E, const float* x,
                             const float* pos, const int32_t* row_ptr, const int32_t* src,
                             const float* W, float* out, void* ws, size_t ws_bytes,
                             struct CUstream_st* stream) {
  tpconv_status st = common_checks(P, N, E);
  if (st != TPCONV_OK) return st;
  if (N == 0) return TPCONV_OK;
  st = check_ptrs({x, pos, row_ptr, W, out}, {src});
  if (st != TPCONV_OK) return st;
  if (E > 0 && !src) return TPCONV_ERR_INVALID_ARG;
  const Layout L = make_layout(P, N, E, TPCONV_PASS_FORWARD);
  st = check_ws(L, ws, ws_bytes);
  if (st != TPCONV_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int n = (int)N;
  if (P->mode == TPCONV_UVU) {
    TPC_RUN(PC_UVU_FWD, 1, launch_uvu_fwd(P->dev, P->bp_out, P->t_bo, 0, x, nullptr, pos, nullptr, row_ptr, src, W,
                           nullptr, n, out, s));
    return TPCONV_OK;
  }
  if (!every_block_reached(P, true)) TPC_TRY(cudaMemsetAsync(out, 0, sizeof(float) * (size_t)N * P->dim_out, s));
  float* S = fptr(ws, L.state_a);
  DevPlan D = P->dev;
  TPC_RUN(PC_UVW_STATE, 1, attach_order(D, L, ws, n, row_ptr, s));
  for (int n0 = 0; n0 < n; n0 += L.recv_chunk) {
    const int cn = std::min(L.recv_chunk, n - n0);
    TPC_RUN(PC_UVW_STATE, 1, launch_uvw_state(D, P->t_in, 0, x, nullptr, pos, nullptr, row_ptr, src, n0, cn, S,
                             nullptr, s));
    TPC_RUN(PC_GEMM, 0, gemm_state_times_A(P, S, W, nullptr, nullptr, out, n0, cn, fptr(ws, L.part), s));
  }
  return TPCONV_OK;
}

static tpconv_status backward_ir_mul(tpconv_plan_t P, int64_t N, int64_t E, const float* x,
                              const float* pos, const int32_t* row_ptr, const int32_t* src,
                              const int32_t* t_ptr, const int32_t* t_eid, const int32_t* t_dst,
                              const float* W, const float* grad_out, float* grad_x,
                              float* grad_pos, float* grad_W, void* ws, size_t ws_bytes,
                              struct CUstream_st* stream) {
  tpconv_status st = common_checks(P, N, E);
  if (st != TPCONV_OK) return st;
  st = check_ptrs({}, {x, pos, row_ptr, src, t_ptr, t_eid, t_dst, W, grad_out, grad_x, grad_pos, grad_W});
  if (st != TPCONV_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (N == 0) {
    if (grad_W) TPC_TRY(cudaMemsetAsync(grad_W, 0, sizeof(float) * (size_t)P->K * P->n_w, s));
    return TPCONV_OK;
  }
  if (!x || !pos || !row_ptr || !W || !grad_out || (E > 0 && !src)) return TPCONV_ERR_INVALID_ARG;
  if ((grad_x || grad_pos || grad_W) && (!t_ptr || (E > 0 && (!t_eid || !t_dst)))) return TPCONV_ERR_INVALID_ARG;
  const Layout L = make_layout(P, N, E, TPCONV_PASS_BACKWARD);
  st = check_ws(L, ws, ws_bytes);
  if (st != TPCONV_OK) return st;
  const int n = (int)N;
  float4* gbuf = reinterpret_cast<float4*>(static_cast<char*>(ws) + L.gbuf);
  float* part = fptr(ws, L.part);

  // CTAs per receiver in the receiver backward: about four times the mean number of
  // 32-edge chunks per receiver (at most 16), so that receivers far above the mean
  // degree are shared
  const int edge_split = (int)std::max<long long>(1, std::min<long long>(16, (4 * E / std::max<int64_t>(N, 1) + 31) / 32));
  if (P->mode == TPCONV_UVU) {
    if (grad_pos) {
      TPC_TRY(cudaMemsetAsync(grad_pos, 0, sizeof(float) * 3 * (size_t)N, s));
      int* cursor = reinterpret_cast<int*>(static_cast<char*>(ws) + L.cursor);
      TPC_TRY(cudaMemcpyAsync(cursor, t_ptr, sizeof(int) * (size_t)N, cudaMemcpyDeviceToDevice, s));
      for (int w = 0; w < windows_per_range(E, L.win_edges); ++w) {
        const EdgeWindow win{0, n, w, L.win_edges};
        TPC_RUN(PC_UVU_RECV_BWD, 1, launch_uvu_recv_bwd(P->dev, P->t_in, x, pos, row_ptr, src, W, grad_out, n, gbuf,
                                                        win, edge_split, s));
        TPC_RUN(PC_POS, 1, launch_pos_window(n, row_ptr, t_ptr, t_eid, gbuf, win, cursor, grad_pos, s));
      }
    }
    if (grad_W) {
      const int nr = std::min(kUvuRanges, n);
      TPC_RUN(PC_UVU_GRADW, 1, launch_uvu_gradw(P->dev, P->t_in, 0, x, nullptr, pos, nullptr, row_ptr, src, grad_out, n,
                               nr, part, s));
      TPC_RUN(PC_UVU_GRADW, 1, launch_reduce_partials(part, nr, (long long)P->K * P->n_w, grad_W, 0, s));
    }
    if (grad_x)
      TPC_RUN(PC_UVU_SRC, 1, launch_uvu_src(P->dev, P->bp_in, P->t_bi, 0, pos, nullptr, t_ptr, t_eid, t_dst, W,
                             nullptr, grad_out, n, grad_x, s));
    return TPCONV_OK;
  }

  float* state = fptr(ws, L.state_a);
  if (grad_pos) {
    DevPlan D = P->dev;
    TPC_RUN(PC_UVW_RECV_BWD, 1, attach_order(D, L, ws, n, row_ptr, s));
    TPC_TRY(cudaMemsetAsync(grad_pos, 0, sizeof(float) * 3 * (size_t)N, s));
    int* cursor = reinterpret_cast<int*>(static_cast<char*>(ws) + L.cursor);
    TPC_TRY(cudaMemcpyAsync(cursor, t_ptr, sizeof(int) * (size_t)N, cudaMemcpyDeviceToDevice, s));
    for (int n0 = 0; n0 < n; n0 += L.recv_chunk) {
      const int cn = std::min(L.recv_chunk, n - n0);
      TPC_RUN(PC_GEMM, 0, gemm_sbar(P, grad_out, W, state, n0, cn, s));
      for (int w = 0; w < windows_per_range(E, L.win_edges); ++w) {
        const EdgeWindow win{n0, cn, w, L.win_edges};
        TPC_RUN(PC_UVW_RECV_BWD, 1, launch_uvw_recv_edge(D, x, pos, row_ptr, src, state, n0, cn, gbuf, win,
                                                         chunk_split(N, E), s));
        TPC_RUN(PC_POS, 1, launch_pos_window(n, row_ptr, t_ptr, t_eid, gbuf, win, cursor, grad_pos, s));
      }
    }
  }
  if (grad_x && !every_block_reached(P, false))
    TPC_TRY(cudaMemsetAsync(grad_x, 0, sizeof(float) * (size_t)N * P->dim_in, s));
  if (grad_x || grad_W) {
    for (int n0 = 0; n0 < n; n0 += L.src_chunk) {
      const int cn = std::min(L.src_chunk, n - n0);
      TPC_RUN(PC_UVW_SRC, 1, launch_uvw_src_state(P->dev, P->t_out, 0, pos, nullptr, t_ptr, t_eid, t_dst, grad_out, n0,
                                   cn, state, nullptr, s));
      if (grad_x) TPC_RUN(PC_GEMM, 0, gemm_xbar(P, state, W, nullptr, nullptr, grad_x, n0, cn, part, s));
      if (grad_W) TPC_RUN(PC_GEMM, 0, gemm_abar_src(P, x, state, grad_W, n0, cn, n0 > 0, part, s));
    }
  }
  return TPCONV_OK;
}

static tpconv_status forward_embedded_ir_mul(tpconv_plan_t P, int64_t N, int64_t E, const float* x,
                                      const float* Y, const float* phi, const int32_t* row_ptr,
                                      const int32_t* src, const float* W, float* out, void* ws,
                                      size_t ws_bytes, struct CUstream_st* stream) {
  tpconv_status st = common_checks(P, N, E);
  if (st != TPCONV_OK) return st;
  if (N == 0) return TPCONV_OK;
  st = check_ptrs({x, row_ptr, W, out}, {src, Y, phi});
  if (st != TPCONV_OK) return st;
  if (E > 0 && (!src || !Y || !phi)) return TPCONV_ERR_INVALID_ARG;
  const Layout L = make_layout(P, N, E, TPCONV_PASS_FORWARD);
  st = check_ws(L, ws, ws_bytes);
  if (st != TPCONV_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int n = (int)N;
  DevPlan D = P->dev;
  D.emb_Y = Y;
  D.emb_phi = phi;
  if (P->mode == TPCONV_UVU) {
    TPC_RUN(PC_UVU_FWD, 1, launch_uvu_fwd(D, P->bp_out, P->t_bo, 0, x, nullptr, nullptr, nullptr, row_ptr, src, W,
                           nullptr, n, out, s));
    return TPCONV_OK;
  }
  TPC_RUN(PC_UVW_STATE, 1, attach_order(D, L, ws, n, row_ptr, s));
  if (!every_block_reached(P, true)) TPC_TRY(cudaMemsetAsync(out, 0, sizeof(float) * (size_t)N * P->dim_out, s));
  float* S = fptr(ws, L.state_a);
  for (int n0 = 0; n0 < n; n0 += L.recv_chunk) {
    const int cn = std::min(L.recv_chunk, n - n0);
    TPC_RUN(PC_UVW_STATE, 1, launch_uvw_state(D, P->t_in, 0, x, nullptr, nullptr, nullptr, row_ptr, src, n0, cn, S,
                             nullptr, s));
    TPC_RUN(PC_GEMM, 0, gemm_state_times_A(P, S, W, nullptr, nullptr, out, n0, cn, fptr(ws, L.part), s));
  }
  return TPCONV_OK;
}

static tpconv_status backward_embedded_ir_mul(tpconv_plan_t P, int64_t N, int64_t E, const float* x,
                                       const float* Y, const float* phi, const int32_t* row_ptr,
                                       const int32_t* src, const int32_t* t_ptr, const int32_t* t_eid,
                                       const int32_t* t_dst, const float* W, const float* grad_out,
                                       float* grad_x, float* grad_W, float* grad_phi, float* grad_Y,
                                       void* ws, size_t ws_bytes, struct CUstream_st* stream) {
  tpconv_status st = common_checks(P, N, E);
  if (st != TPCONV_OK) return st;
  st = check_ptrs({}, {x, Y, phi, row_ptr, src, t_ptr, t_eid, t_dst, W, grad_out, grad_x, grad_W, grad_phi, grad_Y});
  if (st != TPCONV_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (N == 0) {
    if (grad_W) TPC_TRY(cudaMemsetAsync(grad_W, 0, sizeof(float) * (size_t)P->K * P->n_w, s));
    return TPCONV_OK;
  }
  if (!x || !row_ptr || !W || !grad_out || (E > 0 && (!src || !Y || !phi))) return TPCONV_ERR_INVALID_ARG;
  if ((grad_x || grad_W) && (!t_ptr || (E > 0 && (!t_eid || !t_dst)))) return TPCONV_ERR_INVALID_ARG;
  const Layout L = make_layout(P, N, E, TPCONV_PASS_BACKWARD);
  st = check_ws(L, ws, ws_bytes);
  if (st != TPCONV_OK) return st;
  const int n = (int)N;
  float* part = fptr(ws, L.part);
  DevPlan D = P->dev;
  D.emb_Y = Y;
  D.emb_phi = phi;
  D.emb_eid = t_eid;
  D.emb_gY = grad_Y;
  D.emb_gphi = grad_phi;
  const int edge_split = (int)std::max<long long>(1, std::min<long long>(16, (4 * E / std::max<int64_t>(N, 1) + 31) / 32));
  if (P->mode == TPCONV_UVU) {
    if ((grad_phi || grad_Y) && E > 0)
      TPC_RUN(PC_UVU_RECV_BWD, 1, launch_uvu_recv_bwd(D, P->t_in, x, nullptr, row_ptr, src, W, grad_out, n, nullptr,
                                    whole_range(0, n), edge_split, s));
    if (grad_W) {
      const int nr = std::min(kUvuRanges, n);
      TPC_RUN(PC_UVU_GRADW, 1, launch_uvu_gradw(D, P->t_in, 0, x, nullptr, nullptr, nullptr, row_ptr, src, grad_out,
                               n, nr, part, s));
      TPC_RUN(PC_UVU_GRADW, 1, launch_reduce_partials(part, nr, (long long)P->K * P->n_w, grad_W, 0, s));
    }
    if (grad_x)
      TPC_RUN(PC_UVU_SRC, 1, launch_uvu_src(D, P->bp_in, P->t_bi, 0, nullptr, nullptr, t_ptr, t_eid, t_dst, W,
                             nullptr, grad_out, n, grad_x, s));
    return TPCONV_OK;
  }
  float* state = fptr(ws, L.state_a);
  if ((grad_phi || grad_Y) && E > 0) {
    TPC_RUN(PC_UVW_RECV_BWD, 1, attach_order(D, L, ws, n, row_ptr, s));
    for (int n0 = 0; n0 < n; n0 += L.recv_chunk) {
      const int cn = std::min(L.recv_chunk, n - n0);
      TPC_RUN(PC_GEMM, 0, gemm_sbar(P, grad_out, W, state, n0, cn, s));
      TPC_RUN(PC_UVW_RECV_BWD, 1, launch_uvw_recv_edge(D, x, nullptr, row_ptr, src, state, n0, cn, nullptr,
                                                       whole_range(n0, cn), chunk_split(N, E), s));
    }
  }
  if (grad_x && !every_block_reached(P, false))
    TPC_TRY(cudaMemsetAsync(grad_x, 0, sizeof(float) * (size_t)N * P->dim_in, s));
  if (grad_x || grad_W) {
    for (int n0 = 0; n0 < n; n0 += L.src_chunk) {
      const int cn = std::min(L.src_chunk, n - n0);
      TPC_RUN(PC_UVW_SRC, 1, launch_uvw_src_state(D, P->t_out, 0, nullptr, nullptr, t_ptr, t_eid, t_dst, grad_out, n0,
                                   cn, state, nullptr, s));
      if (grad_x) TPC_RUN(PC_GEMM, 0, gemm_xbar(P, state, W, nullptr, nullptr, grad_x, n0, cn, part, s));
      if (grad_W) TPC_RUN(PC_GEMM, 0, gemm_abar_src(P, x, state, grad_W, n0, cn, n0 > 0, part, s));
    }
  }
  return TPCONV_OK;
}

static tpconv_status double_backward_ir_mul(tpconv_plan_t P, int64_t N, int64_t E, const float* x,
                                     const float* pos, const int32_t* row_ptr, const int32_t* src,
                                     const int32_t* t_ptr, const int32_t* t_eid,
                                     const int32_t* t_dst, const float* W, const float* grad_out,
                                     const float* gg_x, const float* gg_pos, const float* gg_W,
                                     float* grad_x, float* grad_W, float* grad_grad_out,
                                     float* grad_pos, void* ws, size_t ws_bytes,
                                     struct CUstream_st* stream) {
  tpconv_status st = common_checks(P, N, E);
  if (st != TPCONV_OK) return st;
  st = check_ptrs({}, {x, pos, row_ptr, src, t_ptr, t_eid, t_dst, W, grad_out, gg_x, gg_pos, gg_W, grad_x,
                       grad_W, grad_grad_out, grad_pos});
  if (st != TPCONV_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (N == 0) {
    if (grad_W) TPC_TRY(cudaMemsetAsync(grad_W, 0, sizeof(float) * (size_t)P->K * P->n_w, s));
    return TPCONV_OK;
  }
  if (!x || !pos || !row_ptr || !W || !grad_out || (E > 0 && !src)) return TPCONV_ERR_INVALID_ARG;
  if (grad_x && (!t_ptr || (E > 0 && !t_dst))) return TPCONV_ERR_INVALID_ARG;
  if (grad_pos && (!t_ptr || (E > 0 && !t_eid))) return TPCONV_ERR_INVALID_ARG;
  const Layout L = make_layout(P, N, E, TPCONV_PASS_DOUBLE_BACKWARD);
  st = check_ws(L, ws, ws_bytes);
  if (st != TPCONV_OK) return st;
  const int n = (int)N;
  float* part = fptr(ws, L.part);
  const bool tan_xp = gg_x || gg_pos;
  float4* gbuf = reinterpret_cast<float4*>(static_cast<char*>(ws) + L.gbuf);
  const int edge_split = (int)std::max<long long>(1, std::min<long long>(16, (4 * E / std::max<int64_t>(N, 1) + 31) / 32));
  const bool any_tan = gg_x || gg_pos || gg_W;
  if (grad_pos && !any_tan) TPC_TRY(cudaMemsetAsync(grad_pos, 0, sizeof(float) * 3 * (size_t)N, s));

  if (P->mode == TPCONV_UVU) {
    if (grad_grad_out)
      TPC_RUN(PC_UVU_FWD, 1, launch_uvu_fwd(P->dev, P->bp_out, P->t_bo, 1, x, gg_x, pos, gg_pos, row_ptr, src, W, gg_W,
                             n, grad_grad_out, s));
    if (grad_W) {
      const int nr = std::min(kUvuRanges, n);
      TPC_RUN(PC_UVU_GRADW, 1, launch_uvu_gradw(P->dev, P->t_in, 1, x, gg_x, pos, gg_pos, row_ptr, src, grad_out, n, nr,
                               part, s));
      TPC_RUN(PC_UVU_GRADW, 1, launch_reduce_partials(part, nr, (long long)P->K * P->n_w, grad_W, 0, s));
    }
    if (grad_x)
      TPC_RUN(PC_UVU_SRC, 1, launch_uvu_src(P->dev, P->bp_in, P->t_bi, 1, pos, gg_pos, t_ptr, t_eid, t_dst, W, gg_W,
                             grad_out, n, grad_x, s));
    if (grad_pos && any_tan) {
      // the tangent of the first-order position gradient (second derivatives of Y, phi)
      TPC_TRY(cudaMemsetAsync(grad_pos, 0, sizeof(float) * 3 * (size_t)N, s));
      int* cursor = reinterpret_cast<int*>(static_cast<char*>(ws) + L.cursor);
      TPC_TRY(cudaMemcpyAsync(cursor, t_ptr, sizeof(int) * (size_t)N, cudaMemcpyDeviceToDevice, s));
      for (int w = 0; w < windows_per_range(E, L.win_edges); ++w) {
        const EdgeWindow win{0, n, w, L.win_edges};
        TPC_RUN(PC_RECV_TAN, 1, launch_uvu_recv_dbl(P->dev, P->t_in, x, gg_x, pos, gg_pos, row_ptr, src, W, gg_W,
                                                   grad_out, n, gbuf, win, edge_split, s));
        TPC_RUN(PC_POS, 1, launch_pos_window(n, row_ptr, t_ptr, t_eid, gbuf, win, cursor, grad_pos, s));
      }
    }
    return TPCONV_OK;
  }

  float* sa = fptr(ws, L.state_a);
  float* sb = fptr(ws, L.state_b);
  const bool need_S = grad_grad_out && gg_W;
  const bool gout_direct = grad_grad_out && (tan_xp || need_S) && every_block_reached(P, true);
  if (grad_grad_out && !gout_direct)
    TPC_TRY(cudaMemsetAsync(grad_grad_out, 0, sizeof(float) * (size_t)N * P->dim_out, s));
  if (grad_W && !tan_xp) TPC_TRY(cudaMemsetAsync(grad_W, 0, sizeof(float) * (size_t)P->K * P->n_w, s));
  if ((grad_grad_out || grad_W) && (tan_xp || need_S)) {
    DevPlan D = P->dev;
    TPC_RUN(PC_UVW_STATE_TAN, 1, attach_order(D, L, ws, n, row_ptr, s));
    for (int n0 = 0; n0 < n; n0 += L.recv_chunk) {
      const int cn = std::min(L.recv_chunk, n - n0);
      // sa = dS (tangent of eq. 33), sb = S (needed for S dA in eq. 37)
      TPC_RUN(PC_UVW_STATE_TAN, 1, launch_uvw_state(D, P->t_in, 1, x, gg_x, pos, gg_pos, row_ptr, src, n0, cn,
                               need_S ? sb : nullptr, sa, s));
      if (grad_grad_out)
        TPC_RUN(PC_GEMM, 0, gemm_state_times_A(P, tan_xp ? sa : nullptr, W, need_S ? sb : nullptr, gg_W, grad_grad_out, n0,
                                   cn, part, s));
      if (grad_W && tan_xp) TPC_RUN(PC_GEMM, 0, gemm_abar_recv(P, sa, grad_out, grad_W, n0, cn, n0 > 0, part, s));
    }
  }
  if (grad_x) {
    const bool direct = (gg_pos || gg_W) && every_block_reached(P, false);
    if (!direct) TPC_TRY(cudaMemsetAsync(grad_x, 0, sizeof(float) * (size_t)N * P->dim_in, s));
    if (gg_pos || gg_W) {
      for (int n0 = 0; n0 < n; n0 += L.src_chunk) {
        const int cn = std::min(L.src_chunk, n - n0);
        // sa = X' (tangent of the source state), sb = X
        TPC_RUN(PC_UVW_SRC_TAN, 1, launch_uvw_src_state(P->dev, P->t_out, 1, pos, gg_pos, t_ptr, t_eid, t_dst, grad_out, n0,
                                     cn, gg_W ? sb : nullptr, sa, s));
        TPC_RUN(PC_GEMM, 0, gemm_xbar(P, gg_pos ? sa : nullptr, W, gg_W ? sb : nullptr, gg_W, grad_x, n0, cn, part, s));
      }
    }
  }
  if (grad_pos && any_tan) {
    // the tangent of the first-order position gradient: per receiver range S_bar = m_bar A^T
    // (sa) and S_bar_dot = m_bar A_dot^T (sb), then per edge through second derivatives
    // of Y and phi, then the fixed-order scatter of the backward
    DevPlan D = P->dev;
    TPC_RUN(PC_RECV_TAN, 1, attach_order(D, L, ws, n, row_ptr, s));
    TPC_TRY(cudaMemsetAsync(grad_pos, 0, sizeof(float) * 3 * (size_t)N, s));
    int* cursor = reinterpret_cast<int*>(static_cast<char*>(ws) + L.cursor);
    TPC_TRY(cudaMemcpyAsync(cursor, t_ptr, sizeof(int) * (size_t)N, cudaMemcpyDeviceToDevice, s));
    for (int n0 = 0; n0 < n; n0 += L.recv_chunk) {
      const int cn = std::min(L.recv_chunk, n - n0);
      TPC_RUN(PC_GEMM, 0, gemm_sbar(P, grad_out, W, sa, n0, cn, s));
      if (gg_W) TPC_RUN(PC_GEMM, 0, gemm_sbar(P, grad_out, gg_W, sb, n0, cn, s));
      for (int w = 0; w < windows_per_range(E, L.win_edges); ++w) {
        const EdgeWindow win{n0, cn, w, L.win_edges};
        TPC_RUN(PC_RECV_TAN, 1, launch_uvw_recv_dbl(D, P->t_in, x, gg_x, pos, gg_pos, row_ptr, src, sa,
                                                   gg_W ? sb : nullptr, n0, cn, gbuf, win, edge_split, s));
        TPC_RUN(PC_POS, 1, launch_pos_window(n, row_ptr, t_ptr, t_eid, gbuf, win, cursor, grad_pos, s));
      }
    }
  }
  return TPCONV_OK;
}

// Public passes: the ir_mul implementations above, with the node arrays converted at the
// boundary when the plan's layout is mul_ir.
tpconv_status tpconv_forward(tpconv_plan_t P, int64_t N, int64_t E, const float* x, const float* pos,
                             const int32_t* row_ptr, const int32_t* src, const float* W, float* out, void* ws,
                             size_t ws_bytes, struct CUstream_st* stream) {
  if (!P || P->layout == TPCONV_LAYOUT_IR_MUL || N <= 0)
    return forward_ir_mul(P, N, E, x, pos, row_ptr, src, W, out, ws, ws_bytes, stream);
  if (!x || !out || N > 0x7ffffffe) return TPCONV_ERR_INVALID_ARG;
  ConvBufs B;
  tpconv_status st = conversion_setup(P, N, E, TPCONV_PASS_FORWARD, ws, ws_bytes, B);
  if (st != TPCONV_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  const float* xi = to_ir_mul(P, true, N, x, B.xin[0], s, e);
  if (e != cudaSuccess) return TPCONV_ERR_CUDA;
  st = forward_ir_mul(P, N, E, xi, pos, row_ptr, src, W, B.xout[0], ws, B.inner, stream);
  if (st != TPCONV_OK) return st;
  from_ir_mul(P, false, N, B.xout[0], out, s, e);
  return e == cudaSuccess ? TPCONV_OK : TPCONV_ERR_CUDA;
}

tpconv_status tpconv_backward(tpconv_plan_t P, int64_t N, int64_t E, const float* x, const float* pos,
                              const int32_t* row_ptr, const int32_t* src, const int32_t* t_ptr,
                              const int32_t* t_eid, const int32_t* t_dst, const float* W, const float* grad_out,
                              float* grad_x, float* grad_pos, float* grad_W, void* ws, size_t ws_bytes,
                              struct CUstream_st* stream) {
  if (!P || P->layout == TPCONV_LAYOUT_IR_MUL || N <= 0)
    return backward_ir_mul(P, N, E, x, pos, row_ptr, src, t_ptr, t_eid, t_dst, W, grad_out, grad_x, grad_pos,
                           grad_W, ws, ws_bytes, stream);
  if (!x || !grad_out || N > 0x7ffffffe) return TPCONV_ERR_INVALID_ARG;
  ConvBufs B;
  tpconv_status st = conversion_setup(P, N, E, TPCONV_PASS_BACKWARD, ws, ws_bytes, B);
  if (st != TPCONV_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  const float* xi = to_ir_mul(P, true, N, x, B.xin[0], s, e);
  const float* gi = to_ir_mul(P, false, N, grad_out, B.xout[0], s, e);
  if (e != cudaSuccess) return TPCONV_ERR_CUDA;
  st = backward_ir_mul(P, N, E, xi, pos, row_ptr, src, t_ptr, t_eid, t_dst, W, gi, grad_x ? B.xin[1] : nullptr,
                       grad_pos, grad_W, ws, B.inner, stream);
  if (st != TPCONV_OK) return st;
  from_ir_mul(P, true, N, B.xin[1], grad_x, s, e);
  return e == cudaSuccess ? TPCONV_OK : TPCONV_ERR_CUDA;
}

tpconv_status tpconv_double_backward(tpconv_plan_t P, int64_t N, int64_t E, const float* x, const float* pos,
                                     const int32_t* row_ptr, const int32_t* src, const int32_t* t_ptr,
                                     const int32_t* t_eid, const int32_t* t_dst, const float* W,
                                     const float* grad_out, const float* gg_x, const float* gg_pos,
                                     const float* gg_W, float* grad_x, float* grad_W, float* grad_grad_out,
                                     float* grad_pos, void* ws, size_t ws_bytes, struct CUstream_st* stream) {
  if (!P || P->layout == TPCONV_LAYOUT_IR_MUL || N <= 0)
    return double_backward_ir_mul(P, N, E, x, pos, row_ptr, src, t_ptr, t_eid, t_dst, W, grad_out, gg_x, gg_pos,
                                  gg_W, grad_x, grad_W, grad_grad_out, grad_pos, ws, ws_bytes, stream);
  if (!x || !grad_out || N > 0x7ffffffe) return TPCONV_ERR_INVALID_ARG;
  ConvBufs B;
  tpconv_status st = conversion_setup(P, N, E, TPCONV_PASS_DOUBLE_BACKWARD, ws, ws_bytes, B);
  if (st != TPCONV_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  const float* xi = to_ir_mul(P, true, N, x, B.xin[0], s, e);
  const float* gi = to_ir_mul(P, false, N, grad_out, B.xout[0], s, e);
  const float* ggi = to_ir_mul(P, true, N, gg_x, B.xin[1], s, e);
  if (e != cudaSuccess) return TPCONV_ERR_CUDA;
  st = double_backward_ir_mul(P, N, E, xi, pos, row_ptr, src, t_ptr, t_eid, t_dst, W, gi, ggi, gg_pos, gg_W,
                              grad_x ? B.xin[2] : nullptr, grad_W, grad_grad_out ? B.xout[1] : nullptr, grad_pos,
                              ws, B.inner, stream);
  if (st != TPCONV_OK) return st;
  from_ir_mul(P, true, N, B.xin[2], grad_x, s, e);
  from_ir_mul(P, false, N, B.xout[1], grad_grad_out, s, e);
  return e == cudaSuccess ? TPCONV_OK : TPCONV_ERR_CUDA;
}

tpconv_status tpconv_forward_embedded(tpconv_plan_t P, int64_t N, int64_t E, const float* x, const float* Y,
                                      const float* phi, const int32_t* row_ptr, const int32_t* src, const float* W,
                                      float* out, void* ws, size_t ws_bytes, struct CUstream_st* stream) {
  if (!P || P->layout == TPCONV_LAYOUT_IR_MUL || N <= 0)
    return forward_embedded_ir_mul(P, N, E, x, Y, phi, row_ptr, src, W, out, ws, ws_bytes, stream);
  if (!x || !out || N > 0x7ffffffe) return TPCONV_ERR_INVALID_ARG;
  ConvBufs B;
  tpconv_status st = conversion_setup(P, N, E, TPCONV_PASS_FORWARD, ws, ws_bytes, B);
  if (st != TPCONV_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  const float* xi = to_ir_mul(P, true, N, x, B.xin[0], s, e);
  if (e != cudaSuccess) return TPCONV_ERR_CUDA;
  st = forward_embedded_ir_mul(P, N, E, xi, Y, phi, row_ptr, src, W, B.xout[0], ws, B.inner, stream);
  if (st != TPCONV_OK) return st;
  from_ir_mul(P, false, N, B.xout[0], out, s, e);
  return e == cudaSuccess ? TPCONV_OK : TPCONV_ERR_CUDA;
}

tpconv_status tpconv_backward_embedded(tpconv_plan_t P, int64_t N, int64_t E, const float* x, const float* Y,
                                       const float* phi, const int32_t* row_ptr, const int32_t* src,
                                       const int32_t* t_ptr, const int32_t* t_eid, const int32_t* t_dst,
                                       const float* W, const float* grad_out, float* grad_x, float* grad_W,
                                       float* grad_phi, float* grad_Y, void* ws, size_t ws_bytes,
                                       struct CUstream_st* stream) {
  if (!P || P->layout == TPCONV_LAYOUT_IR_MUL || N <= 0)
    return backward_embedded_ir_mul(P, N, E, x, Y, phi, row_ptr, src, t_ptr, t_eid, t_dst, W, grad_out, grad_x,
                                    grad_W, grad_phi, grad_Y, ws, ws_bytes, stream);
  if (!x || !grad_out || N > 0x7ffffffe) return TPCONV_ERR_INVALID_ARG;
  ConvBufs B;
  tpconv_status st = conversion_setup(P, N, E, TPCONV_PASS_BACKWARD, ws, ws_bytes, B);
  if (st != TPCONV_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  const float* xi = to_ir_mul(P, true, N, x, B.xin[0], s, e);
  const float* gi = to_ir_mul(P, false, N, grad_out, B.xout[0], s, e);
  if (e != cudaSuccess) return TPCONV_ERR_CUDA;
  st = backward_embedded_ir_mul(P, N, E, xi, Y, phi, row_ptr, src, t_ptr, t_eid, t_dst, W, gi,
                                grad_x ? B.xin[1] : nullptr, grad_W, grad_phi, grad_Y, ws, B.inner, stream);
  if (st != TPCONV_OK) return st;
  from_ir_mul(P, true, N, B.xin[1], grad_x, s, e);
  return e == cudaSuccess ? TPCONV_OK : TPCONV_ERR_CUDA;
}

tpconv_status tpconv_profile_begin(int32_t max_records) {
  if (max_records < 1 || max_records > (1 << 20)) return TPCONV_ERR_INVALID_ARG;
  Prof& P = prof();
  std::lock_guard<std::mutex> g(P.mu);
  const size_t want = size_t(2) * max_records;
  while (P.pool.size() < want) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return TPCONV_ERR_CUDA;
    P.pool.push_back(e);
  }
  P.cat.assign(max_records, 0);
  P.used = 0;
  for (long long& v : P.launches) v = 0;
  P.on = true;
  return TPCONV_OK;
}

tpconv_status tpconv_profile_end(double* ms, int64_t* launches, int32_t n) {
  if (n < 0 || n > PC_COUNT) return TPCONV_ERR_INVALID_ARG;
  Prof& P = prof();
  std::lock_guard<std::mutex> g(P.mu);
  double tot[PC_COUNT] = {};
  tpconv_status st = TPCONV_OK;
  for (size_t r = 0; r < P.used; ++r) {
    float t = 0.f;
    if (cudaEventSynchronize(P.pool[2 * r + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&t, P.pool[2 * r], P.pool[2 * r + 1]) != cudaSuccess) {
      st = TPCONV_ERR_CUDA;
      continue;
    }
    tot[P.cat[r]] += t;
  }
  for (int c = 0; c < n; ++c) {
    if (ms) ms[c] = tot[c];
    if (launches) launches[c] = P.launches[c];
  }
  P.on = false;
  P.used = 0;
  return st;
}

tpconv_status tpconv_device_error(int32_t* out) {
  if (!out) return TPCONV_ERR_INVALID_ARG;
  int v = 0;
  if (read_and_clear_device_error(&v) != cudaSuccess) return TPCONV_ERR_CUDA;
  *out = v;
  return TPCONV_OK;
}

const char* tpconv_profile_category_name(int32_t c) {
  return (c >= 0 && c < PC_COUNT) ? kProfNames[c] : "unknown";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// forward with library-owned static scratch (no allocation anywhere)
// ---------------------------------------------------------------------------

static __device__ __align__(256) unsigned char g_static_scratch[TPCONV_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 256;
std::mutex g_static_mu;
void* g_static_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device, looked up once per device
// (per process: a cudaDeviceReset discards the module, so the library must not be used
// across one).
tpconv_status static_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return TPCONV_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TPCONV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> g(g_static_mu);
  if (!g_static_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return TPCONV_ERR_CUDA;
    g_static_addr[dev] = p;
  }
  *out = g_static_addr[dev];
  return TPCONV_OK;
}

// Forward layout (uvw) sized for a fixed scratch: receiver ranges of node state plus
// the split-K slices of the channel contraction.  The two arrays are each padded to
// 256 bytes, so the range is sized for the scratch less those paddings and then shrunk
// while the padded total still exceeds it.
Layout forward_layout_for(const tpconv_plan* P, long long N, size_t bytes) {
  const long long st = P->dev.state_per_node;
  const long long per_node = st + (long long)kSplits * P->dim_out;
  const size_t usable = bytes > 512 ? bytes - 512 : 0;
  long long fit = std::max<long long>(0, std::min<long long>((long long)(usable / 4) / per_node, N));
  auto make = [&](long long chunk) {
    Layout L;
    L.recv_chunk = (int)chunk;
    L.state_a = 0;
    const size_t one = align256(size_t(4) * chunk * st);
    L.has_part = true;
    L.part = one;
    L.total = one + align256(size_t(4) * kSplits * chunk * P->dim_out);
    return L;
  };
  Layout L = make(fit);
  while (fit > 0 && L.total > bytes) L = make(--fit);
  return L;
}

}  // namespace

extern "C" tpconv_status tpconv_forward_no_alloc(tpconv_plan_t P, int64_t N, int64_t E, const float* x,
                                                 const float* pos, const int32_t* row_ptr,
                                                 const int32_t* src, const float* W, float* out,
                                                 struct CUstream_st* stream) {
  if (P && P->layout != TPCONV_LAYOUT_IR_MUL) return TPCONV_ERR_UNSUPPORTED;  // ir_mul boundary only
  tpconv_status st = common_checks(P, N, E);
  if (st != TPCONV_OK) return st;
  if (N == 0) return TPCONV_OK;
  st = check_ptrs({x, pos, row_ptr, W, out}, {src});
  if (st != TPCONV_OK) return st;
  if (E > 0 && !src) return TPCONV_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  const int n = (int)N;
  if (P->mode == TPCONV_UVU) {  // channelwise forward keeps no scratch
    TPC_RUN(PC_UVU_FWD, 1, launch_uvu_fwd(P->dev, P->bp_out, P->t_bo, 0, x, nullptr, pos, nullptr, row_ptr, src,
                                          W, nullptr, n, out, s));
    return TPCONV_OK;
  }
  const Layout L = forward_layout_for(P, N, TPCONV_STATIC_SCRATCH_BYTES);
  if (L.recv_chunk < 1 || L.total > TPCONV_STATIC_SCRATCH_BYTES) return TPCONV_ERR_WORKSPACE_TOO_SMALL;
  void* ws = nullptr;
  st = static_scratch_address(&ws);
  if (st != TPCONV_OK) return st;
  // every element of the state and of the split-K slices is written before it is read
  if (!every_block_reached(P, true)) TPC_TRY(cudaMemsetAsync(out, 0, sizeof(float) * (size_t)N * P->dim_out, s));
  float* S = fptr(ws, L.state_a);
  for (int n0 = 0; n0 < n; n0 += L.recv_chunk) {
    const int cn = std::min(L.recv_chunk, n - n0);
    TPC_RUN(PC_UVW_STATE, 1, launch_uvw_state(P->dev, P->t_in, 0, x, nullptr, pos, nullptr, row_ptr, src, n0, cn, S,
                                              nullptr, s));
    TPC_RUN(PC_GEMM, 0, gemm_state_times_A(P, S, W, nullptr, nullptr, out, n0, cn, fptr(ws, L.part), s));
  }
  return TPCONV_OK;
}
