// Internal types shared by the host plan/launch code and the kernels (the kernel
// launchers are declared in launch.h, which kernel sources do not include, so that a new
// launcher does not rebuild every kernel unit).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace tpc {

constexpr int MAX_PATHS = 64;
constexpr int MAX_TASKS = 256;
constexpr int MAX_BLOCKS = 16;
constexpr int WARPS_PER_CTA = 4;
// Resident CTAs per SM requested by the streaming kernels (second launch-bounds argument,
// a register cap of 65536 / (128 x blocks)): 4 or 5 where that measured faster, else left
// to the compiler.

// One path of the plan as the kernels see it.
struct DevPath {
  int type;            // index into tpc_tab::TRIPLES (the (l_in, l_sh, l_out) triple)
  int l_in, l_sh, l_out;
  int c_in, c_out;
  int in_off, out_off; // float offsets of the input / output block inside a node row
  int w_off;           // first weight column
  int st_off;          // offset of the path inside a receiver-state row  (R_out*K*C_in floats)
  int xst_off;         // offset of the path inside a source-state row    (R_in*K*C_out floats)
  int b_in, b_out;
};

struct DevPlan {
  int n_paths, dim_in, dim_out, n_w, K, lmax, mode;
  int radial_kind, poly_p;
  float r_cut, inv_r_cut, bessel_pref, g_mu0, g_step, g_inv_sigma2;
  float env_a, env_b, env_c;
  int state_per_node;   // sum_pi R_out * K * C_in
  int xstate_per_node;  // sum_pi R_in * K * C_out
  int n_sh;             // (lmax + 1)^2
  // embedded-input calls only (all NULL otherwise): per-edge Y [E][n_sh] and phi [E][K]
  // in receiver-CSR edge order, the source view's edge ids, and the edge-owned adjoints
  const float* emb_Y;
  const float* emb_phi;
  const int* emb_eid;
  float* emb_gY;
  float* emb_gphi;
  // receiver processing order of a pass (NULL: node order): within every chunk of
  // `order_chunk` nodes, the chunk's nodes by descending in-degree class
  const int* order;
  DevPath p[MAX_PATHS];
};

// One window of the position-gradient staging: the edges of receivers
// [n0, n0 + n_nodes) are cut into consecutive windows of `size` edge ids, and window
// `index` covers [row_ptr[n0] + index * size, min(that + size, row_ptr[n0 + n_nodes])).
// The receiver kernels stage g_e of the window's edges at gbuf[e - window start]; the
// host loops over an upper bound of the window count (empty windows do nothing), since
// the edge count of a receiver range is known on the device only.
struct EdgeWindow {
  int n0, n_nodes, index;
  long long size;
};

__host__ __device__ inline EdgeWindow whole_range(int n0, int n_nodes) {
  return EdgeWindow{n0, n_nodes, 0, 0x7fffffffLL};
}

// A list of warp tasks: (a, b) pairs whose meaning depends on the kernel
// (path & 32-channel chunk, or block & chunk).
struct Tasks {
  int n;
  short a[MAX_TASKS];
  short b[MAX_TASKS];
};

// Paths grouped by an irrep block (output block for uvu forward, input block for the
// uvu source pass).
struct BlockPaths {
  int n_blocks;
  int l[MAX_BLOCKS];
  int c[MAX_BLOCKS];
  int off[MAX_BLOCKS];
  int count[MAX_BLOCKS];
  short list[MAX_BLOCKS][MAX_PATHS];
};

// Two-level affine index map f(i) = (i / d) * s1 + (i % d) * s2.
struct Idx2 {
  int d;
  long long s1, s2;
};
inline Idx2 idx1(long long s) { return Idx2{0x7fffffff, 0, s}; }
inline Idx2 idx2(int d, long long s1, long long s2) { return Idx2{d, s1, s2}; }

// Grouped, multi-segment GEMM.  Problem p computes
//   C_p(m, n) (+)= sum over its segments s of sum_k A_s(m, k) B_s(k, n)
// with every operand addressed through two-level affine maps, so node rows of the
// ir_mul tensors, the weight matrix and workspace states are read in place.  Problems
// write disjoint outputs; one launch covers all problems.  With splits > 1 each
// problem's contraction is split and reduced in a fixed order from `partial`.
constexpr int MAX_GEMM_PROBLEMS = 64;
constexpr int MAX_GEMM_SEGS = 128;

struct GemmSeg {
  const float* A; Idx2 Am, Ak;   // A(m, k)
  const float* B; Idx2 Bk, Bn;   // B(k, n)
  int K;
  int a_vec4;                    // A rows are 16-byte aligned and contiguous in k
  int b_vec4;                    // B columns are 16-byte aligned and contiguous in k
  int a_mvec4;                   // A is contiguous in m (unit m stride), 16-byte aligned at every k
};

struct GemmProblem {
  float* C; Idx2 Cm, Cn;         // C(m, n)
  int M, N;
  int seg0, nseg;                // segments [seg0, seg0 + nseg)
  int Ktot;                      // sum of the segments' K
  int tile0;                     // first global tile of this problem
  long long part_off;            // offset of this problem in `partial` (splits * M * N floats)
};

struct GemmBatch {
  int n_problems, n_segs, splits, total_tiles, accumulate;
  int math;                      // TPCONV_MATH_FP32 (3xTF32), _TF32 (one TF32 product) or _BF16
  float* partial;
  GemmProblem pr[MAX_GEMM_PROBLEMS];
  GemmSeg sg[MAX_GEMM_SEGS];
};

// Irrep blocks of a node row, for converting between the ir_mul layout (block [2l+1][C])
// and the mul_ir layout (block [C][2l+1]).
struct LayoutMap {
  int n;
  int off[MAX_BLOCKS], l[MAX_BLOCKS], mul[MAX_BLOCKS];
};
}  // namespace tpc
