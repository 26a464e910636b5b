// Dispatch of the streaming kernels on the padded radial size KP (8 or 16) and on the
// pass mode (0: primal, 1: tangent for the double backward).
#include "launch.h"

namespace tpc {

#define TPC_BY_KP_MODE(RUN, ...)                                      \
  if (P.K <= 8) return mode == 0 ? RUN<8, 0>(__VA_ARGS__) : RUN<8, 1>(__VA_ARGS__); \
  return mode == 0 ? RUN<16, 0>(__VA_ARGS__) : RUN<16, 1>(__VA_ARGS__);

cudaError_t launch_uvw_state(const DevPlan& P, const Tasks& T, int mode, const float* x,
                             const float* xdot, const float* pos, const float* posdot,
                             const int* row_ptr, const int* src, int node0, int n_nodes,
                             float* S, float* Sdot, cudaStream_t s) {
  if (n_nodes <= 0 || T.n == 0) return cudaSuccess;
  TPC_BY_KP_MODE(run_uvw_state, P, T, x, xdot, pos, posdot, row_ptr, src, node0, n_nodes, S, Sdot, s)
}

cudaError_t launch_uvw_recv_edge(const DevPlan& P, const float* x, const float* pos, const int* row_ptr,
                                 const int* src, const float* Sbar, int node0, int n_nodes, float4* gbuf,
                                 EdgeWindow win, int split, cudaStream_t s) {
  if (n_nodes <= 0) return cudaSuccess;
  if (split < 1) split = 1;
  // the fast variant needs every channel count and offset of x and of the state to be a
  // multiple of 4 floats
  bool fast = P.dim_in % 4 == 0 && P.state_per_node % 4 == 0;
  for (int k = 0; k < P.n_paths; ++k)
    fast = fast && P.p[k].c_in % 4 == 0 && P.p[k].in_off % 4 == 0 && P.p[k].st_off % 4 == 0;
  if (P.K <= 8)
    return fast ? run_uvw_recv_edge<8, true>(P, x, pos, row_ptr, src, Sbar, node0, n_nodes, gbuf, win, split, s)
                : run_uvw_recv_edge<8, false>(P, x, pos, row_ptr, src, Sbar, node0, n_nodes, gbuf, win, split, s);
  return fast ? run_uvw_recv_edge<16, true>(P, x, pos, row_ptr, src, Sbar, node0, n_nodes, gbuf, win, split, s)
              : run_uvw_recv_edge<16, false>(P, x, pos, row_ptr, src, Sbar, node0, n_nodes, gbuf, win, split, s);
}

cudaError_t launch_uvw_recv_dbl(const DevPlan& P, const Tasks& T, const float* x, const float* xdot,
                                const float* pos, const float* posdot, const int* row_ptr, const int* src,
                                const float* Sbar, const float* Sbard, int node0, int n_nodes, float4* gbuf,
                                EdgeWindow win, int edge_split, cudaStream_t s) {
  if (n_nodes <= 0) return cudaSuccess;
  if (edge_split < 1) edge_split = 1;
#define TPC_RUN_DBL(KP, AD) \
  return run_uvw_recv_dbl<KP, AD>(P, T, x, xdot, pos, posdot, row_ptr, src, Sbar, Sbard, node0, n_nodes, gbuf, win, \
                                  edge_split, s)
  if (P.K <= 8) {
    if (Sbard) TPC_RUN_DBL(8, true);
    TPC_RUN_DBL(8, false);
  }
  if (Sbard) TPC_RUN_DBL(16, true);
  TPC_RUN_DBL(16, false);
#undef TPC_RUN_DBL
}

cudaError_t launch_uvu_recv_dbl(const DevPlan& P, const Tasks& T, const float* x, const float* xdot,
                                const float* pos, const float* posdot, const int* row_ptr, const int* src,
                                const float* W, const float* Wdot, const float* grad_out, int N, float4* gbuf,
                                EdgeWindow win, int edge_split, cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  if (edge_split < 1) edge_split = 1;
#define TPC_RUN_DBL(KP, AD) \
  return run_uvu_recv_dbl<KP, AD>(P, T, x, xdot, pos, posdot, row_ptr, src, W, Wdot, grad_out, N, gbuf, win, \
                                  edge_split, s)
  if (P.K <= 8) {
    if (Wdot) TPC_RUN_DBL(8, true);
    TPC_RUN_DBL(8, false);
  }
  if (Wdot) TPC_RUN_DBL(16, true);
  TPC_RUN_DBL(16, false);
#undef TPC_RUN_DBL
}

cudaError_t launch_uvw_src_state(const DevPlan& P, const Tasks& T, int mode,
                                 const float* pos, const float* posdot, const int* t_ptr,
                                 const int* t_eid, const int* t_dst, const float* grad_out,
                                 int node0, int n_nodes, float* X, float* Xdot,
                                 cudaStream_t s) {
  (void)t_eid;
  if (n_nodes <= 0 || T.n == 0) return cudaSuccess;
  TPC_BY_KP_MODE(run_uvw_src_state, P, T, pos, posdot, t_ptr, t_dst, grad_out, node0, n_nodes, X, Xdot, s)
}

cudaError_t launch_uvu_fwd(const DevPlan& P, const BlockPaths& BP, const Tasks& T, int mode,
                           const float* x, const float* xdot, const float* pos,
                           const float* posdot, const int* row_ptr, const int* src,
                           const float* W, const float* Wdot, int N, float* out,
                           cudaStream_t s) {
  if (N <= 0 || T.n == 0) return cudaSuccess;
  TPC_BY_KP_MODE(run_uvu_fwd, P, BP, T, x, xdot, pos, posdot, row_ptr, src, W, Wdot, N, out, s)
}

cudaError_t launch_uvu_recv_bwd(const DevPlan& P, const Tasks& T, const float* x,
                                const float* pos, const int* row_ptr, const int* src,
                                const float* W, const float* grad_out, int N, float4* gbuf,
                                EdgeWindow win, int edge_split, cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  if (edge_split < 1) edge_split = 1;
  if (P.K <= 8) return run_uvu_recv_bwd<8>(P, T, x, pos, row_ptr, src, W, grad_out, N, gbuf, win, edge_split, s);
  return run_uvu_recv_bwd<16>(P, T, x, pos, row_ptr, src, W, grad_out, N, gbuf, win, edge_split, s);
}

cudaError_t launch_uvu_gradw(const DevPlan& P, const Tasks& T, int mode, const float* x,
                             const float* xdot, const float* pos, const float* posdot,
                             const int* row_ptr, const int* src, const float* grad_out,
                             int N, int n_ranges, float* partial, cudaStream_t s) {
  if (N <= 0 || T.n == 0) return cudaSuccess;
  TPC_BY_KP_MODE(run_uvu_gradw, P, T, x, xdot, pos, posdot, row_ptr, src, grad_out, N, n_ranges, partial, s)
}

cudaError_t launch_uvu_src(const DevPlan& P, const BlockPaths& BP, const Tasks& T, int mode,
                           const float* pos, const float* posdot, const int* t_ptr,
                           const int* t_eid, const int* t_dst, const float* W,
                           const float* Wdot, const float* grad_out, int N, float* grad_x,
                           cudaStream_t s) {
  (void)t_eid;
  if (N <= 0 || T.n == 0) return cudaSuccess;
  TPC_BY_KP_MODE(run_uvu_src, P, BP, T, pos, posdot, t_ptr, t_dst, W, Wdot, grad_out, N, grad_x, s)
}

}  // namespace tpc
