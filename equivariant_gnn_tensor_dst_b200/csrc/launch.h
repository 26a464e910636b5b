// Kernel runners and launchers (host side): included by the launch, API, graph and
// contraction sources, not by the streaming-kernel units.
#pragma once
#include "internal.h"

namespace tpc {

// Per-(KP, MODE) kernel runners.  Each is explicitly instantiated in its own
// translation unit (the build compiles k_uvw.cu / k_uvu.cu once per unit) so that the
// heavily unrolled kernels compile in parallel.
template <int KP, int MODE>
cudaError_t run_uvw_state(const DevPlan& P, const Tasks& T, const float* x, const float* xdot,
                          const float* pos, const float* posdot, const int* row_ptr,
                          const int* src, int node0, int n_nodes, float* S, float* Sdot,
                          cudaStream_t s);
template <int KP, bool FAST>  // FAST: every channel count and offset a multiple of 4 floats
cudaError_t run_uvw_recv_edge(const DevPlan& P, const float* x, const float* pos, const int* row_ptr,
                              const int* src, const float* Sbar, int node0, int n_nodes, float4* gbuf,
                              EdgeWindow win, int split, cudaStream_t s);
template <int KP, bool AD>   // AD: the A_dot tangent is present (its own build unit)
cudaError_t run_uvw_recv_dbl(const DevPlan& P, const Tasks& T, const float* x, const float* xdot,
                             const float* pos, const float* posdot, const int* row_ptr, const int* src,
                             const float* Sbar, const float* Sbard, int node0, int n_nodes, float4* gbuf,
                             EdgeWindow win, int edge_split, cudaStream_t s);
template <int KP, bool AD>
cudaError_t run_uvu_recv_dbl(const DevPlan& P, const Tasks& T, const float* x, const float* xdot,
                             const float* pos, const float* posdot, const int* row_ptr, const int* src,
                             const float* W, const float* Wdot, const float* grad_out, int N, float4* gbuf,
                             EdgeWindow win, int edge_split, cudaStream_t s);
template <int KP, int MODE>
cudaError_t run_uvw_src_state(const DevPlan& P, const Tasks& T, const float* pos,
                              const float* posdot, const int* t_ptr, const int* t_dst,
                              const float* grad_out, int node0, int n_nodes, float* X,
                              float* Xdot, cudaStream_t s);
template <int KP, int MODE>
cudaError_t run_uvu_fwd(const DevPlan& P, const BlockPaths& BP, const Tasks& T, const float* x,
                        const float* xdot, const float* pos, const float* posdot,
                        const int* row_ptr, const int* src, const float* W, const float* Wdot,
                        int N, float* out, cudaStream_t s);
template <int KP>
cudaError_t run_uvu_recv_bwd(const DevPlan& P, const Tasks& T, const float* x, const float* pos,
                             const int* row_ptr, const int* src, const float* W,
                             const float* grad_out, int N, float4* gbuf, EdgeWindow win, int edge_split,
                             cudaStream_t s);
template <int KP, int MODE>
cudaError_t run_uvu_gradw(const DevPlan& P, const Tasks& T, const float* x, const float* xdot,
                          const float* pos, const float* posdot, const int* row_ptr,
                          const int* src, const float* grad_out, int N, int n_ranges,
                          float* partial, cudaStream_t s);
template <int KP, int MODE>
cudaError_t run_uvu_src(const DevPlan& P, const BlockPaths& BP, const Tasks& T, const float* pos,
                        const float* posdot, const int* t_ptr, const int* t_dst, const float* W,
                        const float* Wdot, const float* grad_out, int N, float* grad_x,
                        cudaStream_t s);

// kernel launchers (dispatch on K and mode; defined in launch.cu and k_misc.cu)
cudaError_t launch_gemm(GemmBatch& g, cudaStream_t s);     // tensor cores; fills tile0 / total_tiles
cudaError_t launch_gemm_tc(GemmBatch& g, int* err, cudaStream_t s);
int gemm_tiles(const GemmBatch& g);                             // output tiles of the tensor-core kernel
int* device_error_word();                                       // set by bounded waits that give up
cudaError_t read_and_clear_device_error(int* host_value);

cudaError_t launch_uvw_state(const DevPlan& P, const Tasks& T, int mode, const float* x,
                             const float* xdot, const float* pos, const float* posdot,
                             const int* row_ptr, const int* src, int node0, int n_nodes,
                             float* S, float* Sdot, cudaStream_t s);
// receiver backward, one lane per edge (phi_bar, Y_bar summed in registers): g_e of the
// window's edges into gbuf, or the edge-owned adjoints of the embedded interface
cudaError_t launch_uvw_recv_edge(const DevPlan& P, const float* x, const float* pos, const int* row_ptr,
                                 const int* src, const float* Sbar, int node0, int n_nodes, float4* gbuf,
                                 EdgeWindow win, int split, cudaStream_t s);
// double backward position gradient: per-edge tangent of g_e into gbuf (then pos_window)
cudaError_t launch_uvw_recv_dbl(const DevPlan& P, const Tasks& T, const float* x, const float* xdot,
                                const float* pos, const float* posdot, const int* row_ptr, const int* src,
                                const float* Sbar, const float* Sbard, int node0, int n_nodes, float4* gbuf,
                                EdgeWindow win, int edge_split, cudaStream_t s);
cudaError_t launch_uvu_recv_dbl(const DevPlan& P, const Tasks& T, const float* x, const float* xdot,
                                const float* pos, const float* posdot, const int* row_ptr, const int* src,
                                const float* W, const float* Wdot, const float* grad_out, int N, float4* gbuf,
                                EdgeWindow win, int edge_split, cudaStream_t s);
cudaError_t launch_uvw_src_state(const DevPlan& P, const Tasks& T, int mode,
                                 const float* pos, const float* posdot, const int* t_ptr,
                                 const int* t_eid, const int* t_dst, const float* grad_out,
                                 int node0, int n_nodes, float* X, float* Xdot,
                                 cudaStream_t s);
cudaError_t launch_uvu_fwd(const DevPlan& P, const BlockPaths& BP, const Tasks& T, int mode,
                           const float* x, const float* xdot, const float* pos,
                           const float* posdot, const int* row_ptr, const int* src,
                           const float* W, const float* Wdot, int N, float* out,
                           cudaStream_t s);
cudaError_t launch_uvu_recv_bwd(const DevPlan& P, const Tasks& T, const float* x,
                                const float* pos, const int* row_ptr, const int* src,
                                const float* W, const float* grad_out, int N, float4* gbuf,
                                EdgeWindow win, int edge_split, cudaStream_t s);
cudaError_t launch_uvu_gradw(const DevPlan& P, const Tasks& T, int mode, const float* x,
                             const float* xdot, const float* pos, const float* posdot,
                             const int* row_ptr, const int* src, const float* grad_out,
                             int N, int n_ranges, float* partial, cudaStream_t s);
cudaError_t launch_uvu_src(const DevPlan& P, const BlockPaths& BP, const Tasks& T, int mode,
                           const float* pos, const float* posdot, const int* t_ptr,
                           const int* t_eid, const int* t_dst, const float* W,
                           const float* Wdot, const float* grad_out, int N, float* grad_x,
                           cudaStream_t s);
cudaError_t launch_reduce_partials(const float* partial, int n_parts, long long n, float* out,
                                   int accumulate, cudaStream_t s);
// grad_pos[n] += sum_{e out of n, e in win} g_e - sum_{e into n, e in win} g_e; cursor [N]
// starts as a copy of t_ptr and is advanced window by window
cudaError_t launch_pos_window(int N, const int* row_ptr, const int* t_ptr, const int* t_eid,
                              const float4* gbuf, EdgeWindow win, int* cursor, float* grad_pos, cudaStream_t s);
cudaError_t launch_csr_transpose(int N, int E, const int* row_ptr, const int* src, int* t_ptr,
                                 int* t_eid, int* t_dst, int* cursor, cudaStream_t s);
cudaError_t launch_degree_order(int N, const int* row_ptr, int chunk, int* order, cudaStream_t s);

cudaError_t launch_layout_convert(int N, int dim, const LayoutMap& M, int to_ir_mul, const float* src,
                                  float* dst, cudaStream_t s);
cudaError_t launch_validate_graph(int N, int E, const int* row_ptr, const int* src, int* err,
                                  cudaStream_t s);

}  // namespace tpc
