// Double backward of the fully connected (uvw) convolution, position gradient.
//
// Sobek: Streaming Equivariant Tensor Product Convolutions, section 3 (eqs. 23-31) read
// through to positions: the tangent of the receiver backward (k_recv_edge.cu) along
// (x_dot, pos_dot, A_dot).  One CTA per (receiver, share of its 32-edge chunks); warps
// take the (path, 32-channel chunk) tasks, lane = channel; per-edge sums of the warps
// are added in warp order.  Compiled once per radial width and with / without the
// A_dot term (build units of their own: these are the slowest units to compile).
#include "common.cuh"

namespace tpc {

// ---------------------------------------------------------------------------
// double backward, position gradient: the tangent of the receiver backward along
// (x_dot, pos_dot, A_dot).  With S_bar = m_bar A^T and S_bar_dot = m_bar A_dot^T per
// receiver, each edge needs phi_bar, Y_bar and their tangents
//   phi_bar_dot_q = <S_bar_q, C(x_dot, Y) + C(x, Y_dot)> + <S_bar_dot_q, C(x, Y)>
//   Y_bar_dot     = D_Y C(x_dot)^T T_bar + D_Y C(x)^T T_bar_dot,
//   T_bar = sum_q phi_q S_bar_q,  T_bar_dot = sum_q (phi_dot_q S_bar_q + phi_q S_bar_dot_q),
// then the tangent of g_e (position_tangent), staged per edge like the backward's g_e.
// ---------------------------------------------------------------------------

#define TPC_MINB_RECV_DBL ((KP == 8 || !AD) ? 2 : 1)

template <int LI, int LS, int LO, int KP, bool AD>
__device__ __forceinline__ void uvw_recv_dbl_body(const DevPlan& P, const DevPath& p, int chunk,
                                                  int node_local, int ne,
                                                  const float* __restrict__ x,
                                                  const float* __restrict__ xdot,
                                                  const float* __restrict__ Sbar,
                                                  const float* __restrict__ Sbard,
                                                  RecvDblSmem<KP>& sm) {
  constexpr int RI = 2 * LI + 1, RS = 2 * LS + 1, RO = 2 * LO + 1;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = chunk * 32 + lane;
  const bool act = u < p.c_in;
  const float* xb = x + p.in_off + (act ? u : 0);
  const bool XD = xdot != nullptr;   // warp-uniform: the x_dot terms are skipped when absent
  const float* xdb = XD ? xdot + p.in_off + (act ? u : 0) : nullptr;
  float sb[KP][RO], sbd[AD ? KP : 1][RO];
  {
    const long long base = (long long)node_local * P.state_per_node + p.st_off + u;
    const int rs = P.K * p.c_in;
#pragma unroll
    for (int o = 0; o < RO; ++o)
#pragma unroll
      for (int q = 0; q < KP; ++q) {
        const bool ok = act && q < P.K;
        sb[q][o] = ok ? Sbar[base + (long long)o * rs + q * p.c_in] : 0.f;
        if constexpr (AD) sbd[q][o] = ok ? Sbard[base + (long long)o * rs + q * p.c_in] : 0.f;
      }
  }
  constexpr int NY = RS <= 1 ? 1 : RS <= 2 ? 2 : RS <= 4 ? 4 : 8;
  const int yw = reduce_multi_index<NY>(lane), pw_ = reduce_multi_index<KP>(lane);
  const bool ywr = reduce_multi_writer<NY>(lane), pwr = reduce_multi_writer<KP>(lane);
  for (int t = 0; t < ne; ++t) {
    const long long row = (long long)sm.j[t] * P.dim_in;
    float xv[RI], xdv[RI];
#pragma unroll
    for (int m = 0; m < RI; ++m) xv[m] = act ? __ldg(xb + row + m * p.c_in) : 0.f;
    if (XD) {
#pragma unroll
      for (int m = 0; m < RI; ++m) xdv[m] = act ? __ldg(xdb + row + m * p.c_in) : 0.f;
    }
    float Y[RS], Yd[RS], phi[KP], phid[KP];
#pragma unroll
    for (int k = 0; k < RS; ++k) {
      Y[k] = sm.Y[t][LS * LS + k];
      Yd[k] = sm.Yd[t][LS * LS + k];
    }
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      phi[q] = sm.phi[t][q];
      phid[q] = sm.phid[t][q];
    }
    float C[RO], Cd[RO];
    cg_couple<LI, LS, LO>(xv, Y, C);
    cg_couple<LI, LS, LO>(xv, Yd, Cd);
    if (XD) {
      float Ct[RO];
      cg_couple<LI, LS, LO>(xdv, Y, Ct);
#pragma unroll
      for (int o = 0; o < RO; ++o) Cd[o] += Ct[o];
    }
    float pp[KP], ppd[KP];
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      float a = 0.f, b = 0.f;
#pragma unroll
      for (int o = 0; o < RO; ++o) {
        a = fmaf(sb[q][o], C[o], a);
        b = fmaf(sb[q][o], Cd[o], b);
        if constexpr (AD) b = fmaf(sbd[q][o], C[o], b);
      }
      pp[q] = a;
      ppd[q] = b;
    }
    float Tb[RO], Tbd[RO];
#pragma unroll
    for (int o = 0; o < RO; ++o) {
      float a = 0.f, b = 0.f;
#pragma unroll
      for (int q = 0; q < KP; ++q) {
        a = fmaf(phi[q], sb[q][o], a);
        b = fmaf(phid[q], sb[q][o], b);
        if constexpr (AD) b = fmaf(phi[q], sbd[q][o], b);
      }
      Tb[o] = a;
      Tbd[o] = b;
    }
    float py[NY], pyd[NY];
#pragma unroll
    for (int k = 0; k < NY; ++k) {
      py[k] = 0.f;
      pyd[k] = 0.f;
    }
    cg_adj_y<LI, LS, LO>(xv, Tb, py);
    cg_adj_y<LI, LS, LO>(xv, Tbd, pyd);
    if (XD) cg_adj_y<LI, LS, LO>(xdv, Tb, pyd);
    const float rphi = warp_reduce_multi<KP>(pp);
    const float rphid = warp_reduce_multi<KP>(ppd);
    const float ry = warp_reduce_multi<NY>(py);
    const float ryd = warp_reduce_multi<NY>(pyd);
    if (pwr) {
      sm.accphi[w][t][pw_] += rphi;
      sm.accphid[w][t][pw_] += rphid;
    }
    if (ywr && yw < RS) {
      sm.accY[w][t][LS * LS + yw] += ry;
      sm.accYd[w][t][LS * LS + yw] += ryd;
    }
    __syncwarp();
  }
}

// Same grid as k_uvw_recv_bwd: one CTA per (receiver, share of its 32-edge chunks).
// AD: an A_dot tangent is present (S_bar_dot is read); without it those terms are zero.
template <int KP, bool AD>
__global__ void __launch_bounds__(WARPS_PER_CTA * 32, TPC_MINB_RECV_DBL)
    k_uvw_recv_dbl(DevPlan P, Tasks T, const float* __restrict__ x, const float* __restrict__ xdot,
                   const float* __restrict__ pos, const float* __restrict__ posdot,
                   const int* __restrict__ row_ptr, const int* __restrict__ src,
                   const float* __restrict__ Sbar, const float* __restrict__ Sbard, int node0, int n_nodes,
                   float4* gbuf, EdgeWindow win) {
  __shared__ RecvDblSmem<KP> sm;
  const int w = threadIdx.x >> 5;
  if ((int)blockIdx.x >= n_nodes) return;
  const int node_local = P.order ? __ldg(P.order + node0 + blockIdx.x) - node0 : (int)blockIdx.x;
  const int i = node0 + node_local;
  int w0, w1;
  window_bounds(row_ptr, win, w0, w1);
  const int eb = max(__ldg(row_ptr + i), w0), ee = min(__ldg(row_ptr + i + 1), w1);
  for (int e0 = eb + 32 * blockIdx.y; e0 < ee; e0 += 32 * gridDim.y) {
    const int ne = min(32, ee - e0);
    recv_dbl_prep<KP>(P, pos, posdot, src, i, e0, ne, sm);
    __syncthreads();
    for (int task = w; task < T.n; task += WARPS_PER_CTA) {
      const DevPath& p = P.p[T.a[task]];
      const int chunk = T.b[task];
      dispatch_type(p.type, [&](auto tr) {
        using TR = decltype(tr);
        uvw_recv_dbl_body<TR::li, TR::ls, TR::lo, KP, AD>(P, p, chunk, node_local, ne, x, xdot, Sbar, Sbard, sm);
      });
    }
    __syncthreads();
    recv_dbl_finish<KP>(P, pos, posdot, i, e0, ne, sm, gbuf, w0);
    __syncthreads();
  }
}

template <int KP, bool AD>
cudaError_t run_uvw_recv_dbl(const DevPlan& P, const Tasks& T, const float* x, const float* xdot,
                             const float* pos, const float* posdot, const int* row_ptr, const int* src,
                             const float* Sbar, const float* Sbard, int node0, int n_nodes, float4* gbuf,
                             EdgeWindow win, int edge_split, cudaStream_t s) {
  k_uvw_recv_dbl<KP, AD><<<dim3((unsigned)n_nodes, (unsigned)edge_split), WARPS_PER_CTA * 32, 0, s>>>(
      P, T, x, xdot, pos, posdot, row_ptr, src, Sbar, AD ? Sbard : nullptr, node0, n_nodes, gbuf, win);
  return cudaGetLastError();
}


#if defined(TPC_UNIT_KP) && defined(TPC_UNIT_MODE) && (TPC_UNIT_MODE == 1 || TPC_UNIT_MODE == 2)
template cudaError_t run_uvw_recv_dbl<TPC_UNIT_KP, TPC_UNIT_MODE == 2>(const DevPlan&, const Tasks&, const float*, const float*,
                                                   const float*, const float*, const int*, const int*,
                                                   const float*, const float*, int, int, float4*, EdgeWindow, int,
                                                   cudaStream_t);
#endif

}  // namespace tpc
