// Double backward of the channelwise (uvu) convolution, position gradient.
//
// Sobek: Streaming Equivariant Tensor Product Convolutions, section 3 (eqs. 23-31) read
// through to positions: the tangent of the uvu receiver backward along (x_dot, pos_dot,
// A_dot), with the edge weight w = phi . a formed in registers.  Compiled once per radial
// width and with / without the A_dot term (build units of their own).
#include "common.cuh"

namespace tpc {

// ---------------------------------------------------------------------------
// double backward, position gradient: the tangent of the receiver backward along
// (x_dot, pos_dot, A_dot).  Per channel u of path pi, with a = A_{., pi, u}:
//   h = <m_bar, C(x, Y)>,   h_dot = <m_bar, C(x_dot, Y) + C(x, Y_dot)>         (eqs. 18, 26)
//   phi_bar_dot_q = a_q h_dot + a_dot_q h                                      (eq. 20)
//   Y_bar_dot = D_Y C(x_dot)^T (w m_bar) + D_Y C(x)^T (w_dot m_bar)            (eq. 22)
// with w = phi . a and w_dot = phi_dot . a + phi . a_dot (eq. 23); then the tangent of
// g_e per edge (position_tangent).
// ---------------------------------------------------------------------------

template <int LI, int LS, int LO, int KP, bool AD>
__device__ __forceinline__ void uvu_recv_dbl_body(const DevPlan& P, const DevPath& p, int chunk, int i,
                                                  int ne, const float* __restrict__ x,
                                                  const float* __restrict__ xdot,
                                                  const float* __restrict__ W,
                                                  const float* __restrict__ Wdot,
                                                  const float* __restrict__ gout, RecvDblSmem<KP>& sm) {
  constexpr int RI = 2 * LI + 1, RS = 2 * LS + 1, RO = 2 * LO + 1;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = chunk * 32 + lane;
  const bool act = u < p.c_in;
  float a[KP], ad[AD ? KP : 1], mb[RO];
#pragma unroll
  for (int q = 0; q < KP; ++q) {
    const bool ok = act && q < P.K;
    a[q] = ok ? __ldg(W + (long long)q * P.n_w + p.w_off + u) : 0.f;
    if constexpr (AD) ad[q] = ok ? __ldg(Wdot + (long long)q * P.n_w + p.w_off + u) : 0.f;
  }
#pragma unroll
  for (int o = 0; o < RO; ++o)
    mb[o] = act ? __ldg(gout + (long long)i * P.dim_out + p.out_off + o * p.c_out + u) : 0.f;
  const float* xb = x + p.in_off + (act ? u : 0);
  const bool XD = xdot != nullptr;   // warp-uniform: the x_dot terms are skipped when absent
  const float* xdb = XD ? xdot + p.in_off + (act ? u : 0) : nullptr;
  constexpr int NY = RS <= 1 ? 1 : RS <= 2 ? 2 : RS <= 4 ? 4 : 8;
  const int yw = reduce_multi_index<NY>(lane), pw_ = reduce_multi_index<KP>(lane);
  const bool ywr = reduce_multi_writer<NY>(lane), pwr = reduce_multi_writer<KP>(lane);
  for (int t = 0; t < ne; ++t) {
    const long long row = (long long)sm.j[t] * P.dim_in;
    float xv[RI], xdv[RI], Y[RS], Yd[RS];
#pragma unroll
    for (int k = 0; k < RI; ++k) xv[k] = act ? __ldg(xb + row + k * p.c_in) : 0.f;
    if (XD) {
#pragma unroll
      for (int k = 0; k < RI; ++k) xdv[k] = act ? __ldg(xdb + row + k * p.c_in) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < RS; ++k) {
      Y[k] = sm.Y[t][LS * LS + k];
      Yd[k] = sm.Yd[t][LS * LS + k];
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
    float h = 0.f, hd = 0.f;
#pragma unroll
    for (int o = 0; o < RO; ++o) {
      h = fmaf(mb[o], C[o], h);
      hd = fmaf(mb[o], Cd[o], hd);
    }
    float we = 0.f, wed = 0.f;
    float pp[KP], ppd[KP];
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      const float ph = sm.phi[t][q], phd = sm.phid[t][q];
      we = fmaf(ph, a[q], we);
      wed = fmaf(phd, a[q], wed);
      pp[q] = a[q] * h;
      ppd[q] = a[q] * hd;
      if constexpr (AD) {
        wed = fmaf(ph, ad[q], wed);
        ppd[q] = fmaf(ad[q], h, ppd[q]);
      }
    }
    float G[RO], Gd[RO], py[NY], pyd[NY];
#pragma unroll
    for (int o = 0; o < RO; ++o) {
      G[o] = mb[o] * we;
      Gd[o] = mb[o] * wed;
    }
#pragma unroll
    for (int k = 0; k < NY; ++k) {
      py[k] = 0.f;
      pyd[k] = 0.f;
    }
    cg_adj_y<LI, LS, LO>(xv, G, py);
    cg_adj_y<LI, LS, LO>(xv, Gd, pyd);
    if (XD) cg_adj_y<LI, LS, LO>(xdv, G, pyd);
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

// Same grid as k_uvu_recv_bwd: one CTA per (receiver, share of its 32-edge chunks).
// AD: an A_dot tangent is present; without it those terms are zero.
template <int KP, bool AD>
__global__ void __launch_bounds__(WARPS_PER_CTA * 32, 2)
    k_uvu_recv_dbl(DevPlan P, Tasks T, const float* __restrict__ x, const float* __restrict__ xdot,
                   const float* __restrict__ pos, const float* __restrict__ posdot,
                   const int* __restrict__ row_ptr, const int* __restrict__ src,
                   const float* __restrict__ W, const float* __restrict__ Wdot,
                   const float* __restrict__ gout, int N, float4* gbuf, EdgeWindow win) {
  __shared__ RecvDblSmem<KP> sm;
  const int w = threadIdx.x >> 5;
  const int i = blockIdx.x;
  if (i >= N) return;
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
        uvu_recv_dbl_body<TR::li, TR::ls, TR::lo, KP, AD>(P, p, chunk, i, ne, x, xdot, W, Wdot, gout, sm);
      });
    }
    __syncthreads();
    recv_dbl_finish<KP>(P, pos, posdot, i, e0, ne, sm, gbuf, w0);
    __syncthreads();
  }
}

template <int KP, bool AD>
cudaError_t run_uvu_recv_dbl(const DevPlan& P, const Tasks& T, const float* x, const float* xdot,
                             const float* pos, const float* posdot, const int* row_ptr, const int* src,
                             const float* W, const float* Wdot, const float* grad_out, int N, float4* gbuf,
                             EdgeWindow win, int edge_split, cudaStream_t s) {
  k_uvu_recv_dbl<KP, AD><<<dim3((unsigned)N, (unsigned)edge_split), WARPS_PER_CTA * 32, 0, s>>>(
      P, T, x, xdot, pos, posdot, row_ptr, src, W, AD ? Wdot : nullptr, grad_out, N, gbuf, win);
  return cudaGetLastError();
}


#if defined(TPC_UNIT_KP) && defined(TPC_UNIT_MODE) && (TPC_UNIT_MODE == 1 || TPC_UNIT_MODE == 2)
template cudaError_t run_uvu_recv_dbl<TPC_UNIT_KP, TPC_UNIT_MODE == 2>(const DevPlan&, const Tasks&, const float*, const float*,
                                                   const float*, const float*, const int*, const int*,
                                                   const float*, const float*, const float*, int, float4*,
                                                   EdgeWindow, int, cudaStream_t);
#endif

}  // namespace tpc
