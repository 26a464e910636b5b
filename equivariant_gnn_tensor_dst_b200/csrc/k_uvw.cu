// Fully connected (uvw) streaming kernels.
//
// Sobek: Streaming Equivariant Tensor Product Convolutions, section 4.
//  * k_uvw_state      -- receiver traversal building the state of eq. 33,
//                        S_{i,pi,q,u,mo} = sum_j phi_{ij,q} C_{pi,u,mo}(x_j, Y_ij),
//                        or (double backward) its directional derivative dS along
//                        (x_dot, pos_dot) as used in eq. 37/39.
//  * k_uvw_recv_bwd   -- receiver traversal differentiating eq. 33 given S_bar = m_bar A^T
//                        (eq. 36): per edge phi_bar (eq. 20) and Y_bar (eq. 22), carried
//                        to the edge vector r_e and staged per edge for the positions.
//  * k_uvw_recv_dbl   -- its tangent along (x_dot, pos_dot, A_dot): the position gradient
//                        of the double backward, through second derivatives of Y and phi.
//  * k_uvw_src_state  -- source traversal (source-contiguous CSR owns x_bar):
//                        X_{j,pi,q,w,mi} = sum_{e out of j} phi_{e,q} U_{e,pi,w,mi},
//                        U = adjoint of the coupling in x applied to m_bar of the
//                        receiver; then x_bar = X A^T (eq. 21) and A_bar = x^T X (eq. 19).
//
// One warp owns one (node, path, 32-channel chunk) task; lane = channel.  Edge
// geometry, harmonics and radial values are computed lane-per-edge for 32 edges at a
// time and broadcast through shared memory.  Per-lane state lives in registers and is
// written once to the caller's workspace; nothing is accumulated with atomics.
#include "common.cuh"

namespace tpc {

// Per-warp edge data in shared memory (dynamic: the tangent variant exceeds 48 KB).
template <int KP, bool TAN>
struct GeoSmem {
  static constexpr int WT = TAN ? WARPS_PER_CTA : 1;
  int j[WARPS_PER_CTA][32];
  alignas(16) float cy[WARPS_PER_CTA][32][CY_MAX];    // c_n * Y[my_n] per edge
  alignas(16) float phi[WARPS_PER_CTA][32][KP];
  alignas(16) float cyd[WT][32][CY_MAX];               // c_n * Y_dot[my_n] (tangent only)
  alignas(16) float phid[WT][32][KP];
};

// lane-per-edge preparation for one path: coupling products c*Y, radial values (and
// their tangents along r_dot)
template <int LI, int LS, int LO, int KP, bool TAN>
__device__ __forceinline__ void prep_edge(const DevPlan& P, const float* __restrict__ pos,
                                          const float* __restrict__ posdot, int i, int j,
                                          int store, int e, GeoSmem<KP, TAN>& sm, int w, int lane) {
  constexpr int RS = 2 * LS + 1;
  constexpr int N4 = CgInfo<LI, LS, LO>::n4;
  if (!TAN && P.emb_Y) {
    // embedded input: Y_e and phi_e of edge e as given
    float Y[RS], cy[4 * N4];
#pragma unroll
    for (int k = 0; k < RS; ++k) Y[k] = __ldg(P.emb_Y + (long long)e * P.n_sh + LS * LS + k);
    sm.j[w][lane] = store;
    cg_products<LI, LS, LO>(Y, cy);
#pragma unroll
    for (int b = 0; b < N4; ++b)
      reinterpret_cast<float4*>(sm.cy[w][lane])[b] = make_float4(cy[4 * b], cy[4 * b + 1], cy[4 * b + 2], cy[4 * b + 3]);
#pragma unroll
    for (int q = 0; q < KP; ++q) sm.phi[w][lane][q] = q < P.K ? __ldg(P.emb_phi + (long long)e * P.K + q) : 0.f;
    return;
  }
  const EdgeGeo g = edge_geo(pos, i, j);
  const Pow3 pw(g.ux, g.uy, g.uz);
  float Y[RS];
  sh_block<LS>(pw, Y);
  float phi[KP], dphi[KP];
  radial<KP, TAN>(P, g.d, phi, dphi);
  sm.j[w][lane] = store;
  float cy[4 * N4];
  cg_products<LI, LS, LO>(Y, cy);
#pragma unroll
  for (int b = 0; b < N4; ++b)
    reinterpret_cast<float4*>(sm.cy[w][lane])[b] = make_float4(cy[4 * b], cy[4 * b + 1], cy[4 * b + 2], cy[4 * b + 3]);
#pragma unroll
  for (int q = 0; q < KP; q += 4)
    reinterpret_cast<float4*>(sm.phi[w][lane])[q / 4] = make_float4(phi[q], phi[q + 1], phi[q + 2], phi[q + 3]);
  if (TAN) {
    float vx = 0.f, vy = 0.f, vz = 0.f;
    if (posdot) {
      vx = __ldg(posdot + 3 * j) - __ldg(posdot + 3 * i);
      vy = __ldg(posdot + 3 * j + 1) - __ldg(posdot + 3 * i + 1);
      vz = __ldg(posdot + 3 * j + 2) - __ldg(posdot + 3 * i + 2);
    }
    const float s = g.ux * vx + g.uy * vy + g.uz * vz;     // d|r| along r_dot
    const float tx = (vx - s * g.ux) * g.inv_d;            // d r_hat along r_dot
    const float ty = (vy - s * g.uy) * g.inv_d;
    const float tz = (vz - s * g.uz) * g.inv_d;
    float Yd[RS];
    sh_block_dir<LS>(pw, tx, ty, tz, Yd);
    cg_products<LI, LS, LO>(Yd, cy);
#pragma unroll
    for (int b = 0; b < N4; ++b)
      reinterpret_cast<float4*>(sm.cyd[w][lane])[b] = make_float4(cy[4 * b], cy[4 * b + 1], cy[4 * b + 2], cy[4 * b + 3]);
#pragma unroll
    for (int q = 0; q < KP; q += 4)
      reinterpret_cast<float4*>(sm.phid[w][lane])[q / 4] =
          make_float4(dphi[q] * s, dphi[q + 1] * s, dphi[q + 2] * s, dphi[q + 3] * s);
  }
}

// ---------------------------------------------------------------------------
// receiver state (eq. 33) and its tangent
// ---------------------------------------------------------------------------

// Resident CTAs per SM requested by the streaming kernels (register cap 65536 / (128 x
// blocks)), chosen per radial width KP and pass: the fewest registers that do not spill
// the KP x R accumulators (and their tangents in MODE 1), or that measured faster.
#define TPC_MINB_STATE (KP == 8 ? (MODE == 0 ? 5 : 3) : (MODE == 0 ? 3 : 2))
#define TPC_MINB_RECV (KP == 8 ? 4 : 3)

template <int LI, int LS, int LO, int KP, int MODE>
__device__ __forceinline__ void uvw_state_body(const DevPlan& P, const DevPath& p, int chunk, int i,
                                               int node_local, const float* __restrict__ x,
                                               const float* __restrict__ xdot,
                                               const float* __restrict__ pos,
                                               const float* __restrict__ posdot,
                                               const int* __restrict__ row_ptr,
                                               const int* __restrict__ src, float* S, float* Sd,
                                               GeoSmem<KP, MODE == 1>& sm) {
  constexpr int RI = 2 * LI + 1, RS = 2 * LS + 1, RO = 2 * LO + 1;
  constexpr bool TAN = MODE == 1;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = chunk * 32 + lane;
  const bool act = u < p.c_in;
  const float* xb = x + p.in_off + (act ? u : 0);
  const float* xdb = xdot ? xdot + p.in_off + (act ? u : 0) : nullptr;
  float acc[KP][RO], acc0[KP][RO];
#pragma unroll
  for (int q = 0; q < KP; ++q)
#pragma unroll
    for (int o = 0; o < RO; ++o) { acc[q][o] = 0.f; acc0[q][o] = 0.f; }

  const int eb = __ldg(row_ptr + i), ee = __ldg(row_ptr + i + 1);
  for (int e0 = eb; e0 < ee; e0 += 32) {
    const int ne = min(32, ee - e0);
    if (lane < ne) {
      const int j = __ldg(src + e0 + lane);
      prep_edge<LI, LS, LO, KP, TAN>(P, pos, posdot, i, j, j, e0 + lane, sm, w, lane);
    }
    __syncwarp();
    // x of the next edge is loaded while the current one is consumed
    float xn[RI], xdn[RI];
    {
      const long long row = (long long)sm.j[w][0] * P.dim_in;
#pragma unroll
      for (int m = 0; m < RI; ++m) {
        xn[m] = act ? __ldg(xb + row + m * p.c_in) : 0.f;
        xdn[m] = (TAN && xdb && act) ? __ldg(xdb + row + m * p.c_in) : 0.f;
      }
    }
    for (int t = 0; t < ne; ++t) {
      float xv[RI], xdv[RI];
#pragma unroll
      for (int m = 0; m < RI; ++m) { xv[m] = xn[m]; xdv[m] = xdn[m]; }
      if (t + 1 < ne) {
        const long long row = (long long)sm.j[w][t + 1] * P.dim_in;
#pragma unroll
        for (int m = 0; m < RI; ++m) {
          xn[m] = act ? __ldg(xb + row + m * p.c_in) : 0.f;
          if (TAN && xdb) xdn[m] = act ? __ldg(xdb + row + m * p.c_in) : 0.f;
        }
      }
      float phi[KP];
#pragma unroll
      for (int q = 0; q < KP; q += 4) {
        const float4 v = reinterpret_cast<const float4*>(sm.phi[w][t])[q / 4];
        phi[q] = v.x; phi[q + 1] = v.y; phi[q + 2] = v.z; phi[q + 3] = v.w;
      }
      float C[RO];
      cg_couple_cy<LI, LS, LO>(xv, sm.cy[w][t], C);
      if (!TAN) {
#pragma unroll
        for (int q = 0; q < KP; ++q)
#pragma unroll
          for (int o = 0; o < RO; ++o) acc[q][o] = fmaf(phi[q], C[o], acc[q][o]);
      } else {
        float phid[KP], Cd[RO], C2[RO];
#pragma unroll
        for (int q = 0; q < KP; q += 4) {
          const float4 v = reinterpret_cast<const float4*>(sm.phid[w][t])[q / 4];
          phid[q] = v.x; phid[q + 1] = v.y; phid[q + 2] = v.z; phid[q + 3] = v.w;
        }
        cg_couple_cy<LI, LS, LO>(xv, sm.cyd[w][t], Cd);
        if (xdb) {
          cg_couple_cy<LI, LS, LO>(xdv, sm.cy[w][t], C2);
#pragma unroll
          for (int o = 0; o < RO; ++o) Cd[o] += C2[o];
        }
#pragma unroll
        for (int q = 0; q < KP; ++q)
#pragma unroll
          for (int o = 0; o < RO; ++o) {
            acc[q][o] = fmaf(phid[q], C[o], fmaf(phi[q], Cd[o], acc[q][o]));
            acc0[q][o] = fmaf(phi[q], C[o], acc0[q][o]);
          }
      }
    }
    __syncwarp();
  }
  if (!act) return;
  const long long base = (long long)node_local * P.state_per_node + p.st_off + u;
  const int rs = P.K * p.c_in;
  float* out = TAN ? Sd : S;
#pragma unroll
  for (int o = 0; o < RO; ++o)
#pragma unroll
    for (int q = 0; q < KP; ++q)
      if (q < P.K) out[base + (long long)o * rs + q * p.c_in] = acc[q][o];
  if (TAN && S) {
#pragma unroll
    for (int o = 0; o < RO; ++o)
#pragma unroll
      for (int q = 0; q < KP; ++q)
        if (q < P.K) S[base + (long long)o * rs + q * p.c_in] = acc0[q][o];
  }
}

template <int KP, int MODE>
__global__ void __launch_bounds__(WARPS_PER_CTA * 32, TPC_MINB_STATE)
    k_uvw_state(DevPlan P, Tasks T, const float* __restrict__ x, const float* __restrict__ xdot,
                const float* __restrict__ pos, const float* __restrict__ posdot,
                const int* __restrict__ row_ptr, const int* __restrict__ src, int node0,
                int n_nodes, float* S, float* Sd) {
  extern __shared__ __align__(16) char dyn_smem[];
  GeoSmem<KP, MODE == 1>& sm = *reinterpret_cast<GeoSmem<KP, MODE == 1>*>(dyn_smem);
  // task-major order: co-resident warps run the same (l_in, l_sh, l_out) body, which keeps
  // the instruction working set small
  const long long gw = (long long)blockIdx.x * WARPS_PER_CTA + (threadIdx.x >> 5);
  const int task = (int)(gw / n_nodes);
  const int slot = (int)(gw % n_nodes);
  if (task >= T.n) return;
  const int node_local = P.order ? __ldg(P.order + node0 + slot) - node0 : slot;
  const DevPath& p = P.p[T.a[task]];
  const int chunk = T.b[task];
  const int i = node0 + node_local;
  dispatch_type(p.type, [&](auto tr) {
    using TR = decltype(tr);
    uvw_state_body<TR::li, TR::ls, TR::lo, KP, MODE>(P, p, chunk, i, node_local, x, xdot, pos,
                                                     posdot, row_ptr, src, S, Sd, sm);
  });
}

// ---------------------------------------------------------------------------
// receiver backward: phi_bar and Y_bar per edge -> d L / d r_e
// ---------------------------------------------------------------------------

template <int KP>
struct RecvSmem {
  int j[32];
  float Y[32][16];
  float phi[32][KP];
  float accY[WARPS_PER_CTA][32][16];   // per-warp partial sums, combined in warp order
  float accphi[WARPS_PER_CTA][32][KP];
};

template <int LI, int LS, int LO, int KP>
__device__ __forceinline__ void uvw_recv_body(const DevPlan& P, const DevPath& p, int chunk,
                                              int node_local, int ne,
                                              const float* __restrict__ x,
                                              const float* __restrict__ Sbar, RecvSmem<KP>& sm) {
  constexpr int RI = 2 * LI + 1, RS = 2 * LS + 1, RO = 2 * LO + 1;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = chunk * 32 + lane;
  const bool act = u < p.c_in;
  const float* xb = x + p.in_off + (act ? u : 0);
  float sb[KP][RO];
  {
    const long long base = (long long)node_local * P.state_per_node + p.st_off + u;
    const int rs = P.K * p.c_in;
#pragma unroll
    for (int o = 0; o < RO; ++o)
#pragma unroll
      for (int q = 0; q < KP; ++q)
        sb[q][o] = (act && q < P.K) ? Sbar[base + (long long)o * rs + q * p.c_in] : 0.f;
  }
  // Y_bar has RS components: reduce the next power of two of them
  constexpr int NY = RS <= 1 ? 1 : RS <= 2 ? 2 : RS <= 4 ? 4 : 8;
  const int yw = reduce_multi_index<NY>(lane), pw_ = reduce_multi_index<KP>(lane);
  const bool ywr = reduce_multi_writer<NY>(lane), pwr = reduce_multi_writer<KP>(lane);
  // x rows of the chunk's sources, one edge ahead of the arithmetic
  float xn[RI];
  {
    const long long row = (long long)sm.j[0] * P.dim_in;
#pragma unroll
    for (int m = 0; m < RI; ++m) xn[m] = act ? __ldg(xb + row + m * p.c_in) : 0.f;
  }
  for (int t = 0; t < ne; ++t) {
    float xv[RI];
#pragma unroll
    for (int m = 0; m < RI; ++m) xv[m] = xn[m];
    if (t + 1 < ne) {
      const long long row = (long long)sm.j[t + 1] * P.dim_in;
#pragma unroll
      for (int m = 0; m < RI; ++m) xn[m] = act ? __ldg(xb + row + m * p.c_in) : 0.f;
    }
    float Y[RS], phi[KP];
#pragma unroll
    for (int k = 0; k < RS; ++k) Y[k] = sm.Y[t][LS * LS + k];
#pragma unroll
    for (int q = 0; q < KP; ++q) phi[q] = sm.phi[t][q];
    float C[RO];
    cg_couple<LI, LS, LO>(xv, Y, C);
    float pp[KP];
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      float s = 0.f;
#pragma unroll
      for (int o = 0; o < RO; ++o) s = fmaf(sb[q][o], C[o], s);
      pp[q] = s;
    }
    float Tb[RO];
#pragma unroll
    for (int o = 0; o < RO; ++o) {
      float s = 0.f;
#pragma unroll
      for (int q = 0; q < KP; ++q) s = fmaf(phi[q], sb[q][o], s);
      Tb[o] = s;
    }
    float py[NY];
#pragma unroll
    for (int k = 0; k < NY; ++k) py[k] = 0.f;
    cg_adj_y<LI, LS, LO>(xv, Tb, py);
    const float rphi = warp_reduce_multi<KP>(pp);
    const float ry = warp_reduce_multi<NY>(py);
    if (pwr) sm.accphi[w][t][pw_] += rphi;
    if (ywr && yw < RS) sm.accY[w][t][LS * LS + yw] += ry;
    __syncwarp();
  }
}

// One CTA per (receiver, share of its 32-edge chunks); its warps split the (path,
// channel chunk) tasks and keep per-warp partial sums of phi_bar and Y_bar per edge,
// added in warp order.
template <int KP>
__global__ void __launch_bounds__(WARPS_PER_CTA * 32, TPC_MINB_RECV)
    k_uvw_recv_bwd(DevPlan P, Tasks T, const float* __restrict__ x, const float* __restrict__ pos,
                   const int* __restrict__ row_ptr, const int* __restrict__ src,
                   const float* __restrict__ Sbar, int node0, int n_nodes, float4* gbuf) {
  __shared__ RecvSmem<KP> sm;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if ((int)blockIdx.x >= n_nodes) return;
  const int node_local = P.order ? __ldg(P.order + node0 + blockIdx.x) - node0 : (int)blockIdx.x;
  const int i = node0 + node_local;
  const int eb = __ldg(row_ptr + i), ee = __ldg(row_ptr + i + 1);
  // the 32-edge chunks of one receiver are shared by gridDim.y CTAs (their per-edge
  // results are independent), which keeps high-degree receivers off the critical path
  for (int e0 = eb + 32 * blockIdx.y; e0 < ee; e0 += 32 * gridDim.y) {
    const int ne = min(32, ee - e0);
    if (w == 0 && lane < ne) {
      const int j = __ldg(src + e0 + lane);
      float Y[16], phi[KP], dphi[KP];
      if (P.emb_Y) {   // embedded input: Y_e and phi_e as given
        const long long e = e0 + lane;
#pragma unroll
        for (int k = 0; k < 16; ++k) Y[k] = k < P.n_sh ? __ldg(P.emb_Y + e * P.n_sh + k) : 0.f;
#pragma unroll
        for (int q = 0; q < KP; ++q) phi[q] = q < P.K ? __ldg(P.emb_phi + e * P.K + q) : 0.f;
      } else {
        const EdgeGeo g = edge_geo(pos, i, j);
        const Pow3 pw(g.ux, g.uy, g.uz);
        sh_all(pw, Y);
        radial<KP, false>(P, g.d, phi, dphi);
      }
      sm.j[lane] = j;
#pragma unroll
      for (int k = 0; k < 16; ++k) sm.Y[lane][k] = Y[k];
#pragma unroll
      for (int q = 0; q < KP; ++q) sm.phi[lane][q] = phi[q];
    }
    for (int k = threadIdx.x; k < WARPS_PER_CTA * 32 * 16; k += blockDim.x) (&sm.accY[0][0][0])[k] = 0.f;
    for (int k = threadIdx.x; k < WARPS_PER_CTA * 32 * KP; k += blockDim.x) (&sm.accphi[0][0][0])[k] = 0.f;
    __syncthreads();
    for (int task = w; task < T.n; task += WARPS_PER_CTA) {
      const DevPath& p = P.p[T.a[task]];
      const int chunk = T.b[task];
      dispatch_type(p.type, [&](auto tr) {
        using TR = decltype(tr);
        uvw_recv_body<TR::li, TR::ls, TR::lo, KP>(P, p, chunk, node_local, ne, x, Sbar, sm);
      });
    }
    __syncthreads();
    if (w == 0 && lane < ne && (P.emb_gY || P.emb_gphi)) {
      // embedded input: the edge-owned adjoints Y_bar (eq. 22) and phi_bar (eq. 20)
      const long long e = e0 + lane;
      if (P.emb_gY)
        for (int k = 0; k < P.n_sh; ++k) {
          float s = 0.f;
#pragma unroll
          for (int ww = 0; ww < WARPS_PER_CTA; ++ww) s += sm.accY[ww][lane][k];
          P.emb_gY[e * P.n_sh + k] = s;
        }
      if (P.emb_gphi)
        for (int q = 0; q < P.K; ++q) {
          float s = 0.f;
#pragma unroll
          for (int ww = 0; ww < WARPS_PER_CTA; ++ww) s += sm.accphi[ww][lane][q];
          P.emb_gphi[e * P.K + q] = s;
        }
    } else if (w == 0 && lane < ne) {
      const int j = sm.j[lane];
      const EdgeGeo g = edge_geo(pos, i, j);
      const Pow3 pw(g.ux, g.uy, g.uz);
      float phi[KP], dphi[KP], Yb[16];
      radial<KP, true>(P, g.d, phi, dphi);
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        float s = 0.f;
#pragma unroll
        for (int ww = 0; ww < WARPS_PER_CTA; ++ww) s += sm.accY[ww][lane][k];
        Yb[k] = s;
      }
      float vx = 0.f, vy = 0.f, vz = 0.f;
      sh_vjp_all(pw, Yb, vx, vy, vz);
      const float vr = vx * g.ux + vy * g.uy + vz * g.uz;
      float s = 0.f;
#pragma unroll
      for (int q = 0; q < KP; ++q) {
        float a = 0.f;
#pragma unroll
        for (int ww = 0; ww < WARPS_PER_CTA; ++ww) a += sm.accphi[ww][lane][q];
        s = fmaf(a, dphi[q], s);
      }
      float4 out;
      out.x = (vx - vr * g.ux) * g.inv_d + s * g.ux;
      out.y = (vy - vr * g.uy) * g.inv_d + s * g.uy;
      out.z = (vz - vr * g.uz) * g.inv_d + s * g.uz;
      out.w = 0.f;
      gbuf[e0 + lane] = out;
    }
    __syncthreads();
  }
}

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
                   float4* gbuf) {
  __shared__ RecvDblSmem<KP> sm;
  const int w = threadIdx.x >> 5;
  if ((int)blockIdx.x >= n_nodes) return;
  const int node_local = P.order ? __ldg(P.order + node0 + blockIdx.x) - node0 : (int)blockIdx.x;
  const int i = node0 + node_local;
  const int eb = __ldg(row_ptr + i), ee = __ldg(row_ptr + i + 1);
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
    recv_dbl_finish<KP>(P, pos, posdot, i, e0, ne, sm, gbuf);
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// source state X (and its tangent for the double backward)
// ---------------------------------------------------------------------------

template <int LI, int LS, int LO, int KP, int MODE>
__device__ __forceinline__ void uvw_src_body(const DevPlan& P, const DevPath& p, int chunk, int j,
                                             int node_local, const float* __restrict__ pos,
                                             const float* __restrict__ posdot,
                                             const int* __restrict__ t_ptr,
                                             const int* __restrict__ t_dst,
                                             const float* __restrict__ gout, float* X, float* Xd,
                                             GeoSmem<KP, MODE == 1>& sm) {
  constexpr int RI = 2 * LI + 1, RS = 2 * LS + 1, RO = 2 * LO + 1;
  constexpr bool TAN = MODE == 1;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = chunk * 32 + lane;
  const bool act = c < p.c_out;
  const float* gb = gout + p.out_off + (act ? c : 0);
  float acc[KP][RI], acc0[KP][RI];
#pragma unroll
  for (int q = 0; q < KP; ++q)
#pragma unroll
    for (int m = 0; m < RI; ++m) { acc[q][m] = 0.f; acc0[q][m] = 0.f; }
  const int kb = __ldg(t_ptr + j), ke = __ldg(t_ptr + j + 1);
  for (int k0 = kb; k0 < ke; k0 += 32) {
    const int ne = min(32, ke - k0);
    // edge j -> i seen from its source: r = pos[j] - pos[i]; keep the receiver index
    if (lane < ne) {
      const int i = __ldg(t_dst + k0 + lane);
      const int e = P.emb_eid ? __ldg(P.emb_eid + k0 + lane) : 0;
      prep_edge<LI, LS, LO, KP, TAN>(P, pos, posdot, i, j, i, e, sm, w, lane);
    }
    __syncwarp();
    float mn[RO];
    {
      const long long row = (long long)sm.j[w][0] * P.dim_out;
#pragma unroll
      for (int o = 0; o < RO; ++o) mn[o] = act ? __ldg(gb + row + o * p.c_out) : 0.f;
    }
    for (int t = 0; t < ne; ++t) {
      float mb[RO];
#pragma unroll
      for (int o = 0; o < RO; ++o) mb[o] = mn[o];
      if (t + 1 < ne) {
        const long long row = (long long)sm.j[w][t + 1] * P.dim_out;
#pragma unroll
        for (int o = 0; o < RO; ++o) mn[o] = act ? __ldg(gb + row + o * p.c_out) : 0.f;
      }
      float phi[KP];
#pragma unroll
      for (int q = 0; q < KP; q += 4) {
        const float4 v = reinterpret_cast<const float4*>(sm.phi[w][t])[q / 4];
        phi[q] = v.x; phi[q + 1] = v.y; phi[q + 2] = v.z; phi[q + 3] = v.w;
      }
      float U[RI];
      cg_adj_x_cy<LI, LS, LO>(sm.cy[w][t], mb, U);
      if (!TAN) {
#pragma unroll
        for (int q = 0; q < KP; ++q)
#pragma unroll
          for (int m = 0; m < RI; ++m) acc[q][m] = fmaf(phi[q], U[m], acc[q][m]);
      } else {
        float phid[KP], Ud[RI];
#pragma unroll
        for (int q = 0; q < KP; q += 4) {
          const float4 v = reinterpret_cast<const float4*>(sm.phid[w][t])[q / 4];
          phid[q] = v.x; phid[q + 1] = v.y; phid[q + 2] = v.z; phid[q + 3] = v.w;
        }
        cg_adj_x_cy<LI, LS, LO>(sm.cyd[w][t], mb, Ud);
#pragma unroll
        for (int q = 0; q < KP; ++q)
#pragma unroll
          for (int m = 0; m < RI; ++m) {
            acc[q][m] = fmaf(phid[q], U[m], fmaf(phi[q], Ud[m], acc[q][m]));
            acc0[q][m] = fmaf(phi[q], U[m], acc0[q][m]);
          }
      }
    }
    __syncwarp();
  }
  if (!act) return;
  const long long base = (long long)node_local * P.xstate_per_node + p.xst_off + c;
  const int rs = P.K * p.c_out;
  float* out = TAN ? Xd : X;
#pragma unroll
  for (int m = 0; m < RI; ++m)
#pragma unroll
    for (int q = 0; q < KP; ++q)
      if (q < P.K) out[base + (long long)m * rs + q * p.c_out] = acc[q][m];
  if (TAN && X) {
#pragma unroll
    for (int m = 0; m < RI; ++m)
#pragma unroll
      for (int q = 0; q < KP; ++q)
        if (q < P.K) X[base + (long long)m * rs + q * p.c_out] = acc0[q][m];
  }
}

template <int KP, int MODE>
__global__ void __launch_bounds__(WARPS_PER_CTA * 32, TPC_MINB_STATE)
    k_uvw_src_state(DevPlan P, Tasks T, const float* __restrict__ pos,
                    const float* __restrict__ posdot, const int* __restrict__ t_ptr,
                    const int* __restrict__ t_dst, const float* __restrict__ gout, int node0,
                    int n_nodes, float* X, float* Xd) {
  extern __shared__ __align__(16) char dyn_smem[];
  GeoSmem<KP, MODE == 1>& sm = *reinterpret_cast<GeoSmem<KP, MODE == 1>*>(dyn_smem);
  // task-major order: co-resident warps run the same (l_in, l_sh, l_out) body, which keeps
  // the instruction working set small
  const long long gw = (long long)blockIdx.x * WARPS_PER_CTA + (threadIdx.x >> 5);
  const int task = (int)(gw / n_nodes);
  const int node_local = (int)(gw % n_nodes);
  if (task >= T.n) return;
  const DevPath& p = P.p[T.a[task]];
  const int chunk = T.b[task];
  const int j = node0 + node_local;
  dispatch_type(p.type, [&](auto tr) {
    using TR = decltype(tr);
    uvw_src_body<TR::li, TR::ls, TR::lo, KP, MODE>(P, p, chunk, j, node_local, pos, posdot, t_ptr,
                                                   t_dst, gout, X, Xd, sm);
  });
}

// ---------------------------------------------------------------------------
// runners, explicitly instantiated per translation unit
// ---------------------------------------------------------------------------

static inline unsigned grid_for(long long warps) {
  return (unsigned)((warps + WARPS_PER_CTA - 1) / WARPS_PER_CTA);
}

template <int KP, int MODE>
cudaError_t run_uvw_state(const DevPlan& P, const Tasks& T, const float* x, const float* xdot,
                          const float* pos, const float* posdot, const int* row_ptr,
                          const int* src, int node0, int n_nodes, float* S, float* Sdot,
                          cudaStream_t s) {
  constexpr int smem = sizeof(GeoSmem<KP, MODE == 1>);
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_uvw_state<KP, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  k_uvw_state<KP, MODE><<<grid_for((long long)n_nodes * T.n), WARPS_PER_CTA * 32, smem, s>>>(
      P, T, x, xdot, pos, posdot, row_ptr, src, node0, n_nodes, S, Sdot);
  return cudaGetLastError();
}

template <int KP>
cudaError_t run_uvw_recv_bwd(const DevPlan& P, const Tasks& T, const float* x, const float* pos,
                             const int* row_ptr, const int* src, const float* Sbar, int node0,
                             int n_nodes, float4* gbuf, int edge_split, cudaStream_t s) {
  k_uvw_recv_bwd<KP><<<dim3((unsigned)n_nodes, (unsigned)edge_split), WARPS_PER_CTA * 32, 0, s>>>(P, T, x, pos, row_ptr, src,
                                                                     Sbar, node0, n_nodes, gbuf);
  return cudaGetLastError();
}

template <int KP, bool AD>
cudaError_t run_uvw_recv_dbl(const DevPlan& P, const Tasks& T, const float* x, const float* xdot,
                             const float* pos, const float* posdot, const int* row_ptr, const int* src,
                             const float* Sbar, const float* Sbard, int node0, int n_nodes, float4* gbuf,
                             int edge_split, cudaStream_t s) {
  k_uvw_recv_dbl<KP, AD><<<dim3((unsigned)n_nodes, (unsigned)edge_split), WARPS_PER_CTA * 32, 0, s>>>(
      P, T, x, xdot, pos, posdot, row_ptr, src, Sbar, AD ? Sbard : nullptr, node0, n_nodes, gbuf);
  return cudaGetLastError();
}

template <int KP, int MODE>
cudaError_t run_uvw_src_state(const DevPlan& P, const Tasks& T, const float* pos,
                              const float* posdot, const int* t_ptr, const int* t_dst,
                              const float* grad_out, int node0, int n_nodes, float* X,
                              float* Xdot, cudaStream_t s) {
  constexpr int smem = sizeof(GeoSmem<KP, MODE == 1>);
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_uvw_src_state<KP, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  k_uvw_src_state<KP, MODE><<<grid_for((long long)n_nodes * T.n), WARPS_PER_CTA * 32, smem, s>>>(
      P, T, pos, posdot, t_ptr, t_dst, grad_out, node0, n_nodes, X, Xdot);
  return cudaGetLastError();
}

#if defined(TPC_UNIT_KP) && defined(TPC_UNIT_MODE) && defined(TPC_UNIT_PART)
#define TPC_PART_STATE 1
#define TPC_PART_SRC 2
#define TPC_PART_RECV 3
#define TPC_PART_FWD 4
#define TPC_PART_GRADW 5
#if TPC_UNIT_PART == TPC_PART_STATE
template cudaError_t run_uvw_state<TPC_UNIT_KP, TPC_UNIT_MODE>(
    const DevPlan&, const Tasks&, const float*, const float*, const float*, const float*,
    const int*, const int*, int, int, float*, float*, cudaStream_t);
#endif
#if TPC_UNIT_PART == TPC_PART_SRC
template cudaError_t run_uvw_src_state<TPC_UNIT_KP, TPC_UNIT_MODE>(
    const DevPlan&, const Tasks&, const float*, const float*, const int*, const int*,
    const float*, int, int, float*, float*, cudaStream_t);
#endif
#if TPC_UNIT_PART == TPC_PART_RECV && TPC_UNIT_MODE == 0
template cudaError_t run_uvw_recv_bwd<TPC_UNIT_KP>(const DevPlan&, const Tasks&, const float*,
                                                   const float*, const int*, const int*,
                                                   const float*, int, int, float4*, int,
                                                   cudaStream_t);
#endif
#if TPC_UNIT_PART == TPC_PART_RECV && (TPC_UNIT_MODE == 1 || TPC_UNIT_MODE == 2)
template cudaError_t run_uvw_recv_dbl<TPC_UNIT_KP, TPC_UNIT_MODE == 2>(const DevPlan&, const Tasks&, const float*, const float*,
                                                   const float*, const float*, const int*, const int*,
                                                   const float*, const float*, int, int, float4*, int,
                                                   cudaStream_t);
#endif
#endif

}  // namespace tpc
