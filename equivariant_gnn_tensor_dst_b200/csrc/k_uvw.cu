// Fully connected (uvw) streaming kernels.
//
// Sobek: Streaming Equivariant Tensor Product Convolutions, section 4.
//  * k_uvw_state      -- receiver traversal building the state of eq. 33,
//                        S_{i,pi,q,u,mo} = sum_j phi_{ij,q} C_{pi,u,mo}(x_j, Y_ij),
//                        or (double backward) its directional derivative dS along
//                        (x_dot, pos_dot) as used in eq. 37/39.
//  * k_uvw_src_state  -- source traversal (source-contiguous CSR owns x_bar):
//                        X_{j,pi,q,w,mi} = sum_{e out of j} phi_{e,q} U_{e,pi,w,mi},
//                        U = adjoint of the coupling in x applied to m_bar of the
//                        receiver; then x_bar = X A^T (eq. 21) and A_bar = x^T X (eq. 19).
// (The receiver backward is k_recv_edge.cu; its tangent, k_uvw_dbl.cu.)
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

// SQ (primal pass, paths of at most 16 input channels): the two half-warps take the two
// halves of the radial index q for the same 16 channels, instead of leaving half of the
// lanes idle; each lane then keeps KP / 2 accumulators per output component.
template <int LI, int LS, int LO, int KP, int MODE, bool SQ>
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
  static_assert(!(SQ && TAN), "the radial split is for the primal pass");
  constexpr int KQ = SQ ? KP / 2 : KP;   // radial values per lane
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = SQ ? (lane >> 4) * KQ : 0;
  const int u = SQ ? (lane & 15) : chunk * 32 + lane;
  const bool act = u < p.c_in;
  const float* xb = x + p.in_off + (act ? u : 0);
  const float* xdb = xdot ? xdot + p.in_off + (act ? u : 0) : nullptr;
  float acc[KQ][RO], acc0[KQ][RO];
#pragma unroll
  for (int q = 0; q < KQ; ++q)
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
      float phi[KQ];
#pragma unroll
      for (int q = 0; q < KQ; q += 4) {
        const float4 v = reinterpret_cast<const float4*>(sm.phi[w][t] + q0)[q / 4];
        phi[q] = v.x; phi[q + 1] = v.y; phi[q + 2] = v.z; phi[q + 3] = v.w;
      }
      float C[RO];
      cg_couple_cy<LI, LS, LO>(xv, sm.cy[w][t], C);
      if constexpr (!TAN) {
#pragma unroll
        for (int q = 0; q < KQ; ++q)
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
    for (int q = 0; q < KQ; ++q)
      if (q0 + q < P.K) out[base + (long long)o * rs + (q0 + q) * p.c_in] = acc[q][o];
  if constexpr (TAN) {
    if (S) {
#pragma unroll
      for (int o = 0; o < RO; ++o)
#pragma unroll
        for (int q = 0; q < KP; ++q)
          if (q < P.K) S[base + (long long)o * rs + q * p.c_in] = acc0[q][o];
    }
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
  if constexpr (MODE == 0) {
    if (p.c_in <= 16) {
      dispatch_type(p.type, [&](auto tr) {
        using TR = decltype(tr);
        uvw_state_body<TR::li, TR::ls, TR::lo, KP, MODE, true>(P, p, chunk, i, node_local, x, xdot, pos,
                                                               posdot, row_ptr, src, S, Sd, sm);
      });
      return;
    }
  }
  dispatch_type(p.type, [&](auto tr) {
    using TR = decltype(tr);
    uvw_state_body<TR::li, TR::ls, TR::lo, KP, MODE, false>(P, p, chunk, i, node_local, x, xdot, pos,
                                                            posdot, row_ptr, src, S, Sd, sm);
  });
}

// ---------------------------------------------------------------------------
// source state X (and its tangent for the double backward)
// ---------------------------------------------------------------------------

// SQ: as for the receiver state, for paths of at most 16 output channels.
template <int LI, int LS, int LO, int KP, int MODE, bool SQ>
__device__ __forceinline__ void uvw_src_body(const DevPlan& P, const DevPath& p, int chunk, int j,
                                             int node_local, const float* __restrict__ pos,
                                             const float* __restrict__ posdot,
                                             const int* __restrict__ t_ptr,
                                             const int* __restrict__ t_dst,
                                             const float* __restrict__ gout, float* X, float* Xd,
                                             GeoSmem<KP, MODE == 1>& sm) {
  constexpr int RI = 2 * LI + 1, RS = 2 * LS + 1, RO = 2 * LO + 1;
  constexpr bool TAN = MODE == 1;
  static_assert(!(SQ && TAN), "the radial split is for the primal pass");
  constexpr int KQ = SQ ? KP / 2 : KP;   // radial values per lane
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = SQ ? (lane >> 4) * KQ : 0;
  const int c = SQ ? (lane & 15) : chunk * 32 + lane;
  const bool act = c < p.c_out;
  const float* gb = gout + p.out_off + (act ? c : 0);
  float acc[KQ][RI], acc0[KQ][RI];
#pragma unroll
  for (int q = 0; q < KQ; ++q)
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
      float phi[KQ];
#pragma unroll
      for (int q = 0; q < KQ; q += 4) {
        const float4 v = reinterpret_cast<const float4*>(sm.phi[w][t] + q0)[q / 4];
        phi[q] = v.x; phi[q + 1] = v.y; phi[q + 2] = v.z; phi[q + 3] = v.w;
      }
      float U[RI];
      cg_adj_x_cy<LI, LS, LO>(sm.cy[w][t], mb, U);
      if constexpr (!TAN) {
#pragma unroll
        for (int q = 0; q < KQ; ++q)
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
    for (int q = 0; q < KQ; ++q)
      if (q0 + q < P.K) out[base + (long long)m * rs + (q0 + q) * p.c_out] = acc[q][m];
  if constexpr (TAN) {
    if (X) {
#pragma unroll
      for (int m = 0; m < RI; ++m)
#pragma unroll
        for (int q = 0; q < KP; ++q)
          if (q < P.K) X[base + (long long)m * rs + q * p.c_out] = acc0[q][m];
    }
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
  if constexpr (MODE == 0) {
    if (p.c_out <= 16) {
      dispatch_type(p.type, [&](auto tr) {
        using TR = decltype(tr);
        uvw_src_body<TR::li, TR::ls, TR::lo, KP, MODE, true>(P, p, chunk, j, node_local, pos, posdot, t_ptr,
                                                             t_dst, gout, X, Xd, sm);
      });
      return;
    }
  }
  dispatch_type(p.type, [&](auto tr) {
    using TR = decltype(tr);
    uvw_src_body<TR::li, TR::ls, TR::lo, KP, MODE, false>(P, p, chunk, j, node_local, pos, posdot, t_ptr,
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

#endif

}  // namespace tpc
