// Channelwise (uvu) streaming kernels.
//
// Sobek: Streaming Equivariant Tensor Product Convolutions, eq. 7 (uvu ties the output
// channel to the input channel) and section 4, which builds channelwise products as a
// kernel of their own rather than as a masked fully connected one, with no per-edge
// workspace.  With one weight per (path, channel), the edge weight
// w_{e,pi,u} = sum_q phi_q A_{q,pi,u} (eq. 17) is formed in registers and consumed at
// once; there is no receiver state and no channel GEMM.
//
//  * k_uvu_fwd      -- m_i (eq. 11), or its tangent m_dot (eq. 25) for the double backward
//  * k_uvu_recv_bwd -- per edge phi_bar (eq. 20) and Y_bar (eq. 22) -> d L / d r_e
//  * k_uvu_gradw    -- A_bar (eq. 19), or its directional derivative (eq. 27), as
//                      deterministic per-receiver-range partials
//  * k_uvu_src      -- x_bar (eq. 21), or eq. 30, owned by the source CSR
// (The tangent of the receiver backward, for the double backward's position gradient,
// is k_uvu_dbl.cu.)
#include "common.cuh"

namespace tpc {

template <int KP>
struct USmem {
  int j[WARPS_PER_CTA][32];
  float Y[WARPS_PER_CTA][32][8];
  float phi[WARPS_PER_CTA][32][KP];
  float Yd[WARPS_PER_CTA][32][8];
  float phid[WARPS_PER_CTA][32][KP];
};

template <int LS, int KP, bool TAN>
__device__ __forceinline__ void uprep(const DevPlan& P, const float* __restrict__ pos,
                                      const float* __restrict__ posdot, int i, int j, int store, int e,
                                      USmem<KP>& sm, int w, int lane) {
  constexpr int RS = 2 * LS + 1;
  if (!TAN && P.emb_Y) {
    // embedded input: Y_e and phi_e of edge e as given
    sm.j[w][lane] = store;
#pragma unroll
    for (int k = 0; k < RS; ++k) sm.Y[w][lane][k] = __ldg(P.emb_Y + (long long)e * P.n_sh + LS * LS + k);
#pragma unroll
    for (int q = 0; q < KP; ++q) sm.phi[w][lane][q] = q < P.K ? __ldg(P.emb_phi + (long long)e * P.K + q) : 0.f;
    return;
  }
  const EdgeGeo g = edge_geo(pos, i, j);
  const Pow3 pw(g.ux, g.uy, g.uz);
  float Y[RS], phi[KP], dphi[KP];
  sh_block<LS>(pw, Y);
  radial<KP, TAN>(P, g.d, phi, dphi);
  sm.j[w][lane] = store;
#pragma unroll
  for (int k = 0; k < RS; ++k) sm.Y[w][lane][k] = Y[k];
#pragma unroll
  for (int q = 0; q < KP; ++q) sm.phi[w][lane][q] = phi[q];
  if (TAN) {
    float vx = 0.f, vy = 0.f, vz = 0.f;
    if (posdot) {
      vx = __ldg(posdot + 3 * j) - __ldg(posdot + 3 * i);
      vy = __ldg(posdot + 3 * j + 1) - __ldg(posdot + 3 * i + 1);
      vz = __ldg(posdot + 3 * j + 2) - __ldg(posdot + 3 * i + 2);
    }
    const float s = g.ux * vx + g.uy * vy + g.uz * vz;
    const float tx = (vx - s * g.ux) * g.inv_d, ty = (vy - s * g.uy) * g.inv_d,
                tz = (vz - s * g.uz) * g.inv_d;
    float Yd[RS];
    sh_block_dir<LS>(pw, tx, ty, tz, Yd);
#pragma unroll
    for (int k = 0; k < RS; ++k) sm.Yd[w][lane][k] = Yd[k];
#pragma unroll
    for (int q = 0; q < KP; ++q) sm.phid[w][lane][q] = dphi[q] * s;
  }
}

// ---------------------------------------------------------------------------
// forward (MODE 0) and forward tangent (MODE 1)
// ---------------------------------------------------------------------------

template <int LI, int LS, int LO, int KP, int MODE>
__device__ __forceinline__ void uvu_fwd_body(const DevPlan& P, const DevPath& p, int u, bool act,
                                             int i, const float* __restrict__ x,
                                             const float* __restrict__ xdot,
                                             const float* __restrict__ pos,
                                             const float* __restrict__ posdot,
                                             const int* __restrict__ row_ptr,
                                             const int* __restrict__ src,
                                             const float* __restrict__ W,
                                             const float* __restrict__ Wdot, float* m,
                                             USmem<KP>& sm) {
  constexpr int RI = 2 * LI + 1, RS = 2 * LS + 1, RO = 2 * LO + 1;
  constexpr bool TAN = MODE == 1;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float a[KP], ad[KP];
#pragma unroll
  for (int q = 0; q < KP; ++q) {
    a[q] = (act && q < P.K) ? __ldg(W + (long long)q * P.n_w + p.w_off + u) : 0.f;
    ad[q] = (TAN && Wdot && act && q < P.K) ? __ldg(Wdot + (long long)q * P.n_w + p.w_off + u) : 0.f;
  }
  const float* xb = x + p.in_off + (act ? u : 0);
  const float* xdb = xdot ? xdot + p.in_off + (act ? u : 0) : nullptr;
  const int eb = __ldg(row_ptr + i), ee = __ldg(row_ptr + i + 1);
  for (int e0 = eb; e0 < ee; e0 += 32) {
    const int ne = min(32, ee - e0);
    if (lane < ne) {
      const int j = __ldg(src + e0 + lane);
      uprep<LS, KP, TAN>(P, pos, posdot, i, j, j, e0 + lane, sm, w, lane);
    }
    __syncwarp();
    for (int t = 0; t < ne; ++t) {
      const long long row = (long long)sm.j[w][t] * P.dim_in;
      float xv[RI], Y[RS], C[RO];
#pragma unroll
      for (int k = 0; k < RI; ++k) xv[k] = act ? __ldg(xb + row + k * p.c_in) : 0.f;
#pragma unroll
      for (int k = 0; k < RS; ++k) Y[k] = sm.Y[w][t][k];
      float we = 0.f;
#pragma unroll
      for (int q = 0; q < KP; ++q) we = fmaf(sm.phi[w][t][q], a[q], we);
      cg_couple<LI, LS, LO>(xv, Y, C);
      if (!TAN) {
#pragma unroll
        for (int o = 0; o < RO; ++o) m[o] = fmaf(we, C[o], m[o]);
      } else {
        float Yd[RS], Cd[RO], C2[RO];
        float wd = 0.f;
#pragma unroll
        for (int q = 0; q < KP; ++q) wd = fmaf(sm.phid[w][t][q], a[q], fmaf(sm.phi[w][t][q], ad[q], wd));
#pragma unroll
        for (int k = 0; k < RS; ++k) Yd[k] = sm.Yd[w][t][k];
        cg_couple<LI, LS, LO>(xv, Yd, Cd);
        if (xdb) {
          float xdv[RI];
#pragma unroll
          for (int k = 0; k < RI; ++k) xdv[k] = act ? __ldg(xdb + row + k * p.c_in) : 0.f;
          cg_couple<LI, LS, LO>(xdv, Y, C2);
#pragma unroll
          for (int o = 0; o < RO; ++o) Cd[o] += C2[o];
        }
#pragma unroll
        for (int o = 0; o < RO; ++o) m[o] = fmaf(wd, C[o], fmaf(we, Cd[o], m[o]));
      }
    }
    __syncwarp();
  }
}

template <int KP, int MODE>
__global__ void __launch_bounds__(WARPS_PER_CTA * 32)
    k_uvu_fwd(DevPlan P, BlockPaths BP, Tasks T, const float* __restrict__ x,
              const float* __restrict__ xdot, const float* __restrict__ pos,
              const float* __restrict__ posdot, const int* __restrict__ row_ptr,
              const int* __restrict__ src, const float* __restrict__ W,
              const float* __restrict__ Wdot, int N, float* out) {
  __shared__ USmem<KP> sm;
  const long long gw = (long long)blockIdx.x * WARPS_PER_CTA + (threadIdx.x >> 5);
  const int task = (int)(gw / N);   // task-major: co-resident warps share code
  const int i = (int)(gw % N);
  if (task >= T.n) return;
  const int bo = T.a[task];
  const int lane = threadIdx.x & 31;
  const int u = T.b[task] * 32 + lane;
  const int c = BP.c[bo];
  const bool act = u < c;
  float m[7];
#pragma unroll
  for (int o = 0; o < 7; ++o) m[o] = 0.f;
  for (int k = 0; k < BP.count[bo]; ++k) {
    const DevPath& p = P.p[BP.list[bo][k]];
    dispatch_type(p.type, [&](auto tr) {
      using TR = decltype(tr);
      uvu_fwd_body<TR::li, TR::ls, TR::lo, KP, MODE>(P, p, u, act, i, x, xdot, pos, posdot, row_ptr,
                                                     src, W, Wdot, m, sm);
    });
  }
  if (!act) return;
  const int ro = 2 * BP.l[bo] + 1;
  float* dst = out + (long long)i * P.dim_out + BP.off[bo] + u;
#pragma unroll
  for (int o = 0; o < 7; ++o)
    if (o < ro) dst[o * c] = m[o];
}

// ---------------------------------------------------------------------------
// receiver backward: phi_bar, Y_bar -> d L / d r_e
// ---------------------------------------------------------------------------

template <int KP>
struct URecvSmem {
  int j[32];
  float Y[32][16];
  float phi[32][KP];
  float accY[WARPS_PER_CTA][32][16];   // per-warp partial sums, combined in warp order
  float accphi[WARPS_PER_CTA][32][KP];
};

template <int LI, int LS, int LO, int KP>
__device__ __forceinline__ void uvu_recv_body(const DevPlan& P, const DevPath& p, int chunk, int i,
                                              int ne, const float* __restrict__ x,
                                              const float* __restrict__ W,
                                              const float* __restrict__ gout,
                                              URecvSmem<KP>& sm) {
  constexpr int RI = 2 * LI + 1, RS = 2 * LS + 1, RO = 2 * LO + 1;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = chunk * 32 + lane;
  const bool act = u < p.c_in;
  float a[KP], mb[RO];
#pragma unroll
  for (int q = 0; q < KP; ++q) a[q] = (act && q < P.K) ? __ldg(W + (long long)q * P.n_w + p.w_off + u) : 0.f;
#pragma unroll
  for (int o = 0; o < RO; ++o)
    mb[o] = act ? __ldg(gout + (long long)i * P.dim_out + p.out_off + o * p.c_out + u) : 0.f;
  const float* xb = x + p.in_off + (act ? u : 0);
  // Y_bar has RS components: reduce the next power of two of them
  constexpr int NY = RS <= 1 ? 1 : RS <= 2 ? 2 : RS <= 4 ? 4 : 8;
  const int yw = reduce_multi_index<NY>(lane), pw_ = reduce_multi_index<KP>(lane);
  const bool ywr = reduce_multi_writer<NY>(lane), pwr = reduce_multi_writer<KP>(lane);
  // x rows of the chunk's sources, one edge ahead of the arithmetic
  float xn[RI];
  {
    const long long row = (long long)sm.j[0] * P.dim_in;
#pragma unroll
    for (int k = 0; k < RI; ++k) xn[k] = act ? __ldg(xb + row + k * p.c_in) : 0.f;
  }
  for (int t = 0; t < ne; ++t) {
    float xv[RI], Y[RS], C[RO];
#pragma unroll
    for (int k = 0; k < RI; ++k) xv[k] = xn[k];
    if (t + 1 < ne) {
      const long long row = (long long)sm.j[t + 1] * P.dim_in;
#pragma unroll
      for (int k = 0; k < RI; ++k) xn[k] = act ? __ldg(xb + row + k * p.c_in) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < RS; ++k) Y[k] = sm.Y[t][LS * LS + k];
    cg_couple<LI, LS, LO>(xv, Y, C);
    float h = 0.f;
#pragma unroll
    for (int o = 0; o < RO; ++o) h = fmaf(mb[o], C[o], h);   // eq. 18
    float we = 0.f;
    float pp[KP];
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      we = fmaf(sm.phi[t][q], a[q], we);
      pp[q] = a[q] * h;                                        // eq. 20 (per channel)
    }
    float G[RO], py[NY];
#pragma unroll
    for (int o = 0; o < RO; ++o) G[o] = mb[o] * we;
#pragma unroll
    for (int k = 0; k < NY; ++k) py[k] = 0.f;
    cg_adj_y<LI, LS, LO>(xv, G, py);                            // eq. 22 (per channel)
    const float rphi = warp_reduce_multi<KP>(pp);
    const float ry = warp_reduce_multi<NY>(py);
    if (pwr) sm.accphi[w][t][pw_] += rphi;
    if (ywr && yw < RS) sm.accY[w][t][LS * LS + yw] += ry;
    __syncwarp();
  }
}

// One CTA per (receiver, share of its 32-edge chunks); its warps split the (path,
// channel chunk) tasks.
template <int KP>
__global__ void __launch_bounds__(WARPS_PER_CTA * 32, 5)
    k_uvu_recv_bwd(DevPlan P, Tasks T, const float* __restrict__ x, const float* __restrict__ pos,
                   const int* __restrict__ row_ptr, const int* __restrict__ src,
                   const float* __restrict__ W, const float* __restrict__ gout, int N,
                   float4* gbuf, EdgeWindow win) {
  __shared__ URecvSmem<KP> sm;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x;
  if (i >= N) return;
  int w0, w1;
  window_bounds(row_ptr, win, w0, w1);
  // the receiver's edges inside the staging window
  const int eb = max(__ldg(row_ptr + i), w0), ee = min(__ldg(row_ptr + i + 1), w1);
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
        uvu_recv_body<TR::li, TR::ls, TR::lo, KP>(P, p, chunk, i, ne, x, W, gout, sm);
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
      float4 o;
      o.x = (vx - vr * g.ux) * g.inv_d + s * g.ux;
      o.y = (vy - vr * g.uy) * g.inv_d + s * g.uy;
      o.z = (vz - vr * g.uz) * g.inv_d + s * g.uz;
      o.w = 0.f;
      gbuf[e0 + lane - w0] = o;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// radial-parameter gradient (eq. 19; MODE 1: eq. 27) as per-range partials
// ---------------------------------------------------------------------------

template <int LI, int LS, int LO, int KP, int MODE>
__device__ __forceinline__ void uvu_gradw_body(const DevPlan& P, const DevPath& p, int chunk, int r0,
                                               int r1, const float* __restrict__ x,
                                               const float* __restrict__ xdot,
                                               const float* __restrict__ pos,
                                               const float* __restrict__ posdot,
                                               const int* __restrict__ row_ptr,
                                               const int* __restrict__ src,
                                               const float* __restrict__ gout, float* part,
                                               USmem<KP>& sm) {
  constexpr int RI = 2 * LI + 1, RS = 2 * LS + 1, RO = 2 * LO + 1;
  constexpr bool TAN = MODE == 1;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = chunk * 32 + lane;
  const bool act = u < p.c_in;
  const float* xb = x + p.in_off + (act ? u : 0);
  const float* xdb = xdot ? xdot + p.in_off + (act ? u : 0) : nullptr;
  float acc[KP];
#pragma unroll
  for (int q = 0; q < KP; ++q) acc[q] = 0.f;
  for (int i = r0; i < r1; ++i) {
    float mb[RO];
#pragma unroll
    for (int o = 0; o < RO; ++o)
      mb[o] = act ? __ldg(gout + (long long)i * P.dim_out + p.out_off + o * p.c_out + u) : 0.f;
    const int eb = __ldg(row_ptr + i), ee = __ldg(row_ptr + i + 1);
    for (int e0 = eb; e0 < ee; e0 += 32) {
      const int ne = min(32, ee - e0);
      if (lane < ne) {
        const int j = __ldg(src + e0 + lane);
        uprep<LS, KP, TAN>(P, pos, posdot, i, j, j, e0 + lane, sm, w, lane);
      }
      __syncwarp();
      for (int t = 0; t < ne; ++t) {
        const long long row = (long long)sm.j[w][t] * P.dim_in;
        float xv[RI], Y[RS], C[RO];
#pragma unroll
        for (int k = 0; k < RI; ++k) xv[k] = act ? __ldg(xb + row + k * p.c_in) : 0.f;
#pragma unroll
        for (int k = 0; k < RS; ++k) Y[k] = sm.Y[w][t][k];
        cg_couple<LI, LS, LO>(xv, Y, C);
        float h = 0.f;
#pragma unroll
        for (int o = 0; o < RO; ++o) h = fmaf(mb[o], C[o], h);
        if (!TAN) {
#pragma unroll
          for (int q = 0; q < KP; ++q) acc[q] = fmaf(sm.phi[w][t][q], h, acc[q]);
        } else {
          float Yd[RS], Cd[RO], C2[RO];
#pragma unroll
          for (int k = 0; k < RS; ++k) Yd[k] = sm.Yd[w][t][k];
          cg_couple<LI, LS, LO>(xv, Yd, Cd);
          if (xdb) {
            float xdv[RI];
#pragma unroll
            for (int k = 0; k < RI; ++k) xdv[k] = act ? __ldg(xdb + row + k * p.c_in) : 0.f;
            cg_couple<LI, LS, LO>(xdv, Y, C2);
#pragma unroll
            for (int o = 0; o < RO; ++o) Cd[o] += C2[o];
          }
          float hd = 0.f;
#pragma unroll
          for (int o = 0; o < RO; ++o) hd = fmaf(mb[o], Cd[o], hd);
#pragma unroll
          for (int q = 0; q < KP; ++q) acc[q] = fmaf(sm.phid[w][t][q], h, fmaf(sm.phi[w][t][q], hd, acc[q]));
        }
      }
      __syncwarp();
    }
  }
  if (!act) return;
#pragma unroll
  for (int q = 0; q < KP; ++q)
    if (q < P.K) part[(long long)q * P.n_w + p.w_off + u] = acc[q];
}

template <int KP, int MODE>
__global__ void __launch_bounds__(WARPS_PER_CTA * 32)
    k_uvu_gradw(DevPlan P, Tasks T, const float* __restrict__ x, const float* __restrict__ xdot,
                const float* __restrict__ pos, const float* __restrict__ posdot,
                const int* __restrict__ row_ptr, const int* __restrict__ src,
                const float* __restrict__ gout, int N, int n_ranges, float* partial) {
  __shared__ USmem<KP> sm;
  const long long gw = (long long)blockIdx.x * WARPS_PER_CTA + (threadIdx.x >> 5);
  const int task = (int)(gw / n_ranges);
  const int range = (int)(gw % n_ranges);
  if (task >= T.n) return;
  const int r0 = (int)((long long)N * range / n_ranges);
  const int r1 = (int)((long long)N * (range + 1) / n_ranges);
  const DevPath& p = P.p[T.a[task]];
  const int chunk = T.b[task];
  float* part = partial + (long long)range * P.K * P.n_w;
  dispatch_type(p.type, [&](auto tr) {
    using TR = decltype(tr);
    uvu_gradw_body<TR::li, TR::ls, TR::lo, KP, MODE>(P, p, chunk, r0, r1, x, xdot, pos, posdot,
                                                     row_ptr, src, gout, part, sm);
  });
}

// ---------------------------------------------------------------------------
// source pass: x_bar (eq. 21; MODE 1: eq. 30)
// ---------------------------------------------------------------------------

template <int LI, int LS, int LO, int KP, int MODE>
__device__ __forceinline__ void uvu_src_body(const DevPlan& P, const DevPath& p, int u, bool act,
                                             int j, const float* __restrict__ pos,
                                             const float* __restrict__ posdot,
                                             const int* __restrict__ t_ptr,
                                             const int* __restrict__ t_dst,
                                             const float* __restrict__ W,
                                             const float* __restrict__ Wdot,
                                             const float* __restrict__ gout, float* xb_acc,
                                             USmem<KP>& sm) {
  constexpr int RI = 2 * LI + 1, RS = 2 * LS + 1, RO = 2 * LO + 1;
  constexpr bool TAN = MODE == 1;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float a[KP], ad[KP];
#pragma unroll
  for (int q = 0; q < KP; ++q) {
    a[q] = (act && q < P.K) ? __ldg(W + (long long)q * P.n_w + p.w_off + u) : 0.f;
    ad[q] = (TAN && Wdot && act && q < P.K) ? __ldg(Wdot + (long long)q * P.n_w + p.w_off + u) : 0.f;
  }
  const float* gb = gout + p.out_off + (act ? u : 0);
  const int kb = __ldg(t_ptr + j), ke = __ldg(t_ptr + j + 1);
  for (int k0 = kb; k0 < ke; k0 += 32) {
    const int ne = min(32, ke - k0);
    if (lane < ne) {
      const int i = __ldg(t_dst + k0 + lane);
      const int e = P.emb_eid ? __ldg(P.emb_eid + k0 + lane) : 0;
      uprep<LS, KP, TAN>(P, pos, posdot, i, j, i, e, sm, w, lane);
    }
    __syncwarp();
    for (int t = 0; t < ne; ++t) {
      const long long row = (long long)sm.j[w][t] * P.dim_out;
      float mb[RO], Y[RS], U[RI];
#pragma unroll
      for (int o = 0; o < RO; ++o) mb[o] = act ? __ldg(gb + row + o * p.c_out) : 0.f;
#pragma unroll
      for (int k = 0; k < RS; ++k) Y[k] = sm.Y[w][t][k];
      float we = 0.f;
#pragma unroll
      for (int q = 0; q < KP; ++q) we = fmaf(sm.phi[w][t][q], a[q], we);
      cg_adj_x<LI, LS, LO>(Y, mb, U);
      if (!TAN) {
#pragma unroll
        for (int k = 0; k < RI; ++k) xb_acc[k] = fmaf(we, U[k], xb_acc[k]);
      } else {
        float Yd[RS], Ud[RI];
        float wd = 0.f;
#pragma unroll
        for (int q = 0; q < KP; ++q) wd = fmaf(sm.phid[w][t][q], a[q], fmaf(sm.phi[w][t][q], ad[q], wd));
#pragma unroll
        for (int k = 0; k < RS; ++k) Yd[k] = sm.Yd[w][t][k];
        cg_adj_x<LI, LS, LO>(Yd, mb, Ud);
#pragma unroll
        for (int k = 0; k < RI; ++k) xb_acc[k] = fmaf(wd, U[k], fmaf(we, Ud[k], xb_acc[k]));
      }
    }
    __syncwarp();
  }
}

template <int KP, int MODE>
__global__ void __launch_bounds__(WARPS_PER_CTA * 32)
    k_uvu_src(DevPlan P, BlockPaths BP, Tasks T, const float* __restrict__ pos,
              const float* __restrict__ posdot, const int* __restrict__ t_ptr,
              const int* __restrict__ t_dst, const float* __restrict__ W,
              const float* __restrict__ Wdot, const float* __restrict__ gout, int N,
              float* grad_x) {
  __shared__ USmem<KP> sm;
  const long long gw = (long long)blockIdx.x * WARPS_PER_CTA + (threadIdx.x >> 5);
  const int task = (int)(gw / N);
  const int j = (int)(gw % N);
  if (task >= T.n) return;
  const int bi = T.a[task];
  const int lane = threadIdx.x & 31;
  const int u = T.b[task] * 32 + lane;
  const int c = BP.c[bi];
  const bool act = u < c;
  float acc[7];
#pragma unroll
  for (int k = 0; k < 7; ++k) acc[k] = 0.f;
  for (int k = 0; k < BP.count[bi]; ++k) {
    const DevPath& p = P.p[BP.list[bi][k]];
    dispatch_type(p.type, [&](auto tr) {
      using TR = decltype(tr);
      uvu_src_body<TR::li, TR::ls, TR::lo, KP, MODE>(P, p, u, act, j, pos, posdot, t_ptr, t_dst, W,
                                                     Wdot, gout, acc, sm);
    });
  }
  if (!act) return;
  const int ri = 2 * BP.l[bi] + 1;
  float* dst = grad_x + (long long)j * P.dim_in + BP.off[bi] + u;
#pragma unroll
  for (int k = 0; k < 7; ++k)
    if (k < ri) dst[k * c] = acc[k];
}

// ---------------------------------------------------------------------------
// runners, explicitly instantiated per translation unit
// ---------------------------------------------------------------------------

static inline unsigned ugrid(long long warps) {
  return (unsigned)((warps + WARPS_PER_CTA - 1) / WARPS_PER_CTA);
}

template <int KP, int MODE>
cudaError_t run_uvu_fwd(const DevPlan& P, const BlockPaths& BP, const Tasks& T, const float* x,
                        const float* xdot, const float* pos, const float* posdot,
                        const int* row_ptr, const int* src, const float* W, const float* Wdot,
                        int N, float* out, cudaStream_t s) {
  k_uvu_fwd<KP, MODE><<<ugrid((long long)N * T.n), WARPS_PER_CTA * 32, 0, s>>>(
      P, BP, T, x, xdot, pos, posdot, row_ptr, src, W, Wdot, N, out);
  return cudaGetLastError();
}

template <int KP>
cudaError_t run_uvu_recv_bwd(const DevPlan& P, const Tasks& T, const float* x, const float* pos,
                             const int* row_ptr, const int* src, const float* W,
                             const float* grad_out, int N, float4* gbuf, EdgeWindow win, int edge_split,
                             cudaStream_t s) {
  k_uvu_recv_bwd<KP><<<dim3((unsigned)N, (unsigned)edge_split), WARPS_PER_CTA * 32, 0, s>>>(P, T, x, pos, row_ptr, src, W,
                                                            grad_out, N, gbuf, win);
  return cudaGetLastError();
}

template <int KP, int MODE>
cudaError_t run_uvu_gradw(const DevPlan& P, const Tasks& T, const float* x, const float* xdot,
                          const float* pos, const float* posdot, const int* row_ptr,
                          const int* src, const float* grad_out, int N, int n_ranges,
                          float* partial, cudaStream_t s) {
  k_uvu_gradw<KP, MODE><<<ugrid((long long)n_ranges * T.n), WARPS_PER_CTA * 32, 0, s>>>(
      P, T, x, xdot, pos, posdot, row_ptr, src, grad_out, N, n_ranges, partial);
  return cudaGetLastError();
}

template <int KP, int MODE>
cudaError_t run_uvu_src(const DevPlan& P, const BlockPaths& BP, const Tasks& T, const float* pos,
                        const float* posdot, const int* t_ptr, const int* t_dst, const float* W,
                        const float* Wdot, const float* grad_out, int N, float* grad_x,
                        cudaStream_t s) {
  k_uvu_src<KP, MODE><<<ugrid((long long)N * T.n), WARPS_PER_CTA * 32, 0, s>>>(
      P, BP, T, pos, posdot, t_ptr, t_dst, W, Wdot, grad_out, N, grad_x);
  return cudaGetLastError();
}

#if defined(TPC_UNIT_KP) && defined(TPC_UNIT_MODE) && defined(TPC_UNIT_PART)
#define TPC_PART_STATE 1
#define TPC_PART_SRC 2
#define TPC_PART_RECV 3
#define TPC_PART_FWD 4
#define TPC_PART_GRADW 5
#if TPC_UNIT_PART == TPC_PART_FWD
template cudaError_t run_uvu_fwd<TPC_UNIT_KP, TPC_UNIT_MODE>(
    const DevPlan&, const BlockPaths&, const Tasks&, const float*, const float*, const float*,
    const float*, const int*, const int*, const float*, const float*, int, float*, cudaStream_t);
#endif
#if TPC_UNIT_PART == TPC_PART_GRADW
template cudaError_t run_uvu_gradw<TPC_UNIT_KP, TPC_UNIT_MODE>(
    const DevPlan&, const Tasks&, const float*, const float*, const float*, const float*,
    const int*, const int*, const float*, int, int, float*, cudaStream_t);
#endif
#if TPC_UNIT_PART == TPC_PART_SRC
template cudaError_t run_uvu_src<TPC_UNIT_KP, TPC_UNIT_MODE>(
    const DevPlan&, const BlockPaths&, const Tasks&, const float*, const float*, const int*,
    const int*, const float*, const float*, const float*, int, float*, cudaStream_t);
#endif
#if TPC_UNIT_PART == TPC_PART_RECV && TPC_UNIT_MODE == 0
template cudaError_t run_uvu_recv_bwd<TPC_UNIT_KP>(const DevPlan&, const Tasks&, const float*,
                                                   const float*, const int*, const int*,
                                                   const float*, const float*, int, float4*, EdgeWindow, int,
                                                   cudaStream_t);
#endif
#endif

}  // namespace tpc
