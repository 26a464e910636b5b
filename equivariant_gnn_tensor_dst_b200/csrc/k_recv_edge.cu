// Receiver backward of the fully connected (uvw) convolution, one lane per edge.
//
// Sobek: Streaming Equivariant Tensor Product Convolutions, section 3 (eqs. 18-22) in
// the receiver-factorised form of section 4 (eq. 36).  Given the receiver's state
// adjoint S_bar = m_bar A^T (a channel contraction on the tensor cores), every edge e
// of receiver i needs
//     phi_bar_{e,q} = sum_pi sum_u sum_mo  S_bar_{i,pi,q,mo,u} C_{e,pi,u,mo}        (eq. 20)
//     Y_bar_e      = sum_pi sum_u  D_Y C_{e,pi,u}(x_j)^T T_bar_{e,pi,u},
//     T_bar_{e,pi,u,mo} = sum_q phi_{e,q} S_bar_{i,pi,q,mo,u}                          (eq. 22)
// with C = the coupling of x_j with Y_e (eq. 32), and then the edge's position gradient
// g_e = (d phi / d r)^T phi_bar + (d Y / d r)^T Y_bar, staged for the fixed-order node
// sums (or, for the embedded-input interface, the edge-owned phi_bar and Y_bar).
//
// Layout of the work: a CTA owns up to 32 consecutive edges of one receiver, one edge per
// lane, and its four warps split the input channels of every path four ways.  phi_bar
// and Y_bar are sums over channels and paths, so each lane accumulates its own edge's
// partial sums in registers, with no cross-lane reduction; the four warps' partials are
// added in warp order once per chunk.  No atomics.  S_bar of the receiver is the same for
// all lanes: each warp stages its channel slice of it in shared memory (asynchronous
// copies, double buffered across the (path, slice) pieces it owns) and reads it back as
// broadcasts; x_j differs per lane and is read through L1, where the four warps' slices
// of the same 32 rows meet.  Edges with d >= r_cut have phi = 0 and contribute 0.
#include "common.cuh"

namespace tpc {

// Per-warp staging of S_bar: one slice of up to CHMAX channels of one path, rows
// (m_out, q) padded to KP rows per m_out, double buffered (7 KB per warp for either
// radial width).  red: per-warp partial phi_bar and Y_bar of each lane's edge (row
// stride KP + 17: conflict-free columns).
template <int KP>
struct RecvEdgeSmem {
  static constexpr int CHMAX = 128 / KP;
  alignas(16) float sb[4][2][7 * KP][CHMAX];
  float red[4][32][KP + 17];
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Channel slice width of a path of C input channels: a quarter of C (each warp of the
// CTA takes every fourth slice), at most CHMAX, a multiple of 4 when FAST.
template <int KP, bool FAST>
__device__ __forceinline__ int slice_width(int C) {
  constexpr int CHMAX = RecvEdgeSmem<KP>::CHMAX;
  const int q = (C + 3) >> 2;
  return FAST ? min(CHMAX, max(4, (q + 3) & ~3)) : min(CHMAX, max(1, q));
}

// Copy channels [c0, c0 + cw) of the (m_out, q) rows of one path's S_bar into `dst`
// (FAST: 16-byte asynchronous copies, every offset a multiple of 4 floats).
template <int KP, bool FAST>
__device__ __forceinline__ void stage_slice(const DevPlan& P, const DevPath& p, const float* __restrict__ sbn,
                                            int c0, int cw, float (*dst)[RecvEdgeSmem<KP>::CHMAX]) {
  const int lane = threadIdx.x & 31;
  const int K = P.K, C = p.c_in, ro = 2 * p.l_out + 1;
  const float* __restrict__ sb = sbn + p.st_off;
  const long long KC = (long long)K * C;
  if (FAST) {
    const int per_row = cw >> 2, n = ro * K * per_row;
    for (int t = lane; t < n; t += 32) {
      const int row = t / per_row, part = t - row * per_row;
      const int o = row / K, q = row - o * K;
      cp_async16(&dst[o * KP + q][4 * part], sb + o * KC + (long long)q * C + c0 + 4 * part);
    }
    cp_async_commit();
  } else {
    const int n = ro * K * cw;
    for (int t = lane; t < n; t += 32) {
      const int row = t / cw, c = t - row * cw;
      const int o = row / K, q = row - o * K;
      dst[o * KP + q][c] = __ldg(sb + o * KC + (long long)q * C + c0 + c);
    }
  }
}

// One piece (a path and one channel slice of it): accumulate phi_bar (pb) and the path's
// block of Y_bar (yb) of this lane's edge from the staged slice S.  FAST: two channels
// per step with 8-byte loads; otherwise one.
template <int LI, int LS, int LO, int KP, bool FAST>
__device__ __forceinline__ void recv_edge_piece(const DevPlan& P, const DevPath& p, const float* __restrict__ xrow,
                                                const float* Y, const float* phi, int c0, int cw,
                                                const float (*S)[RecvEdgeSmem<KP>::CHMAX], float* pb, float* yb) {
  using T = tpc_tab::CG<LI, LS, LO>;
  constexpr int RI = 2 * LI + 1, RS = 2 * LS + 1, RO = 2 * LO + 1, NZ = T::nnz;
  constexpr int U = FAST ? 2 : 1;
  const int C = p.c_in, K = P.K;
  const float* __restrict__ xb = xrow + p.in_off + c0;
  float cy[NZ];
#pragma unroll
  for (int n = 0; n < NZ; ++n) cy[n] = T::val(n) * Y[LS * LS + T::my(n)];
  float ybl[RS];
#pragma unroll
  for (int k = 0; k < RS; ++k) ybl[k] = 0.f;
#pragma unroll 1
  for (int cc = 0; cc < cw; cc += U) {
    float xv[U][RI];
#pragma unroll
    for (int mi = 0; mi < RI; ++mi) {
      if (FAST) {
        const float2 v = __ldg(reinterpret_cast<const float2*>(xb + mi * C + cc));
        xv[0][mi] = v.x;
        xv[U - 1][mi] = v.y;
      } else {
        xv[0][mi] = __ldg(xb + mi * C + cc);
      }
    }
    // coupled message C_{e,pi,u,mo} (eq. 32)
    float cm[U][RO];
#pragma unroll
    for (int c = 0; c < U; ++c)
#pragma unroll
      for (int o = 0; o < RO; ++o) cm[c][o] = 0.f;
#pragma unroll
    for (int n = 0; n < NZ; ++n)
#pragma unroll
      for (int c = 0; c < U; ++c) cm[c][T::mo(n)] = fmaf(cy[n], xv[c][T::mi(n)], cm[c][T::mo(n)]);
    // phi_bar += <S_bar_q, C> and T_bar = sum_q phi_q S_bar_q
    float tb[U][RO];
#pragma unroll
    for (int c = 0; c < U; ++c)
#pragma unroll
      for (int o = 0; o < RO; ++o) tb[c][o] = 0.f;
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      if (q < K) {
#pragma unroll
        for (int o = 0; o < RO; ++o) {
          float sv[U];
          if (FAST) {
            const float2 v = *reinterpret_cast<const float2*>(&S[o * KP + q][cc]);
            sv[0] = v.x;
            sv[U - 1] = v.y;
          } else {
            sv[0] = S[o * KP + q][cc];
          }
#pragma unroll
          for (int c = 0; c < U; ++c) {
            pb[q] = fmaf(sv[c], cm[c][o], pb[q]);
            tb[c][o] = fmaf(phi[q], sv[c], tb[c][o]);
          }
        }
      }
    }
    // Y_bar_my += sum_n c_n x_mi T_bar_mo (the adjoint of eq. 32 in Y)
#pragma unroll
    for (int n = 0; n < NZ; ++n) {
      float v = xv[0][T::mi(n)] * tb[0][T::mo(n)];
#pragma unroll
      for (int c = 1; c < U; ++c) v = fmaf(xv[c][T::mi(n)], tb[c][T::mo(n)], v);
      ybl[T::my(n)] = fmaf(T::val(n), v, ybl[T::my(n)]);
    }
  }
#pragma unroll
  for (int k = 0; k < RS; ++k) yb[LS * LS + k] += ybl[k];
}

// The pieces of warp w in order: for every path, its slices w, w + 4, ...  Returns false
// past the last one.
template <int KP, bool FAST>
__device__ __forceinline__ bool next_piece(const DevPlan& P, int w, int& pi, int& slice) {
  if (pi >= 0) {
    slice += 4;
    const int C = P.p[pi].c_in;
    if (slice * slice_width<KP, FAST>(C) < C) return true;
  }
  for (++pi; pi < P.n_paths; ++pi) {
    const int C = P.p[pi].c_in;
    if (w * slice_width<KP, FAST>(C) < C) {
      slice = w;
      return true;
    }
  }
  return false;
}

// Grid: CTAs enumerate (receiver slot, share); share s of a receiver takes its 32-edge
// chunks s, s + split, ...  Four CTAs per SM for K <= 8, three for K <= 16 (its
// accumulators need more registers).
template <int KP, bool FAST>
__global__ void __launch_bounds__(128, KP == 8 ? 4 : 3)
    k_uvw_recv_edge(DevPlan P, const float* __restrict__ x, const float* __restrict__ pos,
                    const int* __restrict__ row_ptr, const int* __restrict__ src, const float* __restrict__ Sbar,
                    int node0, int n_nodes, float4* gbuf, EdgeWindow win, int split) {
  __shared__ RecvEdgeSmem<KP> sm;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int slot = (int)(blockIdx.x / split), share = (int)(blockIdx.x % split);
  if (slot >= n_nodes) return;
  const int node_local = P.order ? __ldg(P.order + node0 + slot) - node0 : slot;
  const int i = node0 + node_local;
  int w0, w1;
  window_bounds(row_ptr, win, w0, w1);
  const int eb = max(__ldg(row_ptr + i), w0), ee = min(__ldg(row_ptr + i + 1), w1);
  const float* __restrict__ sbn = Sbar + (long long)node_local * P.state_per_node;
  for (int e0 = eb + 32 * share; e0 < ee; e0 += 32 * split) {
    const int e = e0 + lane;
    const bool act = e < ee;
    const int j = __ldg(src + (act ? e : e0));   // idle lanes shadow the chunk's first edge
    float Y[16], phi[KP];
    if (P.emb_Y) {
#pragma unroll
      for (int k = 0; k < 16; ++k) Y[k] = k < P.n_sh ? __ldg(P.emb_Y + (long long)(act ? e : e0) * P.n_sh + k) : 0.f;
#pragma unroll
      for (int q = 0; q < KP; ++q) phi[q] = q < P.K ? __ldg(P.emb_phi + (long long)(act ? e : e0) * P.K + q) : 0.f;
    } else {
      const EdgeGeo g = edge_geo(pos, i, j);
      const Pow3 pw(g.ux, g.uy, g.uz);
      sh_all(pw, Y);
      float dphi[KP];
      radial<KP, false>(P, g.d, phi, dphi);
    }
    float pb[KP], yb[16];
#pragma unroll
    for (int q = 0; q < KP; ++q) pb[q] = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) yb[k] = 0.f;
    const float* __restrict__ xrow = x + (long long)j * P.dim_in;
    // pieces of this warp, software-pipelined: the next piece's S_bar slice is copied
    // while the current one is consumed
    int pi = -1, slice = 0;
    bool have = next_piece<KP, FAST>(P, w, pi, slice);
    int buf = 0;
    if (have) {
      const int cw = slice_width<KP, FAST>(P.p[pi].c_in);
      const int c0 = slice * cw;
      stage_slice<KP, FAST>(P, P.p[pi], sbn, c0, min(cw, P.p[pi].c_in - c0), sm.sb[w][0]);
    }
    while (have) {
      int npi = pi, nslice = slice;
      const bool more = next_piece<KP, FAST>(P, w, npi, nslice);
      if (more) {
        const int ncw = slice_width<KP, FAST>(P.p[npi].c_in);
        const int nc0 = nslice * ncw;
        stage_slice<KP, FAST>(P, P.p[npi], sbn, nc0, min(ncw, P.p[npi].c_in - nc0), sm.sb[w][buf ^ 1]);
      }
      if (FAST) {
        if (more) cp_async_wait<1>(); else cp_async_wait<0>();
      }
      __syncwarp();
      const DevPath& p = P.p[pi];
      const int cwid = slice_width<KP, FAST>(p.c_in);
      const int c0 = slice * cwid, cw = min(cwid, p.c_in - c0);
      dispatch_type(p.type, [&](auto tr) {
        using TR = decltype(tr);
        recv_edge_piece<TR::li, TR::ls, TR::lo, KP, FAST>(P, p, xrow, Y, phi, c0, cw, sm.sb[w][buf], pb, yb);
      });
      __syncwarp();   // this buffer is refilled two pieces later
      pi = npi;
      slice = nslice;
      have = more;
      buf ^= 1;
    }
    // the four warps' partial sums of this lane's edge, added in warp order
#pragma unroll
    for (int q = 0; q < KP; ++q) sm.red[w][lane][q] = pb[q];
#pragma unroll
    for (int k = 0; k < 16; ++k) sm.red[w][lane][KP + k] = yb[k];
    __syncthreads();
    if (w == 0 && act) {
#pragma unroll
      for (int q = 0; q < KP; ++q)
        pb[q] = ((sm.red[0][lane][q] + sm.red[1][lane][q]) + sm.red[2][lane][q]) + sm.red[3][lane][q];
#pragma unroll
      for (int k = 0; k < 16; ++k)
        yb[k] = ((sm.red[0][lane][KP + k] + sm.red[1][lane][KP + k]) + sm.red[2][lane][KP + k]) +
                sm.red[3][lane][KP + k];
      if (P.emb_gY || P.emb_gphi) {
        // embedded input: the edge-owned adjoints Y_bar (eq. 22) and phi_bar (eq. 20)
        // (compile-time indices keep yb and pb in registers)
        if (P.emb_gY) {
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if (k < P.n_sh) P.emb_gY[(long long)e * P.n_sh + k] = yb[k];
        }
        if (P.emb_gphi) {
#pragma unroll
          for (int q = 0; q < KP; ++q)
            if (q < P.K) P.emb_gphi[(long long)e * P.K + q] = pb[q];
        }
      } else {
        // g_e = (d phi/d r)^T phi_bar + (d Y/d r)^T Y_bar, through r_hat = r / |r|
        const EdgeGeo g = edge_geo(pos, i, j);
        const Pow3 pw(g.ux, g.uy, g.uz);
        float phi2[KP], dphi[KP];
        radial<KP, true>(P, g.d, phi2, dphi);
        float vx = 0.f, vy = 0.f, vz = 0.f;
        sh_vjp_all(pw, yb, vx, vy, vz);
        const float vr = vx * g.ux + vy * g.uy + vz * g.uz;
        float s = 0.f;
#pragma unroll
        for (int q = 0; q < KP; ++q) s = fmaf(pb[q], dphi[q], s);
        float4 out;
        out.x = (vx - vr * g.ux) * g.inv_d + s * g.ux;
        out.y = (vy - vr * g.uy) * g.inv_d + s * g.uy;
        out.z = (vz - vr * g.uz) * g.inv_d + s * g.uz;
        out.w = 0.f;
        gbuf[e - w0] = out;
      }
    }
    __syncthreads();   // red is rewritten by the next chunk
  }
}

// FAST: every path's channel count, input offset and state offset, the node row width
// and the node state stride are multiples of 4 floats (16-byte copies of S_bar, 8-byte
// loads of x); otherwise the generic variant (one channel per step).
template <int KP, bool FAST>
cudaError_t run_uvw_recv_edge(const DevPlan& P, const float* x, const float* pos, const int* row_ptr,
                              const int* src, const float* Sbar, int node0, int n_nodes, float4* gbuf,
                              EdgeWindow win, int split, cudaStream_t s) {
  const long long ctas = (long long)n_nodes * split;
  k_uvw_recv_edge<KP, FAST><<<(unsigned)ctas, 128, 0, s>>>(P, x, pos, row_ptr, src, Sbar, node0, n_nodes, gbuf,
                                                             win, split);
  return cudaGetLastError();
}

#if defined(TPC_UNIT_KP) && defined(TPC_UNIT_MODE)
template cudaError_t run_uvw_recv_edge<TPC_UNIT_KP, TPC_UNIT_MODE == 1>(const DevPlan&, const float*, const float*,
                                                                      const int*, const int*, const float*, int, int,
                                                                      float4*, EdgeWindow, int, cudaStream_t);
#endif

}  // namespace tpc
