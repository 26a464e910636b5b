// Device helpers shared by the streaming kernels: edge geometry (eq. 8), real
// spherical harmonics and their derivatives, the radial basis, the sparse coupling
// of eq. 32 and its two adjoints, warp reductions and the dispatch from a runtime
// path type to a kernel body specialised on (l_in, l_sh, l_out).
#pragma once
#include <cuda_runtime.h>
#include <type_traits>
#include "internal.h"
#include "tables.inc"

namespace tpc {

#define TPC_FULL 0xffffffffu

// ---------------------------------------------------------------------------
// spherical harmonics (polynomials in the unit direction, from the generated tables)
// ---------------------------------------------------------------------------

struct Pow3 {
  float x[4], y[4], z[4];
  __device__ __forceinline__ Pow3(float a, float b, float c) {
    x[0] = 1.f; x[1] = a; x[2] = a * a; x[3] = x[2] * a;
    y[0] = 1.f; y[1] = b; y[2] = b * b; y[3] = y[2] * b;
    z[0] = 1.f; z[1] = c; z[2] = c * c; z[3] = z[2] * c;
  }
};

template <int L>
__device__ __forceinline__ void sh_block(const Pow3& p, float* Y) {
  using T = tpc_tab::SH<L>;
#pragma unroll
  for (int k = 0; k < 2 * L + 1; ++k) Y[k] = 0.f;
#pragma unroll
  for (int t = 0; t < T::nterm; ++t)
    Y[T::k(t)] = fmaf(T::coef(t), p.x[T::ex(t)] * p.y[T::ey(t)] * p.z[T::ez(t)], Y[T::k(t)]);
}

// d/d(unit vector) of block L, contracted with a direction v: Yd[k] = grad P_k . v
template <int L>
__device__ __forceinline__ void sh_block_dir(const Pow3& p, float vx, float vy, float vz, float* Yd) {
  using T = tpc_tab::SH<L>;
#pragma unroll
  for (int k = 0; k < 2 * L + 1; ++k) Yd[k] = 0.f;
#pragma unroll
  for (int t = 0; t < T::nterm; ++t) {
    constexpr int dummy = 0; (void)dummy;
    const int ex = T::ex(t), ey = T::ey(t), ez = T::ez(t);
    float g = 0.f;
    if (ex > 0) g = fmaf((float)ex * p.x[ex > 0 ? ex - 1 : 0] * p.y[ey] * p.z[ez], vx, g);
    if (ey > 0) g = fmaf((float)ey * p.x[ex] * p.y[ey > 0 ? ey - 1 : 0] * p.z[ez], vy, g);
    if (ez > 0) g = fmaf((float)ez * p.x[ex] * p.y[ey] * p.z[ez > 0 ? ez - 1 : 0], vz, g);
    Yd[T::k(t)] = fmaf(T::coef(t), g, Yd[T::k(t)]);
  }
}

// v += sum_k w[k] grad P_k  for block L (w has 2L+1 entries)
template <int L>
__device__ __forceinline__ void sh_block_vjp(const Pow3& p, const float* w, float& gx, float& gy,
                                             float& gz) {
  using T = tpc_tab::SH<L>;
#pragma unroll
  for (int t = 0; t < T::nterm; ++t) {
    const int ex = T::ex(t), ey = T::ey(t), ez = T::ez(t);
    const float c = T::coef(t) * w[T::k(t)];
    if (ex > 0) gx = fmaf(c * (float)ex, p.x[ex > 0 ? ex - 1 : 0] * p.y[ey] * p.z[ez], gx);
    if (ey > 0) gy = fmaf(c * (float)ey, p.x[ex] * p.y[ey > 0 ? ey - 1 : 0] * p.z[ez], gy);
    if (ez > 0) gz = fmaf(c * (float)ez, p.x[ex] * p.y[ey] * p.z[ez > 0 ? ez - 1 : 0], gz);
  }
}

// all blocks l = 0..3 into Y[16]
__device__ __forceinline__ void sh_all(const Pow3& p, float* Y) {
  sh_block<0>(p, Y);
  sh_block<1>(p, Y + 1);
  sh_block<2>(p, Y + 4);
  sh_block<3>(p, Y + 9);
}

__device__ __forceinline__ void sh_vjp_all(const Pow3& p, const float* w, float& gx, float& gy,
                                           float& gz) {
  sh_block_vjp<1>(p, w + 1, gx, gy, gz);
  sh_block_vjp<2>(p, w + 4, gx, gy, gz);
  sh_block_vjp<3>(p, w + 9, gx, gy, gz);
}

template <int L>
__device__ __forceinline__ void sh_block_any(int l, const Pow3& p, float* Y);

// ---------------------------------------------------------------------------
// edge geometry: r = pos[src] - pos[dst], d = |r|, r_hat = r / d (0 when d = 0)
// ---------------------------------------------------------------------------

struct EdgeGeo {
  float rx, ry, rz, d, inv_d, ux, uy, uz;
};

__device__ __forceinline__ EdgeGeo edge_geo(const float* __restrict__ pos, int i, int j) {
  EdgeGeo g;
  g.rx = __ldg(pos + 3 * j) - __ldg(pos + 3 * i);
  g.ry = __ldg(pos + 3 * j + 1) - __ldg(pos + 3 * i + 1);
  g.rz = __ldg(pos + 3 * j + 2) - __ldg(pos + 3 * i + 2);
  float d2 = g.rx * g.rx + g.ry * g.ry + g.rz * g.rz;
  if (d2 > 1e-30f) {
    g.d = sqrtf(d2);
    g.inv_d = 1.0f / g.d;
  } else {
    g.d = 0.f;
    g.inv_d = 0.f;
  }
  g.ux = g.rx * g.inv_d;
  g.uy = g.ry * g.inv_d;
  g.uz = g.rz * g.inv_d;
  return g;
}

// ---------------------------------------------------------------------------
// radial basis phi_q(d), q < K (zero for K <= q < KP), and d phi_q / d d
// ---------------------------------------------------------------------------

__device__ __forceinline__ void envelope(const DevPlan& P, float t, float& u, float& du) {
  if (t >= 1.f) { u = 0.f; du = 0.f; return; }
  float tpm1 = 1.f;
  for (int k = 0; k < P.poly_p - 1; ++k) tpm1 *= t;
  const float tp = tpm1 * t, tp1 = tp * t, tp2 = tp1 * t;
  u = 1.f - P.env_a * tp + P.env_b * tp1 - P.env_c * tp2;
  const float p = (float)P.poly_p;
  du = -P.env_a * p * tpm1 + P.env_b * (p + 1.f) * tp - P.env_c * (p + 2.f) * tp1;
}

template <int KP, bool DERIV>
__device__ __forceinline__ void radial(const DevPlan& P, float d, float* phi, float* dphi) {
  const float t = d * P.inv_r_cut;
  float u, du;
  envelope(P, t, u, du);
  du *= P.inv_r_cut;  // d u / d d
  if (P.radial_kind == 0) {
    const float inv_d = d > 0.f ? 1.f / d : 0.f;
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      float f = 0.f, df = 0.f;
      if (q < P.K && u != 0.f) {
        const float b = (float)(q + 1);
        if (d > 0.f) {
          float s, c;
          sincospif(b * t, &s, &c);
          const float base = P.bessel_pref * s * inv_d;  // sqrt(2/rc) sin(b pi t)/d
          f = base * u;
          if (DERIV) {
            const float dbase = P.bessel_pref * (b * 3.14159265358979f * P.inv_r_cut * c - s * inv_d) * inv_d;
            df = dbase * u + base * du;
          }
        } else {
          f = P.bessel_pref * b * 3.14159265358979f * P.inv_r_cut * u;
        }
      }
      phi[q] = f;
      if (DERIV) dphi[q] = df;
    }
  } else {
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      float f = 0.f, df = 0.f;
      if (q < P.K && u != 0.f) {
        const float dm = d - (P.g_mu0 + P.g_step * (float)q);
        const float e = expf(-0.5f * dm * dm * P.g_inv_sigma2);
        f = e * u;
        if (DERIV) df = e * (du - u * dm * P.g_inv_sigma2);
      }
      phi[q] = f;
      if (DERIV) dphi[q] = df;
    }
  }
}

// ---------------------------------------------------------------------------
// eq. 32: C[mo] = sum c[mi][my][mo] x[mi] Y[my], and its adjoints
// ---------------------------------------------------------------------------

template <int LI, int LS, int LO>
__device__ __forceinline__ void cg_couple(const float* xv, const float* Y, float* C) {
  using T = tpc_tab::CG<LI, LS, LO>;
#pragma unroll
  for (int o = 0; o < 2 * LO + 1; ++o) C[o] = 0.f;
#pragma unroll
  for (int n = 0; n < T::nnz; ++n) C[T::mo(n)] = fmaf(T::val(n) * Y[T::my(n)], xv[T::mi(n)], C[T::mo(n)]);
}

// Per-edge products cy[n] = c_n * Y[my_n] of one path (n < nnz, padded with zeros to a
// multiple of 4); every lane then needs only these and its own x values.
constexpr int CY_MAX = 44;   // max nnz over l <= 3 triples (42), padded to a multiple of 4

template <int LI, int LS, int LO>
struct CgInfo {
  static constexpr int nnz = tpc_tab::CG<LI, LS, LO>::nnz;
  static constexpr int n4 = (nnz + 3) / 4;
};

template <int LI, int LS, int LO>
__device__ __forceinline__ void cg_products(const float* Y, float* cy) {
  using T = tpc_tab::CG<LI, LS, LO>;
  constexpr int n4 = CgInfo<LI, LS, LO>::n4;
#pragma unroll
  for (int n = 0; n < 4 * n4; ++n) cy[n] = n < T::nnz ? T::val(n < T::nnz ? n : 0) * Y[T::my(n < T::nnz ? n : 0)] : 0.f;
}

// C[mo] = sum_n cy[n] x[mi_n] with cy read from shared memory (broadcast)
template <int LI, int LS, int LO>
__device__ __forceinline__ void cg_couple_cy(const float* xv, const float* cy, float* C) {
  using T = tpc_tab::CG<LI, LS, LO>;
  constexpr int n4 = CgInfo<LI, LS, LO>::n4;
#pragma unroll
  for (int o = 0; o < 2 * LO + 1; ++o) C[o] = 0.f;
#pragma unroll
  for (int b = 0; b < n4; ++b) {
    const float4 v = reinterpret_cast<const float4*>(cy)[b];
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int n = 4 * b + k;
      if (n < T::nnz) C[T::mo(n < T::nnz ? n : 0)] = fmaf(vv[k], xv[T::mi(n < T::nnz ? n : 0)], C[T::mo(n < T::nnz ? n : 0)]);
    }
  }
}

// U[mi] = sum_n cy[n] g[mo_n]   (adjoint in x, products from shared memory)
template <int LI, int LS, int LO>
__device__ __forceinline__ void cg_adj_x_cy(const float* cy, const float* g, float* U) {
  using T = tpc_tab::CG<LI, LS, LO>;
  constexpr int n4 = CgInfo<LI, LS, LO>::n4;
#pragma unroll
  for (int i = 0; i < 2 * LI + 1; ++i) U[i] = 0.f;
#pragma unroll
  for (int b = 0; b < n4; ++b) {
    const float4 v = reinterpret_cast<const float4*>(cy)[b];
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int n = 4 * b + k;
      if (n < T::nnz) U[T::mi(n < T::nnz ? n : 0)] = fmaf(vv[k], g[T::mo(n < T::nnz ? n : 0)], U[T::mi(n < T::nnz ? n : 0)]);
    }
  }
}

// U[mi] = sum c Y[my] g[mo]  (adjoint in x)
template <int LI, int LS, int LO>
__device__ __forceinline__ void cg_adj_x(const float* Y, const float* g, float* U) {
  using T = tpc_tab::CG<LI, LS, LO>;
#pragma unroll
  for (int i = 0; i < 2 * LI + 1; ++i) U[i] = 0.f;
#pragma unroll
  for (int n = 0; n < T::nnz; ++n) U[T::mi(n)] = fmaf(T::val(n) * Y[T::my(n)], g[T::mo(n)], U[T::mi(n)]);
}

// Yb[my] += sum c x[mi] g[mo]  (adjoint in Y)
template <int LI, int LS, int LO>
__device__ __forceinline__ void cg_adj_y(const float* xv, const float* g, float* Yb) {
  using T = tpc_tab::CG<LI, LS, LO>;
#pragma unroll
  for (int n = 0; n < T::nnz; ++n) Yb[T::my(n)] = fmaf(T::val(n) * xv[T::mi(n)], g[T::mo(n)], Yb[T::my(n)]);
}

// ---------------------------------------------------------------------------
// warp reductions
// ---------------------------------------------------------------------------

template <int N>
struct Log2 { static constexpr int v = (N <= 1) ? 0 : 1 + Log2<N / 2>::v; };
template <>
struct Log2<1> { static constexpr int v = 0; };

// Sum N values (N a power of two <= 32) over the 32 lanes.  Returns, in every lane L,
// the total of value index (L >> (5 - log2 N)) & (N - 1).  Fixed shuffle order, so the
// result is deterministic.
template <int N>
__device__ __forceinline__ float warp_reduce_multi(float (&v)[N]) {
  const int lane = threadIdx.x & 31;
  constexpr int LG = Log2<N>::v;
#pragma unroll
  for (int s = 0; s < LG; ++s) {
    const int o = 16 >> s;
    const int half = N >> (s + 1);
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(TPC_FULL, send, o);
    }
  }
#pragma unroll
  for (int o = 16 >> LG; o >= 1; o >>= 1) v[0] += __shfl_xor_sync(TPC_FULL, v[0], o);
  return v[0];
}

template <int N>
__device__ __forceinline__ int reduce_multi_index(int lane) {
  return (lane >> (5 - Log2<N>::v)) & (N - 1);
}
template <int N>
__device__ __forceinline__ bool reduce_multi_writer(int lane) {
  return (lane & ((1 << (5 - Log2<N>::v)) - 1)) == 0;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(TPC_FULL, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// runtime path type -> compile-time (l_in, l_sh, l_out)
// ---------------------------------------------------------------------------

template <int A, int B, int C>
struct Triple {
  static constexpr int li = A, ls = B, lo = C;
};

static_assert(tpc_tab::NTRIPLES == 34, "dispatch table expects l <= 3");

#define TPC_CASE(n)                                                                          \
  case n:                                                                                    \
    f(Triple<tpc_tab::TRIPLES[n][0], tpc_tab::TRIPLES[n][1], tpc_tab::TRIPLES[n][2]>{});     \
    break;

template <class F>
__device__ __forceinline__ void dispatch_type(int type, F&& f) {
  switch (type) {
    TPC_CASE(0) TPC_CASE(1) TPC_CASE(2) TPC_CASE(3) TPC_CASE(4) TPC_CASE(5) TPC_CASE(6)
    TPC_CASE(7) TPC_CASE(8) TPC_CASE(9) TPC_CASE(10) TPC_CASE(11) TPC_CASE(12) TPC_CASE(13)
    TPC_CASE(14) TPC_CASE(15) TPC_CASE(16) TPC_CASE(17) TPC_CASE(18) TPC_CASE(19) TPC_CASE(20)
    TPC_CASE(21) TPC_CASE(22) TPC_CASE(23) TPC_CASE(24) TPC_CASE(25) TPC_CASE(26) TPC_CASE(27)
    TPC_CASE(28) TPC_CASE(29) TPC_CASE(30) TPC_CASE(31) TPC_CASE(32) TPC_CASE(33)
    default: break;
  }
}

// compile-time l -> block of Y[16]
template <int L>
struct ShOff { static constexpr int v = L * L; };

}  // namespace tpc
