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

// Powers of the unit direction (a, b, c).  A zero-length edge arrives as (0, 0, 0) and
// has no direction: `dir` is 0 there (1 for a unit vector), and every l > 0 harmonic
// is scaled by it, so only the invariant Y_0 survives (the rotation-invariant value).
struct Pow3 {
  float x[4], y[4], z[4];
  float dir;
  __device__ __forceinline__ Pow3(float a, float b, float c) {
    x[0] = 1.f; x[1] = a; x[2] = a * a; x[3] = x[2] * a;
    y[0] = 1.f; y[1] = b; y[2] = b * b; y[3] = y[2] * b;
    z[0] = 1.f; z[1] = c; z[2] = c * c; z[3] = z[2] * c;
    dir = (x[2] + y[2] + z[2] > 0.5f) ? 1.f : 0.f;
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
  if (L > 0) {
#pragma unroll
    for (int k = 0; k < 2 * L + 1; ++k) Y[k] *= p.dir;
  }
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

// v += sum_k w[k] (Hess P_k) t  for block L (the derivative of sh_block_vjp's sum along
// a direction t of the unit vector)
template <int L>
__device__ __forceinline__ void sh_block_hvp(const Pow3& p, const float* w, float tx, float ty, float tz,
                                             float& gx, float& gy, float& gz) {
  using T = tpc_tab::SH<L>;
#pragma unroll
  for (int t = 0; t < T::nterm; ++t) {
    const int ex = T::ex(t), ey = T::ey(t), ez = T::ez(t);
    const float c = T::coef(t) * w[T::k(t)];
    const int ex1 = ex > 0 ? ex - 1 : 0, ey1 = ey > 0 ? ey - 1 : 0, ez1 = ez > 0 ? ez - 1 : 0;
    const int ex2 = ex > 1 ? ex - 2 : 0, ey2 = ey > 1 ? ey - 2 : 0, ez2 = ez > 1 ? ez - 2 : 0;
    const float hxx = ex > 1 ? (float)(ex * (ex - 1)) * p.x[ex2] * p.y[ey] * p.z[ez] : 0.f;
    const float hyy = ey > 1 ? (float)(ey * (ey - 1)) * p.x[ex] * p.y[ey2] * p.z[ez] : 0.f;
    const float hzz = ez > 1 ? (float)(ez * (ez - 1)) * p.x[ex] * p.y[ey] * p.z[ez2] : 0.f;
    const float hxy = (ex > 0 && ey > 0) ? (float)(ex * ey) * p.x[ex1] * p.y[ey1] * p.z[ez] : 0.f;
    const float hxz = (ex > 0 && ez > 0) ? (float)(ex * ez) * p.x[ex1] * p.y[ey] * p.z[ez1] : 0.f;
    const float hyz = (ey > 0 && ez > 0) ? (float)(ey * ez) * p.x[ex] * p.y[ey1] * p.z[ez1] : 0.f;
    gx = fmaf(c, hxx * tx + hxy * ty + hxz * tz, gx);
    gy = fmaf(c, hxy * tx + hyy * ty + hyz * tz, gy);
    gz = fmaf(c, hxz * tx + hyz * ty + hzz * tz, gz);
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

__device__ __forceinline__ void sh_hvp_all(const Pow3& p, const float* w, float tx, float ty, float tz,
                                           float& gx, float& gy, float& gz) {
  sh_block_hvp<1>(p, w + 1, tx, ty, tz, gx, gy, gz);
  sh_block_hvp<2>(p, w + 4, tx, ty, tz, gx, gy, gz);
  sh_block_hvp<3>(p, w + 9, tx, ty, tz, gx, gy, gz);
}

// Yd[k] = grad P_k . t for all blocks l = 0..3
__device__ __forceinline__ void sh_dir_all(const Pow3& p, float tx, float ty, float tz, float* Yd) {
  Yd[0] = 0.f;
  sh_block_dir<1>(p, tx, ty, tz, Yd + 1);
  sh_block_dir<2>(p, tx, ty, tz, Yd + 4);
  sh_block_dir<3>(p, tx, ty, tz, Yd + 9);
}

template <int L>
__device__ __forceinline__ void sh_block_any(int l, const Pow3& p, float* Y);

// ---------------------------------------------------------------------------
// edge geometry: r = pos[src] - pos[dst], d = |r|, r_hat = r / d (0 when d = 0; the
// harmonics of that zero direction are 1 for l = 0 and 0 for l > 0, see Pow3)
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

// Edge ids [w0, w1) of a staging window (w0 >= w1: empty).
__device__ __forceinline__ void window_bounds(const int* __restrict__ row_ptr, const EdgeWindow& win, int& w0,
                                              int& w1) {
  const long long lo = __ldg(row_ptr + win.n0), hi = __ldg(row_ptr + win.n0 + win.n_nodes);
  const long long a = lo + (long long)win.index * win.size;
  w0 = (int)min(a, hi);
  w1 = (int)min(a + win.size, hi);
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

// sin(b pi t) and cos(b pi t) for b = 1..KP from one sincospif: the three-term recurrence
// sin((b+1)a) = 2 cos(a) sin(b a) - sin((b-1)a) (and the same for cos), exact in exact
// arithmetic; in fp32 its absolute error grows like b^2 times the rounding of cos(a): below
// 3e-6 for b <= 8 and 1.1e-5 for b <= 16 on t in (0, 1) (values bounded by 1).
template <int KP>
__device__ __forceinline__ void sincos_multiples(float t, float* sn, float* cs) {
  float s1, c1;
  sincospif(t, &s1, &c1);
  const float two_c = 2.f * c1;
  float sp = 0.f, cp = 1.f, sc = s1, cc = c1;   // b - 1 and b
#pragma unroll
  for (int q = 0; q < KP; ++q) {
    sn[q] = sc;
    cs[q] = cc;
    const float sn1 = fmaf(two_c, sc, -sp), cn1 = fmaf(two_c, cc, -cp);
    sp = sc; cp = cc; sc = sn1; cc = cn1;
  }
}

template <int KP, bool DERIV>
__device__ __forceinline__ void radial(const DevPlan& P, float d, float* phi, float* dphi) {
  const float t = d * P.inv_r_cut;
  float u, du;
  envelope(P, t, u, du);
  du *= P.inv_r_cut;  // d u / d d
  if (P.radial_kind == 0) {
    const float inv_d = d > 0.f ? 1.f / d : 0.f;
    float sn[KP], cs[KP];
    sincos_multiples<KP>(t, sn, cs);
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      float f = 0.f, df = 0.f;
      if (q < P.K && u != 0.f) {
        const float b = (float)(q + 1);
        if (d > 0.f) {
          const float s = sn[q], c = cs[q];
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

// phi_q(d) with its first and second derivatives in d (the double backward's position
// gradient).  The same basis as radial(); the envelope's second derivative is
// u''(t) = -a p (p-1) t^(p-2) + b (p+1) p t^(p-1) - c (p+2)(p+1) t^p  for t < 1, else 0.
template <int KP>
__device__ __forceinline__ void radial2(const DevPlan& P, float d, float* phi, float* dphi, float* d2phi) {
  const float t = d * P.inv_r_cut;
  float u = 0.f, du = 0.f, ddu = 0.f;
  if (t < 1.f) {
    envelope(P, t, u, du);
    const int pp = P.poly_p;
    const float p = (float)pp;
    float tpm1 = 1.f;
    for (int k = 0; k < pp - 1; ++k) tpm1 *= t;
    float tpm2 = 0.f;
    if (pp >= 2) {
      tpm2 = 1.f;
      for (int k = 0; k < pp - 2; ++k) tpm2 *= t;
    }
    ddu = -P.env_a * p * (p - 1.f) * tpm2 + P.env_b * (p + 1.f) * p * tpm1 - P.env_c * (p + 2.f) * (p + 1.f) * tpm1 * t;
  }
  du *= P.inv_r_cut;
  ddu *= P.inv_r_cut * P.inv_r_cut;
  if (P.radial_kind == 0) {
    const float inv_d = d > 0.f ? 1.f / d : 0.f;
    float sn[KP], cs[KP];
    sincos_multiples<KP>(t, sn, cs);
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      float f = 0.f, df = 0.f, d2f = 0.f;
      if (q < P.K && t < 1.f) {
        const float b = (float)(q + 1);
        const float k = b * 3.14159265358979f * P.inv_r_cut;
        if (d > 0.f) {
          const float s = sn[q], c = cs[q];
          const float base = P.bessel_pref * s * inv_d;
          const float g1 = (k * c - s * inv_d) * inv_d;   // d/dd of sin(kd)/d
          const float dbase = P.bessel_pref * g1;
          const float d2base = P.bessel_pref * (-k * k * s - 2.f * g1) * inv_d;
          f = base * u;
          df = dbase * u + base * du;
          d2f = d2base * u + 2.f * dbase * du + base * ddu;
        } else {
          f = P.bessel_pref * k * u;
        }
      }
      phi[q] = f;
      dphi[q] = df;
      d2phi[q] = d2f;
    }
  } else {
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      float f = 0.f, df = 0.f, d2f = 0.f;
      if (q < P.K && t < 1.f) {
        const float dm = d - (P.g_mu0 + P.g_step * (float)q);
        const float g2 = P.g_inv_sigma2;
        const float e = expf(-0.5f * dm * dm * g2);
        const float e1 = -e * dm * g2;
        const float e2 = e * (dm * dm * g2 * g2 - g2);
        f = e * u;
        df = e1 * u + e * du;
        d2f = e2 * u + 2.f * e1 * du + e * ddu;
      }
      phi[q] = f;
      dphi[q] = df;
      d2phi[q] = d2f;
    }
  }
}

// The tangent of the first-order position gradient of one edge (double backward):
//   g = (dphi/dr)^T phi_bar + (dY/dr)^T Y_bar, with phi(|r|) and Y(r / |r|),
// differentiated along r_dot (v) with phi_bar and Y_bar moving by phi_bar_dot, Y_bar_dot:
//   radial part  (sum pbd phi' + d_dot sum pb phi'') r_hat + (sum pb phi') r_hat_dot
//   harmonic part, with G = grad_u F . Y_bar and Gt = grad_u F . Y_bar_dot + Hess_u F (Y_bar) r_hat_dot:
//     (1/d) [Gt - (r_hat.Gt) r_hat - (r_hat_dot.G) r_hat - (r_hat.G) r_hat_dot - (d_dot/d)(G - (r_hat.G) r_hat)]
// where d_dot = r_hat . v and r_hat_dot = (v - d_dot r_hat) / d.  Zero for a zero-length edge.
template <int KP>
__device__ __forceinline__ float3 position_tangent(const DevPlan& P, const EdgeGeo& g, float vx, float vy, float vz,
                                                   const float* Yb, const float* Ybd, const float* pb,
                                                   const float* pbd) {
  const Pow3 pw(g.ux, g.uy, g.uz);
  float phi[KP], dphi[KP], d2phi[KP];
  radial2<KP>(P, g.d, phi, dphi, d2phi);
  const float dd = g.ux * vx + g.uy * vy + g.uz * vz;
  const float tx = (vx - dd * g.ux) * g.inv_d, ty = (vy - dd * g.uy) * g.inv_d, tz = (vz - dd * g.uz) * g.inv_d;
  float s0 = 0.f, s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int q = 0; q < KP; ++q) {
    s0 = fmaf(pb[q], dphi[q], s0);
    s1 = fmaf(pbd[q], dphi[q], s1);
    s2 = fmaf(pb[q], d2phi[q], s2);
  }
  s1 = fmaf(dd, s2, s1);
  float Gx = 0.f, Gy = 0.f, Gz = 0.f, Hx = 0.f, Hy = 0.f, Hz = 0.f;
  sh_vjp_all(pw, Yb, Gx, Gy, Gz);
  sh_vjp_all(pw, Ybd, Hx, Hy, Hz);
  sh_hvp_all(pw, Yb, tx, ty, tz, Hx, Hy, Hz);
  const float uG = g.ux * Gx + g.uy * Gy + g.uz * Gz;
  const float uH = g.ux * Hx + g.uy * Hy + g.uz * Hz;
  const float tG = tx * Gx + ty * Gy + tz * Gz;
  const float k = dd * g.inv_d;
  float3 o;
  o.x = s1 * g.ux + s0 * tx + g.inv_d * (Hx - uH * g.ux - tG * g.ux - uG * tx - k * (Gx - uG * g.ux));
  o.y = s1 * g.uy + s0 * ty + g.inv_d * (Hy - uH * g.uy - tG * g.uy - uG * ty - k * (Gy - uG * g.uy));
  o.z = s1 * g.uz + s0 * tz + g.inv_d * (Hz - uH * g.uz - tG * g.uz - uG * tz - k * (Gz - uG * g.uz));
  return o;
}

// Per-CTA edge data of the double backward's position-gradient kernels (one 32-edge
// chunk of a receiver): Y, phi and their tangents along r_dot, and per-warp partial sums
// of phi_bar, Y_bar and their tangents, combined in warp order.
template <int KP>
struct RecvDblSmem {
  int j[32];
  float Y[32][16], Yd[32][16];
  float phi[32][KP], phid[32][KP];
  float accY[WARPS_PER_CTA][32][16], accYd[WARPS_PER_CTA][32][16];
  float accphi[WARPS_PER_CTA][32][KP], accphid[WARPS_PER_CTA][32][KP];
};

__device__ __forceinline__ float3 edge_rdot(const float* __restrict__ posdot, int i, int j) {
  if (!posdot) return make_float3(0.f, 0.f, 0.f);
  return make_float3(__ldg(posdot + 3 * j) - __ldg(posdot + 3 * i), __ldg(posdot + 3 * j + 1) - __ldg(posdot + 3 * i + 1),
                     __ldg(posdot + 3 * j + 2) - __ldg(posdot + 3 * i + 2));
}

// lane-per-edge staging of edges e0 .. e0+ne-1 of receiver i (warp 0), and zeroed sums
template <int KP>
__device__ __forceinline__ void recv_dbl_prep(const DevPlan& P, const float* __restrict__ pos,
                                              const float* __restrict__ posdot, const int* __restrict__ src,
                                              int i, int e0, int ne, RecvDblSmem<KP>& sm) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (w == 0 && lane < ne) {
    const int j = __ldg(src + e0 + lane);
    const EdgeGeo g = edge_geo(pos, i, j);
    const Pow3 pw(g.ux, g.uy, g.uz);
    float Y[16], Yd[16], phi[KP], dphi[KP];
    sh_all(pw, Y);
    radial<KP, true>(P, g.d, phi, dphi);
    const float3 v = edge_rdot(posdot, i, j);
    const float dd = g.ux * v.x + g.uy * v.y + g.uz * v.z;   // d|r| along r_dot
    sh_dir_all(pw, (v.x - dd * g.ux) * g.inv_d, (v.y - dd * g.uy) * g.inv_d, (v.z - dd * g.uz) * g.inv_d, Yd);
    sm.j[lane] = j;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      sm.Y[lane][k] = Y[k];
      sm.Yd[lane][k] = Yd[k];
    }
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      sm.phi[lane][q] = phi[q];
      sm.phid[lane][q] = dphi[q] * dd;
    }
  }
  for (int k = threadIdx.x; k < WARPS_PER_CTA * 32 * 16; k += blockDim.x) {
    (&sm.accY[0][0][0])[k] = 0.f;
    (&sm.accYd[0][0][0])[k] = 0.f;
  }
  for (int k = threadIdx.x; k < WARPS_PER_CTA * 32 * KP; k += blockDim.x) {
    (&sm.accphi[0][0][0])[k] = 0.f;
    (&sm.accphid[0][0][0])[k] = 0.f;
  }
}

// per edge (warp 0): the warp-ordered sums, then the tangent of g_e into gbuf (at the
// edge id less gbase, the start of the staging window)
template <int KP>
__device__ __forceinline__ void recv_dbl_finish(const DevPlan& P, const float* __restrict__ pos,
                                                const float* __restrict__ posdot, int i, int e0, int ne,
                                                const RecvDblSmem<KP>& sm, float4* gbuf, int gbase) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (w != 0 || lane >= ne) return;
  const int j = sm.j[lane];
  const EdgeGeo g = edge_geo(pos, i, j);
  const float3 v = edge_rdot(posdot, i, j);
  float Yb[16], Ybd[16], pb[KP], pbd[KP];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    float a = 0.f, b = 0.f;
#pragma unroll
    for (int ww = 0; ww < WARPS_PER_CTA; ++ww) {
      a += sm.accY[ww][lane][k];
      b += sm.accYd[ww][lane][k];
    }
    Yb[k] = a;
    Ybd[k] = b;
  }
#pragma unroll
  for (int q = 0; q < KP; ++q) {
    float a = 0.f, b = 0.f;
#pragma unroll
    for (int ww = 0; ww < WARPS_PER_CTA; ++ww) {
      a += sm.accphi[ww][lane][q];
      b += sm.accphid[ww][lane][q];
    }
    pb[q] = a;
    pbd[q] = b;
  }
  const float3 o = position_tangent<KP>(P, g, v.x, v.y, v.z, Yb, Ybd, pb, pbd);
  gbuf[e0 + lane - gbase] = make_float4(o.x, o.y, o.z, 0.f);
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
