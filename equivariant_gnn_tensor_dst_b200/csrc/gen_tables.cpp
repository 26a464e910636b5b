// Build-time generator of the compile-time tables used by the CUDA kernels:
//   * real spherical harmonics of order l <= TPC_LMAX as polynomials in the unit
//     direction (x, y, z);
//   * the real coupling tensors c[m_in][m_sh][m_out] of every order triple allowed by
//     the triangle rule (Sobek, section 2, eq. 5; eq. 32's c^pi).
//
// Conventions (shared with the rest of the library): component index k = m + l,
// m = -l..l; real harmonics with z as polar axis, no Condon-Shortley phase,
// normalised so that the mean of Y_lm^2 over the sphere is 1 (sum_m Y_lm^2 = 2l+1):
//     Y_{l, m}  ~ Q_l^m(z) Re((x + i y)^m),   Y_{l,-m} ~ Q_l^m(z) Im((x + i y)^m)
// with Q_l^m the m-th z-derivative of the Legendre polynomial, built here by the
// three-term recurrence in l and normalised numerically by exact sphere integrals.
// The coupling tensor of (l1, l2, l3) is the unit-norm vector annihilated by the
// three infinitesimal rotation generators acting on l1 (x) l2 (x) l3 (it is unique up
// to sign), signed so that its first entry above 1e-9 in row-major (m_in, m_sh,
// m_out) order is positive, then multiplied by sqrt(2 l3 + 1).
//
// Output: a C++17 header of constexpr tables (argv[1]).

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <vector>
#include <algorithm>
#include <string>

static const int LMAX = 3;
static const int D = LMAX + 1;  // exponents 0..LMAX per variable

struct Poly {  // dense coefficients c[a][b][c] of x^a y^b z^c, total degree <= LMAX
  double c[D][D][D];
  Poly() { for (int a = 0; a < D; ++a) for (int b = 0; b < D; ++b) for (int k = 0; k < D; ++k) c[a][b][k] = 0; }
};

static Poly add(const Poly& p, const Poly& q, double s = 1.0) {
  Poly r;
  for (int a = 0; a < D; ++a) for (int b = 0; b < D; ++b) for (int k = 0; k < D; ++k)
    r.c[a][b][k] = p.c[a][b][k] + s * q.c[a][b][k];
  return r;
}
static Poly scale(const Poly& p, double s) { Poly r; return add(r, p, s); }
static Poly mul(const Poly& p, const Poly& q) {
  Poly r;
  for (int a = 0; a < D; ++a) for (int b = 0; b < D; ++b) for (int k = 0; k < D; ++k) {
    if (p.c[a][b][k] == 0) continue;
    for (int a2 = 0; a2 < D; ++a2) for (int b2 = 0; b2 < D; ++b2) for (int k2 = 0; k2 < D; ++k2) {
      if (q.c[a2][b2][k2] == 0) continue;
      if (a + a2 >= D || b + b2 >= D || k + k2 >= D) { fprintf(stderr, "degree overflow\n"); exit(2); }
      r.c[a + a2][b + b2][k + k2] += p.c[a][b][k] * q.c[a2][b2][k2];
    }
  }
  return r;
}
static Poly mono(int a, int b, int k, double v = 1.0) { Poly p; p.c[a][b][k] = v; return p; }

// d/dx_var of a polynomial (var 0,1,2); degree never grows
static Poly deriv(const Poly& p, int var) {
  Poly r;
  for (int a = 0; a < D; ++a) for (int b = 0; b < D; ++b) for (int k = 0; k < D; ++k) {
    double v = p.c[a][b][k];
    if (v == 0) continue;
    int e[3] = {a, b, k};
    if (e[var] == 0) continue;
    double f = v * e[var];
    e[var] -= 1;
    r.c[e[0]][e[1]][e[2]] += f;
  }
  return r;
}

// Exact integral of x^a y^b z^c over the unit sphere.
static double sphere_int(int a, int b, int c) {
  if ((a & 1) || (b & 1) || (c & 1)) return 0.0;
  return 2.0 * std::tgamma((a + 1) / 2.0) * std::tgamma((b + 1) / 2.0) * std::tgamma((c + 1) / 2.0) /
         std::tgamma((a + b + c + 3) / 2.0);
}
static double inner(const Poly& p, const Poly& q) {  // (1/4pi) int p q
  double s = 0;
  for (int a = 0; a < D; ++a) for (int b = 0; b < D; ++b) for (int k = 0; k < D; ++k) {
    if (p.c[a][b][k] == 0) continue;
    for (int a2 = 0; a2 < D; ++a2) for (int b2 = 0; b2 < D; ++b2) for (int k2 = 0; k2 < D; ++k2) {
      if (q.c[a2][b2][k2] == 0) continue;
      // products may exceed LMAX per variable: integrate directly
      s += p.c[a][b][k] * q.c[a2][b2][k2] * sphere_int(a + a2, b + b2, k + k2);
    }
  }
  return s / (4.0 * M_PI);
}

// Y[l][k] as polynomials
static std::vector<std::vector<Poly>> build_sh() {
  std::vector<std::vector<Poly>> Y(LMAX + 1);
  for (int l = 0; l <= LMAX; ++l) Y[l].resize(2 * l + 1);
  // (x + i y)^m
  std::vector<Poly> re(LMAX + 1), im(LMAX + 1);
  re[0] = mono(0, 0, 0);
  for (int m = 1; m <= LMAX; ++m) {
    re[m] = add(mul(re[m - 1], mono(1, 0, 0)), mul(im[m - 1], mono(0, 1, 0)), -1.0);
    im[m] = add(mul(re[m - 1], mono(0, 1, 0)), mul(im[m - 1], mono(1, 0, 0)));
  }
  for (int m = 0; m <= LMAX; ++m) {
    // Q_l^m(z) for l = m..LMAX: Q_m^m = (2m-1)!!, Q_{m+1}^m = (2m+1) z Q_m^m,
    // (l-m) Q_l^m = (2l-1) z Q_{l-1}^m - (l+m-1) Q_{l-2}^m
    std::vector<Poly> Q(LMAX + 1);
    double dfact = 1.0;
    for (int t = 2 * m - 1; t > 1; t -= 2) dfact *= t;
    Q[m] = mono(0, 0, 0, dfact);
    if (m + 1 <= LMAX) Q[m + 1] = mul(mono(0, 0, 1, 2.0 * m + 1), Q[m]);
    for (int l = m + 2; l <= LMAX; ++l)
      Q[l] = scale(add(mul(mono(0, 0, 1, 2.0 * l - 1), Q[l - 1]), Q[l - 2], -(l + m - 1.0)), 1.0 / (l - m));
    for (int l = m; l <= LMAX; ++l) {
      if (m == 0) {
        Y[l][l] = Q[l];
      } else {
        Y[l][l + m] = mul(Q[l], re[m]);
        Y[l][l - m] = mul(Q[l], im[m]);
      }
    }
  }
  for (int l = 0; l <= LMAX; ++l)
    for (int k = 0; k < 2 * l + 1; ++k) {
      double n2 = inner(Y[l][k], Y[l][k]);
      Y[l][k] = scale(Y[l][k], 1.0 / std::sqrt(n2));
    }
  return Y;
}

// generators G_k (k = x, y, z) in the basis Y[l]: L_k Y_b = sum_a G[a][b] Y_a
static void generators(const std::vector<Poly>& Yl, std::vector<double> G[3]) {
  int d = (int)Yl.size();
  for (int k = 0; k < 3; ++k) G[k].assign(d * d, 0.0);
  for (int b = 0; b < d; ++b) {
    const Poly& p = Yl[b];
    Poly dx = deriv(p, 0), dy = deriv(p, 1), dz = deriv(p, 2);
    Poly L[3];
    L[0] = add(mul(mono(0, 1, 0), dz), mul(mono(0, 0, 1), dy), -1.0);  // y d/dz - z d/dy
    L[1] = add(mul(mono(0, 0, 1), dx), mul(mono(1, 0, 0), dz), -1.0);  // z d/dx - x d/dz
    L[2] = add(mul(mono(1, 0, 0), dy), mul(mono(0, 1, 0), dx), -1.0);  // x d/dy - y d/dx
    for (int k = 0; k < 3; ++k) {
      Poly resid = L[k];
      for (int a = 0; a < d; ++a) {
        double g = inner(Yl[a], L[k]);  // basis is orthonormal under inner()
        G[k][a * d + b] = g;
        resid = add(resid, Yl[a], -g);
      }
      if (std::fabs(inner(resid, resid)) > 1e-12) { fprintf(stderr, "generator not closed\n"); exit(3); }
    }
  }
}

// Unit null vector of M (rows x cols) by Gaussian elimination with full pivoting.
static std::vector<double> null_vector(std::vector<double> M, int rows, int cols) {
  std::vector<int> colperm(cols);
  for (int i = 0; i < cols; ++i) colperm[i] = i;
  int rank = 0;
  for (int piv = 0; piv < cols && piv < rows; ++piv) {
    int br = -1, bc = -1;
    double best = 0;
    for (int r = piv; r < rows; ++r)
      for (int c = piv; c < cols; ++c)
        if (std::fabs(M[r * cols + c]) > best) { best = std::fabs(M[r * cols + c]); br = r; bc = c; }
    if (best < 1e-9) break;
    if (br != piv) for (int c = 0; c < cols; ++c) std::swap(M[br * cols + c], M[piv * cols + c]);
    if (bc != piv) { for (int r = 0; r < rows; ++r) std::swap(M[r * cols + bc], M[r * cols + piv]); std::swap(colperm[bc], colperm[piv]); }
    double p = M[piv * cols + piv];
    for (int c = piv; c < cols; ++c) M[piv * cols + c] /= p;
    for (int r = 0; r < rows; ++r) {
      if (r == piv) continue;
      double f = M[r * cols + piv];
      if (f == 0) continue;
      for (int c = piv; c < cols; ++c) M[r * cols + c] -= f * M[piv * cols + c];
    }
    ++rank;
  }
  if (rank != cols - 1) { fprintf(stderr, "null space dimension %d != 1\n", cols - rank); exit(4); }
  // reduced form: x_piv + M[piv][cols-1] * x_free = 0, free variable = last permuted column
  std::vector<double> v(cols, 0.0);
  v[colperm[cols - 1]] = 1.0;
  for (int r = 0; r < rank; ++r) v[colperm[r]] = -M[r * cols + (cols - 1)];
  double n = 0;
  for (double t : v) n += t * t;
  n = std::sqrt(n);
  for (double& t : v) t /= n;
  return v;
}

int main(int argc, char** argv) {
  if (argc < 2) { fprintf(stderr, "usage: gen_tables out.inc\n"); return 1; }
  auto Y = build_sh();
  std::vector<std::vector<double>> G(LMAX + 1);
  std::vector<double> Gl[LMAX + 1][3];
  for (int l = 0; l <= LMAX; ++l) generators(Y[l], Gl[l]);

  FILE* f = fopen(argv[1], "w");
  if (!f) return 1;
  fprintf(f, "// Generated by gen_tables.cpp at build time. Do not edit.\n");
  fprintf(f, "#pragma once\n#define TPC_LMAX %d\nnamespace tpc_tab {\n", LMAX);

  // ---- spherical harmonics: for block l, terms (k, a, b, c, coef)
  for (int l = 0; l <= LMAX; ++l) {
    std::vector<int> tk, ta, tb, tc;
    std::vector<double> tv;
    for (int k = 0; k < 2 * l + 1; ++k)
      for (int a = 0; a < D; ++a) for (int b = 0; b < D; ++b) for (int c = 0; c < D; ++c) {
        double v = Y[l][k].c[a][b][c];
        if (std::fabs(v) < 1e-13) continue;
        tk.push_back(k); ta.push_back(a); tb.push_back(b); tc.push_back(c); tv.push_back(v);
      }
    int n = (int)tk.size();
    fprintf(f, "struct SH%d {\n  static constexpr int nterm = %d;\n", l, n);
    auto emit_int = [&](const char* name, const std::vector<int>& v) {
      fprintf(f, "  __host__ __device__ static constexpr int %s(int t) { constexpr int a[] = {", name);
      for (int i = 0; i < n; ++i) fprintf(f, "%s%d", i ? "," : "", v[i]);
      fprintf(f, "}; return a[t]; }\n");
    };
    emit_int("k", tk); emit_int("ex", ta); emit_int("ey", tb); emit_int("ez", tc);
    fprintf(f, "  __host__ __device__ static constexpr float coef(int t) { constexpr float a[] = {");
    for (int i = 0; i < n; ++i) fprintf(f, "%s%.9ef", i ? "," : "", tv[i]);
    fprintf(f, "}; return a[t]; }\n");
    fprintf(f, "  static constexpr double coef_d(int t) { constexpr double a[] = {");
    for (int i = 0; i < n; ++i) fprintf(f, "%s%.17e", i ? "," : "", tv[i]);
    fprintf(f, "}; return a[t]; }\n};\n");
  }
  fprintf(f, "template <int L> struct SH;\n");
  for (int l = 0; l <= LMAX; ++l) fprintf(f, "template <> struct SH<%d> : SH%d {};\n", l, l);

  // ---- coupling tensors
  fprintf(f, "template <int L1, int L2, int L3> struct CG { static constexpr int nnz = 0; };\n");
  int ntrip = 0;
  std::string table = "";
  for (int l1 = 0; l1 <= LMAX; ++l1)
    for (int l2 = 0; l2 <= LMAX; ++l2)
      for (int l3 = std::abs(l1 - l2); l3 <= std::min(LMAX, l1 + l2); ++l3) {
        int d1 = 2 * l1 + 1, d2 = 2 * l2 + 1, d3 = 2 * l3 + 1, n = d1 * d2 * d3;
        std::vector<double> M((size_t)3 * n * n, 0.0);
        for (int k = 0; k < 3; ++k)
          for (int a = 0; a < d1; ++a) for (int b = 0; b < d2; ++b) for (int c = 0; c < d3; ++c) {
            int row = k * n + (a * d2 + b) * d3 + c;
            for (int a2 = 0; a2 < d1; ++a2) M[(size_t)row * n + (a2 * d2 + b) * d3 + c] += Gl[l1][k][a * d1 + a2];
            for (int b2 = 0; b2 < d2; ++b2) M[(size_t)row * n + (a * d2 + b2) * d3 + c] += Gl[l2][k][b * d2 + b2];
            for (int c2 = 0; c2 < d3; ++c2) M[(size_t)row * n + (a * d2 + b) * d3 + c2] += Gl[l3][k][c * d3 + c2];
          }
        std::vector<double> w = null_vector(M, 3 * n, n);
        int first = 0;
        while (first < n && std::fabs(w[first]) <= 1e-9) ++first;
        double s = (w[first] < 0 ? -1.0 : 1.0) * std::sqrt((double)d3);
        std::vector<int> im, iy, io;
        std::vector<double> v;
        for (int a = 0; a < d1; ++a) for (int b = 0; b < d2; ++b) for (int c = 0; c < d3; ++c) {
          double t = w[(a * d2 + b) * d3 + c] * s;
          if (std::fabs(t) < 1e-12) continue;
          im.push_back(a); iy.push_back(b); io.push_back(c); v.push_back(t);
        }
        int nz = (int)v.size();
        fprintf(f, "template <> struct CG<%d, %d, %d> {\n  static constexpr int nnz = %d;\n", l1, l2, l3, nz);
        auto emit_int = [&](const char* name, const std::vector<int>& vv) {
          fprintf(f, "  __host__ __device__ static constexpr int %s(int t) { constexpr int a[] = {", name);
          for (int i = 0; i < nz; ++i) fprintf(f, "%s%d", i ? "," : "", vv[i]);
          fprintf(f, "}; return a[t]; }\n");
        };
        emit_int("mi", im); emit_int("my", iy); emit_int("mo", io);
        fprintf(f, "  __host__ __device__ static constexpr float val(int t) { constexpr float a[] = {");
        for (int i = 0; i < nz; ++i) fprintf(f, "%s%.9ef", i ? "," : "", v[i]);
        fprintf(f, "}; return a[t]; }\n");
        fprintf(f, "  static constexpr double val_d(int t) { constexpr double a[] = {");
        for (int i = 0; i < nz; ++i) fprintf(f, "%s%.17e", i ? "," : "", v[i]);
        fprintf(f, "}; return a[t]; }\n};\n");
        char buf[64];
        snprintf(buf, sizeof buf, "  {%d, %d, %d},\n", l1, l2, l3);
        table += buf;
        ++ntrip;
      }
  fprintf(f, "static constexpr int NTRIPLES = %d;\n", ntrip);
  fprintf(f, "static constexpr int TRIPLES[NTRIPLES][3] = {\n%s};\n", table.c_str());
  fprintf(f, "}  // namespace tpc_tab\n");
  fclose(f);
  return 0;
}
