// Node-level contractions and graph utilities.
//
//  * k_gemm / k_gemm_reduce -- the channel contractions of Sobek section 4
//    (m = S A, eq. 35; S_bar = m_bar A^T and A_bar = S^T m_bar, eq. 36; their
//    double-backward forms, eqs. 37-39; and the mirrored source forms x_bar = X A^T,
//    A_bar = x^T X) on operands addressed through two-level affine index maps, so
//    that node rows of the ir_mul tensors, the weight matrix and the workspace
//    states are read in place.  fp32 SIMT tiles; split-K partials are reduced in a
//    fixed order.
//  * k_pos_finish -- position gradient: pos_bar[n] = sum_{e out of n} g_e
//    - sum_{e into n} g_e, in source-CSR and receiver-CSR order (no atomics).
//  * CSR transpose (stable counting sort by source) and the graph validator.
#include <cuda_runtime.h>
#include "internal.h"

namespace tpc {

__device__ __forceinline__ long long ix(const Idx2& f, int i) {
  return (long long)(i / f.d) * f.s1 + (long long)(i % f.d) * f.s2;
}

constexpr int GBM = 64, GBN = 64, GBK = 16;

__global__ void __launch_bounds__(256) k_gemm(const __grid_constant__ GemmBatch g) {
  __shared__ float As[GBK][GBM + 4];
  __shared__ float Bs[GBK][GBN + 4];
  const int tile = blockIdx.x;
  int pi = 0;
  while (pi + 1 < g.n_problems && g.pr[pi + 1].tile0 <= tile) ++pi;
  const GemmProblem& P = g.pr[pi];
  const int lt = tile - P.tile0;
  const int tn = (P.N + GBN - 1) / GBN;
  const int m0 = (lt / tn) * GBM, n0 = (lt % tn) * GBN;
  const int split = blockIdx.y;
  const int kper = (P.Ktot + g.splits - 1) / g.splits;
  const int kb = split * kper, ke = min(P.Ktot, kb + kper);
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  int kbase = 0;
  for (int si = 0; si < P.nseg; ++si) {
    const GemmSeg& S = g.sg[P.seg0 + si];
    const int lo = max(kb - kbase, 0), hi = min(ke - kbase, S.K);
    kbase += S.K;
    for (int k0 = lo; k0 < hi; k0 += GBK) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int idx = tid + r * 256;
        const int kk = idx & 15, mm = idx >> 4;
        const int m = m0 + mm, k = k0 + kk;
        As[kk][mm] = (m < P.M && k < hi) ? __ldg(S.A + ix(S.Am, m) + ix(S.Ak, k)) : 0.f;
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int idx = tid + r * 256;
        const int nn = idx & 63, kk = idx >> 6;
        const int n = n0 + nn, k = k0 + kk;
        Bs[kk][nn] = (n < P.N && k < hi) ? __ldg(S.B + ix(S.Bk, k) + ix(S.Bn, n)) : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < GBK; ++kk) {
        float av[4], bv[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) { av[t] = As[kk][ty * 4 + t]; bv[t] = Bs[kk][tx * 4 + t]; }
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(av[p], bv[q], acc[p][q]);
      }
      __syncthreads();
    }
  }
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int m = m0 + ty * 4 + p;
    if (m >= P.M) continue;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int n = n0 + tx * 4 + q;
      if (n >= P.N) continue;
      if (g.splits > 1) {
        g.partial[P.part_off + ((long long)split * P.M + m) * P.N + n] = acc[p][q];
      } else {
        float* c = P.C + ix(P.Cm, m) + ix(P.Cn, n);
        *c = g.accumulate ? *c + acc[p][q] : acc[p][q];
      }
    }
  }
}

// one thread per output element of every problem; fixed-order sum over splits
__global__ void k_gemm_reduce(const __grid_constant__ GemmBatch g, long long total) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= total) return;
  int pi = 0;
  long long base = 0;
  while (pi < g.n_problems && t >= base + (long long)g.pr[pi].M * g.pr[pi].N) {
    base += (long long)g.pr[pi].M * g.pr[pi].N;
    ++pi;
  }
  const GemmProblem& P = g.pr[pi];
  const long long loc = t - base;
  const long long mn = (long long)P.M * P.N;
  const int m = (int)(loc / P.N), n = (int)(loc % P.N);
  float s = 0.f;
  for (int sp = 0; sp < g.splits; ++sp) s += g.partial[P.part_off + sp * mn + loc];
  float* c = P.C + ix(P.Cm, m) + ix(P.Cn, n);
  *c = g.accumulate ? *c + s : s;
}

cudaError_t launch_gemm_simt(GemmBatch& g, cudaStream_t s) {
  int tiles = 0;
  long long elems = 0;
  for (int p = 0; p < g.n_problems; ++p) {
    g.pr[p].tile0 = tiles;
    g.pr[p].part_off = elems * g.splits;
    tiles += ((g.pr[p].M + GBM - 1) / GBM) * ((g.pr[p].N + GBN - 1) / GBN);
    elems += (long long)g.pr[p].M * g.pr[p].N;
  }
  g.total_tiles = tiles;
  if (tiles == 0) return cudaSuccess;
  k_gemm<<<dim3(tiles, g.splits), 256, 0, s>>>(g);
  if (g.splits > 1) k_gemm_reduce<<<(unsigned)((elems + 255) / 256), 256, 0, s>>>(g, elems);
  return cudaGetLastError();
}

__device__ int g_tpc_error = 0;

int* device_error_word() {
  static int* p = nullptr;
  if (!p) cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_tpc_error);
  return p;
}

cudaError_t launch_gemm(GemmBatch& g, cudaStream_t s) { return launch_gemm_tc(g, device_error_word(), s); }

cudaError_t read_and_clear_device_error(int* host_value) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(host_value, g_tpc_error, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_tpc_error, &zero, sizeof(int));
}

__global__ void k_reduce_partials(const float* __restrict__ partial, int n_parts, long long n,
                                  float* out, int accumulate) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n) return;
  float s = 0.f;
  for (int p = 0; p < n_parts; ++p) s += partial[(long long)p * n + t];
  out[t] = accumulate ? out[t] + s : s;
}

cudaError_t launch_reduce_partials(const float* partial, int n_parts, long long n, float* out,
                                   int accumulate, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  k_reduce_partials<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(partial, n_parts, n, out, accumulate);
  return cudaGetLastError();
}

__global__ void k_pos_finish(int N, const int* __restrict__ row_ptr, const int* __restrict__ t_ptr,
                             const int* __restrict__ t_eid, const float4* __restrict__ gbuf,
                             float* grad_pos) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  float x = 0.f, y = 0.f, z = 0.f;
  for (int k = t_ptr[n]; k < t_ptr[n + 1]; ++k) {
    const float4 g = gbuf[t_eid[k]];
    x += g.x; y += g.y; z += g.z;
  }
  for (int e = row_ptr[n]; e < row_ptr[n + 1]; ++e) {
    const float4 g = gbuf[e];
    x -= g.x; y -= g.y; z -= g.z;
  }
  grad_pos[3 * n] = x;
  grad_pos[3 * n + 1] = y;
  grad_pos[3 * n + 2] = z;
}

cudaError_t launch_pos_finish(int N, const int* row_ptr, const int* t_ptr, const int* t_eid,
                              const float4* gbuf, float* grad_pos, cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  k_pos_finish<<<(N + 255) / 256, 256, 0, s>>>(N, row_ptr, t_ptr, t_eid, gbuf, grad_pos);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// CSR transpose: stable grouping of edge ids by source
// ---------------------------------------------------------------------------

__global__ void k_count_src(int E, const int* __restrict__ src, int* t_ptr) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < E) atomicAdd(t_ptr + src[e] + 1, 1);  // integer counts: order-independent
}

// inclusive scan of t_ptr[1..N] in one block; t_ptr[0] = 0; cursor = exclusive copy
__global__ void k_scan(int N, int* t_ptr, int* cursor) {
  __shared__ int buf[1024];
  __shared__ int carry;
  if (threadIdx.x == 0) { carry = 0; t_ptr[0] = 0; }
  __syncthreads();
  for (int base = 0; base < N; base += 1024) {
    const int i = base + threadIdx.x;
    int v = (i < N) ? t_ptr[i + 1] : 0;
    buf[threadIdx.x] = v;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
      const int add = threadIdx.x >= o ? buf[threadIdx.x - o] : 0;
      __syncthreads();
      buf[threadIdx.x] += add;
      __syncthreads();
    }
    if (i < N) {
      const int incl = buf[threadIdx.x] + carry;
      t_ptr[i + 1] = incl;
      cursor[i] = incl - v;
    }
    __syncthreads();
    if (threadIdx.x == 1023) carry += buf[1023];
    __syncthreads();
  }
}

__global__ void k_scatter_src(int E, const int* __restrict__ src, int* cursor, int* t_eid) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < E) t_eid[atomicAdd(cursor + src[e], 1)] = e;
}

// Sort each source row by edge id (rows are short; insertion sort) and record the
// receiver of every listed edge (binary search in row_ptr).
__global__ void k_sort_rows(int N, const int* __restrict__ row_ptr, const int* __restrict__ t_ptr,
                            int* t_eid, int* t_dst) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const int b = t_ptr[n], e = t_ptr[n + 1];
  for (int k = b + 1; k < e; ++k) {
    const int v = t_eid[k];
    int q = k - 1;
    while (q >= b && t_eid[q] > v) { t_eid[q + 1] = t_eid[q]; --q; }
    t_eid[q + 1] = v;
  }
  for (int k = b; k < e; ++k) {
    const int id = t_eid[k];
    int lo = 0, hi = N;  // last i with row_ptr[i] <= id
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (row_ptr[mid] <= id) lo = mid; else hi = mid;
    }
    t_dst[k] = lo;
  }
}

cudaError_t launch_csr_transpose(int N, int E, const int* row_ptr, const int* src, int* t_ptr,
                                 int* t_eid, int* t_dst, int* cursor, cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(t_ptr, 0, sizeof(int) * (size_t)(N + 1), s);
  if (err != cudaSuccess) return err;
  if (E > 0) k_count_src<<<(E + 255) / 256, 256, 0, s>>>(E, src, t_ptr);
  if (N > 0) k_scan<<<1, 1024, 0, s>>>(N, t_ptr, cursor);
  if (E > 0) k_scatter_src<<<(E + 255) / 256, 256, 0, s>>>(E, src, cursor, t_eid);
  if (N > 0) k_sort_rows<<<(N + 127) / 128, 128, 0, s>>>(N, row_ptr, t_ptr, t_eid, t_dst);
  return cudaGetLastError();
}

// Receiver order for load balance: within each chunk of `chunk` nodes (one CTA per
// chunk), the nodes grouped by in-degree class floor(log2(degree + 1)), heaviest class
// first (longest work first).  The order inside a class is arbitrary; results do not
// depend on it, since every receiver's output is computed independently.
__global__ void k_degree_order(int N, const int* __restrict__ row_ptr, int chunk, int* __restrict__ order) {
  constexpr int NB = 32;
  __shared__ int count[NB], cursor[NB];
  const int n0 = blockIdx.x * chunk, n1 = min(N, n0 + chunk);
  if (threadIdx.x < NB) count[threadIdx.x] = 0;
  __syncthreads();
  for (int n = n0 + threadIdx.x; n < n1; n += blockDim.x) {
    const int d = __ldg(row_ptr + n + 1) - __ldg(row_ptr + n);
    atomicAdd(&count[31 - __clz(d + 1)], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int off = n0;
    for (int b = NB - 1; b >= 0; --b) { cursor[b] = off; off += count[b]; }
  }
  __syncthreads();
  for (int n = n0 + threadIdx.x; n < n1; n += blockDim.x) {
    const int d = __ldg(row_ptr + n + 1) - __ldg(row_ptr + n);
    order[atomicAdd(&cursor[31 - __clz(d + 1)], 1)] = n;
  }
}

cudaError_t launch_degree_order(int N, const int* row_ptr, int chunk, int* order, cudaStream_t s) {
  if (N <= 0 || chunk <= 0) return cudaSuccess;
  k_degree_order<<<(unsigned)((N + chunk - 1) / chunk), 256, 0, s>>>(N, row_ptr, chunk, order);
  return cudaGetLastError();
}

// Layout conversion of node rows: element (m, u) of block b is at off + m*C + u in
// ir_mul and at off + u*(2l+1) + m in mul_ir.  One thread per source element (reads
// coalesced).
__global__ void k_layout_convert(long long total, int dim, const __grid_constant__ LayoutMap M, int to_ir_mul,
                                 const float* __restrict__ src, float* __restrict__ dst) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= total) return;
  const long long row = t / dim;
  const int c = (int)(t - row * dim);
  int b = 0;
  while (b + 1 < M.n && M.off[b + 1] <= c) ++b;
  const int local = c - M.off[b], R = 2 * M.l[b] + 1, C = M.mul[b];
  int d;
  if (to_ir_mul) {   // source mul_ir: local = u*R + m
    const int u = local / R, m = local - u * R;
    d = M.off[b] + m * C + u;
  } else {           // source ir_mul: local = m*C + u
    const int m = local / C, u = local - m * C;
    d = M.off[b] + u * R + m;
  }
  dst[row * dim + d] = src[t];
}

cudaError_t launch_layout_convert(int N, int dim, const LayoutMap& M, int to_ir_mul, const float* src,
                                  float* dst, cudaStream_t s) {
  const long long total = (long long)N * dim;
  if (total <= 0) return cudaSuccess;
  k_layout_convert<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(total, dim, M, to_ir_mul, src, dst);
  return cudaGetLastError();
}

__global__ void k_validate(int N, int E, const int* __restrict__ row_ptr,
                           const int* __restrict__ src, int* err) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t <= N) {
    const int v = row_ptr[t];
    if (t == 0 && v != 0) atomicCAS(err, 0, 1);
    if (t == N && v != E) atomicCAS(err, 0, 1);
    if (v < 0 || v > E) atomicCAS(err, 0, 1);
    if (t < N && row_ptr[t + 1] < v) atomicCAS(err, 0, 2);
  }
  if (t < E) {
    const int j = src[t];
    if (j < 0 || j >= N) atomicCAS(err, 0, 3);
  }
}

cudaError_t launch_validate_graph(int N, int E, const int* row_ptr, const int* src, int* err,
                                  cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  const long long n = (long long)(N > E ? N : E) + 1;
  k_validate<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(N, E, row_ptr, src, err);
  return cudaGetLastError();
}

}  // namespace tpc
