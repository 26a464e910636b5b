// Graph utilities, the position-gradient sums and the library's device error word.
// (The channel contractions themselves run on the tensor cores, k_gemm_tc.cu.)
//
//  * k_pos_window -- position gradient: pos_bar[n] = sum_{e out of n} g_e
//    - sum_{e into n} g_e, one bounded staging window of g_e at a time, in source-CSR
//    and receiver-CSR order (no atomics; a per-node cursor walks the source rows).
//  * CSR transpose (stable counting sort by source) and the graph validator.
#include <cuda_runtime.h>
#include <mutex>
#include "launch.h"

namespace tpc {

__device__ int g_tpc_error = 0;

// Address of g_tpc_error on the current device, looked up once per device (kept for the
// life of the process, like the static scratch of the allocation-free forward).
int* device_error_word() {
  static std::mutex mu;
  static int* addr[256] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return nullptr;
  std::lock_guard<std::mutex> g(mu);
  if (!addr[dev]) {
    int* p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_tpc_error) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
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

// One staging window [w0, w1) of g_e (stored at gbuf[e - w0]): every node adds the g_e of
// its outgoing edges inside the window and subtracts those of its incoming edges inside
// the window (a sub-range of its receiver row).  The windows of a pass cover the edge ids
// in increasing order, and t_eid is increasing within a source, so a node's outgoing
// edges in the window are the next run of its t_eid row: cursor[n] (initialised to
// t_ptr[n]) marks where the run starts and is advanced past it.  Windows are applied in
// a fixed order, so the sums are deterministic.
__global__ void k_pos_window(int N, const int* __restrict__ row_ptr, const int* __restrict__ t_ptr,
                             const int* __restrict__ t_eid, const float4* __restrict__ gbuf, EdgeWindow win,
                             int* cursor, float* grad_pos) {
  const long long lo = __ldg(row_ptr + win.n0), hi = __ldg(row_ptr + win.n0 + win.n_nodes);
  const long long a = lo + (long long)win.index * win.size;
  const int w0 = (int)min(a, hi), w1 = (int)min(a + win.size, hi);
  if (w0 >= w1) return;
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  float x = 0.f, y = 0.f, z = 0.f;
  bool touched = false;
  const int kend = __ldg(t_ptr + n + 1);
  int k = cursor[n];
  for (; k < kend; ++k) {
    const int e = __ldg(t_eid + k);
    if (e >= w1) break;
    const float4 g = gbuf[e - w0];
    x += g.x; y += g.y; z += g.z;
    touched = true;
  }
  if (touched) cursor[n] = k;
  const int eb = max(__ldg(row_ptr + n), w0), ee = min(__ldg(row_ptr + n + 1), w1);
  for (int e = eb; e < ee; ++e) {
    const float4 g = gbuf[e - w0];
    x -= g.x; y -= g.y; z -= g.z;
    touched = true;
  }
  if (touched) {   // nodes without an edge in the window keep their sums untouched
    grad_pos[3 * n] += x;
    grad_pos[3 * n + 1] += y;
    grad_pos[3 * n + 2] += z;
  }
}

cudaError_t launch_pos_window(int N, const int* row_ptr, const int* t_ptr, const int* t_eid,
                              const float4* gbuf, EdgeWindow win, int* cursor, float* grad_pos, cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  k_pos_window<<<(N + 255) / 256, 256, 0, s>>>(N, row_ptr, t_ptr, t_eid, gbuf, win, cursor, grad_pos);
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
