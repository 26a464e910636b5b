// Spatial node order (Morton / Z-order of the positions) and its application to a
// receiver-sorted CSR and to node arrays; declared in include/tpconv_graph.h.
//
// The order is unique: keys (morton_code << 32 | node_id) are distinct, so any correct
// sort gives the same permutation.  The sort is a bitonic network over the keys padded to
// a power of two (one launch per merge step; preprocessing, run once per graph).
#include <cuda_runtime.h>
#include <stdint.h>

#include "tpconv_graph.h"

namespace {

constexpr int kThreads = 256;
constexpr unsigned long long kPad = ~0ull;

size_t pow2_at_least(long long n) {
  size_t p = 1;
  while ((long long)p < n) p <<= 1;
  return p;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// bounding box of pos (one CTA; min / max are exact, so the result is order-independent)
__global__ void k_bbox(int N, const float* __restrict__ pos, float* box) {
  __shared__ float lo[3][kThreads], hi[3][kThreads];
  float l[3] = {3.4e38f, 3.4e38f, 3.4e38f}, h[3] = {-3.4e38f, -3.4e38f, -3.4e38f};
  for (int i = threadIdx.x; i < N; i += blockDim.x)
    for (int a = 0; a < 3; ++a) {
      const float v = pos[3 * (long long)i + a];
      l[a] = fminf(l[a], v);
      h[a] = fmaxf(h[a], v);
    }
  for (int a = 0; a < 3; ++a) {
    lo[a][threadIdx.x] = l[a];
    hi[a][threadIdx.x] = h[a];
  }
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if ((int)threadIdx.x < o)
      for (int a = 0; a < 3; ++a) {
        lo[a][threadIdx.x] = fminf(lo[a][threadIdx.x], lo[a][threadIdx.x + o]);
        hi[a][threadIdx.x] = fmaxf(hi[a][threadIdx.x], hi[a][threadIdx.x + o]);
      }
    __syncthreads();
  }
  if (threadIdx.x < 3) {
    box[threadIdx.x] = lo[threadIdx.x][0];
    box[3 + threadIdx.x] = hi[threadIdx.x][0];
  }
}

// 10 bits of v spread to every third bit
__device__ __forceinline__ unsigned spread3(unsigned v) {
  unsigned r = 0;
  for (int b = 0; b < 10; ++b) r |= ((v >> b) & 1u) << (3 * b);
  return r;
}

__global__ void k_morton_keys(int N, long long n_pad, const float* __restrict__ pos, const float* __restrict__ box,
                              unsigned long long* keys) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_pad) return;
  if (i >= N) {
    keys[i] = kPad;
    return;
  }
  unsigned c[3];
  for (int a = 0; a < 3; ++a) {
    const float lo = box[a], ext = box[3 + a] - box[a];
    const float scale = ext > 0.f ? 1024.f / ext : 0.f;
    const float t = floorf((pos[3 * i + a] - lo) * scale);
    c[a] = t <= 0.f ? 0u : (t >= 1023.f ? 1023u : (unsigned)t);
  }
  const unsigned code = spread3(c[0]) | (spread3(c[1]) << 1) | (spread3(c[2]) << 2);
  keys[i] = ((unsigned long long)code << 32) | (unsigned long long)(unsigned)i;
}

// one compare-exchange step (k: size of the bitonic sequences being merged, j: distance)
__global__ void k_bitonic_step(unsigned long long* keys, long long n_pad, long long j, long long k) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_pad) return;
  const long long l = i ^ j;
  if (l <= i) return;
  const unsigned long long a = keys[i], b = keys[l];
  const bool ascending = (i & k) == 0;
  if (ascending ? (a > b) : (a < b)) {
    keys[i] = b;
    keys[l] = a;
  }
}

__global__ void k_keys_to_perm(int N, const unsigned long long* __restrict__ keys, int32_t* perm) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < N) perm[i] = (int32_t)(keys[i] & 0xffffffffull);
}

__global__ void k_inverse_and_degrees(int N, const int32_t* __restrict__ perm, const int32_t* __restrict__ row_ptr,
                                      int32_t* inv, int32_t* row_ptr_out) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k == 0) row_ptr_out[0] = 0;
  if (k >= N) return;
  const int old = perm[k];
  const bool ok = old >= 0 && old < N;
  if (ok) inv[old] = k;
  row_ptr_out[k + 1] = ok ? row_ptr[old + 1] - row_ptr[old] : 0;
}

// inclusive scan of a[1..N] in place (one CTA of 1024 threads)
__global__ void k_scan_inplace(int N, int32_t* a) {
  __shared__ int32_t buf[1024];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < N; base += 1024) {
    const int i = base + threadIdx.x;
    buf[threadIdx.x] = i < N ? a[i + 1] : 0;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
      const int32_t add = (int)threadIdx.x >= o ? buf[threadIdx.x - o] : 0;
      __syncthreads();
      buf[threadIdx.x] += add;
      __syncthreads();
    }
    if (i < N) a[i + 1] = buf[threadIdx.x] + carry;
    __syncthreads();
    if (threadIdx.x == 1023) carry += buf[1023];
    __syncthreads();
  }
}

// one warp per new receiver: copy the old row, relabelling sources
__global__ void k_copy_rows(int N, int E, const int32_t* __restrict__ perm, const int32_t* __restrict__ row_ptr,
                            const int32_t* __restrict__ src, const int32_t* __restrict__ inv,
                            const int32_t* __restrict__ row_ptr_out, int32_t* src_out) {
  const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= N) return;
  const int old = perm[w];
  if (old < 0 || old >= N) return;
  const int b = row_ptr[old], len = row_ptr[old + 1] - b, o = row_ptr_out[w];
  for (int t = lane; t < len; t += 32) {
    const int s = src[b + t];
    if (o + t < E && s >= 0 && s < N) src_out[o + t] = inv[s];
  }
}

__global__ void k_gather_rows(long long rows, long long width, const float* __restrict__ in,
                              const int32_t* __restrict__ perm, float* out) {
  const long long r = blockIdx.y * (long long)gridDim.x + blockIdx.x;
  if (r >= rows) return;
  const int p = perm[r];
  const bool ok = p >= 0 && p < rows;
  for (long long c = threadIdx.x; c < width; c += blockDim.x)
    out[r * width + c] = ok ? in[(long long)p * width + c] : 0.f;
}

tpconv_status launched() {
  return cudaGetLastError() == cudaSuccess ? TPCONV_OK : TPCONV_ERR_CUDA;
}

}  // namespace

extern "C" {

tpconv_status tpconv_spatial_order_workspace_bytes(int64_t N, size_t* bytes) {
  if (!bytes || N < 0 || N >= 0x7fffffffLL) return TPCONV_ERR_INVALID_ARG;
  *bytes = align256(8 * pow2_at_least(N > 0 ? N : 1)) + 256;
  return TPCONV_OK;
}

tpconv_status tpconv_spatial_order(int64_t N, const float* pos, int32_t* perm, void* ws, size_t ws_bytes,
                                   struct CUstream_st* stream) {
  size_t need = 0;
  if (tpconv_spatial_order_workspace_bytes(N, &need) != TPCONV_OK) return TPCONV_ERR_INVALID_ARG;
  if (N == 0) return TPCONV_OK;
  if (!pos || !perm || !ws) return TPCONV_ERR_INVALID_ARG;
  if (ws_bytes < need) return TPCONV_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = (cudaStream_t)stream;
  const long long n_pad = (long long)pow2_at_least(N);
  auto* keys = static_cast<unsigned long long*>(ws);
  float* box = reinterpret_cast<float*>(static_cast<char*>(ws) + align256(8 * (size_t)n_pad));
  const int n = (int)N;
  const unsigned blocks = (unsigned)((n_pad + kThreads - 1) / kThreads);
  k_bbox<<<1, kThreads, 0, s>>>(n, pos, box);
  k_morton_keys<<<blocks, kThreads, 0, s>>>(n, n_pad, pos, box, keys);
  for (long long k = 2; k <= n_pad; k <<= 1)
    for (long long j = k >> 1; j > 0; j >>= 1) k_bitonic_step<<<blocks, kThreads, 0, s>>>(keys, n_pad, j, k);
  k_keys_to_perm<<<(n + kThreads - 1) / kThreads, kThreads, 0, s>>>(n, keys, perm);
  return launched();
}

tpconv_status tpconv_permute_graph(int64_t N, int64_t E, const int32_t* row_ptr, const int32_t* src,
                                   const int32_t* perm, int32_t* row_ptr_out, int32_t* src_out,
                                   int32_t* inv, struct CUstream_st* stream) {
  if (N < 0 || E < 0 || N >= 0x7fffffffLL || E >= 0x7fffffffLL) return TPCONV_ERR_INVALID_ARG;
  if (!row_ptr || !row_ptr_out) return TPCONV_ERR_INVALID_ARG;
  if (N > 0 && (!perm || !inv)) return TPCONV_ERR_INVALID_ARG;
  if (E > 0 && (!src || !src_out)) return TPCONV_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  const int n = (int)N;
  if (N == 0) {
    if (cudaMemsetAsync(row_ptr_out, 0, sizeof(int32_t), s) != cudaSuccess) return TPCONV_ERR_CUDA;
    return TPCONV_OK;
  }
  k_inverse_and_degrees<<<(n + kThreads - 1) / kThreads, kThreads, 0, s>>>(n, perm, row_ptr, inv, row_ptr_out);
  k_scan_inplace<<<1, 1024, 0, s>>>(n, row_ptr_out);
  if (E > 0)
    k_copy_rows<<<(unsigned)(((long long)n * 32 + kThreads - 1) / kThreads), kThreads, 0, s>>>(
        n, (int)E, perm, row_ptr, src, inv, row_ptr_out, src_out);
  return launched();
}

tpconv_status tpconv_gather_rows(int64_t rows, int64_t width, const float* in, const int32_t* perm, float* out,
                                 struct CUstream_st* stream) {
  if (rows < 0 || width < 0 || rows >= 0x7fffffffLL) return TPCONV_ERR_INVALID_ARG;
  if (rows == 0 || width == 0) return TPCONV_OK;
  if (!in || !perm || !out) return TPCONV_ERR_INVALID_ARG;
  const unsigned gx = (unsigned)(rows < 65535 ? rows : 65535);
  const unsigned gy = (unsigned)((rows + gx - 1) / gx);
  k_gather_rows<<<dim3(gx, gy), 128, 0, (cudaStream_t)stream>>>(rows, width, in, perm, out);
  return launched();
}

}  // extern "C"
