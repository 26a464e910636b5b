// Channel contractions on the 5th-generation tensor cores (tcgen05, accumulator in TMEM).
//
// Sobek, section 4: the receiver state S is contracted with the radial parameters A
// as one matrix product per output group (m = S A, eqs. 34-35); backward uses
// S_bar = m_bar A^T and A_bar = S^T m_bar (eq. 36), double backward eqs. 37-39, and the
// source side the mirrored x_bar = X A^T and A_bar = x^T X.  These are the only dense
// contractions of the method.
//
// fp32 accuracy from TF32 tensor cores: every operand value a is split as
// a = hi + lo with hi = a truncated to TF32 and lo = a - hi; each k-step
// issues hi*hi + hi*lo + lo*hi into the same fp32 accumulator ("3xTF32", the
// decomposition of Ootomo and Yokota, 2022), which keeps the relative error near
// 2^-21 instead of TF32's 2^-11.  The TF32 MMA reads only the top 19 bits of each
// 32-bit operand, so the raw fp32 tile itself serves as "hi"; only "lo" is computed.
//
// Structure: one CTA of 256 threads per 128 x NT output tile (NT = 64 or 128) and
// split-K slice.  Operand tiles are copied from global memory with cp.async through
// the same two-level affine index maps as the rest of the library (so ir_mul node
// rows, weight columns and workspace states are read in place) straight into the
// canonical K-major, no-swizzle core-matrix layout (8 rows x 16 bytes per core matrix,
// row groups of a k column contiguous).  Two raw stages: the copies of tile t+1 are in
// flight while tile t is split and multiplied; every thread splits exactly the
// elements it copied, so one barrier per tile suffices.  A tcgen05.commit per tile
// arrives on an mbarrier that frees the raw stage and the lo buffer.  The
// epilogue reads the TMEM accumulator with tcgen05.ld (one TMEM lane = one output row)
// and writes C (or the split-K partial) through the output map.  Every mbarrier wait is
// bounded; a wait that gives up sets *err and the kernel still releases its TMEM.
#include <cuda_runtime.h>
#include <cstdint>
#include "internal.h"

namespace tpc {

namespace {

constexpr int TC_M = 128;
constexpr int TC_K = 32;           // k elements per stage (8 core-matrix columns)
constexpr int TC_THREADS = 256;
constexpr unsigned kWaitLimit = 1u << 20;

__device__ __forceinline__ long long ixd(const Idx2& f, int i) {
  return (long long)(i / f.d) * f.s1 + (long long)(i % f.d) * f.s2;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// TF32 part of a float: keep sign, exponent and the top 10 mantissa bits.  The residual
// a - hi is exact in fp32; the tensor core reads it as TF32 (dropping its low bits),
// which leaves an error below 2^-21 |a|.
__device__ __forceinline__ float tf32_hi(float a) { return __uint_as_float(__float_as_uint(a) & 0xffffe000u); }

// Byte offset of element (row, k) inside a [ROWS x 32] K-major no-swizzle tile.  The 8-row
// core matrices of one 4-wide k column are contiguous (SBO = 128 B), so the tensor core
// reads each k column of the tile as one contiguous block; k columns are ROWS * 16 B
// apart (LBO).
template <int ROWS>
__device__ __forceinline__ uint32_t tile_off(int row, int k) {
  return (uint32_t)((k >> 2) * (ROWS * 16) + (row >> 3) * 128 + (row & 7) * 16 + (k & 3) * 4);
}

template <int ROWS>
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
  // start address, LBO = ROWS * 16 B (next k core matrix), SBO = 128 B (next 8-row
  // group), descriptor version 1, no swizzle
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((ROWS * 16) >> 4) << 16) | ((uint64_t)(128 >> 4) << 32) |
         (1ull << 46);
}

template <int NT>
__host__ __device__ constexpr uint32_t instr_desc() {
  // D fp32 (bits 4-5 = 1), A and B tf32 (bits 7-9, 10-12 = 2), both K-major,
  // N >> 3 at bits 17-22, M >> 4 at bits 24-28
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(NT >> 3) << 17) | ((uint32_t)(TC_M >> 4) << 24);
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (unsigned it = 0; it < kWaitLimit; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

// Asynchronous operand staging: raw fp32 tiles go straight from global to shared memory
// with cp.async (zero-filled outside the operand) into a ring of RING stages, already in
// the canonical core-matrix layout.  A conversion pass then splits a landed stage into
// the hi and lo buffers read by the MMAs.  Thread t owns row t % nrows of an operand
// tile and the contiguous k range [(t / nrows) * KW, +KW).
__device__ __forceinline__ void cp_async4(uint32_t dst, const float* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const float* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}

// Per-thread position of one operand inside the current segment.  The row offset is
// computed once per segment; the k offset is tracked as (kq, kr) = (k / d, k % d) of the
// operand's k map and advanced by additions, so that no division is executed per tile.
struct OpCursor {
  const float* row;     // base + row offset (nullptr: row outside the operand)
  long long s1, s2;     // k map strides
  int d;                // k map block
  int kq, kr;           // (k / d, k % d) of the current tile start
};

__device__ __forceinline__ void op_enter(OpCursor& c, const float* base, const Idx2& mr, const Idx2& mk, int r,
                                         int rmax, int kt) {
  c.row = r < rmax ? base + ixd(mr, r) : nullptr;
  c.s1 = mk.s1;
  c.s2 = mk.s2;
  c.d = mk.d;
  c.kq = kt / mk.d;
  c.kr = kt % mk.d;
}

__device__ __forceinline__ void op_step(OpCursor& c, int dk) {
  c.kr += dk;
  while (c.kr >= c.d) { c.kr -= c.d; ++c.kq; }
}

// Issue the cp.async copies of this thread's share of one operand tile.
template <int KW, int ROWS>
__device__ __forceinline__ void issue_operand(const OpCursor& c, const float* safe, int kt, int khi, int kbeg,
                                              int row, bool vec4, uint32_t dst) {
  const bool lin = c.kr + TC_K <= c.d;
  const float* p = c.row ? c.row + (long long)c.kq * c.s1 + (long long)(c.kr + kbeg) * c.s2 : safe;
  if (vec4 && lin && ((kt & 3) == 0) && kt + kbeg + KW <= khi) {
#pragma unroll
    for (int q = 0; q < KW / 4; ++q) cp_async16(dst + tile_off<ROWS>(row, kbeg + 4 * q), c.row ? p + 4 * q : safe, c.row != nullptr);
    return;
  }
  if (lin) {
#pragma unroll
    for (int j = 0; j < KW; ++j) {
      const bool ok = c.row && kt + kbeg + j < khi;
      cp_async4(dst + tile_off<ROWS>(row, kbeg + j), ok ? p + (long long)j * c.s2 : safe, ok);
    }
    return;
  }
  // the tile crosses a block of the k map: step element by element
  int q = c.kq, r = c.kr + kbeg;
  while (r >= c.d) { r -= c.d; ++q; }
#pragma unroll 1
  for (int j = 0; j < KW; ++j) {
    const bool ok = c.row && kt + kbeg + j < khi;
    cp_async4(dst + tile_off<ROWS>(row, kbeg + j), ok ? c.row + (long long)q * c.s1 + (long long)r * c.s2 : safe, ok);
    if (++r == c.d) { r = 0; ++q; }
  }
}

template <int NT>
struct TcSmem {
  static constexpr int A_BYTES = TC_M * TC_K * 4;
  static constexpr int B_BYTES = NT * TC_K * 4;
  static constexpr int RAW = A_BYTES + B_BYTES;      // one raw fp32 stage [A | B]; also the "hi" operand
  static constexpr int RING = 2;                     // raw stages
  static constexpr int TOTAL = RING * RAW + RAW + 2048;  // + lo buffer, alignment, barriers, TMEM address
};

template <int NT>
__global__ void __launch_bounds__(TC_THREADS) k_gemm_tc(const __grid_constant__ GemmBatch g, int* err) {
  extern __shared__ char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using SM = TcSmem<NT>;
  char* ring = smem;                                  // RING raw stages (the "hi" operands)
  char* lo_buf = smem + SM::RING * SM::RAW;           // "lo" operand of the current tile
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::RING * SM::RAW + SM::RAW);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::RING * SM::RAW + SM::RAW + 64);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // locate (problem, m tile, n tile)
  const int tile = blockIdx.x;
  int pi = 0;
  while (pi + 1 < g.n_problems && g.pr[pi + 1].tile0 <= tile) ++pi;
  const GemmProblem& P = g.pr[pi];
  const int lt = tile - P.tile0;
  const int tn = (P.N + NT - 1) / NT;
  const int m0 = (lt / tn) * TC_M, n0 = (lt % tn) * NT;
  const int split = blockIdx.y;
  const int kper = ((P.Ktot + g.splits - 1) / g.splits + TC_K - 1) / TC_K * TC_K;
  const int kb = split * kper, ke = min(P.Ktot, kb + kper);

  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars[0])));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(NT));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  constexpr uint32_t IDESC = instr_desc<NT>();
  constexpr int KWA = TC_K / (TC_THREADS / TC_M);  // k values per thread for the A operand
  constexpr int KWB = TC_K / (TC_THREADS / NT);    // k values per thread for the B operand
  bool ok = true;

  // The k-tiles of this split, as (segment, kt) pairs, walked by a cursor.
  struct Cursor { int seg, kbase, kt, khi; bool have; };
  auto advance_to_valid = [&](Cursor& c) {
    while (c.seg < P.nseg) {
      const int K = g.sg[P.seg0 + c.seg].K;
      const int lo = max(kb - c.kbase, 0), hi = min(ke - c.kbase, K);
      if (c.kt < lo) c.kt = lo;
      if (c.kt < hi) { c.khi = hi; c.have = true; return; }
      c.kbase += K;
      ++c.seg;
      c.kt = 0;
    }
    c.have = false;
  };
  const int rowA = tid % TC_M, kbegA = (tid / TC_M) * KWA;
  const int rowB = tid % NT, kbegB = (tid / NT) * KWB;
  Cursor ld{0, 0, 0, 0, false};
  OpCursor ca{}, cb{};
  int cur_seg = -1;
  advance_to_valid(ld);
  auto issue_tile = [&](int slot) {
    // always commit a group (possibly empty) so that group counting stays uniform
    if (ld.have) {
      const GemmSeg& S = g.sg[P.seg0 + ld.seg];
      if (ld.seg != cur_seg) {  // entering a segment: row offsets and k positions
        op_enter(ca, S.A, S.Am, S.Ak, m0 + rowA, P.M, ld.kt);
        op_enter(cb, S.B, S.Bn, S.Bk, n0 + rowB, P.N, ld.kt);
        cur_seg = ld.seg;
      }
      const uint32_t dst = smem_u32(ring + slot * SM::RAW);
      issue_operand<KWA, TC_M>(ca, S.A, ld.kt, ld.khi, kbegA, rowA, S.a_vec4 != 0, dst);
      issue_operand<KWB, NT>(cb, S.B, ld.kt, ld.khi, kbegB, rowB, false, dst + SM::A_BYTES);
      const int seg_before = ld.seg;
      ld.kt += TC_K;
      advance_to_valid(ld);
      if (ld.have && ld.seg == seg_before) {
        op_step(ca, TC_K);
        op_step(cb, TC_K);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // number of k-tiles of this split
  int ntiles = 0;
  {
    Cursor c{0, 0, 0, 0, false};
    advance_to_valid(c);
    while (c.have) { ++ntiles; c.kt += TC_K; advance_to_valid(c); }
  }
  issue_tile(0);
  uint32_t phase = 0u;
  int it = 0;
#pragma unroll 1
  for (; it < ntiles; ++it) {
    // MMA(it-1) read raw stage (it+1) % 2 and the lo buffer: wait before reusing them
    if (it >= 1) {
      ok = mbar_wait(smem_u32(&bars[0]), phase) && ok;
      phase ^= 1u;
    }
    issue_tile((it + 1) % SM::RING);
    asm volatile("cp.async.wait_group 1;" ::: "memory");   // this thread's copies of tile `it`
    {
      // split the elements this thread copied: lo = raw - tf32(raw)
      const char* raw = ring + (it % SM::RING) * SM::RAW;
#pragma unroll
      for (int q = 0; q < KWA / 4; ++q) {
        const uint32_t off = tile_off<TC_M>(rowA, kbegA + 4 * q);
        const float4 v = *reinterpret_cast<const float4*>(raw + off);
        float4 l;
        l.x = v.x - tf32_hi(v.x); l.y = v.y - tf32_hi(v.y); l.z = v.z - tf32_hi(v.z); l.w = v.w - tf32_hi(v.w);
        *reinterpret_cast<float4*>(lo_buf + off) = l;
      }
#pragma unroll
      for (int q = 0; q < KWB / 4; ++q) {
        const uint32_t off = SM::A_BYTES + tile_off<NT>(rowB, kbegB + 4 * q);
        const float4 v = *reinterpret_cast<const float4*>(raw + off);
        float4 l;
        l.x = v.x - tf32_hi(v.x); l.y = v.y - tf32_hi(v.y); l.z = v.z - tf32_hi(v.z); l.w = v.w - tf32_hi(v.w);
        *reinterpret_cast<float4*>(lo_buf + off) = l;
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t a_hi = smem_u32(ring + (it % SM::RING) * SM::RAW), b_hi = a_hi + SM::A_BYTES;
      const uint32_t a_lo = smem_u32(lo_buf), b_lo = a_lo + SM::A_BYTES;
#pragma unroll
      for (int ks = 0; ks < TC_K / 8; ++ks) {
        // one K=8 step spans two 4-wide k columns
        const uint32_t ka = ks * 2 * (TC_M * 16), kbo = ks * 2 * (NT * 16);
        const uint64_t dah = smem_desc<TC_M>(a_hi + ka), dal = smem_desc<TC_M>(a_lo + ka);
        const uint64_t dbh = smem_desc<NT>(b_hi + kbo), dbl = smem_desc<NT>(b_lo + kbo);
        const uint32_t acc0 = (it > 0 || ks > 0) ? 1u : 0u;
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
            "l"(dah), "l"(dbh), "r"(IDESC), "r"(acc0));
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
            "l"(dah), "l"(dbl), "r"(IDESC), "r"(1u));
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
            "l"(dal), "l"(dbh), "r"(IDESC), "r"(1u));
      }
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                       smem_u32(&bars[0]))
                   : "memory");
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  // wait for the last commit (tcgen05 operations complete in issue order)
  if (it > 0) ok = mbar_wait(smem_u32(&bars[0]), phase) && ok;
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

  // epilogue.  TMEM lane r holds output row m0 + r; warp w may read lane quadrant w % 4
  // and takes the column half w / 4 of every 64-column slice.  Values pass through
  // shared memory (row stride 65 floats, conflict free) so that each warp then stores
  // consecutive columns of one row; row and column offsets of the output map are
  // tabulated once.
  float* ep = reinterpret_cast<float*>(ring);            // all MMAs are complete here
  long long* rowoff = reinterpret_cast<long long*>(lo_buf);
  long long* coloff = rowoff + TC_M;
  __syncthreads();
  for (int t = tid; t < TC_M; t += TC_THREADS) {
    const int m = m0 + t;
    rowoff[t] = m < P.M ? (g.splits > 1 ? ((long long)split * P.M + m) * P.N : ixd(P.Cm, m)) : 0;
  }
  for (int t = tid; t < NT; t += TC_THREADS) {
    const int n = n0 + t;
    coloff[t] = n < P.N ? (g.splits > 1 ? (long long)n : ixd(P.Cn, n)) : 0;
  }
  float* const outbase = g.splits > 1 ? g.partial + P.part_off : P.C;
  const int quad = warp & 3, half = warp >> 2;
#pragma unroll 1
  for (int c0 = 0; c0 < NT; c0 += 64) {
    uint32_t r[32];
    const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(c0 + half * 32);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    __syncthreads();  // previous slice read out of `ep`; offset tables written
    const int row = quad * 32 + lane;
#pragma unroll
    for (int j = 0; j < 32; ++j) ep[row * 65 + half * 32 + j] = (it > 0) ? __uint_as_float(r[j]) : 0.f;
    __syncthreads();
    const int ncols = min(64, NT - c0);
#pragma unroll 4
    for (int q = 0; q < TC_M / 8; ++q) {
      const int rr = q * 8 + warp;                       // 8 warps store 8 rows per step
      const int m = m0 + rr;
      if (m >= P.M) continue;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int cc = h2 * 32 + lane;
        const int n = n0 + c0 + cc;
        if (cc < ncols && n < P.N) {
          const float v = ep[rr * 65 + cc];
          float* c = outbase + rowoff[rr] + coloff[c0 + cc];
          *c = (g.accumulate && g.splits == 1) ? *c + v : v;
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(NT));
  }
  if (!ok && tid == 0 && err) atomicExch(err, 1);
}

}  // namespace

__global__ void k_gemm_tc_reduce(const __grid_constant__ GemmBatch g, long long total) {
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
  float* c = P.C + ixd(P.Cm, m) + ixd(P.Cn, n);
  *c = g.accumulate ? *c + s : s;
}

template <int NT>
static cudaError_t run_tc(GemmBatch& g, int* err, cudaStream_t s) {
  static bool attr_set = false;  // per device-agnostic process; the attribute is per function
  const int smem = TcSmem<NT>::TOTAL;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k_gemm_tc<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int tiles = 0;
  long long elems = 0;
  for (int p = 0; p < g.n_problems; ++p) {
    g.pr[p].tile0 = tiles;
    g.pr[p].part_off = elems * g.splits;
    tiles += ((g.pr[p].M + TC_M - 1) / TC_M) * ((g.pr[p].N + NT - 1) / NT);
    elems += (long long)g.pr[p].M * g.pr[p].N;
  }
  g.total_tiles = tiles;
  if (tiles == 0) return cudaSuccess;
  k_gemm_tc<NT><<<dim3(tiles, g.splits), TC_THREADS, smem, s>>>(g, err);
  if (g.splits > 1) k_gemm_tc_reduce<<<(unsigned)((elems + 255) / 256), 256, 0, s>>>(g, elems);
  return cudaGetLastError();
}

int gemm_tiles(const GemmBatch& g) {
  int maxN = 0;
  for (int p = 0; p < g.n_problems; ++p) maxN = maxN > g.pr[p].N ? maxN : g.pr[p].N;
  const int nt = maxN <= 64 ? 64 : 128;
  int tiles = 0;
  for (int p = 0; p < g.n_problems; ++p) tiles += ((g.pr[p].M + TC_M - 1) / TC_M) * ((g.pr[p].N + nt - 1) / nt);
  return tiles;
}

cudaError_t launch_gemm_tc(GemmBatch& g, int* err, cudaStream_t s) {
  int maxN = 0;
  for (int p = 0; p < g.n_problems; ++p) maxN = maxN > g.pr[p].N ? maxN : g.pr[p].N;
  if (maxN <= 64) return run_tc<64>(g, err, s);
  return run_tc<128>(g, err, s);
}

}  // namespace tpc
