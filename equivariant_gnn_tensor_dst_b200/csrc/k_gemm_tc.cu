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
// 2^-21 instead of TF32's 2^-11.  The optional TF32 mode issues hi*hi only; the optional
// BF16 mode rounds both operands to bf16 and issues one kind::f16 product per K=16 step
// (relative error near 2^-9).
//
// Structure: one CTA of 288 threads per 128 x NT output tile (NT = 64 or 128) and
// split-K slice, two CTAs per SM, warp-specialised around two rings: raw stages of 32 k
// values, and operand slots (TMEM columns for A, shared memory for B):
//   - warps 0-3 (producers) copy the raw fp32 A and B tiles of a stage from global memory
//     with cp.async, through the same two-level affine index maps as the rest of the
//     library (ir_mul node rows, weight columns and workspace states are read in place);
//     the copies arrive on the stage's "full" mbarrier when they land;
//   - warps 4-7 (converters) split a stage into an operand slot: thread (quadrant w,
//     lane) owns output row 32 w + lane and writes hi(A) and lo(A) of its row into its
//     TMEM lane (tcgen05.st); B hi and B lo are written to shared memory.  The raw stage
//     is released at once ("empty"), the slot handed to the MMA warp ("conv");
//   - warp 8 (one thread) issues hi*hi + hi*lo + lo*hi (A from TMEM, B from shared
//     memory) into the fp32 TMEM accumulator and commits them to the slot's "mdone"
//     mbarrier, which frees the slot for the converters.
// The epilogue reads the accumulator with tcgen05.ld (one TMEM lane = one output row) and
// writes C (or the split-K partial) through the output map.  Every mbarrier wait is
// bounded; a wait that gives up sets *err and the kernel still releases its TMEM.
#include <cuda_runtime.h>
#include <cstdint>
#include "launch.h"
#include "tpconv.h"

namespace tpc {

namespace {

constexpr int TC_M = 128;
constexpr int TC_K = 32;           // k elements per stage (8 core-matrix columns)
constexpr int TC_THREADS = 288;   // 4 producer warps, 4 converter warps, 1 MMA warp
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

template <int NT>
__host__ __device__ constexpr uint32_t instr_desc_bf16() {
  // kind::f16 with D fp32 (bits 4-5 = 1), A and B both bf16 (bits 7-9, 10-12 = 1), both
  // K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NT >> 3) << 17) | ((uint32_t)(TC_M >> 4) << 24);
}

// Two floats rounded to bf16 (nearest even) and packed: the first in the low half, the
// lower k index of an A operand pair in a TMEM cell, of a B pair in shared memory.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Bounded wait for the completion of an mbarrier phase.  SLEEP_NS > 0 backs off between
// polls, for waits off the critical path (a producer ahead of its consumers, threads done
// with their part of the tile), so that spinning threads do not take issue slots from
// the warps doing the work.
template <int SLEEP_NS = 0>
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
    if (SLEEP_NS > 0) __nanosleep(SLEEP_NS);
  }
  return false;
}

// Asynchronous operand staging: raw fp32 values go straight from global to shared memory
// with cp.async, zero-filled outside the operand.
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

// Issue the cp.async copies of one operand tile row owned by this thread: row `row`, k
// range [kbeg, kbeg + KW), into the K-major core-matrix layout (tile_off).
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

// Shared-memory plan (1 KB aligned): a ring of RR raw stages [A raw | B raw], a ring of
// NS operand slots [B hi | B lo], then the mbarriers and the TMEM address.
//   A raw (128 x 32 fp32) is read only by the converter warps, one output row per
//   thread, so its layout is chosen for conflict-free reads: k-contiguous operands are
//   stored row-major with the 16-byte chunks of row r XOR-swizzled by r % 8 ("KM"),
//   m-contiguous operands k-major, [k][128 m] ("MM").
//   B raw, B hi and B lo (NT x 32) are in the tensor core's K-major no-swizzle
//   core-matrix layout (tile_off).
// A raw stage is released as soon as the converters have read it; an operand slot (and
// its TMEM columns) when the MMAs that read it have completed.  The copies therefore run
// ahead of the tensor core by up to RR stages regardless of the MMA latency.
// TMEM: columns [0, NT) the fp32 accumulator; operand slot s holds A hi in columns
// NT + 64 s + [0, 32) and A lo in NT + 64 s + [32, 64).
template <int NT>
struct TcSmem {
  static constexpr int A_BYTES = TC_M * TC_K * 4;
  static constexpr int B_BYTES = NT * TC_K * 4;
  static constexpr int RAW = A_BYTES + B_BYTES;
  static constexpr int RR = NT == 64 ? 3 : 2;         // raw stages (two CTAs share an SM)
  static constexpr int NS = NT == 64 ? 2 : 1;         // operand slots
  static constexpr int OPS_OFF = RR * RAW;
  static constexpr int BAR_OFF = OPS_OFF + NS * 2 * B_BYTES;
  static constexpr int TOTAL = BAR_OFF + 128 + 1024;  // barriers, TMEM address; alignment slack
  static constexpr int TMEM_COLS = 256;
  static_assert(NT + 64 * NS <= TMEM_COLS, "TMEM columns");
  static_assert(2 * (RR + NS) * 8 + 4 <= 128, "barrier area");
};

constexpr int TC_PRODUCERS = 128;  // warps 0-3 copy operand tiles
constexpr int TC_CONVERTERS = 128; // warps 4-7 split tiles, fill TMEM and issue the MMAs

__device__ __forceinline__ void mbar_init(uint32_t bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar) : "memory");
}

// A operands with unit m stride are staged k-major ("MM"), all others row-major ("KM")
__device__ __forceinline__ bool a_is_mm(const GemmSeg& S) { return S.Am.d == 0x7fffffff && S.Am.s2 == 1; }

// byte offset of 16-byte chunk c (k = 4c .. 4c + 3) of row r in a KM stage
__device__ __forceinline__ uint32_t km_off(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// step a (k / d, k % d) position by dk
__device__ __forceinline__ void kstep(int& kq, int& kr, int d, int dk) {
  kr += dk;
  while (kr >= d) { kr -= d; ++kq; }
}

template <int NT>
__global__ void __launch_bounds__(TC_THREADS, 2) k_gemm_tc(const __grid_constant__ GemmBatch g, int* err) {
  extern __shared__ char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using SM = TcSmem<NT>;
  char* ring = smem;
  char* ops = smem + SM::OPS_OFF;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::BAR_OFF);  // raw stage copied (TC_PRODUCERS arrivals)
  uint64_t* empty = full + SM::RR;                    // raw stage read (TC_CONVERTERS arrivals)
  uint64_t* conv = empty + SM::RR;                    // operand slot filled (TC_CONVERTERS arrivals)
  uint64_t* mdone = conv + SM::NS;                    // operand slot consumed by the MMAs (tcgen05.commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + SM::NS);

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
  // Width of the products of this tile: its valid columns rounded up to a multiple of 32
  // (the narrowest width in use), so that the narrow output blocks of a plan (16 or 32
  // channels) do not pay for full-width products, B copies and B splits.  B rows at or
  // beyond `neff` are neither copied nor split (the products do not read them), and the
  // accumulator columns beyond it are neither written nor read.
  const int neff = min(NT, (min(NT, P.N - n0) + 31) & ~31);

  if (tid == 0) {
    for (int i = 0; i < SM::RR; ++i) {
      mbar_init(smem_u32(&full[i]), TC_PRODUCERS);
      mbar_init(smem_u32(&empty[i]), TC_CONVERTERS);
    }
    for (int i = 0; i < SM::NS; ++i) {
      mbar_init(smem_u32(&conv[i]), TC_CONVERTERS);
      mbar_init(smem_u32(&mdone[i]), 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(SM::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  // instruction descriptors with the tile's product width in the N field (bits 17-22)
  const uint32_t IDESC = (instr_desc<NT>() & ~(0x3Fu << 17)) | ((uint32_t)(neff >> 3) << 17);
  const uint32_t IDESC_BF16 = (instr_desc_bf16<NT>() & ~(0x3Fu << 17)) | ((uint32_t)(neff >> 3) << 17);
  const bool tf32 = g.math == TPCONV_MATH_TF32;  // one TF32 product per term, no residuals
  const bool bf16 = g.math == TPCONV_MATH_BF16;  // operands rounded to bf16, one product
  constexpr int KWB = TC_K / (TC_PRODUCERS / NT);    // k values per producer for the B operand
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
  // number of k-tiles of this split
  int ntiles = 0;
  {
    Cursor c{0, 0, 0, 0, false};
    advance_to_valid(c);
    while (c.have) { ++ntiles; c.kt += TC_K; advance_to_valid(c); }
  }

  if (warp < TC_PRODUCERS / 32) {
    // ---- producers: copy stage `it` once the converters have read stage it - RR;
    // up to RR stages are in flight
    const int p = tid;
    const int rowB = p % NT, kbegB = (p / NT) * KWB;
    Cursor ld{0, 0, 0, 0, false};
    OpCursor cb{};
    int cur_seg = -1;
    bool a_mm = false, a_vec = false;
    const float* arow[8];  // KM vector copies: rows 16 q + p / 8
    const float* mrow = nullptr;  // MM copies: row base of this thread's m (or chunk of 4 m)
    long long a_s1 = 0, a_s2 = 0;
    int a_d = 1;
    advance_to_valid(ld);
#pragma unroll 1
    for (int it = 0; it < ntiles; ++it) {
      const int slot = it % SM::RR;
      if (it >= SM::RR) ok = mbar_wait<64>(smem_u32(&empty[slot]), ((it / SM::RR) - 1) & 1) && ok;
      const GemmSeg& S = g.sg[P.seg0 + ld.seg];
      if (ld.seg != cur_seg) {  // entering a segment: layout, row offsets, k map
        cur_seg = ld.seg;
        a_mm = a_is_mm(S);
        a_vec = a_mm ? (S.a_mvec4 != 0 && (P.M & 3) == 0) : (S.a_vec4 != 0);
        a_s1 = S.Ak.s1; a_s2 = S.Ak.s2; a_d = S.Ak.d;
        if (a_mm) {
          const int m = m0 + (a_vec ? 4 * (p & 31) : p);
          mrow = m < P.M ? S.A + m : nullptr;
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int m = m0 + 16 * q + (p >> 3);
            arow[q] = m < P.M ? S.A + ixd(S.Am, m) : nullptr;
          }
          mrow = m0 + p < P.M ? S.A + ixd(S.Am, m0 + p) : nullptr;
        }
        op_enter(cb, S.B, S.Bn, S.Bk, n0 + rowB, P.N, ld.kt);
      }
      char* st = ring + slot * SM::RAW;
      const uint32_t dA = smem_u32(st), dB = dA + SM::A_BYTES;
      const int kt = ld.kt, khi = ld.khi;
      int kq = kt / a_d, kr = kt % a_d;   // k map position of the tile start
      if (!a_mm) {
        const bool lin = kr + TC_K <= a_d;
        if (a_vec && lin && ((kt & 3) == 0) && kt + TC_K <= khi) {
          // 16-byte copies: a warp covers 4 rows x 128 contiguous bytes
          const int c = p & 7;
          const long long ko = (long long)kq * a_s1 + (long long)(kr + 4 * c);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int r = 16 * q + (p >> 3);
            cp_async16(dA + km_off(r, c), arow[q] ? arow[q] + ko : S.A, arow[q] != nullptr);
          }
        } else {
          // 4-byte copies, one row per thread
          int q2 = kq, r2 = kr;
#pragma unroll 1
          for (int j = 0; j < TC_K; ++j) {
            const bool v = mrow && kt + j < khi;
            cp_async4(dA + km_off(p, j >> 2) + (j & 3) * 4, v ? mrow + (long long)q2 * a_s1 + (long long)r2 * a_s2 : S.A,
                      v);
            kstep(q2, r2, a_d, 1);
          }
        }
      } else if (a_vec) {
        // 16-byte copies of 4 consecutive m: thread p takes m chunk p % 32 of k rows
        // 4 q + p / 32; a warp covers 512 contiguous bytes of one k row
        int q2 = kq, r2 = kr;
        kstep(q2, r2, a_d, p >> 5);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int kk = 4 * q + (p >> 5);
          const bool v = mrow && kt + kk < khi;
          cp_async16(dA + kk * 512 + (p & 31) * 16, v ? mrow + (long long)q2 * a_s1 + (long long)r2 * a_s2 : S.A, v);
          kstep(q2, r2, a_d, 4);
        }
      } else {
        // 4-byte copies, lanes along m
        int q2 = kq, r2 = kr;
#pragma unroll 1
        for (int j = 0; j < TC_K; ++j) {
          const bool v = mrow && kt + j < khi;
          cp_async4(dA + j * 512 + p * 4, v ? mrow + (long long)q2 * a_s1 + (long long)r2 * a_s2 : S.A, v);
          kstep(q2, r2, a_d, 1);
        }
      }
      if (rowB < neff) issue_operand<KWB, NT>(cb, S.B, kt, khi, kbegB, rowB, S.b_vec4 != 0, dB);
      // the stage's full barrier completes when this thread's copies (and its earlier
      // ones) have landed; nothing the copies write is read by the tensor core directly
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&full[slot])) : "memory");
      const int seg_before = ld.seg;
      ld.kt += TC_K;
      advance_to_valid(ld);
      if (ld.have && ld.seg == seg_before) op_step(cb, TC_K);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp < (TC_PRODUCERS + TC_CONVERTERS) / 32) {
    // ---- converters: thread (quadrant w, lane) owns output row m = 32 w + lane; it splits
    // its 32 A values of the stage into hi / lo and stores them to its TMEM lane; the B
    // residuals are split cooperatively in shared memory; then the stage is handed to the
    // MMA warp through its conv barrier.
    const int c = tid - TC_PRODUCERS;
    const int quad = warp - TC_PRODUCERS / 32;
    const int m = 32 * quad + lane;
    const uint32_t tlane = tmem + ((uint32_t)(32 * quad) << 16);
    Cursor cv{0, 0, 0, 0, false};  // the same walk as the producers: the A layout of each stage
    advance_to_valid(cv);
#pragma unroll 1
    for (int it = 0; it < ntiles; ++it) {
      const bool mm = a_is_mm(g.sg[P.seg0 + cv.seg]);
      cv.kt += TC_K;
      advance_to_valid(cv);
      const int slot = it % SM::RR, os = it % SM::NS;
      char* st = ring + slot * SM::RAW;
      ok = mbar_wait(smem_u32(&full[slot]), (it / SM::RR) & 1) && ok;
      // the operand slot (and its TMEM columns) is free once the MMAs of stage it - NS
      // have completed
      if (it >= SM::NS) ok = mbar_wait(smem_u32(&mdone[os]), ((it / SM::NS) - 1) & 1) && ok;
      const uint32_t acol = (uint32_t)(NT + 64 * os);
      if (bf16) {
        // the 32 A values of this row as bf16 pairs, k and k + 1 in one TMEM cell
        uint32_t pk[16];
#pragma unroll
        for (int k2 = 0; k2 < 16; ++k2) {
          float v0, v1;
          if (mm) {
            const float* a = reinterpret_cast<const float*>(st);
            v0 = a[(2 * k2) * 128 + m];
            v1 = a[(2 * k2 + 1) * 128 + m];
          } else {
            const float2 v = *reinterpret_cast<const float2*>(st + km_off(m, k2 >> 1) + (k2 & 1) * 8);
            v0 = v.x;
            v1 = v.y;
          }
          pk[k2] = pack_bf16(v0, v1);
        }
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
                tlane + acol),
            "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3]), "r"(pk[4]), "r"(pk[5]), "r"(pk[6]), "r"(pk[7]),
            "r"(pk[8]), "r"(pk[9]), "r"(pk[10]), "r"(pk[11]), "r"(pk[12]), "r"(pk[13]), "r"(pk[14]), "r"(pk[15])
            : "memory");
      }
      // two halves of 16 k values: split, then store hi and lo to this thread's TMEM lane
#pragma unroll
      for (int h = 0; h < (bf16 ? 0 : 2); ++h) {
        uint32_t hi[16], lo[16];
        if (mm) {
          const float* a = reinterpret_cast<const float*>(st);
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float v = a[(16 * h + k) * 128 + m];
            const float t = tf32_hi(v);
            hi[k] = __float_as_uint(t);
            lo[k] = __float_as_uint(v - t);
          }
        } else {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const float4 v = *reinterpret_cast<const float4*>(st + km_off(m, 4 * h + cc));
            const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float t = tf32_hi(vv[e]);
              hi[4 * cc + e] = __float_as_uint(t);
              lo[4 * cc + e] = __float_as_uint(vv[e] - t);
            }
          }
        }
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
                tlane + acol + 16u * h),
            "r"(hi[0]), "r"(hi[1]), "r"(hi[2]), "r"(hi[3]), "r"(hi[4]), "r"(hi[5]), "r"(hi[6]), "r"(hi[7]),
            "r"(hi[8]), "r"(hi[9]), "r"(hi[10]), "r"(hi[11]), "r"(hi[12]), "r"(hi[13]), "r"(hi[14]), "r"(hi[15])
            : "memory");
        if (!tf32) asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
                tlane + acol + 32u + 16u * h),
            "r"(lo[0]), "r"(lo[1]), "r"(lo[2]), "r"(lo[3]), "r"(lo[4]), "r"(lo[5]), "r"(lo[6]), "r"(lo[7]),
            "r"(lo[8]), "r"(lo[9]), "r"(lo[10]), "r"(lo[11]), "r"(lo[12]), "r"(lo[13]), "r"(lo[14]), "r"(lo[15])
            : "memory");
      }
      // B split (layout-agnostic, elementwise) from the raw stage into the operand slot
      const char* braw = st + SM::A_BYTES;
      char* bhi = ops + os * 2 * SM::B_BYTES;
      char* blo = bhi + SM::B_BYTES;
      // 16-byte chunk q of the rows below neff: 4 consecutive k (core column kc4) of one row
      // (neff is 32, 64 or 128 for every plan whose blocks have at most 128 channels: a
      // shift; otherwise a division)
      const int nsh = (neff & (neff - 1)) == 0 ? __ffs(neff) - 1 : -1;
      if (bf16) {
        // fp32 core column kc4 -> 8 bytes of the 16-bit K-major layout (core column kc4 / 2,
        // LBO and SBO as for fp32)
        for (int q = c; q < 8 * neff; q += TC_CONVERTERS) {
          const int kc4 = nsh >= 0 ? q >> nsh : q / neff, row = q - kc4 * neff;
          const int off = kc4 * (NT * 16) + row * 16;
          const float4 v = *reinterpret_cast<const float4*>(braw + off);
          const int dst = (kc4 >> 1) * (NT * 16) + row * 16 + (kc4 & 1) * 8;
          *reinterpret_cast<uint2*>(bhi + dst) = make_uint2(pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
        }
      } else if (tf32) {
        for (int q = c; q < 8 * neff; q += TC_CONVERTERS) {
          const int kc4 = nsh >= 0 ? q >> nsh : q / neff, row = q - kc4 * neff;
          const int off = kc4 * (NT * 16) + row * 16;
          *reinterpret_cast<float4*>(bhi + off) = *reinterpret_cast<const float4*>(braw + off);
        }
      } else {
        for (int q = c; q < 8 * neff; q += TC_CONVERTERS) {
          const int kc4 = nsh >= 0 ? q >> nsh : q / neff, row = q - kc4 * neff;
          const int off = kc4 * (NT * 16) + row * 16;
          const float4 v = *reinterpret_cast<const float4*>(braw + off);
          float4 h, l;
          h.x = tf32_hi(v.x); h.y = tf32_hi(v.y); h.z = tf32_hi(v.z); h.w = tf32_hi(v.w);
          l.x = v.x - h.x; l.y = v.y - h.y; l.z = v.z - h.z; l.w = v.w - h.w;
          *reinterpret_cast<float4*>(bhi + off) = h;
          *reinterpret_cast<float4*>(blo + off) = l;
        }
      }
      // every value read from the raw stage has been used: the producers may refill it
      mbar_arrive(smem_u32(&empty[slot]));
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      mbar_arrive(smem_u32(&conv[os]));
    }
  } else {
    // ---- MMA warp: hi*hi + hi*lo + lo*hi for the stage's four K=8 steps (A from TMEM,
    // B from shared memory), committed to the slot's mdone barrier.  The whole warp runs
    // the loop (no lane spins apart from the others); lane 0 issues.
#pragma unroll 1
    for (int it = 0; it < ntiles; ++it) {
      const int os = it % SM::NS;
      ok = mbar_wait(smem_u32(&conv[os]), (it / SM::NS) & 1) && ok;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      if (lane == 0 && bf16) {
        // two K=16 steps of bf16: 8 TMEM columns of A (two k per cell), two 8-wide k
        // columns of B
        const uint32_t b_hi = smem_u32(ops + os * 2 * SM::B_BYTES);
        const uint32_t acol = (uint32_t)(NT + 64 * os);
#pragma unroll
        for (int ks = 0; ks < TC_K / 16; ++ks) {
          const uint32_t aaddr = tmem + acol + 8 * ks;
          const uint64_t db = smem_desc<NT>(b_hi + ks * 2 * (NT * 16));
          const uint32_t acc0 = (it > 0 || ks > 0) ? 1u : 0u;
          asm volatile(
              "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem),
              "r"(aaddr), "l"(db), "r"(IDESC_BF16), "r"(acc0));
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(&mdone[os]))
                     : "memory");
      } else if (lane == 0) {
        const uint32_t b_hi = smem_u32(ops + os * 2 * SM::B_BYTES), b_lo = b_hi + SM::B_BYTES;
        const uint32_t acol = (uint32_t)(NT + 64 * os);
#pragma unroll
        for (int ks = 0; ks < TC_K / 8; ++ks) {
          // one K=8 step: 8 TMEM columns of A, two 4-wide k columns of B
          const uint32_t ahi = tmem + acol + 8 * ks, alo = ahi + 32;
          const uint32_t kbo = ks * 2 * (NT * 16);
          const uint64_t dbh = smem_desc<NT>(b_hi + kbo), dbl = smem_desc<NT>(b_lo + kbo);
          const uint32_t acc0 = (it > 0 || ks > 0) ? 1u : 0u;
          asm volatile(
              "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem),
              "r"(ahi), "l"(dbh), "r"(IDESC), "r"(acc0));
          if (!tf32) {
            asm volatile(
                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem),
                "r"(ahi), "l"(dbl), "r"(IDESC), "r"(1u));
            asm volatile(
                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem),
                "r"(alo), "l"(dbh), "r"(IDESC), "r"(1u));
          }
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(&mdone[os]))
                     : "memory");
      }
      __syncwarp();
    }
  }
  // the last commit completes after every MMA of the tile (tcgen05 operations complete
  // in issue order).  Only the MMA and converter warps' waits here are exact: a producer
  // warp can run more than one phase ahead of the MMA completions, so its parity wait may
  // pass on an earlier phase.  Every thread therefore reads the accumulator only after the
  // block barrier below, which follows the exact waits.
  if (ntiles > 0) {
    const int j = ntiles - 1;
    ok = mbar_wait<128>(smem_u32(&mdone[j % SM::NS]), (j / SM::NS) & 1) && ok;
  }
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const int it = ntiles;

  // epilogue.  TMEM lane r holds output row m0 + r; warp w may read lane quadrant w % 4
  // and takes the column half w / 4 of every 64-column slice.  Values pass through
  // shared memory (row stride 65 floats, conflict free) so that each warp then stores
  // consecutive columns of one row; row and column offsets of the output map are
  // tabulated once.
  float* ep = reinterpret_cast<float*>(ring);            // all MMAs are complete here
  long long* rowoff = reinterpret_cast<long long*>(ring + 65536);
  long long* coloff = rowoff + TC_M;
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
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
  const bool epi = warp < 8;                             // the MMA warp takes no part
#pragma unroll 1
  for (int c0 = 0; c0 < neff; c0 += 64) {
    uint32_t r[32];
    const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(c0 + half * 32);
    if (epi) asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    if (epi) asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    __syncthreads();  // previous slice read out of `ep`; offset tables written
    const int row = quad * 32 + lane;
    if (epi) {
#pragma unroll
      for (int j = 0; j < 32; ++j) ep[row * 65 + half * 32 + j] = (it > 0) ? __uint_as_float(r[j]) : 0.f;
    }
    __syncthreads();
    const int ncols = min(64, NT - c0);
#pragma unroll 4
    for (int q = 0; q < (epi ? TC_M / 8 : 0); ++q) {
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
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TcSmem<NT>::TMEM_COLS));
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
