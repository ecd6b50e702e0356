// Teacher-forced R-SWA attention on the 5th-generation tensor cores
// (tcgen05 + TMEM), bf16 inputs, head dim 128, float32 accumulation.
//
// Operation ("Unlimited OCR Works：一篇读懂 R-SWA 如何把长文档 OCR 从 for-loop 推向
// one-shot", 方法展开 §3, Eq.(1)-(4), in the packed form used for training on
// 32K sequences, 实验与证据 §1): O = softmax(Q K^T * scale + M) V per head, where
// the query at 0-based row i sees key j iff
//   j <= i  and  (i < L_m  or  j < L_m  or  j > i - n).
//
// Design (B200):
// * One CTA per (pair of 128-query tiles, head), so every K/V tile loaded
//   into shared memory serves 256 queries: half the key/value traffic per
//   FLOP of one tile per CTA, whose delivery from L2 bounded it.  The grid
//   is ordered heaviest pair first so that the hardware block scheduler
//   approximates longest-job-first.
// * The key tiles a pair needs are the reference tiles [0, ceil(L_m/128))
//   plus the tiles of the pair's causal band; every other tile is fully
//   masked and skipped.  Only tiles that are not fully visible to a query
//   tile are masked per element.
// * Warp 0 lane 0 loads both Q tiles, then streams K tiles with TMA
//   (128B-swizzled boxes of 128 rows x 64 columns) into a 2-stage ring freed
//   once both QK^T MMAs of a tile completed; warp 10 lane 0 streams V tiles
//   into a 2-stage ring freed by the PV MMAs.  Warp 1 owns the tensor memory
//   (512 columns: S_a, S_b, O_a, O_b) and one lane issues the MMAs.
// * Warps 2-5 run the softmax of query tile a, warps 6-9 that of tile b, one
//   thread per query row (TMEM lane): it reads its 128 scores into registers
//   with tcgen05.ld, forms p = 2^(s*scale*log2e - m) in one pass against the
//   maximum in use, and writes P (bf16 pairs) over the first 64 columns of
//   its S with tcgen05.st.  The PV MMA reads P from TMEM.  A row sum of at
//   most 2^8 bounds every weight by 2^8, so the row maximum is only taken
//   (and the pass redone) when some row's sum exceeds it.
// * Issue order per key tile j: PV_a(j), S_a(j+1), PV_b(j), S_b(j+1).  While
//   one group computes exponentials, the tensor core runs the other group's
//   products, and vice versa.  S_g(j+1) overwrites P_g(j) only after PV_g(j)
//   in the tensor core's issue order.
// * O_g is rescaled in TMEM only when a row maximum grew by more than 2^8
//   since the last rescale (the stale maximum keeps every exponent <= 2^8,
//   exact in float32).  The commit that signals S_g(j) also covers
//   PV_g(j-1), so the rescale needs no wait of its own.
// * Every wait is bounded; on a timeout the kernel marks its rows with NaN,
//   drains its copies and MMAs, frees its tensor memory and returns.

#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace rswa {
namespace tc {

constexpr int kTile = 128;     // query and key tile
constexpr int kD = 128;        // head dim
constexpr int kQT = 2;         // query tiles per CTA
constexpr int kHalf = 64;      // score columns per pass
constexpr int kBox = 64;       // columns per 128B-swizzled box (bf16)
constexpr int kBoxBytes = kTile * kBox * 2;      // 16 KB
constexpr int kTileBytes = 2 * kBoxBytes;        // 32 KB: 128 rows x 128 cols
constexpr int kKS = 2;                           // K ring stages
constexpr int kVS = 2;                           // V ring stages
constexpr int kSoftmaxThreads = 128 * kQT;       // warps 2 .. 9
constexpr int kVWarp = 2 + kSoftmaxThreads / 32;  // V producer warp (after the softmax warps)
constexpr int kThreads = 64 + kSoftmaxThreads + 32;  // K producer, MMA, softmax, V producer
constexpr int kTmemCols = 512;
// TMEM columns of query tile g: S_g at 128*g (P_g, bf16 pairs, over its first 64), O_g at 256 + 128*g
constexpr uint32_t kColS = 0, kColO = 256;

// Shared memory map (offsets from a 1024-byte aligned base).
constexpr int kSmQ = 0;                          // kQT tiles
constexpr int kSmK = kSmQ + kQT * kTileBytes;
constexpr int kSmV = kSmK + kKS * kTileBytes;
constexpr int kSmBar = kSmV + kVS * kTileBytes;
constexpr int kSmBytes = kSmBar + 256 + 1024;    // + slack for 1024-byte alignment

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, float32 D,
// M = 128, N = 128, A K-major, B K-major (QK^T) or N-major (PV).
constexpr uint32_t kIdescBase = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTile >> 3) << 17) |
                                ((uint32_t)(kTile >> 4) << 24);
constexpr uint32_t kIdescQK = kIdescBase;
constexpr uint32_t kIdescPV = kIdescBase | (1u << 16);

// Shared-memory matrix descriptor, 128B swizzle, sm_100 version bit.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(0), "r"(0), "r"(0), "r"(0)
      : "memory");
}

// The same with A (M x K, bf16 pairs along the columns) read from TMEM.
__device__ __forceinline__ void mma_bf16_ta(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(tmem_d), "r"(tmem_a), "l"(b), "r"(idesc), "r"(acc), "r"(0), "r"(0), "r"(0), "r"(0)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

// 16 consecutive TMEM columns of this thread's lane (load and store).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
      : "memory");
}

// kHalf/2 consecutive TMEM columns of this thread's lane from packed words.
__device__ __forceinline__ void tmem_st_pairs(uint32_t taddr, const uint32_t* w) {
#pragma unroll
  for (int c = 0; c < kHalf / 2; c += 16) {
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(w[c + i]);
    tmem_st16(taddr + c, v);
  }
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// One CTA's work: a pair of query tiles of one document of the pack.
struct TcWork {
  int start;  // first pack row of the document
  int len;    // its rows
  int ref;    // its reference rows (L_m)
  int pair;   // the pair of 128-row query tiles, local rows [256*pair, 256*pair + 256)
};
constexpr int kMaxWork = 1024;  // table entries per launch (16 KB of kernel parameters)

struct TcParams {
  CUtensorMap tmQ, tmK, tmV;  // 3-D maps {d, H, rows} of bf16 over the whole pack, 64x1x128 boxes, 128B swizzle
  __nv_bfloat16* O;
  int n, H;
  int bidir;                  // 1: prefix queries see every reference key
  float scale_log2;
  unsigned long long* timing;  // RSWA_TIMING builds: per-tile cycle stamps of CTA 0
  // Optional cache fill (one sequence): K and V rows into [H][S_cap][d]
  // caches, reference rows at their row, outputs in an n-slot ring that
  // keeps the newest fill_n of them, or (fill_full) every output in order.
  __nv_bfloat16* kc;          // null: no fill
  __nv_bfloat16* vc;
  int S_cap, fill_n, fill_full;
  int n_work;
  TcWork work[kMaxWork];      // heaviest first; CTA c takes entry c / H, head c % H
};

// RSWA_TIMING builds record clock64 stamps of CTA 0 for its first 32 key
// tiles: slot [j][k], k < 8 by softmax warp 2 lane 0 (query tile a), k >= 8
// by the MMA thread.
#ifdef RSWA_TIMING
#define TC_CYC(j, k) \
  do { if (p.timing && blockIdx.x == 0 && (j) < 32) p.timing[(j) * 16 + (k)] = clock64(); } while (0)
#else
#define TC_CYC(j, k) do {} while (0)
#endif

// Key tiles of the query rows [q0, q0 + len): [0, A) then [B0, B1] (B0 > A-1 or empty).
struct TileRange {
  int A, B0, B1;
};

__host__ __device__ __forceinline__ TileRange tile_range(int q0, int len, int L, int L_m, int n, bool bidir) {
  const int q_last = (q0 + len < L ? q0 + len : L) - 1;
  TileRange r;
  if (q_last < L_m) {  // all prefix rows: causal, or every reference key (bidirectional)
    r.A = bidir ? (L_m + kTile - 1) / kTile : q_last / kTile + 1;
    r.B0 = 1;
    r.B1 = 0;
    return r;
  }
  r.A = (L_m + kTile - 1) / kTile;
  const int qs = q0 > L_m ? q0 : L_m;
  const int lo = qs - n + 1 > L_m ? qs - n + 1 : L_m;
  r.B0 = lo / kTile > r.A ? lo / kTile : r.A;
  r.B1 = q_last / kTile;
  return r;
}

__host__ __device__ __forceinline__ int tile_count(const TileRange& r) {
  return r.A + (r.B1 - r.B0 + 1 > 0 ? r.B1 - r.B0 + 1 : 0);
}
__device__ __forceinline__ int tile_at(const TileRange& r, int j) { return j < r.A ? j : r.B0 + (j - r.A); }

// Barrier slots (8 bytes each).
enum : int {
  kBarQ = 0, kBarKFull = 1, kBarKFree = 3, kBarVFull = 5, kBarVFree = 7, kBarSFull = 9, kBarPFull = 11,
  kBarODone = 13, kBarFinal = 15, kSlotTmem = 16, kSlotAbort = 17
};

// 64 columns (starting at col0) of one thread's row of an S tile:
// maximum of the visible scores.  FULL: every column visible; otherwise the
// row's visible columns are [0, ra) and [wb, we] (the reference keys, causal
// for a prefix row, and the output window).
template <bool FULL>
__device__ __forceinline__ float half_max(const float* s, int col0, int ra, int wb, int we) {
  float m8[8];  // independent chains
#pragma unroll
  for (int k = 0; k < 8; ++k) m8[k] = -INFINITY;
  if (FULL) {
#pragma unroll
    for (int e = 0; e < kHalf; e += 2) m8[(e >> 1) & 7] = max3(m8[(e >> 1) & 7], s[e], s[e + 1]);
  } else {
#pragma unroll
    for (int e = 0; e < kHalf; ++e) {
      const int c = col0 + e;
      m8[e & 7] = fmaxf(m8[e & 7], (c < ra || (c >= wb && c <= we)) ? s[e] : -INFINITY);
    }
  }
  return fmaxf(max3(m8[0], m8[1], m8[2]), max3(m8[3], max3(m8[4], m8[5], m8[6]), m8[7]));
}

// Exponentials p = 2^(s*sl2 - msub) of those 64 columns, one XU
// instruction each, packed to bf16 pairs (the PV product's operand); returns
// their float32 sum.  Masked columns get an argument of -inf, so exactly 0.
// Fully visible tiles form two arguments with one fma.rn.f32x2 and add two
// weights to the sums with one add.rn.f32x2 (the same roundings per element).
template <bool FULL>
__device__ __forceinline__ float half_exp(const float* s, int col0, int ra, int wb, int we, float sl2, float msub,
                                          uint32_t* pk) {
  if constexpr (FULL) {
    unsigned long long acc[2] = {0ull, 0ull};  // two pairs of independent sums
    unsigned long long sl2x2, nmx2;
    asm("mov.b64 %0, {%1, %1};" : "=l"(sl2x2) : "f"(sl2));
    asm("mov.b64 %0, {%1, %1};" : "=l"(nmx2) : "f"(-msub));
#pragma unroll
    for (int e = 0; e < kHalf; e += 2) {
      unsigned long long sx, xx, pp;
      asm("mov.b64 %0, {%1, %2};" : "=l"(sx) : "f"(s[e]), "f"(s[e + 1]));
      asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(xx) : "l"(sx), "l"(sl2x2), "l"(nmx2));
      float x0, x1;
      asm("mov.b64 {%0, %1}, %2;" : "=f"(x0), "=f"(x1) : "l"(xx));
      const float p0 = ex2(x0), p1 = ex2(x1);
      asm("mov.b64 %0, {%1, %2};" : "=l"(pp) : "f"(p0), "f"(p1));
      asm("add.rn.f32x2 %0, %0, %1;" : "+l"(acc[(e >> 1) & 1]) : "l"(pp));
      pk[e / 2] = pack_bf16x2(p0, p1);
    }
    float a0, a1, b0, b1;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(acc[0]));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(b0), "=f"(b1) : "l"(acc[1]));
    return (a0 + a1) + (b0 + b1);
  } else {
    float l4[4] = {0.f, 0.f, 0.f, 0.f};  // independent sums
#pragma unroll
    for (int e = 0; e < kHalf; e += 2) {
      const int c = col0 + e;
      float x0 = fmaf(s[e], sl2, -msub), x1 = fmaf(s[e + 1], sl2, -msub);
      x0 = (c < ra || (c >= wb && c <= we)) ? x0 : -INFINITY;
      x1 = (c + 1 < ra || (c + 1 >= wb && c + 1 <= we)) ? x1 : -INFINITY;
      const float p0 = ex2(x0), p1 = ex2(x1);
      l4[(e >> 1) & 3] += p0 + p1;
      pk[e / 2] = pack_bf16x2(p0, p1);
    }
    return (l4[0] + l4[1]) + (l4[2] + l4[3]);
  }
}

__global__ void __launch_bounds__(kThreads, 1) masked_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmBar);
  const uint32_t bar0 = smem_u32(bars);
  auto B = [&](int slot) { return bar0 + 8u * slot; };
  volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(&bars[kSlotTmem]);
  volatile int* s_abort = reinterpret_cast<volatile int*>(&bars[kSlotAbort]);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // the host orders the table heaviest first, so the hardware block
  // scheduler approximates longest-job-first
  const int h = blockIdx.x % p.H;
  const TcWork wk = p.work[blockIdx.x / p.H];
  const int L = wk.len, L_m = wk.ref;  // the document's geometry, in local rows
  const int ds = wk.start;             // its first pack row (TMA and output coordinates)
  const int q0 = wk.pair * kQT * kTile;
  const TileRange tr = tile_range(q0, kQT * kTile, L, L_m, p.n, p.bidir != 0);
  const int nt = tile_count(tr);

  if (threadIdx.x == 0) {
    mbar_init(B(kBarQ), 1);
    for (int s = 0; s < kKS; ++s) {
      mbar_init(B(kBarKFull + s), 1);
      mbar_init(B(kBarKFree + s), 1);
    }
    for (int s = 0; s < kVS; ++s) {
      mbar_init(B(kBarVFull + s), 1);
      mbar_init(B(kBarVFree + s), 1);
    }
    for (int g = 0; g < kQT; ++g) {
      mbar_init(B(kBarSFull + g), 1);
      mbar_init(B(kBarPFull + g), 128);
      mbar_init(B(kBarODone + g), 1);
    }
    mbar_init(B(kBarFinal), 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {  // one warp allocates the tensor memory
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32((const void*)s_tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0 || warp == kVWarp) {
    // ---------------------------------------------------------- producers
    // warp 0: both Q tiles, then the K ring; warp kVWarp: the V ring.  Lane 0
    // issues the copies; with a cache to fill, the whole warp also copies
    // this CTA's own key rows (its query rows, whose tiles it loads anyway)
    // from each staged tile into the cache before the stage is reused.
    const bool is_k = warp == 0;
    const int ns = is_k ? kKS : kVS;
    const uint32_t full0 = B(is_k ? kBarKFull : kBarVFull), free0 = B(is_k ? kBarKFree : kBarVFree);
    const uint32_t dst0 = sbase + (is_k ? kSmK : kSmV);
    const CUtensorMap* map = is_k ? &p.tmK : &p.tmV;
    const bool fill = p.kc != nullptr;
    const int own_lo = q0 / kTile, own_hi = (min(q0 + kQT * kTile, L) - 1) / kTile;  // this CTA's query tiles
    // Rows of tile j (staged in stage s) that belong to this CTA's query rows
    // and to the cache: the reference rows, and the outputs the cache keeps
    // (the newest fill_n in an n-slot ring, or all of them in FULL mode).
    auto fill_tile = [&](int j, int s) {
      const int kt = tile_at(tr, j);
      if (kt < own_lo || kt > own_hi) return;
      const uint8_t* base = smem + (is_k ? kSmK : kSmV) + s * kTileBytes;
      __nv_bfloat16* cache = is_k ? p.kc : p.vc;
#pragma unroll 4
      for (int i = 0; i < kTile / 2; ++i) {
        const int r = 2 * i + (lane >> 4);  // tile row
        const int c = lane & 15;            // 16-byte chunk of the 256-byte row
        const int pos = kt * kTile + r;     // local row
        int crow = -1;
        if (pos < L) {
          if (pos < L_m || p.fill_full) crow = pos;
          else if (pos >= L - p.fill_n) crow = L_m + (pos - L_m) % p.fill_n;
        }
        if (crow >= 0) {
          const uint4 v = *reinterpret_cast<const uint4*>(base + (c >> 3) * kBoxBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
          *reinterpret_cast<uint4*>(cache + ((size_t)h * p.S_cap + crow) * kD + c * 8) = v;
        }
      }
    };
    // A stage's tile is read here only after its full phase completed (the
    // TMA writes are then visible to this warp).
    auto wait_full = [&](int j) -> bool {
      bool ok = true;
      if (lane == 0) ok = mbar_wait_bounded(full0 + 8u * (j % ns), (j / ns) & 1);
      return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    };
    if (lane == 0 && is_k) {
      mbar_arrive_expect_tx(B(kBarQ), kQT * kTileBytes);
      for (int g = 0; g < kQT; ++g) {
        tma_load_3d(sbase + kSmQ + g * kTileBytes, &p.tmQ, 0, h, ds + q0 + g * kTile, B(kBarQ));
        tma_load_3d(sbase + kSmQ + g * kTileBytes + kBoxBytes, &p.tmQ, kBox, h, ds + q0 + g * kTile, B(kBarQ));
      }
    }
    int issued = 0;
    if (fill || lane == 0) {
      for (int j = 0; j < nt; ++j) {
        const int s = j % ns;
        int ok = 1;
        if (lane == 0) ok = !*s_abort && mbar_wait_bounded(free0 + 8u * s, ((j / ns) & 1) ^ 1);
        if (fill) ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) *s_abort = 1;
          break;
        }
        if (fill && j >= ns) {
          if (!wait_full(j - ns)) break;
          fill_tile(j - ns, s);
          __syncwarp();  // every lane's reads of the stage before it is loaded again
        }
        if (lane == 0) {
          // rows past the document's end (the next document's, or zero fill
          // past the pack) are never visible: keys by causality, queries are
          // not stored
          const int k0 = ds + tile_at(tr, j) * kTile;
          mbar_arrive_expect_tx(full0 + 8u * s, kTileBytes);
          tma_load_3d(dst0 + s * kTileBytes, map, 0, h, k0, full0 + 8u * s);
          tma_load_3d(dst0 + s * kTileBytes + kBoxBytes, map, kBox, h, k0, full0 + 8u * s);
        }
        issued = j + 1;
      }
      // the last staged tiles: fill from them once they have landed
      if (fill)
        for (int j = max(0, issued - ns); j < issued; ++j)
          if (wait_full(j)) fill_tile(j, j % ns);
      // drain: every issued copy has landed before the CTA may exit
      if (lane == 0) {
        if (is_k) mbar_wait_bounded(B(kBarQ), 0);
        for (int j = max(0, issued - ns); j < issued; ++j) mbar_wait_bounded(full0 + 8u * (j % ns), (j / ns) & 1);
      }
      // decode kernels may copy reference rows before their dependency wait
      if (fill) __threadfence();
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // S_g(j) = Q_g K_j^T into S_g
      auto issue_s = [&](int g, int j) {
        const uint32_t aQ = sbase + kSmQ + g * kTileBytes;
        const uint32_t aK = sbase + kSmK + (j % kKS) * kTileBytes;
        TC_CYC(j, 8 + g);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
          mma_bf16(tmem + kColS + 128 * g, smem_desc(aQ + off, 16, 1024), smem_desc(aK + off, 16, 1024), kIdescQK,
                   kk > 0);
        }
        mma_commit(B(kBarSFull + g));
      };
      bool ok = mbar_wait_bounded(B(kBarQ), 0) && !*s_abort && mbar_wait_bounded(B(kBarKFull), 0);
      if (ok) {
        tc_fence_after();
        for (int g = 0; g < kQT; ++g) issue_s(g, 0);
        mma_commit(B(kBarKFree));
      }
      for (int j = 0; j < nt && ok; ++j) {
        const int sv = j % kVS;
        for (int g = 0; g < kQT; ++g) {
          // O_g += P_g(j) V_j once group g has written P_g(j)
          ok = !*s_abort && mbar_wait_bounded(B(kBarPFull + g), j & 1) &&
               (g > 0 || mbar_wait_bounded(B(kBarVFull + sv), (j / kVS) & 1));
          if (!ok) break;
          tc_fence_after();
          TC_CYC(j, 10 + g);
          const uint32_t aV = sbase + kSmV + sv * kTileBytes;
          const uint32_t tP = tmem + kColS + 128 * g;
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)  // 16 keys = 8 columns of bf16 pairs per step
            mma_bf16_ta(tmem + kColO + 128 * g, tP + kk * 8, smem_desc(aV + kk * 2048, kBoxBytes, 1024), kIdescPV,
                        (j > 0 || kk > 0));
          if (g == kQT - 1) mma_commit(B(kBarVFree + sv));
          if (j + 1 < nt) {
            // S_g(j+1): issued after PV_g(j), which reads P_g(j) from the same columns
            if (g == 0) {
              ok = !*s_abort && mbar_wait_bounded(B(kBarKFull + (j + 1) % kKS), ((j + 1) / kKS) & 1);
              if (!ok) break;
              tc_fence_after();
            }
            issue_s(g, j + 1);
            if (g == kQT - 1) mma_commit(B(kBarKFree + (j + 1) % kKS));
          } else {
            mma_commit(B(kBarODone + g));
          }
        }
      }
      if (!ok) *s_abort = 1;
      // every MMA issued by this thread has completed before TMEM is freed
      mma_commit(B(kBarFinal));
      mbar_wait_bounded(B(kBarFinal), 0);
    }
  } else {
    // ---------------------------------------------------------- softmax
    const int g = (warp - 2) >> 2;   // query tile of this group
    const int quarter = warp & 3;    // TMEM lanes 32*quarter .. +31
    const int r = quarter * 32 + lane;
    const int q0g = q0 + g * kTile;
    const int i = q0g + r;           // query row
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t colS = kColS + 128 * g, colO = kColO + 128 * g;
    const bool stamp = warp == 2 && lane == 0;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      // After a timed-out wait a thread stops waiting but keeps arriving, so
      // the MMA thread is not left waiting on it; its rows are written as NaN.
      if (stamp) TC_CYC(j, 0);
      if (ok && (*s_abort || !mbar_wait_bounded(B(kBarSFull + g), j & 1))) ok = false;
      if (stamp) TC_CYC(j, 1);
      tc_fence_after();
      const int k0 = tile_at(tr, j) * kTile;
      const bool full = (k0 + kTile - 1 < L_m) && (p.bidir || q0g >= L_m || k0 + kTile - 1 <= q0g);
      int ra = kTile, wb = 1, we = 0;
      if (!full) {
        if (i < L_m) {
          ra = (p.bidir ? L_m : i + 1) - k0;
        } else {
          ra = L_m - k0;
          wb = max(L_m, i - p.n + 1) - k0;
          we = i - k0;
        }
      }
      // the 128 scores into registers once
      float s[kTile];
      tmem_ld32(lane_base + colS, s);
      tmem_ld32(lane_base + colS + 32, s + 32);
      tmem_ld32(lane_base + colS + 64, s + 64);
      tmem_ld32(lane_base + colS + 96, s + 96);
      tmem_wait_ld();
      // Speculative pass (every row of the warp has a maximum in use): the
      // exponentials against it, P kept in registers.  A row sum of at most
      // 2^8 bounds every weight by 2^8, so the maximum in use stands and no
      // row maximum is needed; otherwise S is read again from TMEM, its
      // maximum taken and the pass redone (with the new maximum when it grew
      // by more than 8, log2).
      float lt = 0.f, mh = -INFINITY;
      bool redo = true;
      if (__all_sync(0xffffffffu, m_ref != -INFINITY)) {
        uint32_t pk0[kHalf / 2], pk1[kHalf / 2];
        lt = full ? half_exp<true>(s, 0, ra, wb, we, p.scale_log2, m_ref, pk0)
                  : half_exp<false>(s, 0, ra, wb, we, p.scale_log2, m_ref, pk0);
        lt += full ? half_exp<true>(s + kHalf, kHalf, ra, wb, we, p.scale_log2, m_ref, pk1)
                   : half_exp<false>(s + kHalf, kHalf, ra, wb, we, p.scale_log2, m_ref, pk1);
        redo = __any_sync(0xffffffffu, !(lt <= 256.f));
        if (!redo) {
          tmem_st_pairs(lane_base + colS, pk0);
          tmem_st_pairs(lane_base + colS + kHalf / 2, pk1);
        } else {
#pragma unroll 1
          for (int c0 = 0; c0 < kTile; c0 += kHalf) {
            float s2[kHalf];
            tmem_ld32(lane_base + colS + c0, s2);
            tmem_ld32(lane_base + colS + c0 + 32, s2 + 32);
            tmem_wait_ld();
            mh = fmaxf(mh, full ? half_max<true>(s2, c0, ra, wb, we) : half_max<false>(s2, c0, ra, wb, we));
          }
        }
      } else {
        mh = full ? fmaxf(half_max<true>(s, 0, ra, wb, we), half_max<true>(s + kHalf, kHalf, ra, wb, we))
                  : fmaxf(half_max<false>(s, 0, ra, wb, we), half_max<false>(s + kHalf, kHalf, ra, wb, we));
      }
      if (stamp) TC_CYC(j, 2);
      // lazy rescale: only when the max (log2 units) grew by more than 8
      const float mt_s = mh * p.scale_log2;
      const bool grow = redo && mt_s > m_ref + 8.f;
      const float m_new = grow ? mt_s : m_ref;
      const float corr = grow ? ex2(m_ref - m_new) : 1.f;  // 0 when m_ref was -inf
      const float msub = (m_new == -INFINITY) ? 0.f : m_new;
      if (redo) {
        // pass 2: exponentials; P (bf16 pairs) goes over S columns [0, 64)
        lt = 0.f;
#pragma unroll 1
        for (int c0 = 0; c0 < kTile; c0 += kHalf) {
          float s2[kHalf];
          tmem_ld32(lane_base + colS + c0, s2);
          tmem_ld32(lane_base + colS + c0 + 32, s2 + 32);
          tmem_wait_ld();
          uint32_t pk[kHalf / 2];
          lt += full ? half_exp<true>(s2, c0, ra, wb, we, p.scale_log2, msub, pk)
                     : half_exp<false>(s2, c0, ra, wb, we, p.scale_log2, msub, pk);
          tmem_st_pairs(lane_base + colS + c0 / 2, pk);
        }
      }
      if (stamp) TC_CYC(j, 3);
      // O_g was last written by PV_g(j-1), complete before S_g(j) was signalled
      if (j >= 1 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
        for (int c = 0; c < kD; c += 16) {
          float o[16];
          tmem_ld16(lane_base + colO + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] *= corr;
          tmem_st16(lane_base + colO + c, o);
        }
      }
      tmem_wait_st();
      if (stamp) TC_CYC(j, 4);
      l_sum = l_sum * corr + lt;
      m_ref = m_new;
      tc_fence_before();
      mbar_arrive(B(kBarPFull + g));
    }
    // epilogue: O / l to global memory
    if (ok && (*s_abort || !mbar_wait_bounded(B(kBarODone + g), 0))) ok = false;
    tc_fence_after();
    if (!ok) *s_abort = 1;
    const float inv = (ok && !*s_abort) ? 1.f / l_sum : __int_as_float(0x7fc00000);
    __nv_bfloat16* orow = p.O + ((size_t)(ds + i) * p.H + h) * kD;
#pragma unroll 1
    for (int c = 0; c < kD; c += 32) {
      float o[32];
      tmem_ld32(lane_base + colO + c, o);
      tmem_wait_ld();
      if (i < L) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 w;
          w.x = pack_bf16x2(o[e] * inv, o[e + 1] * inv);
          w.y = pack_bf16x2(o[e + 2] * inv, o[e + 3] * inv);
          w.z = pack_bf16x2(o[e + 4] * inv, o[e + 5] * inv);
          w.w = pack_bf16x2(o[e + 6] * inv, o[e + 7] * inv);
          *reinterpret_cast<uint4*>(orow + c + e) = w;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                              : "memory");
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

static bool make_map(CUtensorMap* m, const void* base, int L, int H) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)L};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2};
  const cuuint32_t box[3] = {(cuuint32_t)kBox, 1, (cuuint32_t)kTile};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

// Launches the kernel over the documents of the pack (one document for the
// single-sequence form): every (document, pair of query tiles, head) is one
// CTA.  Entries are ordered by their number of key tiles, heaviest first;
// a pack with more than kMaxWork pairs is split over several launches.
cudaError_t launch_masked_forward_tc(const MaskedParams& mp, cudaStream_t stream) {
  using namespace tc;
  static TcParams p;  // 16 KB: built in static storage, copied by the launch
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  const int rows = mp.cu[mp.n_docs];
  if (!make_map(&p.tmQ, mp.Q, rows, mp.H) || !make_map(&p.tmK, mp.K, rows, mp.H) ||
      !make_map(&p.tmV, mp.V, rows, mp.H))
    return cudaErrorInvalidValue;
  p.O = static_cast<__nv_bfloat16*>(mp.O);
  p.n = mp.n;
  p.H = mp.H;
  p.scale_log2 = mp.scale_log2;
  p.bidir = mp.bidir_prefix;
  p.timing = mp.timing;
  p.kc = static_cast<__nv_bfloat16*>(mp.fill_kc);
  p.vc = static_cast<__nv_bfloat16*>(mp.fill_vc);
  p.S_cap = mp.fill_S_cap;
  p.fill_n = mp.fill_n;
  p.fill_full = mp.fill_full;
  static PerContextOnce attr_once;
  cudaError_t e = attr_once.run(
      [] { return cudaFuncSetAttribute(masked_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmBytes); });
  if (e != cudaSuccess) return e;
  std::vector<std::pair<int, TcWork>> work;  // (key tiles, entry)
  auto flush = [&]() -> cudaError_t {
    if (work.empty()) return cudaSuccess;
    std::stable_sort(work.begin(), work.end(),
                     [](const std::pair<int, TcWork>& a, const std::pair<int, TcWork>& b) { return a.first > b.first; });
    p.n_work = (int)work.size();
    for (size_t i = 0; i < work.size(); ++i) p.work[i] = work[i].second;
    masked_tc_kernel<<<p.n_work * p.H, kThreads, kSmBytes, stream>>>(p);
    work.clear();
    return cudaGetLastError();
  };
  for (int d = 0; d < mp.n_docs; ++d) {
    const int len = mp.cu[d + 1] - mp.cu[d];
    const int n_pairs = (len + kQT * kTile - 1) / (kQT * kTile);
    for (int pr = 0; pr < n_pairs; ++pr) {
      const TileRange tr = tile_range(pr * kQT * kTile, kQT * kTile, len, mp.refs[d], mp.n, mp.bidir_prefix != 0);
      work.push_back({tile_count(tr), TcWork{mp.cu[d], len, mp.refs[d], pr}});
      if ((int)work.size() == kMaxWork)
        if ((e = flush()) != cudaSuccess) return e;
    }
  }
  return flush();
}

}  // namespace rswa
