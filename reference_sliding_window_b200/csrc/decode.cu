// Split-K decode attention over an R-SWA cache, with an optional fused
// append of the new token's key/value into its ring slot.
//
// Operation ("Unlimited OCR Works：一篇读懂 R-SWA 如何把长文档 OCR 从 for-loop
// 推向 one-shot", 方法展开 §3, Eq.(3)-(4)): for each (b, h),
//   o = sum_j softmax_j(q.k_j * scale) v_j   over the valid cache rows,
// where the valid rows of sequence b are [0, L_m[b] + min(n, T[b])) in RSWA
// mode (reference rows followed by the n-slot output ring, Eq.(6)) and
// [0, L_m[b] + T[b]) in FULL mode (Eq.(5)).  Softmax over a set does not
// depend on storage order, so ring rows can be read in slot order.
//
// Design (B200):
// * Two launch plans (made on the host).  Span plan: the planned rows of all
//   (b, h) slabs are laid end to end and cut into one contiguous span per
//   CTA (one persistent CTA per SM), in 32-row stages; a span splits into
//   items at slab boundaries, so only the first and last item of a CTA can
//   be part of a slab shared with another CTA.  Cluster plan, when every
//   slab can have a resident cluster of its own: slab bh goes to the
//   kDecodeCluster CTAs of cluster bh, one contiguous part each (the leader
//   and the last rank take the short shares).  Each plan is its own kernel
//   instantiation (template parameter CLUSTER).
// * Before waiting on the previous kernel (programmatic dependent launch):
//   barrier set-up, the plan and reference lengths (host-written) staged in
//   shared memory, copies of the leading stages (reference rows, and ring
//   rows when the host allows it: see the prologue), and an L2 prefetch of
//   the remaining rows, q and the new rows.  q, the new rows and the step
//   counter are read after the wait.  The next kernel may launch once this
//   one has passed its own wait.
// * One producer lane streams the stages into a ring of shared-memory
//   buffers with bulk async copies (cp.async.bulk, completion on mbarriers).
// * Stage g (32 rows, counted over the launch) goes to consumer warp group
//   g % kGroups and ring buffer g % kStages; the kSplit warps of a group
//   each take kWarpRows rows of it.  kStages is a multiple of kGroups, so a
//   buffer is only ever consumed by one group, whose warps wait on it only
//   after consuming its previous phase: every mbarrier parity wait is
//   unambiguous.
// * A warp's part of a stage is NV = 8 warp-wide 16-byte loads of K (and of
//   V): 16 rows of bf16 d=128.  The warp reads it from shared memory (one
//   row = LPR lanes), forms NV partial dot products per lane (bf16:
//   mixed-precision FMAs on the packed words) and reduces them with a
//   transposed butterfly over NV lanes plus plain shuffles over the rest of
//   the row's lanes (NV-1 + log2(LPR/NV) shuffles leave every lane one
//   finished score), then updates a float32 online softmax (base 2, with a
//   lazy running maximum) and its slice of the output (bf16 caches: P.V with
//   the weight rounded to bf16, fp32 accumulation).  Rows at or past the
//   current cache length are masked.  Splitting stages over warps keeps the serial work of one warp
//   short (at small cache sizes the launch is latency-bound) while the
//   copies stay 8 KB each.
// * Warps merge per batch of items in shared memory.  Items of a shared
//   slab leave a partial (m, l, o).  Span plan: one release fence and a
//   relaxed ticket per split item; the CTA holding a slab's last ticket
//   acquires and merges the slab's partials with the log-sum-exp rule (one
//   round of independent loads).  Cluster plan: each CTA writes its partial
//   into its own shared memory and one thread sends it to the leader CTA's
//   shared memory with a bulk copy that completes bytes on the leader's
//   mbarrier (no release fence or arrival round trip); the leader, whose
//   barrier expects the other CTAs' bytes, waits and merges.
// * APPEND: the consumer that meets the slot row substitutes the new k/v
//   (the staged copy of that row may predate the write) and stores them into
//   the slot.  The step counter T has one copy per CTA: each CTA reads its
//   own copy and at its end writes T + 1 into copies no other CTA of the
//   launch reads (kStepSlots in internal.h), so advancing T costs no atomic
//   and no fence.  One kernel per decode step, replayable in a CUDA graph.
// * Every wait is bounded; a timeout sets the device error word and the
//   kernel finishes without trapping.

#include <math.h>
#include <stdio.h>

#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace rswa {

constexpr int kStageBudget = 192 * 1024;
constexpr long long kPrefetchBytes = 256 * 1024;  // per CTA and per K/V tensor
constexpr int kPrefetchChunk = 32 * 1024;
// Items per CTA whose descriptor, reference length and query (raw for bf16, scaled for fp32) are
// staged in shared memory by the prologue; later items of a longer span
// read them from global memory when they start.
constexpr int kPreItems = 8;
// Items a CTA processes together: the warps run their stages of both before
// one barrier, so a span that crosses a slab boundary costs one round.
constexpr int kBatch = 2;

template <typename T, int D>
struct DecTraits {
  static constexpr int kRowBytes = D * (int)sizeof(T);
  static constexpr int kEPV = 16 / (int)sizeof(T);     // elements per 16-byte vector
  static constexpr int kLPR = kRowBytes / 16;          // lanes covering one row
  static constexpr int kRPI = 32 / kLPR;               // rows per warp-wide load
  static constexpr int kNV = 8;                        // warp-wide loads per K (or V) part
  static constexpr int kStageRows = 32;                // rows per copied stage
  static constexpr int kWarpRows = kNV * kRPI;         // 16 (bf16 d=128), 32 (bf16 d=64), 8 (f32 d=128)
  static constexpr int kSplit = kStageRows / kWarpRows;  // warps sharing a stage
  static constexpr int kStageBytes = kStageRows * kRowBytes;  // K or V part
  static constexpr int kW = 12;                        // consumer warps
  static constexpr int kGroups = kW / kSplit;          // warp groups, one stage each at a time
  static constexpr int kDepth = kStageBudget / (2 * kStageBytes * kGroups);  // buffers per group
  static constexpr int kStages = kGroups * kDepth;
  static constexpr int kConsumerThreads = kW * 32;
  static constexpr int kThreads = kConsumerThreads + 32;  // + one producer warp
  static_assert(kLPR >= kNV && kLPR <= 32 && (kLPR & (kLPR - 1)) == 0, "unsupported row size");
  static_assert(kStageRows % kWarpRows == 0 && kW % kSplit == 0, "stage split");
  static_assert(kDepth >= 1, "stage budget too small");
  static_assert(kConsumerThreads >= D, "one consumer thread per output dim");
  static constexpr size_t kBarOffset = (size_t)kStages * 2 * kStageBytes;
  static constexpr size_t kRedOffset = kBarOffset + 2 * kStages * 8;
  // staged items: DecodeItem[kPreItems], int32 L_m[kPreItems], float q[kPreItems][D]
  static constexpr size_t kMetaOffset = (kRedOffset + kBatch * (2 * kW + kW * D) * 4 + 16 + 15) / 16 * 16;
  static constexpr size_t kLmOffset = kMetaOffset + sizeof(DecodeItem) * kPreItems;
  static constexpr size_t kQOffset = kLmOffset + 4 * kPreItems;
  // cluster merge: the leader's mbarrier and partials[kDecodeCluster][D + 4]
  // fused append: the new key and value rows of the staged items, [kPreItems][row] each
  static constexpr size_t kKnOffset = (kQOffset + 4 * (size_t)kPreItems * D + 15) / 16 * 16;
  static constexpr size_t kVnOffset = kKnOffset + (size_t)kPreItems * kRowBytes;
  static constexpr size_t kClBarOffset = (kVnOffset + (size_t)kPreItems * kRowBytes + 15) / 16 * 16;
  static constexpr size_t kClBufOffset = kClBarOffset + 16;
  static constexpr size_t kSmemBytes = kClBufOffset + 4 * (size_t)kDecodeCluster * (D + 4);
  static_assert(kSmemBytes <= 227 * 1024, "dynamic shared memory above the per-CTA limit");
  // partials that fit in the stage ring when it doubles as merge buffer
  static constexpr int kMergeCap = (int)(kBarOffset / ((D + 4) * 4));
};

__device__ __forceinline__ int ld_cg(const int32_t* p) { return __ldcg(p); }

// 2^x by the XU instruction (arguments here are at most 8; results below
// 2^-126 flush to zero, negligible beside the weight of the running maximum).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// RSWA_TIMING builds record %globaltimer stamps per CTA (profiling aid).
#ifdef RSWA_TIMING
#define RSWA_STAMP(k) \
  do { if (p.timing) p.timing[blockIdx.x * 32 + (k)] = global_ns(); } while (0)
#define RSWA_CYC(k) \
  do { if (p.timing) p.timing[blockIdx.x * 32 + 16 + (k)] = clock64(); } while (0)
#else
#define RSWA_STAMP(k) do {} while (0)
#define RSWA_CYC(k) do {} while (0)
#endif

__device__ __forceinline__ int atomic_add_acq_rel(int32_t* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Release-only ticket: orders this thread's earlier accesses before the
// increment without making later ones wait; the result is consumed late.
__device__ __forceinline__ int atomic_add_release(int32_t* p, int v) {
  int old;
  asm volatile("atom.release.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Relaxed ticket: no ordering of its own (callers fence where needed).
__device__ __forceinline__ int atomic_add_relaxed(int32_t* p, int v) {
  int old;
  asm volatile("atom.relaxed.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// acc + a.lo*b.lo + a.hi*b.hi for two packed bf16 pairs, with fp32
// accumulation (each bf16 product is exact in fp32).
__device__ __forceinline__ float fma2_bf16(uint32_t a, uint32_t b, float acc) {
  asm("{.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
      : "+f"(acc)
      : "r"(a), "r"(b));
  return acc;
}

// lo += p2.lo * w.lo, hi += p2.hi * w.hi for packed bf16 pairs, fp32
// accumulation (P.V with the weight rounded to bf16, as a tensor-core P.V
// takes it; each product is exact in fp32).
__device__ __forceinline__ void fma_bf16_pair(uint32_t p2, uint32_t w, float& lo, float& hi) {
  asm("{.reg .b16 pl, ph, wl, wh;\n\t"
      "mov.b32 {pl, ph}, %2;\n\t"
      "mov.b32 {wl, wh}, %3;\n\t"
      "fma.rn.f32.bf16 %0, pl, wl, %0;\n\t"
      "fma.rn.f32.bf16 %1, ph, wh, %1;\n\t}"
      : "+f"(lo), "+f"(hi)
      : "r"(p2), "r"(w));
}
// ---- thread-block cluster helpers (cluster-merge plan)
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// Every thread of every CTA of the cluster (all threads must execute it).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Bounded wait on a local mbarrier phase with cluster-scope acquire (the
// bytes came from other CTAs of the cluster).  Its limit is four times the
// others': a CTA whose own waits timed out still sends its partial, about
// one limit late, and the leader must outlive every copy into its shared
// memory.
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (true) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
    if (clock64() - t0 > 4 * kWaitLimitCycles) return false;
  }
}

__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void bulk_s2cluster(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "r"(src), "r"(bytes), "r"(bar) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// x mod n for 0 <= x < 2^31 by a multiply (the divisor's magic number comes
// with the parameters): q = floor(x * M / 2^k) with k = 32 + ceil(log2 n)
// and M = ceil(2^k / n) is exact there, since M * n - 2^k < n <= 2^(k-32)
// keeps the error of x * M / 2^k below 1 / n (Granlund and Montgomery,
// "Division by invariant integers using multiplication", 1994).
__device__ __forceinline__ int mod_n(const DecodeParams& p, int x) {
  const unsigned q = (unsigned)(((unsigned long long)(unsigned)x * p.n_magic) >> p.n_shift);
  return x - (int)q * p.n;
}

// Valid cache rows of a sequence with Lm reference rows when the step
// counter reads T_now.
__device__ __forceinline__ int valid_rows(const DecodeParams& p, int Lm, int T_now) {
  const int len = p.full_mode ? Lm + T_now : Lm + min(p.n, T_now);
  return min(len, p.S_cap);
}

// Log-sum-exp merge of the partials of up to two slabs into their output
// rows.  A slab's partials are contiguous, so all consumer threads copy both
// slabs' partials into shared memory (the stage ring, idle by then) with
// independent 16-byte loads in one round, then thread x*D + dim folds item x.
// The host planner keeps a slab within kMergeCap / 2 partials, so two always
// fit.
template <typename T, int D, int NT>
__device__ __forceinline__ void merge_partials_joint(const DecodeParams& p, const DecodeItem& i0,
                                                     const DecodeItem& i1, int n_its, int tid, float* buf) {
  constexpr int RW = D + 4;
  const int nv0 = i0.nparts * RW / 4;
  const int nv = nv0 + (n_its > 1 ? i1.nparts * RW / 4 : 0);
  const float4* s0 = reinterpret_cast<const float4*>(p.partials + (size_t)i0.part_first * RW);
  const float4* s1 = reinterpret_cast<const float4*>(p.partials + (size_t)i1.part_first * RW);
  float4* dst = reinterpret_cast<float4*>(buf);
  for (int i = tid; i < nv; i += 4 * NT) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = i + u * NT;
      if (j < nv) v[u] = __ldcg(j < nv0 ? s0 + j : s1 + (j - nv0));
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (i + u * NT < nv) dst[i + u * NT] = v[u];
  }
  named_barrier_sync(1, NT);
  if (tid < n_its * D) {
    const int x = tid / D, dd = tid % D;
    const float* bx = buf + (x ? i0.nparts * RW : 0);
    const int np = x ? i1.nparts : i0.nparts;
    float M = -INFINITY;
    for (int i = 0; i < np; ++i) M = fmaxf(M, bx[i * RW + D]);  // finite: the slab has rows
    float acc = 0.f, L = 0.f;
    for (int i = 0; i < np; ++i) {
      const float w = exp2f(bx[i * RW + D] - M);  // exp2(-inf) = 0 for empty partials
      acc = fmaf(w, bx[i * RW + dd], acc);
      L = fmaf(w, bx[i * RW + D + 1], L);
    }
    store_elem(static_cast<T*>(p.o) + (size_t)(x ? i1.bh : i0.bh) * D + dd, acc / L);
  }
  named_barrier_sync(1, NT);
}

// The fused append's slot row, taken by one lane group of one part per slab
// and step: this lane's 16 bytes of k_new and v_new (staged in shared memory
// for the first kPreItems items) go into the part's registers and the ring
// slot.
template <typename T, int D>
__device__ __forceinline__ void slot_row_kv(const DecodeParams& p, int bh, int slot_row, int li, int sub,
                                            const uint8_t* s_kn, const uint8_t* s_vn, uint4& kn, uint4& vn) {
  constexpr int EPV = 16 / (int)sizeof(T), RB = D * (int)sizeof(T);
  const size_t in_off = (size_t)bh * D + sub * EPV;
  const size_t c_off = ((size_t)bh * p.S_cap + slot_row) * D + sub * EPV;
  if (li < kPreItems) {
    kn = reinterpret_cast<const uint4*>(s_kn + li * RB)[sub];
    vn = reinterpret_cast<const uint4*>(s_vn + li * RB)[sub];
  } else {
    kn = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.k_new) + in_off);
    vn = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.v_new) + in_off);
  }
  *reinterpret_cast<uint4*>(static_cast<T*>(p.kc_w) + c_off) = kn;
  *reinterpret_cast<uint4*>(static_cast<T*>(p.vc_w) + c_off) = vn;
}

// The same, out of line. The cluster plan's short parts run faster with the
// rarely taken copy outside the part loop (4.83 -> 4.78 us per single-document
// launch); the span plan's long streams run faster with it inline (1.8% on a
// ragged batch).
template <typename T, int D>
__device__ __noinline__ void slot_row_kv_outlined(const DecodeParams& p, int bh, int slot_row, int li, int sub,
                                                  const uint8_t* s_kn, const uint8_t* s_vn, uint4& kn,
                                                  uint4& vn) {
  slot_row_kv<T, D>(p, bh, slot_row, li, sub, s_kn, s_vn, kn, vn);
}

// CLUSTER: the cluster plan (a separate instantiation, so that neither plan
// carries the other's code and registers).
template <typename T, int D, bool APPEND, bool CLUSTER>
__global__ void __launch_bounds__(DecTraits<T, D>::kThreads, 1)
decode_kernel(const __grid_constant__ DecodeParams p) {
  using Tr = DecTraits<T, D>;
  constexpr int EPV = Tr::kEPV, LPR = Tr::kLPR, RPI = Tr::kRPI, NS = Tr::kStages, NV = Tr::kNV;
  constexpr int kStageRows = Tr::kStageRows, WR = Tr::kWarpRows, GR = Tr::kGroups;
  // bf16: q.k from the packed words with mixed-precision FMAs (q unscaled,
  // the scale applied to the finished score); fp32: unpacked, q scaled.
  constexpr bool kMixed = std::is_same<T, __nv_bfloat16>::value;
  constexpr int W = Tr::kW, NT = Tr::kConsumerThreads;
  constexpr int RB = Tr::kRowBytes, SB = Tr::kStageBytes;

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + Tr::kBarOffset);
  uint64_t* empty_bar = full_bar + NS;
  float* red_m = reinterpret_cast<float*>(smem + Tr::kRedOffset);  // [kBatch][W]
  float* red_l = red_m + kBatch * W;                                // [kBatch][W]
  float* red_o = red_l + kBatch * W;                                // [kBatch][W][D]
  volatile int* s_flag = reinterpret_cast<volatile int*>(red_o + kBatch * W * D);  // [2]
  volatile int* s_abort = s_flag + 2;
  volatile int* s_T = s_flag + 3;
  DecodeItem* s_items = reinterpret_cast<DecodeItem*>(smem + Tr::kMetaOffset);
  int* s_lm = reinterpret_cast<int*>(smem + Tr::kLmOffset);
  float* s_q = reinterpret_cast<float*>(smem + Tr::kQOffset);
  uint8_t* s_kn = smem + Tr::kKnOffset;
  uint8_t* s_vn = smem + Tr::kVnOffset;
  const uint32_t cl_bar = smem_u32(smem + Tr::kClBarOffset);
  float* cl_buf = reinterpret_cast<float*>(smem + Tr::kClBufOffset);  // [kDecodeCluster][D + 4]
  float* merge_buf = reinterpret_cast<float*>(smem);  // the stage ring, once drained

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  static_assert(kStepSlots <= NT, "one step-counter copy per consumer thread at most");
  if (threadIdx.x == 0) {
    RSWA_STAMP(0);
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 32 * Tr::kSplit);  // every lane of the owning group
    }
    *s_abort = 0;
    if (CLUSTER) mbar_init(cl_bar, 1);  // the leader's own arrival; the others complete bytes
    fence_barrier_init();
  }
  // The plan and the reference lengths are written by host copies ordered
  // before any launch that uses them, so they can be read (and the first
  // kPreItems items staged in shared memory) before waiting on the previous
  // kernel.  So can an L2 prefetch of the rows this CTA will stream: L2 is
  // coherent, so a row the previous kernel still writes is simply fetched
  // again later.
  // Cluster plan: one item per CTA, derived from the CTA index and the
  // per-slab sizes in the parameters exactly as the host planner makes it,
  // so no chain of dependent global loads delays the first copies.
  const int it_begin = CLUSTER ? (int)blockIdx.x : p.cta_begin[blockIdx.x];
  const int it_end = CLUSTER ? (int)blockIdx.x + 1 : p.cta_begin[blockIdx.x + 1];
  const int n_pre = min(it_end - it_begin, kPreItems);
  if ((int)threadIdx.x < n_pre) {
    DecodeItem item;
    int lm;
    if (CLUSTER) {
      const int c = blockIdx.x, bh = c / kDecodeCluster, r = c % kDecodeCluster;
      const int rows_bh = p.cl_rows[bh], S = (rows_bh + 31) / 32;
      const int st0 = cluster_stage_begin(S, r), st1 = cluster_stage_begin(S, r + 1);
      item.bh = bh;
      item.row0 = st0 * 32;
      item.rows = max(0, min(rows_bh, st1 * 32) - item.row0);
      item.part = c;
      item.part_first = bh * kDecodeCluster;
      item.nparts = kDecodeCluster;
      item.last = r == kDecodeCluster - 1;
      item.pad = 0;
      lm = p.cl_lm[bh];
    } else {
      item = p.items[it_begin + threadIdx.x];
      lm = p.Lm[item.bh / p.H];
    }
    s_items[threadIdx.x] = item;
    s_lm[threadIdx.x] = lm;
  }
  __syncthreads();
  // Cluster-merge plan: the leader's barrier must be initialised before any
  // CTA of the cluster arrives on it.  Every thread passes here (no thread
  // has exited yet), so this hardware barrier cannot be left waiting.
  if (CLUSTER) cluster_sync_all();
  auto item_at = [&](int it) -> DecodeItem {
    const int li = it - it_begin;
    return li < kPreItems ? s_items[li] : p.items[it];
  };
  auto lm_at = [&](int it, const DecodeItem& item) -> int {
    const int li = it - it_begin;
    return li < kPreItems ? s_lm[li] : p.Lm[item.bh / p.H];
  };
  // Stage issue, in stage order g over the span: (it, j) is the next stage.
  int p_it = it_begin, p_j = 0;
  uint32_t g = 0;
  auto issue = [&](const DecodeItem& item, int j) {
    const int slot = g % NS;
    const int nr = min(kStageRows, item.rows - j * kStageRows);
    const uint32_t bytes = (uint32_t)(nr * RB);
    const size_t row = (size_t)item.bh * p.S_cap + item.row0 + (size_t)j * kStageRows;
    const uint32_t fb = smem_u32(&full_bar[slot]);
    uint8_t* dst = smem + (size_t)slot * 2 * SB;
    mbar_arrive_expect_tx(fb, 2 * bytes);
    bulk_g2s(smem_u32(dst), static_cast<const uint8_t*>(p.kc) + row * RB, bytes, fb);
    bulk_g2s(smem_u32(dst + SB), static_cast<const uint8_t*>(p.vc) + row * RB, bytes, fb);
    if (g == 0) RSWA_STAMP(2);
    ++g;
  };
  // With ref_stable the leading stages made only of reference rows are
  // copied before the dependency wait, into buffers that are still free
  // (g < NS): only the cache loads and the prefill fill write them, and
  // those kernels never let a dependent start before they retire.  With
  // ring_early, leading stages that hold ring rows are copied early too.
  // Ring rows are written by those kernels and by a fused append+decode,
  // which lets the next kernel start only after its own dependency wait
  // (above), so when this CTA runs, every decode before the previous kernel
  // has retired; the host sets ring_early only when the previous kernel it
  // launched on the stream was not a decode of this handle.
  if (warp == W && lane == 0 && p.ref_stable) {
    while (p_it < it_end && g < (uint32_t)NS) {
      const DecodeItem item = item_at(p_it);
      const int nst = (item.rows + kStageRows - 1) / kStageRows;
      if (p_j >= nst) {
        ++p_it;
        p_j = 0;
        continue;
      }
      const int nr = min(kStageRows, item.rows - p_j * kStageRows);
      if (!p.ring_early && item.row0 + p_j * kStageRows + nr > lm_at(p_it, item)) break;
      issue(item, p_j);
      ++p_j;
    }
  }
  // L2 prefetch of the rows not copied early (bounded so that all CTAs
  // together stay well inside L2).
  if (warp == W && lane == 0) {
    long long budget = kPrefetchBytes;
    for (int it = p_it; it < it_end && budget > 0; ++it) {
      const DecodeItem item = item_at(it);
      const int r0 = it == p_it ? min(p_j * kStageRows, item.rows) : 0;
      const size_t off = ((size_t)item.bh * p.S_cap + item.row0 + r0) * RB;
      const long long bytes = min((long long)(item.rows - r0) * RB, budget);
      for (long long o = 0; o < bytes; o += kPrefetchChunk) {
        const uint32_t nb = (uint32_t)min((long long)kPrefetchChunk, bytes - o);
        bulk_prefetch_l2(static_cast<const uint8_t*>(p.kc) + off + o, nb);
        bulk_prefetch_l2(static_cast<const uint8_t*>(p.vc) + off + o, nb);
      }
      budget -= bytes;
    }
  }
#ifdef RSWA_TIMING
  if (warp == W - 1 && lane == 0 && it_begin < it_end) {  // when the first stage lands
    mbar_wait_bounded(smem_u32(&full_bar[0]), 0);
    RSWA_STAMP(12);
  }
#endif
  // q, the new rows and this CTA's copy of T into L2 (coherent: a value the
  // previous kernel still writes is fetched again when read after the wait).
  if (warp == W && lane == 1) {
    for (int i = 0; i < n_pre; ++i) {
      const size_t off = (size_t)s_items[i].bh * D * sizeof(T);
      bulk_prefetch_l2(static_cast<const uint8_t*>(p.q) + off, D * sizeof(T));
      if (APPEND) {
        bulk_prefetch_l2(static_cast<const uint8_t*>(p.k_new) + off, D * sizeof(T));
        bulk_prefetch_l2(static_cast<const uint8_t*>(p.v_new) + off, D * sizeof(T));
      }
    }
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p.T + (APPEND ? blockIdx.x : 0)));
  }
  griddep_wait();  // everything below may read what the previous kernel wrote
  // Only now may the next kernel start: every kernel before this one has
  // retired by then, which is what lets a decode copy ring rows before its
  // own wait (prologue).
  griddep_launch_dependents();
  if (threadIdx.x == 0) RSWA_STAMP(1);

  // ------------------------------------------------------------ producer
  if (warp == W) {
    if (lane != 0) return;
    bool ok = true;
    while (p_it < it_end && ok) {
      const DecodeItem item = item_at(p_it);
      const int nst = (item.rows + kStageRows - 1) / kStageRows;
      if (p_j >= nst) {
        ++p_it;
        p_j = 0;
        continue;
      }
      const int slot = g % NS;
      if (*s_abort || !mbar_wait_bounded(smem_u32(&empty_bar[slot]), ((g / NS) & 1) ^ 1)) {
        flag_error(p.err, kErrWaitTimeout);
        *s_abort = 1;
        ok = false;
        break;
      }
      issue(item, p_j);
      ++p_j;
    }
    // Drain: never leave the CTA with bulk copies still writing shared memory.
    const uint32_t first = g > (uint32_t)NS ? g - NS : 0;
    for (uint32_t k = first; k < g; ++k) {
      if (!mbar_wait_bounded(smem_u32(&full_bar[k % NS]), (k / NS) & 1)) flag_error(p.err, kErrWaitTimeout);
    }
    RSWA_STAMP(7);
    return;
  }

  // ------------------------------------------------------------ consumers
  // The step counter (this CTA's copy) and the queries of the staged items
  // are outputs of earlier kernels: one round of independent loads, every
  // load issued before any result is used.
  {
    constexpr int VPR = D / EPV;  // 16-byte vectors per query row
    static_assert(kPreItems * VPR <= NT, "one query vector per consumer thread");
    const int x = threadIdx.x;
    int t_val = 0;
    if (x == 0) t_val = ld_cg(p.T + (APPEND ? blockIdx.x : 0));
    uint4 qu = make_uint4(0, 0, 0, 0), kn = qu, vn = qu;
    if (x < n_pre * VPR) {
      const size_t off = (size_t)s_items[x / VPR].bh * D + (x % VPR) * EPV;
      qu = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) + off);
      if (APPEND) {  // the new rows, for the consumer that meets the slot row
        kn = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.k_new) + off);
        vn = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.v_new) + off);
      }
    }
    if (x == 0) *s_T = t_val;
    if (x < n_pre * VPR) {
      const int i = x / VPR, v = x % VPR;
      if (APPEND) {
        reinterpret_cast<uint4*>(s_kn + i * RB)[v] = kn;
        reinterpret_cast<uint4*>(s_vn + i * RB)[v] = vn;
      }
      if (kMixed) {
        reinterpret_cast<uint4*>(s_q + i * D)[v] = qu;  // raw bf16
      } else {
        float f[EPV];
        Vec16<T>::unpack(qu, f);
#pragma unroll
        for (int e = 0; e < EPV; ++e) s_q[i * D + v * EPV + e] = f[e] * p.scale_log2;
      }
    }
  }
  named_barrier_sync(1, NT);
  if (threadIdx.x == 0) {
    RSWA_STAMP(8);
    RSWA_CYC(0);
  }
  const int T0 = *s_T;
  const int T_step = T0 + (APPEND ? 1 : 0);  // outputs in the cache for this step
  const int group = warp / Tr::kSplit;            // stage group of this warp
  const int part_row = (warp % Tr::kSplit) * WR;  // its first row inside a stage
  const int grp = lane / LPR;   // which of the RPI rows of a warp-wide load
  const int sub = lane % LPR;   // which 16-byte slice of the row
  const int tid = threadIdx.x;  // 0 .. NT-1
  uint32_t gctr = 0;
  int pend0 = -1, pend1 = -1;   // split items (at most the first and last of the span)
  int tk0 = 0, tk1 = 0;         // their tickets (valid in thread 0)

  for (int it0 = it_begin; it0 < it_end; it0 += kBatch) {
   const int nb = min(kBatch, it_end - it0);
   for (int x = 0; x < nb; ++x) {
    const int it = it0 + x;
    const int li = it - it_begin;
    // (branches, not selects: the staged case must not wait on a global load)
    DecodeItem item;
    int Lm_b;
    if (li < kPreItems) {
      item = s_items[li];
      Lm_b = s_lm[li];
    } else {
      item = p.items[it];
      Lm_b = p.Lm[item.bh / p.H];
    }
    const int T_now = T_step;
    const int len = valid_rows(p, Lm_b, T_now);
    const int live = max(0, min(len - item.row0, item.rows));  // rows to attend
    const int nst = (item.rows + kStageRows - 1) / kStageRows;  // stages streamed
    if (tid == 0 && item.last && len > item.row0 + item.rows) flag_error(p.err, kErrPlanShort);

    int slot_row = -1;
    if (APPEND) {
      if (p.full_mode) {
        if (T_now <= p.T_cap) slot_row = Lm_b + T_now - 1;
        else if (tid == 0 && item.row0 == 0) flag_error(p.err, kErrCapacity);
      } else {
        slot_row = Lm_b + mod_n(p, T_now - 1);
      }
    }

    float qf[EPV], of[EPV];
    uint4 qraw = make_uint4(0, 0, 0, 0);
    if (kMixed) {
      if (li < kPreItems)
        qraw = reinterpret_cast<const uint4*>(s_q + li * D)[sub];
      else
        qraw = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) + (size_t)item.bh * D + sub * EPV);
    } else if (li < kPreItems) {
#pragma unroll
      for (int e = 0; e < EPV; e += 4) {
        const float4 q4 = *reinterpret_cast<const float4*>(s_q + li * D + sub * EPV + e);
        qf[e] = q4.x;
        qf[e + 1] = q4.y;
        qf[e + 2] = q4.z;
        qf[e + 3] = q4.w;
      }
    } else {
      const uint4 qu =
          *reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) + (size_t)item.bh * D + sub * EPV);
      Vec16<T>::unpack(qu, qf);
#pragma unroll
      for (int e = 0; e < EPV; ++e) qf[e] *= p.scale_log2;
    }
#pragma unroll
    for (int e = 0; e < EPV; ++e) of[e] = 0.f;
    float m = -INFINITY, l = 0.f;

    // this warp group's stages of the item: global stage index = group (mod GR)
    const int j0 = (group - (int)(gctr % GR) + GR) % GR;
    if (tid == 0 && it == it_begin) RSWA_CYC(1);
    for (int j = j0; j < nst; j += GR) {
      const uint32_t gs = gctr + j;
      const int slot = gs % NS;
      if (*s_abort || !mbar_wait_bounded(smem_u32(&full_bar[slot]), (gs / NS) & 1)) {
        if (lane == 0) {
          flag_error(p.err, kErrWaitTimeout);
          *s_abort = 1;
        }
        break;
      }
      if (gs == 0 && lane == 0) {
        RSWA_STAMP(3);
        RSWA_CYC(2);
      }
      // this warp's rows of the stage: [part_row, part_row + WR)
      const int nr = min(WR, live - j * kStageRows - part_row);  // may be <= 0: nothing to attend
      if (nr > 0) {
        const int r_base = item.row0 + j * kStageRows + part_row;
        const uint8_t* Ks = smem + (size_t)slot * 2 * SB + part_row * RB;
        const uint8_t* Vs = Ks + SB;
        float part[NV];
        int sub_k = -1;
        uint4 vsub = make_uint4(0, 0, 0, 0);
        uint4 ku[NV];
#pragma unroll
        for (int k = 0; k < NV; ++k) ku[k] = *reinterpret_cast<const uint4*>(Ks + (k * RPI + grp) * RB + sub * 16);
        if (APPEND) {
          const int rel = slot_row - r_base - grp;
          if (rel >= 0 && rel < NV * RPI && rel % RPI == 0) {
            // The new token: use its k/v from the inputs and store it into its slot.
            sub_k = rel / RPI;
            uint4 kn;
            if constexpr (CLUSTER)
              slot_row_kv_outlined<T, D>(p, item.bh, slot_row, li, sub, s_kn, s_vn, kn, vsub);
            else
              slot_row_kv<T, D>(p, item.bh, slot_row, li, sub, s_kn, s_vn, kn, vsub);
#pragma unroll
            for (int k = 0; k < NV; ++k)
              if (k == sub_k) ku[k] = kn;
          }
        }
#pragma unroll
        for (int k = 0; k < NV; ++k) {
          const uint4 u = ku[k];
          float acc = 0.f;
          if (kMixed) {
            acc = fma2_bf16(qraw.x, u.x, acc);
            acc = fma2_bf16(qraw.y, u.y, acc);
            acc = fma2_bf16(qraw.z, u.z, acc);
            acc = fma2_bf16(qraw.w, u.w, acc);
          } else {
            float f[EPV];
            Vec16<T>::unpack(u, f);
#pragma unroll
            for (int e = 0; e < EPV; ++e) acc = fmaf(qf[e], f[e], acc);
          }
          part[k] = acc;
        }
        if (gs == 0 && lane == 0) RSWA_CYC(3);
        // Transposed butterfly over the low log2(NV) lane bits: lane `sub`
        // keeps value sub % NV summed over its NV-lane group; then plain
        // shuffles sum the groups of the row, so every lane holds the full
        // dot product of row (sub % NV) * RPI + grp.
#pragma unroll
        for (int mk = NV / 2; mk >= 1; mk >>= 1) {
          const bool upper = (sub & mk) != 0;
#pragma unroll
          for (int i = 0; i < mk; ++i) {
            const float send = upper ? part[i] : part[i + mk];
            const float keep = upper ? part[i + mk] : part[i];
            part[i] = keep + __shfl_xor_sync(0xffffffffu, send, mk);
          }
        }
#pragma unroll
        for (int mk = NV; mk < LPR; mk <<= 1) part[0] += __shfl_xor_sync(0xffffffffu, part[0], mk);
        const int my_row = (sub % NV) * RPI + grp;
        const bool valid = my_row < nr;
        const bool owner = sub < NV;  // one lane per row adds to the sum
        if (gs == 0 && lane == 0) RSWA_CYC(4);
        const float sc = valid ? (kMixed ? part[0] * p.scale_log2 : part[0]) : -INFINITY;
        // Lazy running maximum: exponents stay <= 2^8 over the maximum in use,
        // so the maximum is reduced (and o, l rescaled) only when a score
        // exceeds it by more than 8.  A warp's first maximum in use is the
        // score of the part's row 0 (valid here), not a reduction.
        if (m == -INFINITY) m = __shfl_sync(0xffffffffu, sc, 0);
        if (__any_sync(0xffffffffu, sc > m + 8.f)) {
          float mx = sc;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
          const float m_new = fmaxf(m, mx);  // finite: the stage has a valid row
          const float corr = ex2_approx(m - m_new);
          l *= corr;
#pragma unroll
          for (int e = 0; e < EPV; ++e) of[e] *= corr;
          m = m_new;
        }
        const float pr = valid ? ex2_approx(sc - m) : 0.f;
        l += owner ? pr : 0.f;
        if (gs == 0 && lane == 0) RSWA_CYC(5);
        uint4 vu[NV];
        float pk[NV];
#pragma unroll
        for (int k = 0; k < NV; ++k) vu[k] = *reinterpret_cast<const uint4*>(Vs + (k * RPI + grp) * RB + sub * 16);
        // bf16: the weight is rounded once, by the lane that holds it, and
        // broadcast packed
        uint32_t pk2[NV];
        if (kMixed) {
          uint32_t pr2;
          asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(pr2) : "f"(pr));
#pragma unroll
          for (int k = 0; k < NV; ++k) pk2[k] = __shfl_sync(0xffffffffu, pr2, grp * LPR + k);
        } else {
#pragma unroll
          for (int k = 0; k < NV; ++k) pk[k] = __shfl_sync(0xffffffffu, pr, grp * LPR + k);
        }
        if (APPEND && sub_k >= 0) {
#pragma unroll
          for (int k = 0; k < NV; ++k)
            if (k == sub_k) vu[k] = vsub;
        }
#pragma unroll
        for (int k = 0; k < NV; ++k) {
          if (k * RPI + grp < nr) {
            if (kMixed) {
              fma_bf16_pair(pk2[k], vu[k].x, of[0], of[1]);
              fma_bf16_pair(pk2[k], vu[k].y, of[2], of[3]);
              fma_bf16_pair(pk2[k], vu[k].z, of[4], of[5]);
              fma_bf16_pair(pk2[k], vu[k].w, of[6], of[7]);
            } else {
              float f[EPV];
              Vec16<T>::unpack(vu[k], f);
#pragma unroll
              for (int e = 0; e < EPV; ++e) of[e] = fmaf(pk[k], f[e], of[e]);
            }
          }
        }
      }
      if (gs == 0 && lane == 0) {
        RSWA_STAMP(9);
        RSWA_CYC(6);
      }
      // Each lane releases the buffer after its own shared-memory reads.
      mbar_arrive(smem_u32(&empty_bar[slot]));
    }
    gctr += nst;

    // ---- this warp's partial of item x: (m, l, o) into shared memory
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < EPV; ++e) of[e] += __shfl_xor_sync(0xffffffffu, of[e], off);
    }
    if (grp == 0) {
#pragma unroll
      for (int e = 0; e < EPV; ++e) red_o[(x * W + warp) * D + sub * EPV + e] = of[e];
    }
    if (lane == 0) {
      red_m[x * W + warp] = m;
      red_l[x * W + warp] = l;
    }
   }
    // ---- merge the consumer warps of the batch's items (thread x*D + d)
    named_barrier_sync(1, NT);
    if (tid < nb * D) {
      const int x = tid / D, dd = tid % D;
      const DecodeItem item = item_at(it0 + x);
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < W; ++w) M = fmaxf(M, red_m[x * W + w]);
      float acc = 0.f, Ls = 0.f;
#pragma unroll
      for (int w = 0; w < W; ++w) {
        const float mw = red_m[x * W + w];
        const float wt = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        acc = fmaf(wt, red_o[(x * W + w) * D + dd], acc);
        Ls = fmaf(wt, red_l[x * W + w], Ls);
      }
      if (item.nparts == 1) {
        store_elem(static_cast<T*>(p.o) + (size_t)item.bh * D + dd, acc / Ls);
      } else if (CLUSTER) {
        // this CTA's partial into slot `rank` of the cluster leader's buffer
        float* mine = cl_buf + (size_t)cluster_rank() * (D + 4);
        mine[dd] = acc;
        if (dd == 0) {
          mine[D] = M;
          mine[D + 1] = Ls;
        }
        fence_proxy_async_smem();
      } else {
        float* P = p.partials + (size_t)item.part * (D + 4);
        P[dd] = acc;
        if (dd == 0) {
          P[D] = M;
          P[D + 1] = Ls;
        }
      }
    }
    named_barrier_sync(1, NT);  // partials written; red_* are reused by the next batch
    if (tid == 0 && it0 == it_begin) RSWA_STAMP(10);
    if (CLUSTER) {
      // one item per CTA: arrive on the leader's barrier with release at
      // cluster scope (after the barrier, so it covers every thread's stores)
      if (tid == 0 && item_at(it0).nparts > 1) {
        const uint32_t rank = cluster_rank();
        if (rank == 0) {
          mbar_arrive_expect_tx(cl_bar, (kDecodeCluster - 1) * (D + 4) * 4);
        } else {
          const uint32_t src = smem_u32(cl_buf + (size_t)rank * (D + 4));
          bulk_s2cluster(cluster_map(src, 0), src, (D + 4) * 4, cluster_map(cl_bar, 0));
          bulk_commit();
        }
      }
      continue;
    }
    // Tickets of the batch's split items right away: one release fence
    // (after the barrier, so it covers every thread's partial writes), then
    // relaxed increments in flight together; their values are read at the end.
    bool fenced = false;
    for (int x = 0; x < nb; ++x) {
      const int it = it0 + x;
      const DecodeItem item = item_at(it);
      if (item.nparts > 1) {
        if (tid == 0 && !fenced) {
          fence_acq_rel_gpu();
          fenced = true;
        }
        if (pend0 < 0) {
          pend0 = it;
          if (tid == 0) tk0 = atomic_add_relaxed(p.tickets + item.bh, 1);
        } else if (pend1 < 0) {
          pend1 = it;
          if (tid == 0) tk1 = atomic_add_relaxed(p.tickets + item.bh, 1);
        } else if (tid == 0) {  // a span has at most two split items
          flag_error(p.err, kErrPlanShort);
        }
      }
    }
  }

  if (tid == 0) RSWA_STAMP(4);
  // ---- cluster-merge plan: the leader folds the cluster's partials
  if (CLUSTER && it_end > it_begin && cluster_rank() == 0 && item_at(it_begin).nparts > 1 && tid < D) {
    const DecodeItem item = item_at(it_begin);
    const bool ok = mbar_wait_cluster_bounded(cl_bar, 0);
    if (!ok && tid == 0) flag_error(p.err, kErrWaitTimeout);
    if (ok) {
      float M = -INFINITY;
#pragma unroll
      for (int i = 0; i < kDecodeCluster; ++i) M = fmaxf(M, cl_buf[i * (D + 4) + D]);  // finite: the slab has rows
      float acc = 0.f, L = 0.f;
#pragma unroll
      for (int i = 0; i < kDecodeCluster; ++i) {
        const float w = exp2f(cl_buf[i * (D + 4) + D] - M);  // exp2(-inf) = 0 for an empty part
        acc = fmaf(w, cl_buf[i * (D + 4) + tid], acc);
        L = fmaf(w, cl_buf[i * (D + 4) + D + 1], L);
      }
      store_elem(static_cast<T*>(p.o) + (size_t)item.bh * D + tid, acc / L);
    }
  }
  // ---- split items (span plan): the CTA holding the last ticket of a slab
  // merges it.  (The condition is uniform across the CTA.)
  if (!CLUSTER) {
    if (tid == 0) {
      int l0 = 0, l1 = 0;
      if (pend0 >= 0) l0 = tk0 == item_at(pend0).nparts - 1;
      if (pend1 >= 0) l1 = tk1 == item_at(pend1).nparts - 1;
      if (l0 || l1) fence_acq_rel_gpu();  // acquire the other CTAs' partials
      s_flag[0] = l0;
      s_flag[1] = l1;
      RSWA_STAMP(11);
    }
    named_barrier_sync(1, NT);
    {
      // the slabs this CTA merges (uniform across the CTA): m0, then m1
      const int f0 = s_flag[0], f1 = s_flag[1];
      const int nm = f0 + f1;
      if (nm > 0) {
        const DecodeItem m0 = item_at(f0 ? pend0 : pend1);
        const DecodeItem m1 = item_at(pend1 >= 0 ? pend1 : pend0);
        // The host planner keeps every slab within kMergeCap / 2 partials.
        if (m0.nparts + (nm > 1 ? m1.nparts : 0) <= Tr::kMergeCap) {
          merge_partials_joint<T, D, NT>(p, m0, m1, nm, tid, merge_buf);
        } else if (tid == 0) {
          flag_error(p.err, kErrPlanShort);
        }
        if (tid == 0) {
          RSWA_STAMP(13);
          p.tickets[m0.bh] = 0;
          if (nm > 1) p.tickets[m1.bh] = 0;
        }
      }
    }
  }

  if (tid == 0) RSWA_STAMP(5);
  if (CLUSTER && tid == 0) bulk_wait_read();  // the partial has left this CTA's shared memory
  // Advance T: copies blockIdx.x, blockIdx.x + grid, ... (kStepSlots <= NT,
  // one store per thread), none of which another CTA of this launch reads.
  if (APPEND && !(p.full_mode && T0 + 1 > p.T_cap)) {
    const int e = blockIdx.x + tid * gridDim.x;
    if (e < kStepSlots) p.T[e] = T0 + 1;
  }
  if (APPEND && tid == 0 && blockIdx.x == 0 && p.full_mode && T0 + 1 > p.T_cap) flag_error(p.err, kErrCapacity);
  if (tid == 0) RSWA_STAMP(6);
}

template <typename T, int D, bool A>
static cudaError_t launch_one(const DecodeParams& p, int grid, cudaStream_t stream) {
  using Tr = DecTraits<T, D>;
  static PerContextOnce attr_once;
  cudaError_t e = attr_once.run([] {
    cudaError_t e1 = cudaFuncSetAttribute(decode_kernel<T, D, A, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)Tr::kSmemBytes);
    if (e1 != cudaSuccess) return e1;
    return cudaFuncSetAttribute(decode_kernel<T, D, A, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)Tr::kSmemBytes);
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(Tr::kThreads);
  cfg.dynamicSmemBytes = Tr::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = p.cluster_merge ? kDecodeCluster : 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.cluster_merge ? 2 : 1;
  return p.cluster_merge ? cudaLaunchKernelEx(&cfg, decode_kernel<T, D, A, true>, p)
                         : cudaLaunchKernelEx(&cfg, decode_kernel<T, D, A, false>, p);
}

template <typename T, int D>
static int max_clusters(void) {
  using Tr = DecTraits<T, D>;
  if (cudaFuncSetAttribute(decode_kernel<T, D, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Tr::kSmemBytes) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kDecodeCluster);
  cfg.blockDim = dim3(Tr::kThreads);
  cfg.dynamicSmemBytes = Tr::kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kDecodeCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_kernel<T, D, true, true>, &cfg) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error so later calls are unaffected
    return 0;
  }
  return n;
}

int decode_max_active_clusters(int elem, int D) {
  if (elem == kBF16 && D == 128) return max_clusters<__nv_bfloat16, 128>();
  if (elem == kBF16 && D == 64) return max_clusters<__nv_bfloat16, 64>();
  if (elem == kF32 && D == 128) return max_clusters<float, 128>();
  if (elem == kF32 && D == 64) return max_clusters<float, 64>();
  return 0;
}

template <typename T, int D>
static cudaError_t launch_d(bool append, const DecodeParams& p, int grid, cudaStream_t s) {
  return append ? launch_one<T, D, true>(p, grid, s) : launch_one<T, D, false>(p, grid, s);
}

cudaError_t launch_decode(int elem, int D, bool append, const DecodeParams& p, int grid,
                          cudaStream_t stream) {
  if (elem == kBF16 && D == 128) return launch_d<__nv_bfloat16, 128>(append, p, grid, stream);
  if (elem == kBF16 && D == 64) return launch_d<__nv_bfloat16, 64>(append, p, grid, stream);
  if (elem == kF32 && D == 128) return launch_d<float, 128>(append, p, grid, stream);
  if (elem == kF32 && D == 64) return launch_d<float, 64>(append, p, grid, stream);
  return cudaErrorInvalidValue;
}

static_assert(DecTraits<__nv_bfloat16, 128>::kMergeCap >= kMinMergeCap &&
                  DecTraits<__nv_bfloat16, 64>::kMergeCap >= kMinMergeCap &&
                  DecTraits<float, 128>::kMergeCap >= kMinMergeCap && DecTraits<float, 64>::kMergeCap >= kMinMergeCap,
              "the planners' CTA cap assumes every variant merges kMinMergeCap partials");

size_t decode_smem_bytes(int elem, int D) {
  if (elem == kBF16 && D == 128) return DecTraits<__nv_bfloat16, 128>::kSmemBytes;
  if (elem == kBF16 && D == 64) return DecTraits<__nv_bfloat16, 64>::kSmemBytes;
  if (elem == kF32 && D == 128) return DecTraits<float, 128>::kSmemBytes;
  if (elem == kF32 && D == 64) return DecTraits<float, 64>::kSmemBytes;
  return 0;
}

}  // namespace rswa
