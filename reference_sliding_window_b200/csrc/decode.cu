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
// * The planned rows of all (b, h) slabs are laid end to end and cut into
//   one contiguous span per CTA (one persistent CTA per SM), in 32-row
//   stages; a span splits into items at slab boundaries, so only the first
//   and last item of a CTA can be part of a slab shared with another CTA.
// * One producer lane streams the planned K and V stages of its span into a
//   ring of shared-memory buffers with bulk async copies (cp.async.bulk,
//   completion on mbarriers).  It needs no device state, so the first copy
//   is issued right after the plan is read.
// * Stage g (counted over the launch) goes to consumer warp g % kW and ring
//   buffer g % kStages.  kStages is a multiple of kW, so a buffer is only
//   ever consumed by one warp, which waits on it only after consuming its
//   previous phase: every mbarrier parity wait is unambiguous.
// * A consumer warp reads a stage with 16-byte shared loads (one row = LPR
//   lanes), forms LPR partial dot products per lane and reduces them with a
//   transposed butterfly (LPR-1 shuffles leave every lane one finished
//   score), then updates a float32 online softmax (base-2 exponent with the
//   scale folded into q) and its slice of the output.  Rows at or past the
//   current cache length are masked.
// * Warps merge per item in shared memory.  Items of a shared slab leave a
//   partial (m, l, o); at the end of its span a CTA takes one acq_rel ticket
//   per such item and the last CTA of a slab merges its partials with the
//   log-sum-exp rule (one round of independent loads).  Nothing spins.
// * APPEND: the consumer that meets the slot row substitutes the new k/v
//   (the staged copy of that row may predate the write) and stores them into
//   the slot.  Each CTA reads the step counter T once and then takes a
//   launch ticket; the CTA with the last ticket knows every CTA has read T
//   and advances it.  One kernel per decode step, replayable in a CUDA graph.
// * Programmatic dependent launch: barrier set-up, the plan reads and an L2
//   prefetch of the rows to stream happen before waiting on the previous
//   kernel of the stream (the plan is host-written; L2 is coherent), and the
//   next kernel may launch as soon as this one has started.

#include <math.h>
#include <stdio.h>

#include "common.cuh"
#include "internal.h"

namespace rswa {

constexpr int kStageRows = 32;
constexpr int kStageBudget = 192 * 1024;
constexpr long long kPrefetchBytes = 256 * 1024;  // per CTA and per K/V tensor
constexpr int kPrefetchChunk = 32 * 1024;

template <typename T, int D>
struct DecTraits {
  static constexpr int kRowBytes = D * (int)sizeof(T);
  static constexpr int kEPV = 16 / (int)sizeof(T);     // elements per 16-byte vector
  static constexpr int kLPR = kRowBytes / 16;          // lanes covering one row
  static constexpr int kRPI = 32 / kLPR;               // rows per warp-wide load
  static constexpr int kStageBytes = kStageRows * kRowBytes;  // K or V part
  static constexpr int kW = (2 * kStageBytes <= 8192) ? 8 : 6;        // consumer warps
  static constexpr int kDepth = kStageBudget / (2 * kStageBytes * kW);  // buffers per warp
  static constexpr int kStages = kW * kDepth;
  static constexpr int kConsumerThreads = kW * 32;
  static constexpr int kThreads = kConsumerThreads + 32;  // + one producer warp
  static_assert(kLPR >= 8 && kLPR <= 32 && (kLPR & (kLPR - 1)) == 0, "unsupported row size");
  static_assert(kDepth >= 1, "stage budget too small");
  static_assert(kConsumerThreads >= D, "one consumer thread per output dim");
  static constexpr size_t kBarOffset = (size_t)kStages * 2 * kStageBytes;
  static constexpr size_t kRedOffset = kBarOffset + 2 * kStages * 8;
  static constexpr size_t kSmemBytes = kRedOffset + (2 * kW + kW * D) * 4 + 16;
  // partials that fit in the stage ring when it doubles as merge buffer
  static constexpr int kMergeCap = (int)(kBarOffset / ((D + 4) * 4));
};

__device__ __forceinline__ int ld_cg(const int32_t* p) { return __ldcg(p); }

// RSWA_TIMING builds record %globaltimer stamps per CTA (profiling aid).
#ifdef RSWA_TIMING
#define RSWA_STAMP(k) \
  do { if (p.timing) p.timing[blockIdx.x * 8 + (k)] = global_ns(); } while (0)
#else
#define RSWA_STAMP(k) do {} while (0)
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

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Valid cache rows of sequence b when the step counter reads T_now.
__device__ __forceinline__ int valid_rows(const DecodeParams& p, int b, int T_now) {
  const int Lm = p.Lm[b];
  const int len = p.full_mode ? Lm + T_now : Lm + min(p.n, T_now);
  return min(len, p.S_cap);
}

// Log-sum-exp merge of the nparts partials of one slab into its output row.
// A slab's partials are contiguous, so all consumer threads copy them into
// shared memory (the stage ring, idle by then) with independent 16-byte
// loads in one round, then thread `dim` folds them there.  Chunks of
// `cap` partials bound the shared memory used.
template <typename T, int D, int NT>
__device__ __forceinline__ void merge_partials(const DecodeParams& p, const DecodeItem& item, int tid,
                                               float* buf, int cap) {
  constexpr int RW = D + 4;  // floats per partial: o[D], m, l, pad
  const float4* src = reinterpret_cast<const float4*>(p.partials + (size_t)item.part_first * RW);
  float M_run = -INFINITY, L_run = 0.f, o_run = 0.f;
  for (int c0 = 0; c0 < item.nparts; c0 += cap) {
    const int cn = min(cap, item.nparts - c0);
    const int nvec = cn * RW / 4;
    float4* dst = reinterpret_cast<float4*>(buf);
    for (int i = tid; i < nvec; i += NT) dst[i] = __ldcg(src + (size_t)c0 * RW / 4 + i);
    named_barrier_sync(1, NT);
    if (tid < D) {
      float Mc = M_run;
      for (int i = 0; i < cn; ++i) Mc = fmaxf(Mc, buf[i * RW + D]);  // finite: the slab has rows
      const float a = exp2f(M_run - Mc);  // 0 on the first chunk
      float acc = 0.f, Lc = 0.f;
      for (int i = 0; i < cn; ++i) {
        const float w = exp2f(buf[i * RW + D] - Mc);  // exp2(-inf) = 0 for empty partials
        acc = fmaf(w, buf[i * RW + tid], acc);
        Lc = fmaf(w, buf[i * RW + D + 1], Lc);
      }
      o_run = o_run * a + acc;
      L_run = L_run * a + Lc;
      M_run = Mc;
    }
    named_barrier_sync(1, NT);  // buf is reused by the next chunk
  }
  if (tid < D) store_elem(static_cast<T*>(p.o) + (size_t)item.bh * D + tid, o_run / L_run);
}

template <typename T, int D, bool APPEND>
__global__ void __launch_bounds__(DecTraits<T, D>::kThreads, 1)
decode_kernel(const __grid_constant__ DecodeParams p) {
  using Tr = DecTraits<T, D>;
  constexpr int EPV = Tr::kEPV, LPR = Tr::kLPR, RPI = Tr::kRPI, NS = Tr::kStages;
  constexpr int W = Tr::kW, NT = Tr::kConsumerThreads;
  constexpr int RB = Tr::kRowBytes, SB = Tr::kStageBytes;

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + Tr::kBarOffset);
  uint64_t* empty_bar = full_bar + NS;
  float* red_m = reinterpret_cast<float*>(smem + Tr::kRedOffset);
  float* red_l = red_m + W;
  float* red_o = red_l + W;
  volatile int* s_flag = reinterpret_cast<volatile int*>(red_o + W * D);  // [2]
  volatile int* s_abort = s_flag + 2;
  volatile int* s_T = s_flag + 3;
  float* merge_buf = reinterpret_cast<float*>(smem);  // the stage ring, once drained

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    RSWA_STAMP(0);
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 32);  // every lane of the owning warp
    }
    *s_abort = 0;
    fence_barrier_init();
  }
  // The plan is written by the host before any launch that uses it, so it
  // can be read before waiting on the previous kernel.  So can an L2
  // prefetch of the rows this CTA will stream: L2 is coherent, so a row the
  // previous kernel still writes is simply fetched again later.  Bounded so
  // that all CTAs together stay well inside L2.
  const int it_begin = p.cta_begin[blockIdx.x];
  const int it_end = p.cta_begin[blockIdx.x + 1];
  __syncthreads();
  griddep_launch_dependents();
  if (warp == W && lane == 0) {
    long long budget = kPrefetchBytes;
    for (int it = it_begin; it < it_end && budget > 0; ++it) {
      const DecodeItem item = p.items[it];
      const size_t off = ((size_t)item.bh * p.S_cap + item.row0) * RB;
      const long long bytes = min((long long)item.rows * RB, budget);
      for (long long o = 0; o < bytes; o += kPrefetchChunk) {
        const uint32_t nb = (uint32_t)min((long long)kPrefetchChunk, bytes - o);
        bulk_prefetch_l2(static_cast<const uint8_t*>(p.kc) + off + o, nb);
        bulk_prefetch_l2(static_cast<const uint8_t*>(p.vc) + off + o, nb);
      }
      budget -= bytes;
    }
  }
  griddep_wait();  // everything below may read what the previous kernel wrote
  if (threadIdx.x == 0) RSWA_STAMP(1);

  // ------------------------------------------------------------ producer
  if (warp == W) {
    if (lane != 0) return;
    uint32_t g = 0;
    bool ok = true;
    for (int it = it_begin; it < it_end && ok; ++it) {
      const DecodeItem item = p.items[it];
      const int nst = (item.rows + kStageRows - 1) / kStageRows;
      const uint8_t* kb = static_cast<const uint8_t*>(p.kc) + ((size_t)item.bh * p.S_cap + item.row0) * RB;
      const uint8_t* vb = static_cast<const uint8_t*>(p.vc) + ((size_t)item.bh * p.S_cap + item.row0) * RB;
      for (int j = 0; j < nst; ++j, ++g) {
        const int slot = g % NS;
        if (*s_abort || !mbar_wait_bounded(smem_u32(&empty_bar[slot]), ((g / NS) & 1) ^ 1)) {
          flag_error(p.err, kErrWaitTimeout);
          *s_abort = 1;
          ok = false;
          break;
        }
        const int nr = min(kStageRows, item.rows - j * kStageRows);
        const uint32_t bytes = (uint32_t)(nr * RB);
        const uint32_t fb = smem_u32(&full_bar[slot]);
        uint8_t* dst = smem + (size_t)slot * 2 * SB;
        mbar_arrive_expect_tx(fb, 2 * bytes);
        bulk_g2s(smem_u32(dst), kb + (size_t)j * kStageRows * RB, bytes, fb);
        bulk_g2s(smem_u32(dst + SB), vb + (size_t)j * kStageRows * RB, bytes, fb);
        if (g == 0) RSWA_STAMP(2);
      }
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
  if (threadIdx.x == 0) *s_T = ld_cg(p.T);
  named_barrier_sync(1, NT);
  const int T0 = *s_T;
  const int T_step = T0 + (APPEND ? 1 : 0);  // outputs in the cache for this step
  // Launch ticket, taken right after the read of T but only looked at at the
  // end: the CTA holding the last ticket knows every CTA has read T, so it
  // may advance T (the others keep their copy).
  int launch_ticket = 0;
  if (APPEND && threadIdx.x == 0) launch_ticket = atomic_add_release(p.done, 1);
  const int grp = lane / LPR;   // which of the RPI rows of a warp-wide load
  const int sub = lane % LPR;   // which 16-byte slice of the row
  const int tid = threadIdx.x;  // 0 .. NT-1
  uint32_t gctr = 0;
  int pend0 = -1, pend1 = -1;   // split items (at most the first and last of the span)
  int tk0 = 0, tk1 = 0;         // their tickets (valid in thread 0)

  for (int it = it_begin; it < it_end; ++it) {
    const DecodeItem item = p.items[it];
    const int b = item.bh / p.H;
    const int T_now = T_step;
    const int len = valid_rows(p, b, T_now);
    const int live = max(0, min(len - item.row0, item.rows));  // rows to attend
    const int nst = (item.rows + kStageRows - 1) / kStageRows;  // stages streamed
    if (tid == 0 && item.last && len > item.row0 + item.rows) flag_error(p.err, kErrPlanShort);

    int slot_row = -1;
    if (APPEND) {
      const int Lm = p.Lm[b];
      if (p.full_mode) {
        if (T_now <= p.T_cap) slot_row = Lm + T_now - 1;
        else if (tid == 0 && item.row0 == 0) flag_error(p.err, kErrCapacity);
      } else {
        slot_row = Lm + (T_now - 1) % p.n;
      }
    }

    float qf[EPV], of[EPV];
    {
      const uint4 qu =
          *reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) + (size_t)item.bh * D + sub * EPV);
      Vec16<T>::unpack(qu, qf);
#pragma unroll
      for (int e = 0; e < EPV; ++e) {
        qf[e] *= p.scale_log2;
        of[e] = 0.f;
      }
    }
    float m = -INFINITY, l = 0.f;

    // this warp's stages of the item: global stage index = warp (mod W)
    const int j0 = (warp - (int)(gctr % W) + W) % W;
    for (int j = j0; j < nst; j += W) {
      const uint32_t gs = gctr + j;
      const int slot = gs % NS;
      if (*s_abort || !mbar_wait_bounded(smem_u32(&full_bar[slot]), (gs / NS) & 1)) {
        if (lane == 0) {
          flag_error(p.err, kErrWaitTimeout);
          *s_abort = 1;
        }
        break;
      }
      if (gs == 0 && lane == 0) RSWA_STAMP(3);
      const int nr = min(kStageRows, live - j * kStageRows);  // may be <= 0: nothing to attend
      if (nr > 0) {
        const int r_base = item.row0 + j * kStageRows;
        const uint8_t* Ks = smem + (size_t)slot * 2 * SB;
        const uint8_t* Vs = Ks + SB;
        float part[LPR];
        int sub_k = -1;
        uint4 vsub = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int k = 0; k < LPR; ++k) {
          const int row = k * RPI + grp;
          uint4 u = *reinterpret_cast<const uint4*>(Ks + row * RB + sub * 16);
          if (APPEND && r_base + row == slot_row) {
            // The new token: use its k/v from the inputs and store it into its slot.
            const size_t in_off = (size_t)item.bh * D + sub * EPV;
            const size_t c_off = ((size_t)item.bh * p.S_cap + slot_row) * D + sub * EPV;
            u = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.k_new) + in_off);
            vsub = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.v_new) + in_off);
            *reinterpret_cast<uint4*>(static_cast<T*>(p.kc_w) + c_off) = u;
            *reinterpret_cast<uint4*>(static_cast<T*>(p.vc_w) + c_off) = vsub;
            sub_k = k;
          }
          float f[EPV];
          Vec16<T>::unpack(u, f);
          float acc = 0.f;
#pragma unroll
          for (int e = 0; e < EPV; ++e) acc = fmaf(qf[e], f[e], acc);
          part[k] = acc;
        }
        // Transposed butterfly: after log2(LPR) steps lane `sub` of each row
        // group holds the full dot product of row sub*RPI + grp.
#pragma unroll
        for (int mk = LPR / 2; mk >= 1; mk >>= 1) {
          const bool upper = (sub & mk) != 0;
#pragma unroll
          for (int i = 0; i < mk; ++i) {
            const float send = upper ? part[i] : part[i + mk];
            const float keep = upper ? part[i + mk] : part[i];
            part[i] = keep + __shfl_xor_sync(0xffffffffu, send, mk);
          }
        }
        const int my_row = sub * RPI + grp;
        const bool valid = my_row < nr;
        const float sc = valid ? part[0] : -INFINITY;
        float mx = sc;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m, mx);  // finite: the stage has a valid row
        const float corr = exp2f(m - m_new);
        const float pr = valid ? exp2f(sc - m_new) : 0.f;
        l = l * corr + pr;
#pragma unroll
        for (int e = 0; e < EPV; ++e) of[e] *= corr;
#pragma unroll
        for (int k = 0; k < LPR; ++k) {
          const int row = k * RPI + grp;
          const float pk = __shfl_sync(0xffffffffu, pr, grp * LPR + k);
          if (row < nr) {
            uint4 u = *reinterpret_cast<const uint4*>(Vs + row * RB + sub * 16);
            if (APPEND && k == sub_k) u = vsub;
            float f[EPV];
            Vec16<T>::unpack(u, f);
#pragma unroll
            for (int e = 0; e < EPV; ++e) of[e] = fmaf(pk, f[e], of[e]);
          }
        }
        m = m_new;
      }
      // Each lane releases the buffer after its own shared-memory reads.
      mbar_arrive(smem_u32(&empty_bar[slot]));
    }
    gctr += nst;

    // ---- merge the consumer warps of this item
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < EPV; ++e) of[e] += __shfl_xor_sync(0xffffffffu, of[e], off);
    }
    if (grp == 0) {
#pragma unroll
      for (int e = 0; e < EPV; ++e) red_o[warp * D + sub * EPV + e] = of[e];
    }
    if (lane == 0) {
      red_m[warp] = m;
      red_l[warp] = l;
    }
    named_barrier_sync(1, NT);
    if (tid < D) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < W; ++w) M = fmaxf(M, red_m[w]);
      float acc = 0.f, Ls = 0.f;
#pragma unroll
      for (int w = 0; w < W; ++w) {
        const float mw = red_m[w];
        const float wt = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        acc = fmaf(wt, red_o[w * D + tid], acc);
        Ls = fmaf(wt, red_l[w], Ls);
      }
      if (item.nparts == 1) {
        store_elem(static_cast<T*>(p.o) + (size_t)item.bh * D + tid, acc / Ls);
      } else {
        float* P = p.partials + (size_t)item.part * (D + 4);
        P[tid] = acc;
        if (tid == 0) {
          P[D] = M;
          P[D + 1] = Ls;
        }
      }
    }
    named_barrier_sync(1, NT);  // partial written; red_* are reused by the next item
    if (item.nparts > 1) {
      // Ticket with release semantics right away (after the barrier, so it
      // covers every thread's partial writes); its value is read at the end.
      if (pend0 < 0) {
        pend0 = it;
        if (tid == 0) tk0 = atomic_add_release(p.tickets + item.bh, 1);
      } else if (pend1 < 0) {
        pend1 = it;
        if (tid == 0) tk1 = atomic_add_release(p.tickets + item.bh, 1);
      } else if (tid == 0) {  // a span has at most two split items
        flag_error(p.err, kErrPlanShort);
      }
    }
  }

  if (tid == 0) RSWA_STAMP(4);
  // ---- split items: the CTA holding the last ticket of a slab merges it.
  if (tid == 0) {
    int l0 = 0, l1 = 0;
    if (pend0 >= 0) l0 = tk0 == p.items[pend0].nparts - 1;
    if (pend1 >= 0) l1 = tk1 == p.items[pend1].nparts - 1;
    if (l0 || l1) fence_acq_rel_gpu();  // acquire the other CTAs' partials
    s_flag[0] = l0;
    s_flag[1] = l1;
  }
  named_barrier_sync(1, NT);
  for (int i = 0; i < 2; ++i) {
    if (!s_flag[i]) continue;  // uniform across the CTA
    const DecodeItem item = p.items[i == 0 ? pend0 : pend1];
    merge_partials<T, D, NT>(p, item, tid, merge_buf, Tr::kMergeCap);
    if (tid == 0) p.tickets[item.bh] = 0;
    named_barrier_sync(1, NT);
  }

  if (tid == 0) RSWA_STAMP(5);
  if (APPEND && tid == 0 && launch_ticket == (int)gridDim.x - 1) {
    fence_acq_rel_gpu();
    if (p.full_mode && T0 + 1 > p.T_cap) flag_error(p.err, kErrCapacity);
    else *p.T = T0 + 1;
    *p.done = 0;
  }
  if (tid == 0) RSWA_STAMP(6);
}

template <typename T, int D, bool A>
static cudaError_t launch_one(const DecodeParams& p, int grid, cudaStream_t stream) {
  using Tr = DecTraits<T, D>;
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<T, D, A>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Tr::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(Tr::kThreads);
  cfg.dynamicSmemBytes = Tr::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<T, D, A>, p);
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

size_t decode_smem_bytes(int elem, int D) {
  if (elem == kBF16 && D == 128) return DecTraits<__nv_bfloat16, 128>::kSmemBytes;
  if (elem == kBF16 && D == 64) return DecTraits<__nv_bfloat16, 64>::kSmemBytes;
  if (elem == kF32 && D == 128) return DecTraits<float, 128>::kSmemBytes;
  if (elem == kF32 && D == 64) return DecTraits<float, 64>::kSmemBytes;
  return 0;
}

}  // namespace rswa
