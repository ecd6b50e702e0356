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
// Design (B200): the work is a list of items (b, h, run of `chunk` rows),
// statically assigned round-robin to one persistent CTA per SM.  In each CTA
// one producer lane streams 32-row K and V stages from HBM into a ring of
// shared-memory buffers with bulk async copies (cp.async.bulk, completion on
// mbarriers); eight consumer warps take the stages round-robin.  A consumer
// warp reads a stage with 16-byte shared loads (one row = LPR lanes),
// computes the 32 partial dot products per lane, reduces them with a
// transposed butterfly (LPR-1 shuffles give every lane one finished score),
// then updates a float32 online softmax (base-2 exponent with the scale
// folded into q) and its slice of the output.  At the end of an item the
// warps are merged in shared memory; items of one (b, h) are merged by the
// CTA that finishes last (atomic ticket, no spinning) with the log-sum-exp
// rule.  With APPEND the consumer that meets the slot row substitutes the
// new k/v, writes it into the cache, and the last CTA of the launch advances
// the device step counters: one kernel per decode step, replayable in a
// CUDA graph.

#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace rswa {

constexpr int kStageRows = 32;
constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kDecodeThreads = kConsumerThreads + 32;
constexpr int kStageBudget = 192 * 1024;

template <typename T, int D>
struct DecTraits {
  static constexpr int kRowBytes = D * (int)sizeof(T);
  static constexpr int kEPV = 16 / (int)sizeof(T);     // elements per 16-byte vector
  static constexpr int kLPR = kRowBytes / 16;          // lanes covering one row
  static constexpr int kRPI = 32 / kLPR;               // rows per warp-wide load
  static constexpr int kStageBytes = kStageRows * kRowBytes;  // K or V part
  static constexpr int kStages = kStageBudget / (2 * kStageBytes);
  static_assert(kLPR >= 8 && kLPR <= 32 && (kLPR & (kLPR - 1)) == 0, "unsupported row size");
  static constexpr size_t kBarOffset = (size_t)kStages * 2 * kStageBytes;
  static constexpr size_t kRedOffset = kBarOffset + (2 * kStages + 1) * 8;
  static constexpr size_t kSmemBytes =
      kRedOffset + (2 * kConsumerWarps + kConsumerWarps * D) * 4 + 16;
};

__device__ __forceinline__ int ld_cg(const int32_t* p) { return __ldcg(p); }

// Valid cache rows of sequence b when the step counter reads T_now.
__device__ __forceinline__ int valid_rows(const DecodeParams& p, int b, int T_now) {
  const int Lm = p.Lm[b];
  int len = p.full_mode ? Lm + T_now : Lm + min(p.n, T_now);
  return min(len, p.S_cap);
}

template <typename T, int D, bool APPEND>
__global__ void __launch_bounds__(kDecodeThreads, 1)
decode_kernel(const __grid_constant__ DecodeParams p) {
  using Tr = DecTraits<T, D>;
  constexpr int EPV = Tr::kEPV, LPR = Tr::kLPR, RPI = Tr::kRPI, NS = Tr::kStages;
  constexpr int RB = Tr::kRowBytes, SB = Tr::kStageBytes;

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + Tr::kBarOffset);
  uint64_t* empty_bar = full_bar + NS;
  uint64_t* prod_bar = empty_bar + NS;
  float* red_m = reinterpret_cast<float*>(smem + Tr::kRedOffset);
  float* red_l = red_m + kConsumerWarps;
  float* red_o = red_l + kConsumerWarps;
  volatile int* s_flag = reinterpret_cast<volatile int*>(red_o + kConsumerWarps * D);
  volatile int* s_abort = s_flag + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    mbar_init(smem_u32(prod_bar), 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // ------------------------------------------------------------ producer
  if (warp == kConsumerWarps) {
    if (lane != 0) return;
    uint32_t g = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < p.n_items && ok; it += gridDim.x) {
      const DecodeItem item = p.items[it];
      const int b = item.bh / p.H;
      const int T_now = ld_cg(p.T + b) + (APPEND ? 1 : 0);
      const int rows = max(0, min(valid_rows(p, b, T_now) - item.row0, p.chunk));
      const int nst = (rows + kStageRows - 1) / kStageRows;
      const uint8_t* kb = static_cast<const uint8_t*>(p.kc) +
                          ((size_t)item.bh * p.S_cap + item.row0) * RB;
      const uint8_t* vb = static_cast<const uint8_t*>(p.vc) +
                          ((size_t)item.bh * p.S_cap + item.row0) * RB;
      for (int j = 0; j < nst; ++j, ++g) {
        const int slot = g % NS;
        const uint32_t ph = (g / NS) & 1;
        if (*s_abort || !mbar_wait_bounded(smem_u32(&empty_bar[slot]), ph ^ 1)) {
          flag_error(p.err, kErrWaitTimeout);
          *s_abort = 1;
          ok = false;
          break;
        }
        const int nr = min(kStageRows, rows - j * kStageRows);
        const uint32_t bytes = (uint32_t)(nr * RB);
        const uint32_t fb = smem_u32(&full_bar[slot]);
        uint8_t* dst = smem + (size_t)slot * 2 * SB;
        mbar_arrive_expect_tx(fb, 2 * bytes);
        bulk_g2s(smem_u32(dst), kb + (size_t)j * kStageRows * RB, bytes, fb);
        bulk_g2s(smem_u32(dst + SB), vb + (size_t)j * kStageRows * RB, bytes, fb);
      }
    }
    mbar_arrive(smem_u32(prod_bar));  // every read of T by the producer is done
    // Drain: never leave the CTA with bulk copies still writing shared memory.
    const uint32_t first = g > (uint32_t)NS ? g - NS : 0;
    for (uint32_t k = first; k < g; ++k) {
      if (!mbar_wait_bounded(smem_u32(&full_bar[k % NS]), (k / NS) & 1)) {
        flag_error(p.err, kErrWaitTimeout);
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int grp = lane / LPR;   // which of the RPI rows of a warp-wide load
  const int sub = lane % LPR;   // which 16-byte slice of the row
  const int tid = threadIdx.x;  // 0 .. kConsumerThreads-1
  uint32_t gctr = 0;

  for (int it = blockIdx.x; it < p.n_items; it += gridDim.x) {
    const DecodeItem item = p.items[it];
    const int b = item.bh / p.H;
    const int T_now = ld_cg(p.T + b) + (APPEND ? 1 : 0);
    const int len = valid_rows(p, b, T_now);
    const int rows = max(0, min(len - item.row0, p.chunk));
    const int nst = (rows + kStageRows - 1) / kStageRows;
    if (tid == 0 && item.row0 == 0 && len > item.nparts * p.chunk) flag_error(p.err, kErrPlanShort);

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

    for (int j = warp; j < nst; j += kConsumerWarps) {
      const uint32_t gs = gctr + j;
      const int slot = gs % NS;
      if (*s_abort || !mbar_wait_bounded(smem_u32(&full_bar[slot]), (gs / NS) & 1)) {
        if (lane == 0) {
          flag_error(p.err, kErrWaitTimeout);
          *s_abort = 1;
        }
        break;
      }
      const int nr = min(kStageRows, rows - j * kStageRows);
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
          // The new token: use its k/v from the inputs (the staged copy of
          // this row may predate the write) and store it into its slot.
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
      const float m_new = fmaxf(m, mx);  // finite: every stage has a valid row
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
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty_bar[slot]));
    }
    gctr += nst;

    // ---- merge the eight warps of this item
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
    named_barrier_sync(1, kConsumerThreads);

    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, red_m[w]);
    T* out = static_cast<T*>(p.o) + (size_t)item.bh * D;
    if (tid < D) {
      float acc = 0.f, Ls = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float mw = red_m[w];
        const float wt = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        acc = fmaf(wt, red_o[w * D + tid], acc);
        Ls = fmaf(wt, red_l[w], Ls);
      }
      if (item.nparts == 1) {
        store_elem(out + tid, acc / Ls);
      } else {
        float* P = p.partials + (size_t)item.part * (D + 4);
        P[tid] = acc;
        if (tid == 0) {
          P[D] = M;
          P[D + 1] = Ls;
        }
      }
    }
    if (item.nparts > 1) {
      __threadfence();
      named_barrier_sync(1, kConsumerThreads);
      if (tid == 0) {
        const int old = atomicAdd(p.tickets + item.bh, 1);
        *s_flag = (old == item.nparts - 1);
      }
      named_barrier_sync(1, kConsumerThreads);
      if (*s_flag) {
        // Last CTA of this (b, h): log-sum-exp merge of all partials.
        __threadfence();
        const float* P0 = p.partials + (size_t)(item.part - item.row0 / p.chunk) * (D + 4);
        if (tid < D) {
          float Mx = -INFINITY;
          for (int i = 0; i < item.nparts; ++i) Mx = fmaxf(Mx, __ldcg(P0 + (size_t)i * (D + 4) + D));
          float acc = 0.f, Ls = 0.f;
          for (int i = 0; i < item.nparts; ++i) {
            const float* Pi = P0 + (size_t)i * (D + 4);
            const float mi = __ldcg(Pi + D);
            const float wt = (mi == -INFINITY) ? 0.f : exp2f(mi - Mx);
            acc = fmaf(wt, __ldcg(Pi + tid), acc);
            Ls = fmaf(wt, __ldcg(Pi + D + 1), Ls);
          }
          store_elem(out + tid, acc / Ls);
        }
        if (tid == 0) p.tickets[item.bh] = 0;
      }
    }
    named_barrier_sync(1, kConsumerThreads);
  }

  // ---- fused append: the last CTA of the launch advances T.
  if (APPEND && tid == 0) {
    if (!mbar_wait_bounded(smem_u32(prod_bar), 0)) flag_error(p.err, kErrWaitTimeout);
    __threadfence();
    const int old = atomicAdd(p.done, 1);
    if (old == (int)gridDim.x - 1) {
      __threadfence();
      for (int b = 0; b < p.B; ++b) {
        const int Tn = ld_cg(p.T + b) + 1;
        if (p.full_mode && Tn > p.T_cap) {
          flag_error(p.err, kErrCapacity);
        } else {
          p.T[b] = Tn;
        }
      }
      *p.done = 0;
    }
  }
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
  decode_kernel<T, D, A><<<grid, kDecodeThreads, Tr::kSmemBytes, stream>>>(p);
  return cudaGetLastError();
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
