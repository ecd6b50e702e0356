// Teacher-forced R-SWA attention on CUDA cores (float32 inputs, or bf16 with
// head dim 64).  One warp per (query row, head), float32 online softmax.
//
// Mask ("Unlimited OCR Works：一篇读懂 R-SWA 如何把长文档 OCR 从 for-loop 推向
// one-shot", 方法展开 §3, Eq.(1)-(2)): the query at 1-based position p
// produces output t = p - L_m + 1 and sees the reference rows 1..L_m plus
// max(L_m+1, p-n+1)..p; a prefix query (p <= L_m) sees 1..p (1..L_m with a
// bidirectional prefix).  So each row visits at most two contiguous key
// ranges and never tests a mask element.  L_m = 0 leaves the window alone.

#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace rswa {

constexpr int kSimtWarps = 4;

template <typename T, int D>
__global__ void __launch_bounds__(kSimtWarps * 32)
masked_simt_kernel(const __grid_constant__ MaskedParams p) {
  constexpr int DPL = D / 32;  // output elements per lane
  __shared__ float qs[kSimtWarps][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * kSimtWarps + warp;  // 0-based query index
  const int h = blockIdx.y;
  if (row >= p.L) return;
  const T* Q = static_cast<const T*>(p.Q);
  const T* K = static_cast<const T*>(p.K);
  const T* V = static_cast<const T*>(p.V);
  T* O = static_cast<T*>(p.O);
  const size_t hs = (size_t)p.H * D;  // token stride

  for (int c = lane; c < D; c += 32) qs[warp][c] = load_elem(Q + row * hs + (size_t)h * D + c) * p.scale_log2;
  __syncwarp();

  // Visible key ranges, 0-based half-open.
  const int pos = row + 1;
  int r0b = 0, r0e, r1b = 0, r1e = 0;
  if (pos <= p.L_m) {
    r0e = p.bidir_prefix ? p.L_m : pos;
  } else {
    r0e = p.L_m;
    r1b = max(p.L_m, pos - p.n);
    r1e = pos;
  }

  float m = -INFINITY, l = 0.f, acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;

  for (int r = 0; r < 2; ++r) {
    const int beg = r == 0 ? r0b : r1b;
    const int end = r == 0 ? r0e : r1e;
    for (int j0 = beg; j0 < end; j0 += 32) {
      const int j = j0 + lane;
      float s = -INFINITY;
      if (j < end) {
        const T* kr = K + j * hs + (size_t)h * D;
        float a = 0.f;
#pragma unroll 8
        for (int c = 0; c < D; ++c) a = fmaf(qs[warp][c], load_elem(kr + c), a);
        s = a;
      }
      float mx = s;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m, mx);
      const float corr = exp2f(m - m_new);
      const float pj = (j < end) ? exp2f(s - m_new) : 0.f;
      l = l * corr + pj;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] *= corr;
      const int cnt = min(32, end - j0);
      for (int t = 0; t < cnt; ++t) {
        const float pt = __shfl_sync(0xffffffffu, pj, t);
        const T* vr = V + (size_t)(j0 + t) * hs + (size_t)h * D;
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[e] = fmaf(pt, load_elem(vr + lane + 32 * e), acc[e]);
      }
      m = m_new;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < DPL; ++e) store_elem(O + row * hs + (size_t)h * D + lane + 32 * e, acc[e] * inv);
}

cudaError_t launch_masked_forward_simt(const MaskedParams& p, int elem, cudaStream_t stream) {
  dim3 grid((p.L + kSimtWarps - 1) / kSimtWarps, p.H);
  if (elem == kF32 && p.D == 64) masked_simt_kernel<float, 64><<<grid, kSimtWarps * 32, 0, stream>>>(p);
  else if (elem == kF32 && p.D == 128) masked_simt_kernel<float, 128><<<grid, kSimtWarps * 32, 0, stream>>>(p);
  else if (elem == kBF16 && p.D == 64) masked_simt_kernel<__nv_bfloat16, 64><<<grid, kSimtWarps * 32, 0, stream>>>(p);
  else if (elem == kBF16 && p.D == 128) masked_simt_kernel<__nv_bfloat16, 128><<<grid, kSimtWarps * 32, 0, stream>>>(p);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace rswa
