// Cache writes: loading the reference segment, and the standalone append of
// one output token into its slot.
//
// The reference segment (vision tokens + prompt) is "encoded once and never
// updated" ("多模态文档解析开源新进展:Unlimited OCR技术方案", R-SWA section):
// it is copied once into rows [0, L_m[b]) of every (b, h) slab.  Outputs go
// to rows L_m[b] + slot.  In RSWA mode slot = (T-1) mod n for output T, so
// output T overwrites output T-n, the entry the fixed-capacity queue evicts
// ("position m+1", same page, KV cache 恒定 section); in FULL mode slot = T-1.
// Rows are moved as 16-byte vectors (row sizes are multiples of 128 bytes).

#include "common.cuh"
#include "internal.h"

namespace rswa {

// One CTA per sequence b: read T once, write the H new rows of k and v,
// then advance T.  No other CTA touches T[b], so there is no race.
__global__ void __launch_bounds__(256) append_kernel(const __grid_constant__ AppendParams p) {
  __shared__ int s_slot, s_T;
  const int b = blockIdx.x;
  if (threadIdx.x == 0) {
    const int Tn = __ldcg(p.T + b) + 1;
    int slot;
    if (p.full_mode) {
      slot = (Tn <= p.T_cap) ? p.Lm[b] + Tn - 1 : -1;
      if (slot < 0) flag_error(p.err, kErrCapacity);
    } else {
      slot = p.Lm[b] + (Tn - 1) % p.n;
    }
    s_slot = slot;
    s_T = Tn;
  }
  __syncthreads();
  const int slot = s_slot;
  if (slot >= 0) {
    const int vpr = p.row_bytes / 16;
    for (int i = threadIdx.x; i < p.H * vpr; i += blockDim.x) {
      const int h = i / vpr, c = i % vpr;
      const size_t bh = (size_t)b * p.H + h;
      const size_t src = bh * p.row_bytes + (size_t)c * 16;
      const size_t dst = (bh * p.S_cap + slot) * p.row_bytes + (size_t)c * 16;
      *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.kc) + dst) =
          *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.k_new) + src);
      *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.vc) + dst) =
          *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.v_new) + src);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && slot >= 0) p.T[b] = s_T;
}

// grid.y = B*H slabs, grid.x covers max_len rows x vectors; copies rows
// [0, Lm[b]) of each slab from the reference tensor into the cache.
__global__ void __launch_bounds__(256) load_reference_kernel(const __grid_constant__ LoadRefParams p) {
  const int bh = blockIdx.y;
  const int b = bh / p.H;
  const int vpr = p.row_bytes / 16;
  const long long n_vec = (long long)p.Lm[b] * vpr;
  const uint8_t* ks = static_cast<const uint8_t*>(p.K_ref) + (size_t)bh * p.ref_stride * p.row_bytes;
  const uint8_t* vs = static_cast<const uint8_t*>(p.V_ref) + (size_t)bh * p.ref_stride * p.row_bytes;
  uint8_t* kd = static_cast<uint8_t*>(p.kc) + (size_t)bh * p.S_cap * p.row_bytes;
  uint8_t* vd = static_cast<uint8_t*>(p.vc) + (size_t)bh * p.S_cap * p.row_bytes;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_vec;
       i += (long long)gridDim.x * blockDim.x) {
    // rows are contiguous in both tensors, so vector i is at byte 16*i
    *reinterpret_cast<uint4*>(kd + i * 16) = *reinterpret_cast<const uint4*>(ks + i * 16);
    *reinterpret_cast<uint4*>(vd + i * 16) = *reinterpret_cast<const uint4*>(vs + i * 16);
  }
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream) {
  append_kernel<<<p.B, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_load_reference(const LoadRefParams& p, int max_len, cudaStream_t stream) {
  const long long vecs = (long long)max_len * (p.row_bytes / 16);
  long long gx = (vecs + 255) / 256;
  if (gx > 1024) gx = 1024;
  if (gx < 1) gx = 1;
  dim3 grid((unsigned)gx, (unsigned)(p.B * p.H));
  load_reference_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace rswa
