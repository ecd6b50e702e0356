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

#include "cache_copy.h"
#include "common.cuh"
#include "internal.h"

namespace rswa {

// One CTA: read the step counter T once, write the B*H new rows of k and v
// into their slots, then advance every copy of T.  Only this CTA touches T,
// so there is no race.  (Not the hot path: decoding uses the fused kernel.)
__global__ void __launch_bounds__(256) append_kernel(const __grid_constant__ AppendParams p) {
  __shared__ int s_T, s_ok;
  if (threadIdx.x == 0) {
    const int Tn = __ldcg(p.T) + 1;
    const int ok = !p.full_mode || Tn <= p.T_cap;
    if (!ok) flag_error(p.err, kErrCapacity);
    s_T = Tn;
    s_ok = ok;
  }
  __syncthreads();
  const int Tn = s_T;
  if (s_ok) {
    const int vpr = p.row_bytes / 16;
    const long long total = (long long)p.B * p.H * vpr;
    for (long long i = threadIdx.x; i < total; i += blockDim.x) {
      const int bh = (int)(i / vpr), c = (int)(i % vpr);
      const int b = bh / p.H;
      const int slot = p.full_mode ? p.Lm[b] + Tn - 1 : p.Lm[b] + (Tn - 1) % p.n;
      const size_t src = (size_t)bh * p.row_bytes + (size_t)c * 16;
      const size_t dst = ((size_t)bh * p.S_cap + slot) * p.row_bytes + (size_t)c * 16;
      *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.kc) + dst) =
          *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.k_new) + src);
      *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.vc) + dst) =
          *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.v_new) + src);
    }
  }
  __syncthreads();
  if (s_ok)
    for (int e = threadIdx.x; e < kStepSlots; e += blockDim.x) p.T[e] = Tn;
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
  // Decode kernels launched after this one copy reference rows before their
  // dependency wait: make this block's writes visible GPU-wide before it
  // retires.
  __threadfence();
}

// grid.y = B*H slabs, grid.x covers the occupied rows x vectors of a slab.
// Fills the cache as T0 appends after a reference load would have, straight
// from the packed (teacher-forced) layout, where output t of sequence b is
// packed row Lm[b] + t - 1.  Cache row Lm[b] + s (ring slot s) holds the
// newest output t <= T0 with (t - 1) mod n == s; the ring keeps outputs
// T0-W+1 .. T0, W = min(n, T0), so t - 1 = t0 + ((s - t0) mod n) with
// t0 = T0 - W.  In FULL mode slot s holds output s + 1.
__global__ void __launch_bounds__(256) load_packed_kernel(const __grid_constant__ LoadPackedParams p) {
  const int bh = blockIdx.y;
  const int b = bh / p.H, h = bh % p.H;
  const int Lm = p.Lm[b];
  const int W = p.full_mode ? p.T0 : min(p.n, p.T0);
  const int t0 = p.T0 - W;
  const int vpr = p.row_bytes / 16;
  const long long n_vec = (long long)(Lm + W) * vpr;
  const size_t src_row_pitch = (size_t)p.H * p.row_bytes;
  const uint8_t* ks = static_cast<const uint8_t*>(p.K) + (size_t)b * p.seq_stride * src_row_pitch +
                      (size_t)h * p.row_bytes;
  const uint8_t* vs = static_cast<const uint8_t*>(p.V) + (size_t)b * p.seq_stride * src_row_pitch +
                      (size_t)h * p.row_bytes;
  uint8_t* kd = static_cast<uint8_t*>(p.kc) + (size_t)bh * p.S_cap * p.row_bytes;
  uint8_t* vd = static_cast<uint8_t*>(p.vc) + (size_t)bh * p.S_cap * p.row_bytes;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_vec;
       i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / vpr), c = (int)(i % vpr);
    int src = r;
    if (r >= Lm && !p.full_mode) {
      const int s = r - Lm;
      src = Lm + t0 + ((s - t0 % p.n) + p.n) % p.n;
    }
    const size_t so = (size_t)src * src_row_pitch + (size_t)c * 16;
    const size_t dof = (size_t)r * p.row_bytes + (size_t)c * 16;
    *reinterpret_cast<uint4*>(kd + dof) = *reinterpret_cast<const uint4*>(ks + so);
    *reinterpret_cast<uint4*>(vd + dof) = *reinterpret_cast<const uint4*>(vs + so);
  }
  if (blockIdx.x == 0 && blockIdx.y == 0)
    for (int e = threadIdx.x; e < kStepSlots; e += blockDim.x) p.T[e] = p.T0;
  // Same contract as load_reference_kernel: decode kernels may copy
  // reference rows before their dependency wait.
  __threadfence();
}

// grid.y = B*H slabs: appends one chunk of reference rows after the rows
// already loaded ("encoded once": a reference can arrive page by page, each
// page's rows written once and never again).
__global__ void __launch_bounds__(256) load_chunk_kernel(const __grid_constant__ LoadChunkParams p) {
  const int bh = blockIdx.y;
  const int b = bh / p.H;
  const int rows = p.rows[b];
  const int dst0 = p.Lm[b] - rows;
  const int vpr = p.row_bytes / 16;
  const long long n_vec = (long long)rows * vpr;
  const uint8_t* ks = static_cast<const uint8_t*>(p.K) + (size_t)bh * p.chunk_stride * p.row_bytes;
  const uint8_t* vs = static_cast<const uint8_t*>(p.V) + (size_t)bh * p.chunk_stride * p.row_bytes;
  uint8_t* kd = static_cast<uint8_t*>(p.kc) + ((size_t)bh * p.S_cap + dst0) * p.row_bytes;
  uint8_t* vd = static_cast<uint8_t*>(p.vc) + ((size_t)bh * p.S_cap + dst0) * p.row_bytes;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_vec;
       i += (long long)gridDim.x * blockDim.x) {
    *reinterpret_cast<uint4*>(kd + i * 16) = *reinterpret_cast<const uint4*>(ks + i * 16);
    *reinterpret_cast<uint4*>(vd + i * 16) = *reinterpret_cast<const uint4*>(vs + i * 16);
  }
  // Same contract as load_reference_kernel: decode kernels may copy
  // reference rows before their dependency wait.
  __threadfence();
}

cudaError_t launch_load_chunk(const LoadChunkParams& p, int max_rows, cudaStream_t stream) {
  const long long vecs = (long long)max_rows * (p.row_bytes / 16);
  long long gx = (vecs + 255) / 256;
  if (gx > 1024) gx = 1024;
  if (gx < 1) gx = 1;
  dim3 grid((unsigned)gx, (unsigned)(p.B * p.H));
  load_chunk_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream) {
  append_kernel<<<1, 256, 0, stream>>>(p);
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

cudaError_t launch_load_packed(const LoadPackedParams& p, int max_rows, cudaStream_t stream) {
  const long long vecs = (long long)max_rows * (p.row_bytes / 16);
  long long gx = (vecs + 255) / 256;
  if (gx > 1024) gx = 1024;
  if (gx < 1) gx = 1;
  dim3 grid((unsigned)gx, (unsigned)(p.B * p.H));
  load_packed_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace rswa
