// Internal interfaces between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace rswa {

// Bits of the device error word (workspace).  Kernels set them with atomicOr
// and return; they never trap.
enum DeviceError : int {
  kErrWaitTimeout = 1 << 0,     // a bounded mbarrier wait gave up
  kErrPlanShort = 1 << 1,       // cache rows exceed the launch plan
  kErrCapacity = 1 << 2,        // FULL mode: more outputs than T_cap
  kErrTmemAlloc = 1 << 3,       // tensor-memory allocation failed
};


// One unit of decode work: a run of up to `chunk` cache rows of one (b, h).
//   bh:        b * H + h
//   row0:      first cache row of the run
//   part:      index of this item's split-K partial
//   nparts:    number of items (= partials) of this (b, h); its partials are
//              part - row0/chunk ... + nparts - 1
struct DecodeItem {
  int32_t bh, row0, part, nparts;
};

// Device workspace layout (byte offsets from the workspace base).
struct WorkspaceLayout {
  size_t err;        // int32: device error word
  size_t done;       // int32: end-of-launch ticket (fused append+decode)
  size_t T;          // int32[B]: outputs appended so far
  size_t Lm;         // int32[B]: reference rows
  size_t tickets;    // int32[B*H]: split-K tickets
  size_t items;      // DecodeItem[items_cap]
  size_t partials;   // float[items_cap][d + 4]: (o[0..d), m, l, pad)
  size_t total;
  int items_cap;
};

WorkspaceLayout workspace_layout(int B, int H, int d);

enum ElemType : int { kF32 = 0, kBF16 = 1 };

struct DecodeParams {
  const void* kc;        // cache [B][H][S_cap][D]
  const void* vc;
  void* kc_w;            // same buffers, written by the fused append
  void* vc_w;
  const void* q;         // [B][H][D]
  void* o;               // [B][H][D]
  const void* k_new;     // [B][H][D] (fused append only)
  const void* v_new;
  int B, H, S_cap;
  int n;                 // ring size (RSWA mode)
  int full_mode;         // 0: ring of n slots, 1: outputs in order
  int T_cap;             // FULL mode capacity
  int chunk;             // rows per item (multiple of 32)
  int n_items;
  int32_t* T;            // [B]
  const int32_t* Lm;     // [B]
  const DecodeItem* items;
  float* partials;
  int32_t* tickets;
  int32_t* done;
  int32_t* err;
  float scale_log2;      // softmax scale * log2(e)
};

// Launch the split-K decode kernel (append: fused ring write + T advance).
cudaError_t launch_decode(int elem, int D, bool append, const DecodeParams& p, int grid,
                          cudaStream_t stream);
// Dynamic shared memory the decode kernel needs for (elem, D).
size_t decode_smem_bytes(int elem, int D);

struct AppendParams {
  void* kc;
  void* vc;
  const void* k_new;
  const void* v_new;
  int B, H, S_cap, row_bytes, n, full_mode, T_cap;
  int32_t* T;
  const int32_t* Lm;
  int32_t* err;
};
cudaError_t launch_append(const AppendParams& p, cudaStream_t stream);

struct LoadRefParams {
  void* kc;
  void* vc;
  const void* K_ref;
  const void* V_ref;
  int B, H, S_cap, row_bytes, ref_stride;
  const int32_t* Lm;   // device [B]
};
cudaError_t launch_load_reference(const LoadRefParams& p, int max_len, cudaStream_t stream);

struct MaskedParams {
  const void* Q;
  const void* K;
  const void* V;
  void* O;
  int L, L_m, n, H, D;
  float scale_log2;
};
cudaError_t launch_masked_forward_simt(const MaskedParams& p, int elem, cudaStream_t stream);

}  // namespace rswa
