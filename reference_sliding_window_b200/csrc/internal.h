// Internal interfaces between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

namespace rswa {

// Identity of the calling thread's current CUDA context (cuCtxGetId: never
// reused within a process, so a context created after a device reset gets a
// new one), or 0 if none is current or the driver does not provide it.
unsigned long long current_context_id();

// Host set-up that must run once per CUDA context of a device (a kernel's
// shared-memory attribute, a symbol's device address), thread-safe.  run()
// calls f() unless it already succeeded in the current context of the
// current device.
class PerContextOnce {
 public:
  template <typename F>
  cudaError_t run(F&& f) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu_);
    const unsigned long long id = current_context_id();
    if (id != 0 && done_[dev] == id) return cudaSuccess;
    e = f();
    if (e == cudaSuccess) done_[dev] = id != 0 ? id : current_context_id();
    return e;
  }

 private:
  static constexpr int kMaxDevices = 64;
  std::mutex mu_;
  unsigned long long done_[kMaxDevices] = {};
};

// Bits of the device error word (workspace).  Kernels set them with atomicOr
// and return; they never trap.
enum DeviceError : int {
  kErrWaitTimeout = 1 << 0,     // a bounded mbarrier wait gave up
  kErrPlanShort = 1 << 1,       // cache rows exceed the launch plan
  kErrCapacity = 1 << 2,        // FULL mode: more outputs than T_cap
  kErrTmemAlloc = 1 << 3,       // tensor-memory allocation failed
};


// One unit of decode work: a run of cache rows of one (b, h) slab, processed
// by one CTA.  Each CTA owns a contiguous range of items (a span of the
// concatenated slabs), so a CTA has at most a few items and a slab is split
// over at most a few CTAs.
//   bh:          b * H + h
//   row0, rows:  first cache row and planned row count (a multiple of 32
//                except at the end of the slab)
//   part:        index of this item's split-K partial
//   part_first, nparts: the partials of this (b, h)
//   last:        1 if this item ends the planned rows of its slab
struct DecodeItem {
  int32_t bh, row0, rows, part;
  int32_t part_first, nparts, last, pad;
};

// The step counter T is kept as kStepSlots equal copies.  A fused
// append+decode launch has every CTA read its own copy and, when done, write
// T + 1 into the copies c, c + grid, c + 2*grid, ...: no CTA reads a copy
// that another CTA of the same launch writes, so no ticket or fence is needed
// to advance T.  Every other writer sets all copies; readers on the host use
// copy 0.  A decode grid never exceeds kStepSlots CTAs.
constexpr int kStepSlots = 256;

// Slabs (b, h) the cluster plan serves at most (its per-slab sizes travel in
// the kernel parameters).
constexpr int kClusterPlanMaxSlabs = 32;

// Device workspace layout (byte offsets from the workspace base).
struct WorkspaceLayout {
  size_t err;        // int32: device error word
  size_t T;          // int32[kStepSlots]: outputs appended so far (every sequence advances
                     // together), one equal copy per decode CTA
  size_t Lm;         // int32[B]: reference rows
  size_t chunk;      // int32[B]: rows of the reference chunk being appended
  size_t tickets;    // int32[B*H]: split-K tickets
  size_t items;      // DecodeItem[items_cap]
  size_t cta_begin;  // int32[max_ctas + 1]: first item of each CTA
  size_t partials;   // float[items_cap][d + 4]: (o[0..d), m, l, pad)
  size_t total;
  int items_cap;
  int max_ctas;
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
  int n_shift;           // x mod n = x - n * ((x * n_magic) >> n_shift) for 0 <= x < 2^31
  unsigned long long n_magic;
  int full_mode;         // 0: ring of n slots, 1: outputs in order
  int T_cap;             // FULL mode capacity
  int n_ctas;            // grid size; CTA c runs items [cta_begin[c], cta_begin[c+1])
  int n_items_total;
  int32_t* T;            // step counter, kStepSlots equal copies (CTA c reads copy c)
  const int32_t* Lm;     // [B]
  const DecodeItem* items;
  const int32_t* cta_begin;
  float* partials;
  int32_t* tickets;
  int32_t* err;
  int ref_stable;        // 1: the reference rows are final (see decode.cu); 0: read after the wait
  int cluster_merge;     // 1: the kDecodeCluster CTAs of a slab form a cluster and merge in
                         //    the leader's shared memory (one item per CTA)
  int ring_early;        // 1: stages holding ring rows may be copied before the wait too
  float scale_log2;      // softmax scale * log2(e)
  // Cluster plan: the planned rows and the reference length of each slab
  // (at most kClusterPlanMaxSlabs), so that a CTA derives its item from its
  // index with no load from global memory (items/cta_begin then unused).
  int32_t cl_rows[kClusterPlanMaxSlabs];
  int32_t cl_lm[kClusterPlanMaxSlabs];
  unsigned long long* timing;  // profiling stamps (RSWA_TIMING builds), may be null
};

// The decode kernel's magic number for x mod n (mod_n in decode.cu).
inline void set_mod_magic(DecodeParams& p, int n) {
  int s = 0;
  while ((1LL << s) < (long long)n) ++s;
  p.n_shift = 32 + s;
  p.n_magic = ((1ULL << p.n_shift) + (unsigned long long)n - 1) / (unsigned long long)n;
}

// Launch the split-K decode kernel (append: fused ring write + T advance).
// CTAs per cluster in the cluster-merge plan.
constexpr int kDecodeCluster = 8;
// First 32-row stage of cluster rank r's share of a slab with S stages.
// With at least one stage per rank: S / 8 stages each, and the S mod 8
// extra ones to ranks 1, 2, ... (the leader merges the cluster and the last
// rank holds the ring, so both get the short shares when they can).  Fewer
// stages than ranks: floor(S * r / 8), so the last rank still ends the slab.
__host__ __device__ inline int cluster_stage_begin(int S, int r) {
  if (r >= kDecodeCluster) return S;
  if (S < kDecodeCluster) return (int)((long long)S * r / kDecodeCluster);
  const int q = S / kDecodeCluster, rem = S % kDecodeCluster;
  const int extra = r <= 0 ? 0 : (r - 1 < rem ? r - 1 : rem);
  return r * q + extra;
}
// Clusters of kDecodeCluster decode CTAs that can be resident at once (0 on error).
int decode_max_active_clusters(int elem, int D);

cudaError_t launch_decode(int elem, int D, bool append, const DecodeParams& p, int grid,
                          cudaStream_t stream);
// Dynamic shared memory the decode kernel needs for (elem, D).
size_t decode_smem_bytes(int elem, int D);
// Split-K partials the decode kernel can merge in shared memory for two slabs
// at once, for every (elem, D) it supports (checked in decode.cu).  The
// planners use at most kMinMergeCap / 2 CTAs, so a slab never has more.
constexpr int kMinMergeCap = 372;

struct AppendParams {
  void* kc;
  void* vc;
  const void* k_new;
  const void* v_new;
  int B, H, S_cap, row_bytes, n, full_mode, T_cap;
  int32_t* T;  // step counter (kStepSlots copies): copy 0 read, all advanced
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
  int bidir_prefix;             // 1: prefix queries see every reference key
  unsigned long long* timing;  // profiling stamps (RSWA_TIMING builds), may be null
  // Documents of a pack (tensor-core kernel): document i holds rows
  // [cu[i], cu[i+1]) with refs[i] reference rows; HOST arrays.  The
  // single-sequence form is one document {0, L} with L_m reference rows.
  const int32_t* cu;
  const int32_t* refs;
  int n_docs;
  // Cache fill by the tensor-core kernel (one document): null fill_kc for
  // none.  Caches [H][fill_S_cap][D]; reference rows at their row; outputs in
  // a ring of fill_n slots keeping the newest fill_n, or all in order
  // (fill_full).
  void* fill_kc;
  void* fill_vc;
  int fill_S_cap, fill_n, fill_full;
};
// Sets the thread-local message returned by rswa_last_error().
void set_last_error(const char* prefix, const char* msg);

cudaError_t launch_masked_forward_simt(const MaskedParams& p, int elem, cudaStream_t stream);
// bf16, head dim 128: tcgen05 tensor-core kernel.
cudaError_t launch_masked_forward_tc(const MaskedParams& p, cudaStream_t stream);

}  // namespace rswa
