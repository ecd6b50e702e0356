// rswa_decode_noalloc: one-shot decode attention that allocates nothing.
//
// Some callers cannot allocate device memory: a plugin running inside a host
// framework that owns every device allocation (its allocator hands out all
// memory, and a library that called cudaMalloc behind its back would break
// its accounting), or code that must not make the implicitly synchronising
// cudaMalloc / cudaFree calls on a latency-critical path.  The handle API
// needs a caller-provided workspace; this entry point instead keeps the
// decode kernel's scratch (launch plan, split-K partials, tickets, counters)
// in one file-scope device array that every device loading the library holds
// until the process exits.
//
// The caller passes the caches, the query and the output.  Every call reuses
// the same array, so two calls whose kernels overlap on the GPU race; issue
// them on one stream (or otherwise order them).  The parts that must start at
// zero (step counter, split-K tickets) are cleared by every
// call; the device error word is kept until rswa_decode_noalloc_check reads
// and clears it.

#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "rswa.h"

namespace rswa {

// Limits of the static scratch.
constexpr int kNoAllocMaxSlabs = 1024;  // batch * heads
constexpr int kNoAllocMaxCtas = 160;    // >= the SM count of a B200
constexpr int kNoAllocMaxItems = kNoAllocMaxSlabs + kNoAllocMaxCtas;
constexpr int kNoAllocMaxD = 128;

// Scratch layout (bytes), every region 256-byte aligned.
constexpr size_t kNaErr = 0;                                       // int32 error word
constexpr size_t kNaZeroed = 4;                                    // [4, kNaLm) is zeroed before each launch
constexpr size_t kNaT = 256;                                       // int32 step counter (always 0)
constexpr size_t kNaLm = 512;                                      // int32[max slabs]
constexpr size_t kNaTickets = kNaLm + 4 * kNoAllocMaxSlabs;        // int32[max slabs]
constexpr size_t kNaItems = kNaTickets + 4 * kNoAllocMaxSlabs;     // DecodeItem[max items]
constexpr size_t kNaCtaBegin = kNaItems + sizeof(DecodeItem) * kNoAllocMaxItems;
constexpr size_t kNaPartials = (kNaCtaBegin + 4 * (kNoAllocMaxCtas + 1) + 255) / 256 * 256;
constexpr size_t kNaBytes = kNaPartials + 4ull * (kNoAllocMaxD + 4) * kNoAllocMaxItems;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNaBytes];

// Device address of the scratch in the current context of each device.  Host
// code may not use the symbol itself as a device pointer (it names a host-side
// stand-in), so the address is looked up with cudaGetSymbolAddress, with the
// device current, on the first call in each context: a context made after a
// device reset loads the module again and gets its own copy of the array.
constexpr int kMaxDevices = 64;
struct ScratchAddr {
  unsigned long long ctx;
  void* ptr;
};
static ScratchAddr g_scratch_addr[kMaxDevices];
static std::mutex g_scratch_mu;

static cudaError_t scratch_for_current_device(uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long ctx = current_context_id();
  ScratchAddr& a = g_scratch_addr[dev];
  if (ctx == 0 || a.ctx != ctx || !a.ptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    a.ptr = ptr;
    a.ctx = ctx != 0 ? ctx : current_context_id();
  }
  *out = static_cast<uint8_t*>(a.ptr);
  return cudaSuccess;
}

}  // namespace rswa

using namespace rswa;

static thread_local DecodeItem g_na_items[kNoAllocMaxItems];
static thread_local int32_t g_na_begin[kNoAllocMaxCtas + 1];
static thread_local int32_t g_na_lens[kNoAllocMaxSlabs];

// The message is reported by rswa_last_error().
static rswa_status na_fail(rswa_status st, const char* msg) {
  set_last_error("rswa_decode_noalloc: ", msg);
  return st;
}

extern "C" rswa_status rswa_decode_noalloc(const void* k_cache, const void* v_cache, int S_cap,
                                           const int32_t* cache_lens, const void* q, void* o,
                                           int batch, int H, int d, rswa_dtype dtype, float scale,
                                           void* stream) {
  if (!k_cache || !v_cache || !cache_lens || !q || !o) return na_fail(RSWA_ERR_ARG, "null argument");
  const uintptr_t mis = (reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache) |
                         reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(o)) & 15u;
  if (mis) return na_fail(RSWA_ERR_ARG, "pointers must be 16-byte aligned");
  if (dtype != RSWA_F32 && dtype != RSWA_BF16) return na_fail(RSWA_ERR_UNSUPPORTED, "unknown dtype");
  if (d != 64 && d != 128) return na_fail(RSWA_ERR_UNSUPPORTED, "head dim must be 64 or 128");
  if (batch < 1 || H < 1 || S_cap < 1) return na_fail(RSWA_ERR_ARG, "batch, H and S_cap must be >= 1");
  if ((long long)batch * H > kNoAllocMaxSlabs)
    return na_fail(RSWA_ERR_CAPACITY, "batch * H exceeds the static scratch limit of 1024");
  if (!(scale == scale) || isinf(scale)) return na_fail(RSWA_ERR_ARG, "scale is not finite");
  for (int b = 0; b < batch; ++b) {
    if (cache_lens[b] < 1 || cache_lens[b] > S_cap) return na_fail(RSWA_ERR_ARG, "cache_lens[b] outside [1, S_cap]");
    g_na_lens[b] = cache_lens[b];
  }
  int dev = 0, sms = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return na_fail(RSWA_ERR_CUDA, "cannot query the current device");
  if (major != 10 || minor != 0) return na_fail(RSWA_ERR_UNSUPPORTED, "needs an sm_100 device");
  uint8_t* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess)
    return na_fail(RSWA_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed");

  // Span plan over the slabs' rows (32-row stages), one span per CTA.
  const int nbh = batch * H;
  long long total = 0;
  for (int bh = 0; bh < nbh; ++bh) total += (g_na_lens[bh / H] + 31) / 32;
  const int G = (int)std::min<long long>(std::min(std::min(sms, kNoAllocMaxCtas), kMinMergeCap / 2), total);
  int n_items = 0, bh = 0, st = 0;
  int first_item = 0;
  for (int g = 0; g < G; ++g) {
    g_na_begin[g] = n_items;
    long long todo = (total * (g + 1)) / G - (total * g) / G;
    while (todo > 0) {
      const int rows_bh = g_na_lens[bh / H];
      const int stages_bh = (rows_bh + 31) / 32;
      const int take = (int)std::min<long long>(todo, stages_bh - st);
      if (st == 0) first_item = n_items;
      DecodeItem& it = g_na_items[n_items];
      it.bh = bh;
      it.row0 = st * 32;
      it.rows = std::min(rows_bh, (st + take) * 32) - it.row0;
      it.part = n_items;
      it.part_first = first_item;
      it.nparts = 0;  // filled below
      it.last = (st + take == stages_bh) ? 1 : 0;
      it.pad = 0;
      ++n_items;
      todo -= take;
      st += take;
      if (st == stages_bh) {
        for (int i = first_item; i < n_items; ++i) g_na_items[i].nparts = n_items - first_item;
        ++bh;
        st = 0;
      }
    }
  }
  g_na_begin[G] = n_items;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The step counter and the tickets must start at zero (the error word is
  // kept for rswa_decode_noalloc_check); plan and lengths are uploaded.
  if (cudaMemsetAsync(scratch + kNaZeroed, 0, kNaLm - kNaZeroed, s) != cudaSuccess ||
      cudaMemsetAsync(scratch + kNaTickets, 0, 4 * (size_t)nbh, s) != cudaSuccess ||
      cudaMemcpyAsync(scratch + kNaLm, g_na_lens, 4 * (size_t)batch, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(scratch + kNaItems, g_na_items, sizeof(DecodeItem) * n_items, cudaMemcpyHostToDevice, s) !=
          cudaSuccess ||
      cudaMemcpyAsync(scratch + kNaCtaBegin, g_na_begin, 4 * (size_t)(G + 1), cudaMemcpyHostToDevice, s) !=
          cudaSuccess)
    return na_fail(RSWA_ERR_CUDA, "staging the launch plan failed");

  DecodeParams p = {};
  p.kc = k_cache;
  p.vc = v_cache;
  p.q = q;
  p.o = o;
  p.B = batch;
  p.H = H;
  p.S_cap = S_cap;
  p.n = 1;
  set_mod_magic(p, 1);
  p.full_mode = 1;  // with T = 0 the attended rows are exactly cache_lens[b]
  p.T_cap = 0;
  p.n_ctas = G;
  p.n_items_total = n_items;
  p.T = reinterpret_cast<int32_t*>(scratch + kNaT);
  p.Lm = reinterpret_cast<const int32_t*>(scratch + kNaLm);
  p.items = reinterpret_cast<const DecodeItem*>(scratch + kNaItems);
  p.cta_begin = reinterpret_cast<const int32_t*>(scratch + kNaCtaBegin);
  p.partials = reinterpret_cast<float*>(scratch + kNaPartials);
  p.tickets = reinterpret_cast<int32_t*>(scratch + kNaTickets);
  p.err = reinterpret_cast<int32_t*>(scratch + kNaErr);
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
  p.scale_log2 = sc * 1.4426950408889634f;
  p.timing = nullptr;
  if (launch_decode(dtype == RSWA_BF16 ? kBF16 : kF32, d, false, p, G, s) != cudaSuccess)
    return na_fail(RSWA_ERR_CUDA, "decode kernel launch failed");
  return RSWA_OK;
}

extern "C" rswa_status rswa_decode_noalloc_check(void* stream) {
  uint8_t* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess)
    return na_fail(RSWA_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t err = 0;
  if (cudaMemcpyAsync(&err, scratch + kNaErr, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return na_fail(RSWA_ERR_CUDA, "reading the device error word failed");
  if (err == 0) return RSWA_OK;
  if (cudaMemsetAsync(scratch + kNaErr, 0, 4, s) != cudaSuccess)
    return na_fail(RSWA_ERR_CUDA, "clearing the device error word failed");
  char msg[96];
  snprintf(msg, sizeof(msg), "device error word 0x%x%s%s", err, (err & kErrWaitTimeout) ? " wait-timeout" : "",
           (err & kErrPlanShort) ? " plan-short" : "");
  set_last_error("rswa_decode_noalloc: ", msg);
  return RSWA_ERR_DEVICE;
}
