// C ABI of librswa (declared in include/rswa.h): argument and state
// validation, the workspace layout, the split-K launch planner and the
// kernel launches.  Host code only; every step of the attention runs in the
// kernels of decode.cu, append.cu and the masked-forward files.

#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "cache_copy.h"
#include "internal.h"
#include "rswa.h"

using namespace rswa;

// ------------------------------------------------------------------ errors

static thread_local std::string g_last_error = "no error";

static rswa_status fail(rswa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

void rswa::set_last_error(const char* prefix, const char* msg) {
  g_last_error = std::string(prefix) + msg;
}

static rswa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(RSWA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

#define RSWA_CUDA(call, what)              \
  do {                                     \
    cudaError_t e_ = (call);               \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int elem_size(rswa_dtype t) { return t == RSWA_BF16 ? 2 : 4; }

static bool dtype_ok(rswa_dtype t) { return t == RSWA_F32 || t == RSWA_BF16; }

// ------------------------------------------------------------- workspace

namespace rswa {

unsigned long long current_context_id() {
  typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
  static CtxGetIdFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetIdFn>(ptr);
  });
  unsigned long long id = 0;
  if (!fn || fn(nullptr, &id) != CUDA_SUCCESS) return 0;
  return id;
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Split-K partials are bounded: a span plan has at most one item per slab
// plus one per CTA boundary.
static constexpr int kMaxCtas = 1024;

WorkspaceLayout workspace_layout(int B, int H, int d) {
  WorkspaceLayout w{};
  size_t off = 0;
  w.err = off;
  off = 256;
  w.T = off;
  off = align_up(off + 4 * (size_t)kStepSlots, 256);
  w.Lm = off;
  off = align_up(off + 4 * (size_t)B, 256);
  w.chunk = off;
  off = align_up(off + 4 * (size_t)B, 256);
  w.tickets = off;
  off = align_up(off + 4 * (size_t)B * H, 256);
  w.max_ctas = kMaxCtas;
  w.items_cap = B * H + kMaxCtas;
  w.items = off;
  off = align_up(off + sizeof(DecodeItem) * (size_t)w.items_cap, 256);
  w.cta_begin = off;
  off = align_up(off + 4 * (size_t)(kMaxCtas + 1), 256);
  w.partials = off;
  off = align_up(off + 4 * (size_t)(d + 4) * w.items_cap, 256);
  w.total = off;
  return w;
}

}  // namespace rswa

// ------------------------------------------------------------------ handle

struct rswa_ctx {
  rswa_mode mode;
  int L_m_cap, n, T_cap, H, d, B;
  rswa_dtype dtype;
  int window_cap, S_cap, row_bytes;
  int device, num_sms;
  void* kc;
  void* vc;
  uint8_t* ws;
  cudaStream_t stream;
  WorkspaceLayout lay;
  bool loaded;
  int T_host;                 // outputs appended so far (same for every b)
  std::vector<int32_t> Lm;    // host copy of the reference lengths
  int plan_window;            // output rows the current plan covers
  int n_ctas;
  int max_clusters;           // resident clusters of kDecodeCluster decode CTAs
  bool cluster_plan;          // the current plan merges each slab inside one cluster
  std::vector<int32_t> cl_rows, cl_lm;  // cluster plan: planned rows and L_m per slab
  std::vector<DecodeItem> items;
  std::vector<int32_t> cta_begin;
};

static int32_t* ws_i32(rswa_ctx* c, size_t off) { return reinterpret_cast<int32_t*>(c->ws + off); }

static rswa_status check_handle(rswa_handle h) {
  if (!h) return fail(RSWA_ERR_ARG, "null handle");
  return RSWA_OK;
}

static rswa_status use_device(rswa_ctx* c) {
  int cur = -1;
  RSWA_CUDA(cudaGetDevice(&cur), "cudaGetDevice");
  if (cur != c->device) RSWA_CUDA(cudaSetDevice(c->device), "cudaSetDevice");
  return RSWA_OK;
}

// Two planners.
// Cluster plan, when every slab can have a resident cluster of its own
// (few slabs, e.g. one sequence): slab bh goes to the kDecodeCluster CTAs of
// cluster bh, each taking a contiguous eighth of its 32-row stages, and the
// cluster merges its partials in the leader's shared memory.
// Span plan otherwise: the planned rows of every (b, h) slab (b-major, then
// h) are laid end to end in 32-row stages and cut into G nearly equal
// contiguous spans, one per CTA, G = min(#SMs, #stages).  A span splits
// into items at slab boundaries, so every CTA streams the same number of
// stages (+-1) and a slab is merged from only as many partials as spans
// that touch it (through global memory and tickets).
static void make_plan(rswa_ctx* c) {
  const int nbh = c->B * c->H;
  std::vector<int> rows(nbh), stages(nbh);
  long long total = 0;
  for (int b = 0; b < c->B; ++b) {
    const int r = std::min(c->Lm[b] + c->plan_window, c->S_cap);
    for (int h = 0; h < c->H; ++h) {
      rows[b * c->H + h] = r;
      stages[b * c->H + h] = (r + 31) / 32;
      total += (r + 31) / 32;
    }
  }
  const int Gc = nbh * kDecodeCluster;
  c->cluster_plan = nbh <= c->max_clusters && nbh <= kClusterPlanMaxSlabs && Gc <= c->lay.max_ctas &&
                    Gc <= c->lay.items_cap && Gc <= kStepSlots;
  if (c->cluster_plan) {
    c->cl_rows = rows;
    c->cl_lm.assign(nbh, 0);
    for (int bh = 0; bh < nbh; ++bh) c->cl_lm[bh] = c->Lm[bh / c->H];
    c->items.clear();
    c->cta_begin.assign(Gc + 1, 0);
    for (int bh = 0; bh < nbh; ++bh) {
      const int S = stages[bh];
      for (int r = 0; r < kDecodeCluster; ++r) {
        const int g = bh * kDecodeCluster + r;
        const int st0 = cluster_stage_begin(S, r), st1 = cluster_stage_begin(S, r + 1);
        DecodeItem it{};
        it.bh = bh;
        it.row0 = st0 * 32;
        it.rows = std::max(0, std::min(rows[bh], st1 * 32) - it.row0);  // 0 when the slab has < 8 stages
        it.part = g;
        it.part_first = bh * kDecodeCluster;
        it.nparts = kDecodeCluster;
        it.last = (r == kDecodeCluster - 1) ? 1 : 0;
        c->cta_begin[g] = g;
        c->items.push_back(it);
      }
    }
    c->cta_begin[Gc] = Gc;
    c->n_ctas = Gc;
    return;
  }
  static_assert(kMinMergeCap / 2 <= kStepSlots, "a span-plan grid must fit the step-counter copies");
  const int G = (int)std::min<long long>(std::min(std::min(c->num_sms, c->lay.max_ctas), kMinMergeCap / 2), total);
  c->items.clear();
  c->cta_begin.assign(G + 1, 0);
  std::vector<int> first_item(nbh, -1), count(nbh, 0);
  int bh = 0, st_in_bh = 0;  // walk position: slab and stage inside it
  for (int g = 0; g < G; ++g) {
    c->cta_begin[g] = (int)c->items.size();
    long long todo = (total * (g + 1)) / G - (total * g) / G;  // stages of this span
    while (todo > 0) {
      const int take = (int)std::min<long long>(todo, stages[bh] - st_in_bh);
      DecodeItem it{};
      it.bh = bh;
      it.row0 = st_in_bh * 32;
      it.rows = std::min(rows[bh], (st_in_bh + take) * 32) - it.row0;
      it.last = (st_in_bh + take == stages[bh]) ? 1 : 0;
      if (first_item[bh] < 0) first_item[bh] = (int)c->items.size();
      count[bh] += 1;
      c->items.push_back(it);
      todo -= take;
      st_in_bh += take;
      if (st_in_bh == stages[bh]) {
        ++bh;
        st_in_bh = 0;
      }
    }
  }
  c->cta_begin[G] = (int)c->items.size();
  // Partials: item i is partial i; each slab's items are consecutive.
  for (size_t i = 0; i < c->items.size(); ++i) {
    DecodeItem& it = c->items[i];
    it.part = (int)i;
    it.part_first = first_item[it.bh];
    it.nparts = count[it.bh];
  }
  c->n_ctas = G;
}

extern "C" rswa_status rswa_plan_decode(int batch, int H, const int32_t* ref_lens, int window_rows, int S_cap,
                                        int num_sms, int max_clusters, int32_t* items_out, int items_cap,
                                        int32_t* cta_begin_out, int cta_cap, int* n_items, int* n_ctas,
                                        int* cluster_plan) {
  if (!ref_lens || !items_out || !cta_begin_out || !n_items || !n_ctas || !cluster_plan)
    return fail(RSWA_ERR_ARG, "rswa_plan_decode: null argument");
  if (batch < 1 || H < 1 || window_rows < 0 || S_cap < 1 || num_sms < 1 || max_clusters < 0)
    return fail(RSWA_ERR_ARG, "rswa_plan_decode: invalid sizes");
  rswa_ctx c{};
  c.B = batch;
  c.H = H;
  c.S_cap = S_cap;
  c.num_sms = num_sms;
  c.max_clusters = max_clusters;
  c.plan_window = window_rows;
  c.lay = workspace_layout(batch, H, 128);
  for (int b = 0; b < batch; ++b) {
    if (ref_lens[b] < 1 || ref_lens[b] > S_cap) return fail(RSWA_ERR_ARG, "rswa_plan_decode: ref_lens[%d]", b);
    c.Lm.push_back(ref_lens[b]);
  }
  make_plan(&c);
  *n_items = (int)c.items.size();
  *n_ctas = c.n_ctas;
  *cluster_plan = c.cluster_plan ? 1 : 0;
  if ((int)c.items.size() > items_cap || c.n_ctas + 1 > cta_cap)
    return fail(RSWA_ERR_CAPACITY, "rswa_plan_decode: %zu items, %d CTAs", c.items.size(), c.n_ctas);
  static_assert(sizeof(DecodeItem) == 8 * sizeof(int32_t), "item layout");
  memcpy(items_out, c.items.data(), sizeof(DecodeItem) * c.items.size());
  memcpy(cta_begin_out, c.cta_begin.data(), sizeof(int32_t) * (c.n_ctas + 1));
  return RSWA_OK;
}

static rswa_status upload_plan(rswa_ctx* c) {
  if ((int)c->items.size() > c->lay.items_cap)
    return fail(RSWA_ERR_CAPACITY, "decode plan of %zu items exceeds %d", c->items.size(), c->lay.items_cap);
  RSWA_CUDA(cudaMemcpyAsync(c->ws + c->lay.items, c->items.data(),
                            sizeof(DecodeItem) * c->items.size(), cudaMemcpyHostToDevice,
                            c->stream),
            "upload decode plan");
  RSWA_CUDA(cudaMemcpyAsync(c->ws + c->lay.cta_begin, c->cta_begin.data(),
                            sizeof(int32_t) * c->cta_begin.size(), cudaMemcpyHostToDevice, c->stream),
            "upload decode plan");
  return RSWA_OK;
}

// FULL mode: the plan must cover the rows of the next step.
static rswa_status ensure_plan(rswa_ctx* c, int T_next) {
  if (c->mode == RSWA_MODE_RSWA) return RSWA_OK;
  if (T_next <= c->plan_window) return RSWA_OK;
  c->plan_window = std::min(c->T_cap, (T_next + 63) / 64 * 64);
  make_plan(c);
  return upload_plan(c);
}

// ------------------------------------------------------------------ sizing

extern "C" size_t rswa_cache_bytes(int L_m_cap, int window_cap, int H, int d, int batch,
                                   rswa_dtype dtype) {
  if (L_m_cap < 1 || window_cap < 1 || H < 1 || batch < 1 || (d != 64 && d != 128) ||
      !dtype_ok(dtype))
    return 0;
  return (size_t)batch * H * (size_t)(L_m_cap + window_cap) * d * elem_size(dtype);
}

extern "C" size_t rswa_workspace_bytes(int L_m_cap, int window_cap, int H, int d, int batch) {
  if (L_m_cap < 1 || window_cap < 1 || H < 1 || batch < 1 || (d != 64 && d != 128)) return 0;
  return workspace_layout(batch, H, d).total;
}

// ---------------------------------------------------------------- lifetime

extern "C" rswa_status rswa_init(rswa_handle* out, rswa_mode mode, int L_m_cap, int n, int T_cap,
                                 int H, int d, int batch, rswa_dtype dtype, void* k_cache,
                                 void* v_cache, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  if (!out) return fail(RSWA_ERR_ARG, "rswa_init: out is null");
  *out = nullptr;
  if (mode != RSWA_MODE_RSWA && mode != RSWA_MODE_FULL)
    return fail(RSWA_ERR_ARG, "rswa_init: unknown mode %d", (int)mode);
  if (!dtype_ok(dtype)) return fail(RSWA_ERR_UNSUPPORTED, "rswa_init: unknown dtype %d", (int)dtype);
  if (d != 64 && d != 128) return fail(RSWA_ERR_UNSUPPORTED, "rswa_init: head dim %d (64 or 128)", d);
  if (L_m_cap < 1 || H < 1 || batch < 1)
    return fail(RSWA_ERR_ARG, "rswa_init: L_m_cap=%d H=%d batch=%d must be >= 1", L_m_cap, H, batch);
  if ((long long)batch * H > 65535)  // one grid row per (b, h) slab in the cache-fill kernels
    return fail(RSWA_ERR_ARG, "rswa_init: batch*H=%lld above 65535", (long long)batch * H);
  if (mode == RSWA_MODE_RSWA && n < 1) return fail(RSWA_ERR_ARG, "rswa_init: window n=%d must be >= 1", n);
  if (mode == RSWA_MODE_FULL && T_cap < 1)
    return fail(RSWA_ERR_ARG, "rswa_init: T_cap=%d must be >= 1 in FULL mode", T_cap);
  const int window_cap = mode == RSWA_MODE_RSWA ? n : T_cap;
  if ((long long)L_m_cap + window_cap > (1ll << 30))
    return fail(RSWA_ERR_ARG, "rswa_init: L_m_cap + window too large");
  if (!k_cache || !v_cache || !workspace) return fail(RSWA_ERR_ARG, "rswa_init: null buffer");
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(workspace))
    return fail(RSWA_ERR_ARG, "rswa_init: buffers must be 16-byte aligned");
  const WorkspaceLayout lay = workspace_layout(batch, H, d);
  if (workspace_bytes < lay.total)
    return fail(RSWA_ERR_ARG, "rswa_init: workspace of %zu bytes, need %zu", workspace_bytes, lay.total);

  int dev = 0;
  RSWA_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  cudaDeviceProp prop;
  RSWA_CUDA(cudaGetDeviceProperties(&prop, dev), "cudaGetDeviceProperties");
  if (prop.major != 10 || prop.minor != 0)
    return fail(RSWA_ERR_UNSUPPORTED, "rswa_init: device %d is sm_%d%d; this library is built for sm_100a",
                dev, prop.major, prop.minor);
  const size_t smem = decode_smem_bytes(dtype == RSWA_BF16 ? kBF16 : kF32, d);
  if ((size_t)prop.sharedMemPerBlockOptin < smem)
    return fail(RSWA_ERR_UNSUPPORTED, "rswa_init: kernel needs %zu bytes of shared memory", smem);

  rswa_ctx* c = new rswa_ctx();
  c->mode = mode;
  c->L_m_cap = L_m_cap;
  c->n = n;
  c->T_cap = T_cap;
  c->H = H;
  c->d = d;
  c->B = batch;
  c->dtype = dtype;
  c->window_cap = window_cap;
  c->S_cap = L_m_cap + window_cap;
  c->row_bytes = d * elem_size(dtype);
  c->device = dev;
  c->num_sms = prop.multiProcessorCount;
  c->kc = k_cache;
  c->vc = v_cache;
  c->ws = static_cast<uint8_t*>(workspace);
  c->stream = static_cast<cudaStream_t>(stream);
  c->lay = lay;
  c->loaded = false;
  c->T_host = 0;
  c->plan_window = 0;
  c->n_ctas = 0;
  c->max_clusters = decode_max_active_clusters(dtype == RSWA_BF16 ? kBF16 : kF32, d);
  const char* plan = getenv("RSWA_DECODE_PLAN");  // "span": never use the cluster plan
  if (plan && strcmp(plan, "span") == 0) c->max_clusters = 0;
  c->cluster_plan = false;
  cudaError_t e = cudaMemsetAsync(c->ws, 0, lay.total, c->stream);
  if (e != cudaSuccess) {
    delete c;
    return cuda_fail(e, "rswa_init: clear workspace");
  }
  *out = c;
  return RSWA_OK;
}

// The handle of the decode this library last launched on each (device,
// stream).  A decode may copy ring rows before its dependency wait only if
// the previous kernel on its stream is not a decode of the same handle (the
// decode kernel's prologue states why that suffices).  Any kernel launched in
// between, by this library or not, only makes the answer conservative.
// cudaStreamPerThread names a different stream on each host thread, so it
// always answers "same handle".
static std::mutex g_last_decode_mu;
static std::map<std::pair<int, cudaStream_t>, const rswa_ctx*> g_last_decode;

// The caller holds g_last_decode_mu from the query until its launch is
// enqueued and noted, so the record follows the stream's launch order even
// when host threads share a stream; a launch that fails is not noted.
static bool previous_decode_is(const rswa_ctx* c) {
  if (c->stream == cudaStreamPerThread) return true;
  auto it = g_last_decode.find(std::make_pair(c->device, c->stream));
  return it != g_last_decode.end() && it->second == c;
}
static void note_decode(const rswa_ctx* c) { g_last_decode[std::make_pair(c->device, c->stream)] = c; }

extern "C" void rswa_destroy(rswa_handle h) {
  if (!h) return;
  {
    std::lock_guard<std::mutex> lock(g_last_decode_mu);
    for (auto it = g_last_decode.begin(); it != g_last_decode.end();)
      it = it->second == h ? g_last_decode.erase(it) : std::next(it);
  }
  delete h;
}

extern "C" rswa_status rswa_set_stream(rswa_handle h, void* stream) {
  if (rswa_status st = check_handle(h)) return st;
  h->stream = static_cast<cudaStream_t>(stream);
  return RSWA_OK;
}

// ----------------------------------------------------------------- reference

extern "C" rswa_status rswa_load_reference(rswa_handle h, const void* K_ref, const void* V_ref,
                                           int ref_stride, const int32_t* ref_lens) {
  if (rswa_status st = check_handle(h)) return st;
  if (!K_ref || !V_ref || !ref_lens) return fail(RSWA_ERR_ARG, "rswa_load_reference: null argument");
  if (!aligned16(K_ref) || !aligned16(V_ref))
    return fail(RSWA_ERR_ARG, "rswa_load_reference: K_ref/V_ref must be 16-byte aligned");
  if (ref_stride < 1) return fail(RSWA_ERR_ARG, "rswa_load_reference: ref_stride=%d", ref_stride);
  int max_len = 0;
  for (int b = 0; b < h->B; ++b) {
    const int L = ref_lens[b];
    if (L < 1 || L > h->L_m_cap || L > ref_stride)
      return fail(RSWA_ERR_CAPACITY, "rswa_load_reference: ref_lens[%d]=%d outside [1, min(L_m_cap=%d, ref_stride=%d)]",
                  b, L, h->L_m_cap, ref_stride);
    max_len = std::max(max_len, L);
  }
  if (rswa_status st = use_device(h)) return st;
  h->Lm.assign(ref_lens, ref_lens + h->B);
  h->T_host = 0;
  h->plan_window = h->mode == RSWA_MODE_RSWA ? h->n : std::min(h->T_cap, 64);
  make_plan(h);
  RSWA_CUDA(cudaMemcpyAsync(h->ws + h->lay.Lm, h->Lm.data(), 4 * (size_t)h->B, cudaMemcpyHostToDevice,
                            h->stream),
            "upload reference lengths");
  RSWA_CUDA(cudaMemsetAsync(h->ws + h->lay.T, 0, 4 * kStepSlots, h->stream), "reset step counter");
  if (rswa_status st = upload_plan(h)) return st;
  LoadRefParams p;
  p.kc = h->kc;
  p.vc = h->vc;
  p.K_ref = K_ref;
  p.V_ref = V_ref;
  p.B = h->B;
  p.H = h->H;
  p.S_cap = h->S_cap;
  p.row_bytes = h->row_bytes;
  p.ref_stride = ref_stride;
  p.Lm = ws_i32(h, h->lay.Lm);
  RSWA_CUDA(launch_load_reference(p, max_len, h->stream), "load_reference kernel");
  h->loaded = true;
  return RSWA_OK;
}

extern "C" rswa_status rswa_load_reference_chunk(rswa_handle h, const void* K, const void* V, int chunk_stride,
                                                 const int32_t* rows) {
  if (rswa_status st = check_handle(h)) return st;
  if (!K || !V || !rows) return fail(RSWA_ERR_ARG, "rswa_load_reference_chunk: null argument");
  if (!aligned16(K) || !aligned16(V))
    return fail(RSWA_ERR_ARG, "rswa_load_reference_chunk: K/V must be 16-byte aligned");
  if (chunk_stride < 1) return fail(RSWA_ERR_ARG, "rswa_load_reference_chunk: chunk_stride=%d", chunk_stride);
  if (h->T_host != 0)
    return fail(RSWA_ERR_STATE, "rswa_load_reference_chunk: outputs were appended; the reference is complete "
                                "(rswa_reset first)");
  std::vector<int32_t> Lm(h->B, 0);
  if (h->Lm.size() == (size_t)h->B) Lm = h->Lm;
  int max_rows = 0;
  for (int b = 0; b < h->B; ++b) {
    const int r = rows[b];
    if (r < 0 || r > chunk_stride || (long long)Lm[b] + r > h->L_m_cap)
      return fail(RSWA_ERR_CAPACITY,
                  "rswa_load_reference_chunk: rows[%d]=%d outside [0, chunk_stride=%d] or past L_m_cap=%d "
                  "(%d rows loaded)", b, r, chunk_stride, h->L_m_cap, Lm[b]);
    Lm[b] += r;
    max_rows = std::max(max_rows, r);
  }
  if (rswa_status st = use_device(h)) return st;
  h->Lm = Lm;
  bool all = true;
  for (int b = 0; b < h->B; ++b) all = all && Lm[b] >= 1;
  RSWA_CUDA(cudaMemcpyAsync(h->ws + h->lay.Lm, h->Lm.data(), 4 * (size_t)h->B, cudaMemcpyHostToDevice,
                            h->stream),
            "upload reference lengths");
  RSWA_CUDA(cudaMemcpyAsync(h->ws + h->lay.chunk, rows, 4 * (size_t)h->B, cudaMemcpyHostToDevice, h->stream),
            "upload chunk rows");
  RSWA_CUDA(cudaMemsetAsync(h->ws + h->lay.T, 0, 4 * kStepSlots, h->stream), "reset step counter");
  if (all) {
    h->plan_window = h->mode == RSWA_MODE_RSWA ? h->n : std::min(h->T_cap, 64);
    make_plan(h);
    if (rswa_status st = upload_plan(h)) return st;
  }
  LoadChunkParams p;
  p.kc = h->kc;
  p.vc = h->vc;
  p.K = K;
  p.V = V;
  p.B = h->B;
  p.H = h->H;
  p.S_cap = h->S_cap;
  p.row_bytes = h->row_bytes;
  p.chunk_stride = chunk_stride;
  p.Lm = ws_i32(h, h->lay.Lm);
  p.rows = ws_i32(h, h->lay.chunk);
  if (max_rows > 0) RSWA_CUDA(launch_load_chunk(p, max_rows, h->stream), "load_chunk kernel");
  // Decoding needs every sequence's reference to be non-empty.
  h->loaded = all;
  return RSWA_OK;
}

extern "C" rswa_status rswa_load_packed(rswa_handle h, const void* K, const void* V, int seq_stride,
                                        const int32_t* ref_lens, int T0) {
  if (rswa_status st = check_handle(h)) return st;
  if (!K || !V || !ref_lens) return fail(RSWA_ERR_ARG, "rswa_load_packed: null argument");
  if (!aligned16(K) || !aligned16(V))
    return fail(RSWA_ERR_ARG, "rswa_load_packed: K/V must be 16-byte aligned");
  if (seq_stride < 1 || T0 < 0)
    return fail(RSWA_ERR_ARG, "rswa_load_packed: seq_stride=%d T0=%d", seq_stride, T0);
  if (h->mode == RSWA_MODE_FULL && T0 > h->T_cap)
    return fail(RSWA_ERR_CAPACITY, "rswa_load_packed: T0=%d above T_cap=%d", T0, h->T_cap);
  int max_rows = 0;
  const int W = h->mode == RSWA_MODE_RSWA ? std::min(h->n, T0) : T0;
  for (int b = 0; b < h->B; ++b) {
    const int L = ref_lens[b];
    if (L < 1 || L > h->L_m_cap || (long long)L + T0 > seq_stride)
      return fail(RSWA_ERR_CAPACITY,
                  "rswa_load_packed: ref_lens[%d]=%d outside [1, L_m_cap=%d] or ref_lens + T0=%d above seq_stride=%d",
                  b, L, h->L_m_cap, T0, seq_stride);
    max_rows = std::max(max_rows, L + W);
  }
  if (rswa_status st = use_device(h)) return st;
  h->Lm.assign(ref_lens, ref_lens + h->B);
  h->T_host = T0;
  h->plan_window = h->mode == RSWA_MODE_RSWA ? h->n : std::min(h->T_cap, std::max(64, (T0 + 63) / 64 * 64));
  make_plan(h);
  RSWA_CUDA(cudaMemcpyAsync(h->ws + h->lay.Lm, h->Lm.data(), 4 * (size_t)h->B, cudaMemcpyHostToDevice,
                            h->stream),
            "upload reference lengths");
  if (rswa_status st = upload_plan(h)) return st;
  LoadPackedParams p;
  p.kc = h->kc;
  p.vc = h->vc;
  p.K = K;
  p.V = V;
  p.B = h->B;
  p.H = h->H;
  p.S_cap = h->S_cap;
  p.row_bytes = h->row_bytes;
  p.seq_stride = seq_stride;
  p.n = h->n;
  p.T0 = T0;
  p.full_mode = h->mode == RSWA_MODE_FULL;
  p.Lm = ws_i32(h, h->lay.Lm);
  p.T = ws_i32(h, h->lay.T);
  RSWA_CUDA(launch_load_packed(p, max_rows, h->stream), "load_packed kernel");
  h->loaded = true;
  return RSWA_OK;
}

// ------------------------------------------------------------------- steps

static rswa_status check_step(rswa_ctx* c, bool appending, const char* who) {
  if (!c->loaded)
    return fail(RSWA_ERR_STATE, "%s: no reference loaded (rswa_load_reference, rswa_load_packed, or "
                                "rswa_load_reference_chunk until every sequence has a row)", who);
  if (appending && c->mode == RSWA_MODE_FULL && c->T_host + 1 > c->T_cap)
    return fail(RSWA_ERR_CAPACITY, "%s: FULL mode holds at most T_cap=%d outputs", who, c->T_cap);
  return RSWA_OK;
}

extern "C" rswa_status rswa_append(rswa_handle h, const void* k, const void* v) {
  if (rswa_status st = check_handle(h)) return st;
  if (!k || !v) return fail(RSWA_ERR_ARG, "rswa_append: null k/v");
  if (!aligned16(k) || !aligned16(v)) return fail(RSWA_ERR_ARG, "rswa_append: k/v must be 16-byte aligned");
  if (rswa_status st = check_step(h, true, "rswa_append")) return st;
  if (rswa_status st = use_device(h)) return st;
  if (rswa_status st = ensure_plan(h, h->T_host + 1)) return st;
  AppendParams p;
  p.kc = h->kc;
  p.vc = h->vc;
  p.k_new = k;
  p.v_new = v;
  p.B = h->B;
  p.H = h->H;
  p.S_cap = h->S_cap;
  p.row_bytes = h->row_bytes;
  p.n = h->n;
  p.full_mode = h->mode == RSWA_MODE_FULL;
  p.T_cap = h->T_cap;
  p.T = ws_i32(h, h->lay.T);
  p.Lm = ws_i32(h, h->lay.Lm);
  p.err = ws_i32(h, h->lay.err);
  RSWA_CUDA(launch_append(p, h->stream), "append kernel");
  h->T_host += 1;
  return RSWA_OK;
}

// Profiling aid: per-CTA timestamp buffer used by RSWA_TIMING builds.
static unsigned long long* g_timing = nullptr;

#ifdef RSWA_TIMING
extern "C" void rswa_debug_set_timing(void* buf) { g_timing = static_cast<unsigned long long*>(buf); }
#endif

static rswa_status run_decode(rswa_ctx* c, const void* k, const void* v, const void* q, void* o,
                              float scale, bool append, const char* who) {
  if (!q || !o) return fail(RSWA_ERR_ARG, "%s: null q/o", who);
  if (!aligned16(q) || !aligned16(o)) return fail(RSWA_ERR_ARG, "%s: q/o must be 16-byte aligned", who);
  if (append) {
    if (!k || !v) return fail(RSWA_ERR_ARG, "%s: null k/v", who);
    if (!aligned16(k) || !aligned16(v)) return fail(RSWA_ERR_ARG, "%s: k/v must be 16-byte aligned", who);
  }
  if (!(scale == scale) || isinf(scale)) return fail(RSWA_ERR_ARG, "%s: scale is not finite", who);
  if (rswa_status st = check_step(c, append, who)) return st;
  if (rswa_status st = use_device(c)) return st;
  if (rswa_status st = ensure_plan(c, c->T_host + (append ? 1 : 0))) return st;
  DecodeParams p;
  p.kc = c->kc;
  p.vc = c->vc;
  p.kc_w = c->kc;
  p.vc_w = c->vc;
  p.q = q;
  p.o = o;
  p.k_new = k;
  p.v_new = v;
  p.B = c->B;
  p.H = c->H;
  p.S_cap = c->S_cap;
  p.n = c->n;
  set_mod_magic(p, c->n);
  p.full_mode = c->mode == RSWA_MODE_FULL;
  p.T_cap = c->T_cap;
  p.n_ctas = c->n_ctas;
  p.n_items_total = (int)c->items.size();
  p.T = ws_i32(c, c->lay.T);
  p.Lm = ws_i32(c, c->lay.Lm);
  p.items = reinterpret_cast<const DecodeItem*>(c->ws + c->lay.items);
  p.cta_begin = reinterpret_cast<const int32_t*>(c->ws + c->lay.cta_begin);
  p.partials = reinterpret_cast<float*>(c->ws + c->lay.partials);
  p.tickets = ws_i32(c, c->lay.tickets);
  p.err = ws_i32(c, c->lay.err);
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)c->d);
  p.scale_log2 = sc * 1.4426950408889634f;
  p.timing = g_timing;
  p.cluster_merge = c->cluster_plan ? 1 : 0;
  // Reference rows may always be copied before the dependency wait, ring
  // rows unless the previous kernel on the stream is a decode of this handle
  // (decode.cu states the argument).
#ifdef RSWA_NO_EARLY_COPY
  p.ref_stable = 0;
  p.ring_early = 0;
#else
  p.ref_stable = 1;
#endif
  if (c->cluster_plan)
    for (int bh = 0; bh < c->B * c->H; ++bh) {
      p.cl_rows[bh] = c->cl_rows[bh];
      p.cl_lm[bh] = c->cl_lm[bh];
    }
  const int grid = c->n_ctas;
  {
    std::lock_guard<std::mutex> lock(g_last_decode_mu);  // record and launch in one order
#ifndef RSWA_NO_EARLY_COPY
    p.ring_early = previous_decode_is(c) ? 0 : 1;
#endif
    RSWA_CUDA(launch_decode(c->dtype == RSWA_BF16 ? kBF16 : kF32, c->d, append, p, grid, c->stream),
              "decode kernel");
    if (c->stream != cudaStreamPerThread) note_decode(c);
  }
  if (append) c->T_host += 1;
  return RSWA_OK;
}

extern "C" rswa_status rswa_decode(rswa_handle h, const void* q, void* o, float scale) {
  if (rswa_status st = check_handle(h)) return st;
  return run_decode(h, nullptr, nullptr, q, o, scale, false, "rswa_decode");
}

extern "C" rswa_status rswa_append_decode(rswa_handle h, const void* k, const void* v, const void* q,
                                          void* o, float scale) {
  if (rswa_status st = check_handle(h)) return st;
  return run_decode(h, k, v, q, o, scale, true, "rswa_append_decode");
}

extern "C" rswa_status rswa_append_decode_layers(const rswa_handle* hs, int R, const void* const* k,
                                                 const void* const* v, const void* const* q, void* const* o,
                                                 float scale) {
  static const char* who = "rswa_append_decode_layers";
  if (!hs || !k || !v || !q || !o) return fail(RSWA_ERR_ARG, "%s: null argument", who);
  if (R < 1) return fail(RSWA_ERR_ARG, "%s: R=%d layers", who, R);
  if (!(scale == scale) || isinf(scale)) return fail(RSWA_ERR_ARG, "%s: scale is not finite", who);
  // Everything is checked before the first launch.
  for (int r = 0; r < R; ++r) {
    rswa_ctx* c = hs[r];
    if (!c) return fail(RSWA_ERR_ARG, "%s: handle %d is null", who, r);
    if (!k[r] || !v[r] || !q[r] || !o[r]) return fail(RSWA_ERR_ARG, "%s: null tensor for layer %d", who, r);
    if (!aligned16(k[r]) || !aligned16(v[r]) || !aligned16(q[r]) || !aligned16(o[r]))
      return fail(RSWA_ERR_ARG, "%s: tensors of layer %d must be 16-byte aligned", who, r);
    if (c->device != hs[0]->device || c->stream != hs[0]->stream)
      return fail(RSWA_ERR_ARG, "%s: layer %d is on another device or stream than layer 0", who, r);
    for (int r2 = 0; r2 < r; ++r2)
      if (hs[r2] == c) return fail(RSWA_ERR_ARG, "%s: handle of layer %d repeats layer %d", who, r, r2);
    if (rswa_status st = check_step(c, true, who)) return st;
  }
  for (int r = 0; r < R; ++r)
    if (rswa_status st = run_decode(hs[r], k[r], v[r], q[r], o[r], scale, true, who)) return st;
  return RSWA_OK;
}

// ----------------------------------------------------------------- queries

// The device step counter is one int: every sequence advances together.
static rswa_status read_T(rswa_ctx* c, std::vector<int32_t>& T) {
  if (rswa_status st = use_device(c)) return st;
  int32_t t = 0;
  RSWA_CUDA(cudaMemcpyAsync(&t, c->ws + c->lay.T, 4, cudaMemcpyDeviceToHost, c->stream), "read step counter");
  RSWA_CUDA(cudaStreamSynchronize(c->stream), "cudaStreamSynchronize");
  // Graph replays advance the device counter without the host; follow it.
  c->T_host = t;
  T.assign(c->B, t);
  return RSWA_OK;
}

extern "C" rswa_status rswa_step_count(rswa_handle h, int32_t* out) {
  if (rswa_status st = check_handle(h)) return st;
  if (!out) return fail(RSWA_ERR_ARG, "rswa_step_count: null out");
  if (!h->loaded) return fail(RSWA_ERR_STATE, "rswa_step_count: no reference loaded");
  std::vector<int32_t> T;
  if (rswa_status st = read_T(h, T)) return st;
  memcpy(out, T.data(), 4 * (size_t)h->B);
  return RSWA_OK;
}

static int occupancy(const rswa_ctx* c, int b, int T) {
  return c->mode == RSWA_MODE_RSWA ? c->Lm[b] + std::min(c->n, T) : c->Lm[b] + T;
}

extern "C" rswa_status rswa_cache_len(rswa_handle h, int32_t* out) {
  if (rswa_status st = check_handle(h)) return st;
  if (!out) return fail(RSWA_ERR_ARG, "rswa_cache_len: null out");
  if (!h->loaded) return fail(RSWA_ERR_STATE, "rswa_cache_len: no reference loaded");
  std::vector<int32_t> T;
  if (rswa_status st = read_T(h, T)) return st;
  for (int b = 0; b < h->B; ++b) out[b] = occupancy(h, b, T[b]);
  return RSWA_OK;
}

extern "C" rswa_status rswa_cache_positions(rswa_handle h, int b, int64_t* out, int capacity,
                                            int* count) {
  if (rswa_status st = check_handle(h)) return st;
  if (!out || !count) return fail(RSWA_ERR_ARG, "rswa_cache_positions: null out/count");
  if (!h->loaded) return fail(RSWA_ERR_STATE, "rswa_cache_positions: no reference loaded");
  if (b < 0 || b >= h->B) return fail(RSWA_ERR_ARG, "rswa_cache_positions: b=%d outside [0, %d)", b, h->B);
  std::vector<int32_t> T;
  if (rswa_status st = read_T(h, T)) return st;
  const int Tb = T[b];
  const int rows = occupancy(h, b, Tb);
  *count = rows;
  if (capacity < rows) return fail(RSWA_ERR_CAPACITY, "rswa_cache_positions: need %d entries", rows);
  const int Lm = h->Lm[b];
  for (int r = 0; r < Lm; ++r) out[r] = r + 1;
  if (h->mode == RSWA_MODE_FULL) {
    for (int j = 1; j <= Tb; ++j) out[Lm + j - 1] = (int64_t)Lm + j;
  } else {
    // Ring slot s holds the newest output j <= T with (j - 1) mod n == s.
    const int used = std::min(h->n, Tb);
    for (int s = 0; s < used; ++s) {
      const int back = ((Tb - 1 - s) % h->n + h->n) % h->n;
      out[Lm + s] = (int64_t)Lm + (Tb - back);
    }
  }
  return RSWA_OK;
}

extern "C" rswa_status rswa_reset(rswa_handle h) {
  if (rswa_status st = check_handle(h)) return st;
  if (!h->loaded) return fail(RSWA_ERR_STATE, "rswa_reset: no reference loaded");
  if (rswa_status st = use_device(h)) return st;
  RSWA_CUDA(cudaMemsetAsync(h->ws + h->lay.T, 0, 4 * kStepSlots, h->stream), "reset step counter");
  h->T_host = 0;
  return RSWA_OK;
}

extern "C" rswa_status rswa_check(rswa_handle h) {
  if (rswa_status st = check_handle(h)) return st;
  if (rswa_status st = use_device(h)) return st;
  int32_t err = 0;
  RSWA_CUDA(cudaMemcpyAsync(&err, h->ws + h->lay.err, 4, cudaMemcpyDeviceToHost, h->stream),
            "read device error word");
  RSWA_CUDA(cudaStreamSynchronize(h->stream), "cudaStreamSynchronize");
  if (err == 0) return RSWA_OK;
  RSWA_CUDA(cudaMemsetAsync(h->ws + h->lay.err, 0, 4, h->stream), "clear device error word");
  std::string what;
  if (err & kErrWaitTimeout) what += " wait-timeout";
  if (err & kErrPlanShort) what += " plan-short";
  if (err & kErrCapacity) what += " capacity";
  if (err & kErrTmemAlloc) what += " tmem-alloc";
  return fail(RSWA_ERR_DEVICE, "device error word 0x%x:%s", err, what.c_str());
}

// ---------------------------------------------------------- masked forward

extern "C" rswa_status rswa_masked_forward(const void* Q, const void* K, const void* V, void* O, int L,
                                           int L_m, int n, int H, int d, rswa_dtype dtype, float scale,
                                           void* stream) {
  return rswa_masked_forward_ex(Q, K, V, O, L, L_m, n, H, d, dtype, scale, 0, stream);
}

extern "C" rswa_status rswa_masked_forward_ex(const void* Q, const void* K, const void* V, void* O, int L,
                                              int L_m, int n, int H, int d, rswa_dtype dtype, float scale,
                                              int flags, void* stream) {
  if (!Q || !K || !V || !O) return fail(RSWA_ERR_ARG, "rswa_masked_forward: null tensor");
  if (flags & ~(int)RSWA_FLAG_BIDIR_PREFIX) return fail(RSWA_ERR_ARG, "rswa_masked_forward: unknown flags %d", flags);
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return fail(RSWA_ERR_ARG, "rswa_masked_forward: tensors must be 16-byte aligned");
  if (!dtype_ok(dtype)) return fail(RSWA_ERR_UNSUPPORTED, "rswa_masked_forward: unknown dtype");
  if (d != 64 && d != 128) return fail(RSWA_ERR_UNSUPPORTED, "rswa_masked_forward: head dim %d", d);
  if (L < 1 || H < 1) return fail(RSWA_ERR_ARG, "rswa_masked_forward: L=%d H=%d", L, H);
  if (L_m < 0 || L_m > L) return fail(RSWA_ERR_ARG, "rswa_masked_forward: L_m=%d outside [0, L=%d]", L_m, L);
  if (n < 1) return fail(RSWA_ERR_ARG, "rswa_masked_forward: n=%d must be >= 1", n);
  if (!(scale == scale) || isinf(scale)) return fail(RSWA_ERR_ARG, "rswa_masked_forward: scale not finite");
  if ((long long)L * H * d >= (1ll << 31))
    return fail(RSWA_ERR_ARG, "rswa_masked_forward: tensor too large");
  int dev = 0;
  RSWA_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  int major = 0, minor = 0;
  RSWA_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "device attribute");
  RSWA_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev), "device attribute");
  if (major != 10 || minor != 0)
    return fail(RSWA_ERR_UNSUPPORTED, "rswa_masked_forward: device is sm_%d%d; built for sm_100a", major, minor);
  MaskedParams p;
  p.Q = Q;
  p.K = K;
  p.V = V;
  p.O = O;
  p.L = L;
  p.L_m = L_m;
  p.n = n;
  p.H = H;
  p.D = d;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
  p.scale_log2 = sc * 1.4426950408889634f;
  p.bidir_prefix = (flags & RSWA_FLAG_BIDIR_PREFIX) ? 1 : 0;
  p.timing = g_timing;
  const int32_t cu[2] = {0, L}, refs[1] = {L_m};
  p.cu = cu;
  p.refs = refs;
  p.n_docs = 1;
  p.fill_kc = p.fill_vc = nullptr;
  p.fill_S_cap = p.fill_n = p.fill_full = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == RSWA_BF16 && d == 128) {
    RSWA_CUDA(launch_masked_forward_tc(p, s), "masked forward tensor-core kernel");
  } else {
    RSWA_CUDA(launch_masked_forward_simt(p, dtype == RSWA_BF16 ? kBF16 : kF32, s), "masked forward kernel");
  }
  return RSWA_OK;
}

extern "C" rswa_status rswa_masked_forward_varlen(const void* Q, const void* K, const void* V, void* O,
                                                  const int32_t* cu_seqlens, const int32_t* ref_lens,
                                                  int n_docs, int n, int H, int d, rswa_dtype dtype,
                                                  float scale, int flags, void* stream) {
  if (!Q || !K || !V || !O || !cu_seqlens || !ref_lens)
    return fail(RSWA_ERR_ARG, "rswa_masked_forward_varlen: null argument");
  if (n_docs < 1) return fail(RSWA_ERR_ARG, "rswa_masked_forward_varlen: n_docs=%d", n_docs);
  if (flags & ~(int)RSWA_FLAG_BIDIR_PREFIX)
    return fail(RSWA_ERR_ARG, "rswa_masked_forward_varlen: unknown flags %d", flags);
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return fail(RSWA_ERR_ARG, "rswa_masked_forward_varlen: tensors must be 16-byte aligned");
  if (!dtype_ok(dtype)) return fail(RSWA_ERR_UNSUPPORTED, "rswa_masked_forward_varlen: unknown dtype");
  if (d != 64 && d != 128) return fail(RSWA_ERR_UNSUPPORTED, "rswa_masked_forward_varlen: head dim %d", d);
  if (H < 1 || n < 1) return fail(RSWA_ERR_ARG, "rswa_masked_forward_varlen: H=%d n=%d", H, n);
  if (!(scale == scale) || isinf(scale)) return fail(RSWA_ERR_ARG, "rswa_masked_forward_varlen: scale not finite");
  if (cu_seqlens[0] != 0) return fail(RSWA_ERR_ARG, "rswa_masked_forward_varlen: cu_seqlens[0] must be 0");
  for (int i = 0; i < n_docs; ++i) {
    const long long len = (long long)cu_seqlens[i + 1] - cu_seqlens[i];
    if (len < 1)
      return fail(RSWA_ERR_ARG, "rswa_masked_forward_varlen: document %d has %lld rows", i, len);
    if (ref_lens[i] < 0 || ref_lens[i] > len)
      return fail(RSWA_ERR_ARG, "rswa_masked_forward_varlen: ref_lens[%d]=%d outside [0, %lld]", i,
                  ref_lens[i], len);
  }
  if ((long long)cu_seqlens[n_docs] * H * d >= (1ll << 31))
    return fail(RSWA_ERR_ARG, "rswa_masked_forward_varlen: tensor too large");
  if (dtype == RSWA_BF16 && d == 128) {
    // The tensor-core kernel takes the whole pack in one launch: one CTA per
    // (document, pair of query tiles, head).
    int dev = 0, major = 0, minor = 0;
    RSWA_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    RSWA_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "device attribute");
    RSWA_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev), "device attribute");
    if (major != 10 || minor != 0)
      return fail(RSWA_ERR_UNSUPPORTED, "rswa_masked_forward_varlen: device is sm_%d%d; built for sm_100a", major,
                  minor);
    MaskedParams p;
    p.Q = Q;
    p.K = K;
    p.V = V;
    p.O = O;
    p.L = cu_seqlens[n_docs];
    p.L_m = 0;
    p.n = n;
    p.H = H;
    p.D = d;
    const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
    p.scale_log2 = sc * 1.4426950408889634f;
    p.bidir_prefix = (flags & RSWA_FLAG_BIDIR_PREFIX) ? 1 : 0;
    p.timing = g_timing;
    p.cu = cu_seqlens;
    p.refs = ref_lens;
    p.n_docs = n_docs;
    p.fill_kc = p.fill_vc = nullptr;
    p.fill_S_cap = p.fill_n = p.fill_full = 0;
    RSWA_CUDA(launch_masked_forward_tc(p, static_cast<cudaStream_t>(stream)), "masked forward tensor-core kernel");
    return RSWA_OK;
  }
  // CUDA-core kernel: each document is a contiguous [len][H][d] slice of the pack.
  const size_t row_bytes = (size_t)H * d * elem_size(dtype);
  for (int i = 0; i < n_docs; ++i) {
    const size_t off = (size_t)cu_seqlens[i] * row_bytes;
    rswa_status st = rswa_masked_forward_ex(static_cast<const uint8_t*>(Q) + off, static_cast<const uint8_t*>(K) + off,
                                            static_cast<const uint8_t*>(V) + off, static_cast<uint8_t*>(O) + off,
                                            cu_seqlens[i + 1] - cu_seqlens[i], ref_lens[i], n, H, d, dtype,
                                            scale, flags, stream);
    if (st != RSWA_OK) return st;
  }
  return RSWA_OK;
}

extern "C" rswa_status rswa_masked_forward_fill(rswa_handle h, const void* Q, const void* K, const void* V, void* O,
                                               int L, int L_m, float scale, int flags) {
  static const char* who = "rswa_masked_forward_fill";
  if (rswa_status st = check_handle(h)) return st;
  if (!Q || !K || !V || !O) return fail(RSWA_ERR_ARG, "%s: null tensor", who);
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return fail(RSWA_ERR_ARG, "%s: tensors must be 16-byte aligned", who);
  if (flags & ~(int)RSWA_FLAG_BIDIR_PREFIX) return fail(RSWA_ERR_ARG, "%s: unknown flags %d", who, flags);
  if (!(scale == scale) || isinf(scale)) return fail(RSWA_ERR_ARG, "%s: scale not finite", who);
  if (h->B != 1) return fail(RSWA_ERR_UNSUPPORTED, "%s: the packed form is one sequence; the handle has batch %d", who, h->B);
  if (L < 1 || L_m < 1 || L_m > L) return fail(RSWA_ERR_ARG, "%s: L=%d L_m=%d (1 <= L_m <= L)", who, L, L_m);
  if (L_m > h->L_m_cap) return fail(RSWA_ERR_CAPACITY, "%s: L_m=%d above L_m_cap=%d", who, L_m, h->L_m_cap);
  const int T0 = L - L_m;
  if (h->mode == RSWA_MODE_FULL && T0 > h->T_cap)
    return fail(RSWA_ERR_CAPACITY, "%s: %d outputs above T_cap=%d", who, T0, h->T_cap);
  if ((long long)L * h->H * h->d >= (1ll << 31)) return fail(RSWA_ERR_ARG, "%s: tensor too large", who);
  if (rswa_status st = use_device(h)) return st;
  // The attention window: the handle's n, or every output for the full cache.
  const int n_att = h->mode == RSWA_MODE_RSWA ? h->n : L;
  h->Lm.assign(1, L_m);
  h->T_host = T0;
  h->plan_window = h->mode == RSWA_MODE_RSWA ? h->n : std::min(h->T_cap, std::max(64, (T0 + 63) / 64 * 64));
  make_plan(h);
  RSWA_CUDA(cudaMemcpyAsync(h->ws + h->lay.Lm, h->Lm.data(), 4, cudaMemcpyHostToDevice, h->stream),
            "upload reference lengths");
  if (rswa_status st = upload_plan(h)) return st;
  if (h->dtype == RSWA_BF16 && h->d == 128) {
    // One tensor-core launch computes O and writes the cache rows.
    // (pageable source: the copy is staged before the call returns)
    std::vector<int32_t> T0_dev(kStepSlots, T0);
    RSWA_CUDA(cudaMemcpyAsync(h->ws + h->lay.T, T0_dev.data(), 4 * kStepSlots, cudaMemcpyHostToDevice, h->stream),
              "set step counter");
    MaskedParams p;
    p.Q = Q;
    p.K = K;
    p.V = V;
    p.O = O;
    p.L = L;
    p.L_m = L_m;
    p.n = n_att;
    p.H = h->H;
    p.D = h->d;
    const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)h->d);
    p.scale_log2 = sc * 1.4426950408889634f;
    p.bidir_prefix = (flags & RSWA_FLAG_BIDIR_PREFIX) ? 1 : 0;
    p.timing = g_timing;
    const int32_t cu[2] = {0, L}, refs[1] = {L_m};
    p.cu = cu;
    p.refs = refs;
    p.n_docs = 1;
    p.fill_kc = h->kc;
    p.fill_vc = h->vc;
    p.fill_S_cap = h->S_cap;
    p.fill_n = h->mode == RSWA_MODE_RSWA ? h->n : 0;
    p.fill_full = h->mode == RSWA_MODE_FULL ? 1 : 0;
    RSWA_CUDA(launch_masked_forward_tc(p, h->stream), "masked forward tensor-core kernel");
  } else {
    // CUDA-core attention, then the cache from the same packed rows.
    if (rswa_status st = rswa_masked_forward_ex(Q, K, V, O, L, L_m, n_att, h->H, h->d, h->dtype, scale, flags,
                                                h->stream))
      return st;
    LoadPackedParams p;
    p.kc = h->kc;
    p.vc = h->vc;
    p.K = K;
    p.V = V;
    p.B = 1;
    p.H = h->H;
    p.S_cap = h->S_cap;
    p.row_bytes = h->row_bytes;
    p.seq_stride = L;
    p.n = h->n;
    p.T0 = T0;
    p.full_mode = h->mode == RSWA_MODE_FULL;
    p.Lm = ws_i32(h, h->lay.Lm);
    p.T = ws_i32(h, h->lay.T);
    const int W = h->mode == RSWA_MODE_RSWA ? std::min(h->n, T0) : T0;
    RSWA_CUDA(launch_load_packed(p, L_m + W, h->stream), "load_packed kernel");
  }
  h->loaded = true;
  return RSWA_OK;
}

// -------------------------------------------------------------------- misc

extern "C" const char* rswa_last_error(void) { return g_last_error.c_str(); }

extern "C" const char* rswa_version(void) { return "rswa 0.1.0 sm_100a"; }
