/*
 * rswa.h -- C ABI of the B200 (sm_100a) Reference Sliding Window Attention
 * library, librswa.so.
 *
 * R-SWA is defined in "Unlimited OCR Works：一篇读懂 R-SWA 如何把长文档 OCR 从
 * for-loop 推向 one-shot" (WeThinkIn article), 方法展开 §3, Eq.(1)-(4): the
 * query producing output t attends, with softmax weights
 * exp(q.k_j / sqrt(d)) normalised over N(t), to
 *     N(t) = P ∪ D_n(t),  P = {1..L_m},
 *     D_n(t) = {j | max(L_m+1, L_m+t-n) <= j <= L_m+t-1},
 * i.e. every reference token (vision tokens + prompt, encoded once and never
 * updated) and the most recent n outputs.  The decode-side cache therefore
 * holds C(T) = L_m + min(n, T) <= L_m + n rows (方法展开 §4, Eq.(6)) and is
 * managed as a fixed-capacity queue that evicts the oldest output
 * ("多模态文档解析开源新进展:Unlimited OCR技术方案", section
 * "为什么它能“无限”读下去？关键在 KV cache 恒定").
 *
 * Conventions shared by every call
 * --------------------------------
 * - Positions in the pages' notation are 1-based; array indices here are
 *   0-based.  The query that produces output t sits at position L_m+t-1, so
 *   after T outputs were appended the decode query (the newest output T)
 *   sees P and outputs max(1, T+1-n)..T, which is L_m + min(n, T) rows.
 * - MHA: H query heads and H key/value heads.  Head dim d is 64 or 128.
 * - Element types: RSWA_F32 (float) or RSWA_BF16 (bfloat16).  Accumulation
 *   is always float32; outputs are written in the input element type.
 * - scale <= 0 selects 1/sqrt(d) (Eq.(3)).
 * - Every device buffer is allocated and owned by the caller.  The library
 *   never allocates device memory; a handle owns host-side metadata only.
 *   Device pointers must be 16-byte aligned and point at contiguous,
 *   row-major tensors of the stated shapes.
 * - Calls are asynchronous on the CUDA stream given at rswa_init (a
 *   cudaStream_t passed as void*; NULL = the legacy default stream), except
 *   the query calls marked "synchronous".
 * - Argument and state errors are detected on the host, return a status and
 *   launch nothing.  A CUDA launch error returns RSWA_ERR_CUDA.  Anomalies
 *   only a kernel can see (a bounded wait that timed out, a capacity
 *   overflow) set a device error word that rswa_check() reports; kernels
 *   never trap.
 * - A handle is not thread-safe; distinct handles are independent.
 *   rswa_last_error() returns a thread-local message for the last failure.
 */
#ifndef RSWA_H_
#define RSWA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RSWA_OK = 0,
  RSWA_ERR_ARG = 1,          /* invalid argument (null/misaligned pointer, bad size) */
  RSWA_ERR_STATE = 2,        /* call not valid in the handle's current state */
  RSWA_ERR_CAPACITY = 3,     /* would exceed a capacity fixed at rswa_init */
  RSWA_ERR_UNSUPPORTED = 4,  /* head dim / dtype / device not supported */
  RSWA_ERR_CUDA = 5,         /* a CUDA runtime call or kernel launch failed */
  RSWA_ERR_DEVICE = 6        /* a kernel reported an error (see rswa_check) */
} rswa_status;

typedef enum { RSWA_F32 = 0, RSWA_BF16 = 1 } rswa_dtype;

/* RSWA_MODE_RSWA: the output segment is an n-slot ring, cache L_m + n rows
 *                 (Eq.(6)).
 * RSWA_MODE_FULL: full attention over every output (the MHA baseline of
 *                 Eq.(5)), cache L_m + T_cap rows.  Same kernels, used to
 *                 show the growing per-step cost the pages compare against
 *                 (方法展开 §5, Fig.3). */
typedef enum { RSWA_MODE_RSWA = 0, RSWA_MODE_FULL = 1 } rswa_mode;

typedef struct rswa_ctx* rswa_handle;

/* ------------------------------------------------------------------------
 * Sizing.  Pure host functions; no device needed.
 *
 * window_cap is n for RSWA_MODE_RSWA and T_cap (the maximum number of
 * outputs) for RSWA_MODE_FULL.  Returns 0 for invalid arguments.
 * ---------------------------------------------------------------------- */

/* Bytes of ONE of the two cache tensors (K or V):
 * [batch][H][L_m_cap + window_cap][d] elements of dtype. */
size_t rswa_cache_bytes(int L_m_cap, int window_cap, int H, int d, int batch,
                        rswa_dtype dtype);

/* Bytes of the device workspace (step counters, reference lengths, launch
 * plan, split-K partials and tickets).  Must be passed to rswa_init. */
size_t rswa_workspace_bytes(int L_m_cap, int window_cap, int H, int d, int batch);

/* ------------------------------------------------------------------------
 * Decode-side state.
 * ---------------------------------------------------------------------- */

/* Creates a handle over caller-owned device memory.
 *   k_cache, v_cache: rswa_cache_bytes(...) each.  Layout
 *     [batch][H][L_m_cap + window_cap][d]: for sequence b, rows
 *     [0, L_m[b]) hold the reference segment and rows
 *     [L_m[b], L_m[b] + window_cap) the output segment (the n-slot ring in
 *     RSWA mode, outputs in order in FULL mode).
 *   The caches belong to the handle until rswa_destroy: the caller must not
 *     write them.  Decode kernels copy reference rows before waiting on the
 *     preceding kernel of the stream (programmatic dependent launch); this
 *     is safe because only rswa_load_reference and rswa_load_packed write
 *     those rows and their kernels make their writes visible before they
 *     retire.
 *   workspace: rswa_workspace_bytes(...) bytes; zeroed by this call
 *     (stream-ordered).
 *   n: window size (RSWA mode, >= 1).  T_cap: max outputs (FULL mode, >= 1).
 *   The other of n / T_cap is ignored.  batch * H <= 65535.
 *   Decode plan: when every (b, h) slab can have a resident cluster of
 *   8 CTAs, a slab's partial results are merged inside its cluster;
 *   otherwise across CTAs through the workspace.  The environment variable
 *   RSWA_DECODE_PLAN=span, read here, forces the second plan.
 * Requires a CUDA device of compute capability 10.0 (B200). */
rswa_status rswa_init(rswa_handle* out, rswa_mode mode, int L_m_cap, int n, int T_cap,
                      int H, int d, int batch, rswa_dtype dtype,
                      void* k_cache, void* v_cache, void* workspace,
                      size_t workspace_bytes, void* stream);

/* Loads the reference segment ("encoded once and never updated") and
 * resets every sequence to T = 0 outputs.
 *   K_ref, V_ref: device [batch][H][ref_stride][d] (row r of (b, h) at
 *     ((b*H + h)*ref_stride + r)*d); rows [0, ref_lens[b]) are copied.
 *   ref_lens: HOST array [batch], 1 <= ref_lens[b] <= min(L_m_cap, ref_stride). */
rswa_status rswa_load_reference(rswa_handle h, const void* K_ref, const void* V_ref,
                                int ref_stride, const int32_t* ref_lens);

/* Appends one chunk of the reference segment after the rows already loaded,
 * so a reference can be written as it is produced (for example page by page,
 * 256 vision tokens each) and still be "encoded once and never updated":
 * every row is written once, at its final cache row.  A handle starts with
 * an empty reference; rswa_load_reference replaces it, chunks extend it.
 *   K, V: device [batch][H][chunk_stride][d]; rows [0, rows[b]) of sequence
 *     b's chunk become its reference rows L_m[b] .. L_m[b] + rows[b] - 1.
 *   rows: HOST int32[batch], 0 <= rows[b] <= chunk_stride and the total
 *     L_m[b] + rows[b] <= L_m_cap (else RSWA_ERR_CAPACITY, nothing enqueued).
 * Only while no output has been appended (T = 0; else RSWA_ERR_STATE: the
 * output ring starts right after the reference rows).  Sets T = 0.  Decode
 * calls need every sequence to hold at least one reference row.  The result
 * is the cache rswa_load_reference leaves for the concatenated chunks. */
rswa_status rswa_load_reference_chunk(rswa_handle h, const void* K, const void* V, int chunk_stride,
                                      const int32_t* rows);

/* Fills the cache from the packed (teacher-forced) layout, so decoding can
 * continue after a prefill: the result is the cache that
 * rswa_load_reference followed by T0 appends would leave.  The reference
 * rows are written once; the ring keeps the newest min(n, T0) outputs, output
 * t at slot (t-1) mod n (the Eq.(6) cache and its fixed-capacity queue,
 * 方法展开 §4 and the KV-cache section cited above).
 *   K, V: device [batch][seq_stride][H][d], the layout rswa_masked_forward
 *     reads for one sequence ([L][H][d]).  Row p of sequence b is logical
 *     position p+1: reference rows [0, ref_lens[b]), then output t at row
 *     ref_lens[b] + t - 1.  Read only; 16-byte aligned.
 *   ref_lens: HOST array [batch], 1 <= ref_lens[b] <= L_m_cap and
 *     ref_lens[b] + T0 <= seq_stride.
 *   T0 >= 0: outputs already produced (the same for every sequence, as the
 *     step counter is); FULL mode needs T0 <= T_cap.  The next append is
 *     output T0 + 1.
 * Stream-ordered; errors are reported before anything is enqueued. */
rswa_status rswa_load_packed(rswa_handle h, const void* K, const void* V, int seq_stride,
                             const int32_t* ref_lens, int T0);

/* Appends output T+1 of every sequence: k, v device [batch][H][d].  In RSWA
 * mode the row goes to ring slot (T mod n), overwriting the oldest output
 * once the ring is full (the queue's "position m+1"); in FULL mode to row
 * L_m + T.  Then T := T+1 (on the device). */
rswa_status rswa_append(rswa_handle h, const void* k, const void* v);

/* Decode attention of the current step: q, o device [batch][H][d].  Attends
 * to the L_m[b] + min(n, T[b]) cached rows (FULL: L_m[b] + T[b]).  Split-K
 * over the cache rows, float32 online softmax, log-sum-exp combine. */
rswa_status rswa_decode(rswa_handle h, const void* q, void* o, float scale);

/* rswa_append followed by rswa_decode in ONE kernel: the new k, v are
 * written in place into their slot (no compaction copy) while the cache is
 * streamed, and the step counter is advanced on the device, so a captured
 * CUDA graph of this call can be replayed step after step.  In FULL mode
 * the launch plan is made on the host and covers outputs up to the first
 * multiple of 64 at or above the next output; a graph replayed beyond that
 * finds more rows than its plan, and rswa_check then returns
 * RSWA_ERR_DEVICE ("plan-short") rather than the step attending to a
 * subset: re-capture FULL-mode graphs within that range.  RSWA mode has no
 * such limit (its plan covers the whole ring). */
rswa_status rswa_append_decode(rswa_handle h, const void* k, const void* v,
                               const void* q, void* o, float scale);

/* One decode step of an R-layer decoder: rswa_append_decode for layers
 * 0 .. R-1 in order, one kernel each, on the handles' common stream (the
 * handles of one model's attention layers).  Layer r's kernel may start
 * copying its reference rows while layer r-1 still runs (programmatic
 * dependent launch); it reads q, k, v and its ring after layer r-1 has
 * finished.
 *   hs: HOST array of R distinct handles on one device and one stream.
 *   k, v, q, o: HOST arrays of R device pointers, each [batch_r][H_r][d_r] of
 *     its handle.
 * Every argument and every handle's state is checked before the first launch
 * (errors enqueue nothing); a CUDA launch error stops at that layer.  A
 * captured CUDA graph of this call replays whole decode steps. */
rswa_status rswa_append_decode_layers(const rswa_handle* hs, int R, const void* const* k, const void* const* v,
                                      const void* const* q, void* const* o, float scale);

/* Synchronous: cache occupancy L_m[b] + min(n, T[b]) (FULL: L_m[b] + T[b])
 * per sequence, Eq.(6) / Eq.(5).  out: HOST int32[batch]. */
rswa_status rswa_cache_len(rswa_handle h, int32_t* out);

/* Synchronous: number of outputs T[b] appended so far.  out: HOST int32[batch]. */
rswa_status rswa_step_count(rswa_handle h, int32_t* out);

/* Synchronous: the logical 1-based position held by each valid cache row of
 * sequence b, in storage order (reference rows 1..L_m first, then the
 * output rows).  out: HOST int64[capacity]; *count receives the number of
 * rows (= rswa_cache_len()[b]).  RSWA_ERR_CAPACITY if capacity is short. */
rswa_status rswa_cache_positions(rswa_handle h, int b, int64_t* out, int capacity,
                                 int* count);

/* Stream-ordered: T := 0 for every sequence; the reference rows are kept. */
rswa_status rswa_reset(rswa_handle h);

/* Changes the stream later calls are issued on. */
rswa_status rswa_set_stream(rswa_handle h, void* stream);

/* Synchronous: RSWA_ERR_DEVICE if a kernel raised the device error word
 * since the last check (the word is then cleared), else RSWA_OK.  The
 * message names the condition. */
rswa_status rswa_check(rswa_handle h);

/* Frees the handle's host metadata.  Device buffers stay the caller's. */
void rswa_destroy(rswa_handle h);

/* ------------------------------------------------------------------------
 * Teacher-forced (packed prefill / training) form.
 *
 * O = softmax(Q K^T * scale + M) V per head, with M = 0 where key j is
 * visible from query p and -inf elsewhere:
 *   p <= L_m : j <= p                       (causal inside the prefix)
 *   p >  L_m : j <= L_m, or p-n+1 <= j <= p  (Eq.(1)-(2) with t = p-L_m+1)
 * Q, K, V, O: device [L][H][d] (token-major).  0 <= L_m <= L, n >= 1.
 * L_m = 0 leaves no reference segment: every query sees p-n+1 .. p, the
 * plain sliding window the pages contrast R-SWA with ("vanilla SWA",
 * 核心导读 Fig. 1 and 方法展开 §1), for ablation.
 * BF16 with d = 128 runs on the tcgen05 tensor-core kernel.  F32 (d = 64 or
 * 128) and BF16 with d = 64 run on a CUDA-core kernel (one warp per query
 * row and head, float32 online softmax), which is exact to float32 rounding
 * but far slower.  Key tiles (or ranges) the mask fully hides are skipped.
 * ---------------------------------------------------------------------- */
rswa_status rswa_masked_forward(const void* Q, const void* K, const void* V, void* O,
                                int L, int L_m, int n, int H, int d, rswa_dtype dtype,
                                float scale, void* stream);

/* Flags of rswa_masked_forward_ex. */
typedef enum {
  /* Every prefix query p <= L_m sees all reference keys 1..L_m (the pages
   * are silent on prefix queries; without the flag they are causal). */
  RSWA_FLAG_BIDIR_PREFIX = 1
} rswa_forward_flags;

/* rswa_masked_forward with flags (a bitwise OR of rswa_forward_flags; 0
 * gives rswa_masked_forward).  Unknown flag bits return RSWA_ERR_ARG. */
rswa_status rswa_masked_forward_ex(const void* Q, const void* K, const void* V, void* O,
                                   int L, int L_m, int n, int H, int d, rswa_dtype dtype,
                                   float scale, int flags, void* stream);

/* The teacher-forced form over a pack of several documents.  The pages pack
 * training samples to 32K tokens ("Unlimited OCR Works", 实验与证据 §1) and do
 * not say how packed documents see each other; here each document is its own
 * sequence: its queries see only its own keys, under the mask above with its
 * own L_m, at positions local to the document.
 *   Q, K, V, O: device [L][H][d], L = cu_seqlens[n_docs]; document i holds
 *     rows [cu_seqlens[i], cu_seqlens[i+1]).
 *   cu_seqlens: HOST int32[n_docs + 1], cu_seqlens[0] = 0, strictly
 *     increasing (every document has at least one row).
 *   ref_lens: HOST int32[n_docs], 0 <= ref_lens[i] <= length of document i.
 *   n_docs >= 1; n, H, d, dtype, scale, flags as in rswa_masked_forward_ex.
 * Every argument is checked before anything is enqueued.  BF16 with d = 128
 * runs the whole pack in one tensor-core launch (one CTA per document, pair
 * of 128-row query tiles and head, longest first; more than 1024 pairs are
 * split over several launches); the CUDA-core kernel (F32, or d = 64) is
 * launched once per document on its rows. */
rswa_status rswa_masked_forward_varlen(const void* Q, const void* K, const void* V, void* O,
                                       const int32_t* cu_seqlens, const int32_t* ref_lens, int n_docs,
                                       int n, int H, int d, rswa_dtype dtype, float scale, int flags,
                                       void* stream);

/* The teacher-forced form of one sequence that also leaves a handle's cache
 * ready to decode: O as rswa_masked_forward_ex computes it with the handle's
 * window (its n; every output for a FULL-mode handle, i.e. plain causal
 * attention), and the cache rswa_load_reference of rows [0, L_m) followed by
 * L - L_m appends leaves: the reference rows, "encoded once" here, and the
 * newest min(n, L - L_m) outputs in their ring slots (FULL mode: all of
 * them).  The step counter becomes T0 = L - L_m; the next append is output
 * T0 + 1 (方法展开 §4, Eq.(6) and its queue).
 *   h: a handle of batch 1 whose dtype and d the tensors share.
 *   Q, K, V, O: device [L][H][d], as for rswa_masked_forward.
 *   1 <= L_m <= min(L, L_m_cap); FULL mode needs L - L_m <= T_cap.
 *   flags: as rswa_masked_forward_ex.
 * BF16 with d = 128 does both in one tensor-core launch: each CTA copies the
 * key and value rows of its own query tiles from the tiles it has staged
 * for the attention into the cache.  Other types run the CUDA-core kernel
 * and then a copy kernel.  Stream-ordered on the handle's stream; errors are
 * reported before anything is enqueued. */
rswa_status rswa_masked_forward_fill(rswa_handle h, const void* Q, const void* K, const void* V, void* O,
                                     int L, int L_m, float scale, int flags);

/* ------------------------------------------------------------------------
 * Decode without allocation.  The pages have no counterpart to this call;
 * it exists for callers that cannot allocate device memory: a plugin inside
 * a host framework whose own allocator owns every device allocation (memory
 * taken behind its back breaks its accounting), or code that must avoid the
 * implicitly synchronising cudaMalloc / cudaFree on a latency-critical path.
 *
 * One-shot decode attention over caller-owned caches, with no handle and no
 * workspace: the kernel's scratch (launch plan, split-K partials, tickets)
 * lives in a static device array of about 0.7 MB inside the library, which
 * every device that loads the library holds until the process exits.  The
 * library allocates nothing for this call.
 *   k_cache, v_cache: device [batch][H][S_cap][d]; for (b, h), rows
 *     [0, cache_lens[b]) are attended, in any storage order (for example
 *     the reference rows followed by the ring of an RSWA handle).
 *   cache_lens: HOST int32[batch], 1 <= cache_lens[b] <= S_cap.
 *   q, o: device [batch][H][d].  scale <= 0 selects 1/sqrt(d).
 * Limits: batch * H <= 1024; d = 64 or 128.  Larger sizes return
 * RSWA_ERR_CAPACITY with a message in rswa_last_error().
 * The first call on a device (and the first after that device's context was
 * reset) looks up the array's device address (cudaGetSymbolAddress) with
 * that device current.  Every call reuses the same array and clears what
 * must start at zero, so calls whose kernels overlap on the GPU race: order
 * them on one stream.  The plan is staged with stream-ordered copies from
 * host memory.
 * ---------------------------------------------------------------------- */
rswa_status rswa_decode_noalloc(const void* k_cache, const void* v_cache, int S_cap,
                                const int32_t* cache_lens, const void* q, void* o,
                                int batch, int H, int d, rswa_dtype dtype, float scale,
                                void* stream);

/* Synchronous (waits for `stream`): RSWA_ERR_DEVICE if a decode launched by
 * rswa_decode_noalloc on the current device raised the device error word (a
 * bounded wait that timed out) since the last check; the word is then
 * cleared.  Allocates nothing. */
rswa_status rswa_decode_noalloc_check(void* stream);

/* ------------------------------------------------------------------------
 * Introspection (host only; needs no device).
 *
 * The decode launch plan a handle with these sizes uses, for inspection and
 * tests.  ref_lens: HOST int32[batch] (each >= 1); window_rows: output rows
 * the plan covers (n in RSWA mode); S_cap: rows per cache slab; num_sms and
 * max_clusters: the device's SM count and the resident 8-CTA clusters it
 * allows (0: never the cluster plan).
 * Outputs (HOST): items_out int32[items_cap][8], each item
 *   {bh, row0, rows, part, part_first, nparts, last, 0}: CTA c runs items
 *   [cta_begin_out[c], cta_begin_out[c+1]) over rows [row0, row0 + rows) of
 *   slab bh = b*H + h; its partial is number `part` of the slab's `nparts`
 *   partials starting at `part_first`; `last` marks the slab's last item.
 * cta_begin_out: int32[cta_cap] (n_ctas + 1 entries).  *cluster_plan is 1
 * when the slabs are merged inside 8-CTA clusters.  RSWA_ERR_CAPACITY if
 * items_cap or cta_cap is short.
 * ---------------------------------------------------------------------- */
rswa_status rswa_plan_decode(int batch, int H, const int32_t* ref_lens, int window_rows, int S_cap,
                             int num_sms, int max_clusters, int32_t* items_out, int items_cap,
                             int32_t* cta_begin_out, int cta_cap, int* n_items, int* n_ctas,
                             int* cluster_plan);

/* ------------------------------------------------------------------------
 * Misc.
 * ---------------------------------------------------------------------- */

/* Thread-local description of the last non-OK status (never NULL). */
const char* rswa_last_error(void);

/* Library version string, e.g. "rswa 0.1.0 sm_100a". */
const char* rswa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RSWA_H_ */
