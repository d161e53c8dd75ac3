/*
 * mla.h — C ABI of libmla: Multi-Head Latent Attention decode over a paged latent KV cache
 * on NVIDIA B200 (sm_100a), with the MQA-absorb path and the GQLA grouped (GQA) path.
 *
 * Method sources (cited by page title and section):
 *   "MLA and GRPO architecture" (blog), "The Mathematics of MLA": c_t^KV = W_DKV h_t,
 *     k_t^C = W_UK c_t^KV, v_t^C = W_UV c_t^KV; "Decoupled Rotary Position Embeddings":
 *     RoPE only on k_t^R, cached state per token = [c_t^KV, k_t^R].
 *   "How to upgrade GQA models to MLA for massive KV Cache Savings", "Under the hood",
 *     stage "Decompression Multiplex": W_UK folded into the query by associativity, keys
 *     never decompressed.
 *   "GQLA: Group-Query Latent Attention for Hardware-Adaptive Large Language Model Decoding"
 *     (abstract) and the AI Radio episode on GQLA ("Key concepts"; transcript "The paper's
 *     summary"): an MQA-absorb path caching the latent plus the shared RoPE key, and an
 *     algebraically equivalent GQA path caching per-group K and V plus the shared RoPE key;
 *     up-projections shared by groups of query heads.
 *
 * Conventions for every entry point:
 *   - Ownership: the caller owns every buffer.  Device pointers are plain CUDA device
 *     addresses (e.g. from torch).  The library allocates no device or host memory and never
 *     synchronises except in mla_get_device_status().  Scratch comes from a caller-provided
 *     workspace whose size the matching *_workspace_size() call returns.
 *   - Streams: work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and is asynchronous; argument errors are returned before anything is enqueued.  The
 *     kernels are launched with programmatic stream serialisation (programmatic dependent
 *     launch): a kernel may be scheduled while the stream's previous kernel finishes, but it
 *     waits for that kernel's completion before touching memory, so ordering against the
 *     caller's own work on the stream is that of a plain stream.  Stream capture into a CUDA
 *     graph records programmatic edges.
 *   - Layouts are row-major and densely packed unless stated.  bf16 = IEEE bfloat16 bits,
 *     fp32 = IEEE float.  All pointers of one call use the dtype in dims->dtype, except int32
 *     index arrays.  Device pointers must be 16-byte aligned.
 *   - Positions: request b's cache holds seq_lens[b] tokens including its s_q current
 *     tokens (1 <= s_q <= 4: multi-token-prediction depth; the grouped tensor-core kernel
 *     holds 8 heads x 2 queries per 16-row tile and runs two tiles for s_q = 3, 4);
 *     query j (0 <= j < s_q) sits at position seq_lens[b] - s_q + j and attends to
 *     tokens t <= that position (this gives the causal mask between MTP query tokens).
 *     Token t of request b lives in page page_table[b*max_pages + t/page_size], row
 *     t % page_size.
 *   - Errors: every call returns mla_status.  MLA_ERR_CUDA carries detail in
 *     mla_last_error_string().  Conditions only the device can see (a page id or slot out of
 *     range, device seq_lens that contradict the host copy, a pipeline wait that ran out)
 *     set a per-device error word instead of faulting; the offending access is skipped and
 *     mla_get_device_status() reports it.
 *   - Lifetime: on a device's first call the library looks up and keeps that device's address
 *     of its error word and static scratch, and it keeps recent tensor-map encodings keyed by
 *     buffer address.  These stay valid for the life of the device's primary context: do not
 *     use the library across cudaDeviceReset() (or any teardown of the primary context) in
 *     the same process.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols keep default visibility even when the library builds with hidden visibility. */
#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

/* Same object as cudaStream_t / CUstream; declared here so callers need no CUDA headers. */
typedef struct CUstream_st *mla_stream_t;

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, inconsistent lengths            */
    MLA_ERR_UNSUPPORTED = 2,   /* dims/dtype combination this library was not built for   */
    MLA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than *_workspace_size()    */
    MLA_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed (see error string)    */
    MLA_ERR_DEVICE_BOUNDS = 5, /* device saw an index out of range; the access was skipped */
    MLA_ERR_TIMEOUT = 6        /* a bounded device-side wait ran out; the kernel returned  */
} mla_status;

typedef enum { MLA_BF16 = 0, MLA_FP32 = 1 } mla_dtype;

/* Model dimensions, in the pages' notation. */
typedef struct {
    int32_t n_heads;         /* H: query heads                                             */
    int32_t heads_per_group; /* query heads sharing one W_UK / W_UV slice: 1 = MLA, 8 = GQLA */
    int32_t d_c;             /* latent width of c^KV                                        */
    int32_t d_rope;          /* width of the RoPE key k^R and of each head's RoPE query     */
    int32_t d_nope;          /* per-head no-position query/key width                        */
    int32_t d_v;             /* per-head value width                                        */
    int32_t page_size;       /* tokens per cache page                                       */
    float softmax_scale;     /* <= 0 selects 1/sqrt(d_nope + d_rope)                        */
    float rope_base;         /* RoPE base; pair i of a d_rope vector turns by pos*base^(-2i/d_rope) */
    mla_dtype dtype;         /* storage dtype of every float tensor of a call              */
} mla_dims;

/*
 * Supported dims: dtype MLA_BF16 with H=128, d_c=512, d_rope=64, d_nope=128, d_v=128,
 * page_size=64 (DeepSeek-V2 attention shape) runs the tensor-core kernels; any dtype with
 * H <= 128, d_c <= 512, d_rope <= 64 (even), d_nope <= 128, d_v <= 128, page_size in
 * {16, 32, 64, 128} runs the general CUDA-core kernels.  heads_per_group must divide H.
 */

/*
 * mla_cache_append — down-project the new tokens and write them into the paged latent cache.
 * ("MLA and GRPO architecture", "The Mathematics of MLA": c_t^KV = W_DKV h_t; "Decoupled
 *  RoPE": cached state [c_t^KV, k_t^R].  k_t^R = RoPE(W_KR h_t, position) is this library's
 *  reading: the page names no projection for the RoPE key.)
 *
 *   h            device [n_tok, hidden]; with W_dkv == NULL it is [n_tok, d_c + d_rope]
 *                already projected ([c | k_rope before rotation]) and hidden must equal
 *                d_c + d_rope.
 *   W_dkv        device [d_c, hidden] or NULL;  W_kr  device [d_rope, hidden] (NULL iff W_dkv is).
 *   req_idx      device [n_tok] request index of each new token (0 <= req_idx < batch).
 *   positions    device [n_tok] token position inside its request (0 <= pos < max_pages*page).
 *   page_table   device [batch, max_pages] page ids, each < n_pages_total.
 *   latent_cache device [n_pages_total, page_size, d_c + d_rope]; row = [c^KV | k^R].
 * Accumulates in fp32; rounds once to the cache dtype.  Tokens whose indices fail the device
 * bounds checks are skipped and set MLA_ERR_DEVICE_BOUNDS.  Two new tokens that map to the
 * same slot race (last write wins).
 */
MLA_API mla_status mla_cache_append(const mla_dims *dims, const void *h, int32_t hidden,
                            const void *W_dkv, const void *W_kr,
                            const int32_t *req_idx, const int32_t *positions, int32_t n_tok,
                            const int32_t *page_table, int32_t batch, int32_t max_pages,
                            int32_t n_pages_total, void *latent_cache, mla_stream_t stream);

/*
 * mla_decode_workspace_size — bytes of workspace mla_decode_absorbed needs for this batch.
 *   seq_lens_host  host [batch] cache lengths (the same values the device copy will hold).
 * Writes *bytes; the size depends only on (dims, batch, s_q, seq_lens, SM count of the
 * current device).
 */
MLA_API mla_status mla_decode_workspace_size(const mla_dims *dims, int32_t batch, int32_t s_q,
                                     const int32_t *seq_lens_host, size_t *bytes);

/*
 * mla_decode_absorbed — MQA-absorb decode: q absorption, split-KV flash decode over the
 * latent, split combine, output up-projection.
 * ("How to upgrade GQA models to MLA ...", stage "Decompression Multiplex"; "GQLA ..."
 *  abstract: the MQA-absorb path, in which the latent is the key and value shared by all
 *  heads.)  For head h with weight group w = h / heads_per_group and query j at position p:
 *     q_lat   = W_UK[w]^T q_nope                (d_c)
 *     s_t     = scale * (q_lat . c_t + RoPE(q_rope, p) . k^R_t),   t <= p
 *     O_lat   = sum_t softmax(s)_t c_t          (d_c)
 *     out     = W_UV[w] O_lat                   (d_v)
 *
 *   q             device [batch, s_q, H, d_nope + d_rope]; RoPE part NOT yet rotated.
 *   W_uk          device [H / heads_per_group, d_nope, d_c].
 *   W_uv          device [H / heads_per_group, d_v, d_c].
 *   latent_cache  device [n_pages_total, page_size, d_c + d_rope].  Slots past a request's
 *                 length in its last page may hold anything, NaN included: they are never
 *                 read into the softmax or the weighted sum.
 *   page_table    device [batch, max_pages];  seq_lens device [batch];
 *   seq_lens_host host   [batch], equal to the device copy; s_q <= seq_lens[b] <= max_pages*page.
 *   out           device [batch, s_q, H, d_v].
 *   workspace     device, >= mla_decode_workspace_size() bytes, 256-byte aligned; its
 *                 contents are scratch (overwritten; no need to clear).
 * Results are deterministic: the split plan depends only on (seq_lens, s_q, SM count).
 */
MLA_API mla_status mla_decode_absorbed(const mla_dims *dims, const void *q, const void *W_uk,
                               const void *W_uv, const void *latent_cache,
                               const int32_t *page_table, const int32_t *seq_lens,
                               const int32_t *seq_lens_host, int32_t batch, int32_t s_q,
                               int32_t max_pages, int32_t n_pages_total, void *out,
                               void *workspace, size_t workspace_bytes, mla_stream_t stream);

/*
 * gqla_expand_cache — materialise the GQA path's per-group expanded cache from the latent.
 * ("GQLA: Group-Query Latent Attention ..." abstract: a GQA path with a per-group expanded
 *  cache; AI Radio episode transcript: it caches per-group K and V plus the shared RoPE key.)
 *   K_g,t = W_UK[g] c_t  (d_nope),  V_g,t = W_UV[g] c_t  (d_v),  g < H / heads_per_group.
 *
 *   latent_cache    device [n_pages_total, page_size, d_c + d_rope].
 *   page_ids        device [n_ids] pages to expand, or NULL for all pages 0..n_pages_total-1.
 *   expanded_cache  device [n_pages_total, n_groups, page_size, d_nope + d_v]; row =
 *                   [K_g | V_g], same page ids as the latent cache.  The RoPE key is not
 *                   copied: the grouped decode reads it from the latent cache.
 * Accumulates in fp32, rounds once to the cache dtype.  Out-of-range page ids are skipped and
 * set MLA_ERR_DEVICE_BOUNDS.
 */
MLA_API mla_status gqla_expand_cache(const mla_dims *dims, const void *W_uk, const void *W_uv,
                             const void *latent_cache, const int32_t *page_ids, int32_t n_ids,
                             int32_t n_pages_total, void *expanded_cache, mla_stream_t stream);

/*
 * gqla_expand_tokens — gqla_expand_cache for single cache rows: the rows of the tokens that
 * mla_cache_append wrote, given by the same (req_idx, positions) arrays.  A decode step expands
 * exactly its new tokens instead of every row of their pages.  ("GQLA ..." abstract: the GQA
 * path's per-group expanded cache.)
 *   req_idx, positions  device [n_tok]: request and position of each row; the row lives at
 *                       page page_table[req_idx * max_pages + positions / page_size], row
 *                       positions % page_size, of both caches.
 *   page_table          device [batch, max_pages].
 * Writes [K_g | V_g] of those rows for every group and leaves every other row untouched.
 * Same arithmetic and rounding as gqla_expand_cache.  A row whose request, position or page id
 * is out of range is skipped and sets MLA_ERR_DEVICE_BOUNDS; n_tok = 0 is a no-op.
 */
MLA_API mla_status gqla_expand_tokens(const mla_dims *dims, const void *W_uk, const void *W_uv,
                              const void *latent_cache, const int32_t *req_idx,
                              const int32_t *positions, int32_t n_tok, const int32_t *page_table,
                              int32_t batch, int32_t max_pages, int32_t n_pages_total,
                              void *expanded_cache, mla_stream_t stream);

/* gqla_decode_workspace_size — as mla_decode_workspace_size, for gqla_decode_grouped. */
MLA_API mla_status gqla_decode_workspace_size(const mla_dims *dims, int32_t batch, int32_t s_q,
                                      const int32_t *seq_lens_host, size_t *bytes);

/*
 * gqla_decode_grouped — GQA-path decode over the per-group expanded cache.
 * ("GQLA ..." abstract: the GQA path, algebraically equivalent to the MQA-absorb path over
 *  the same weights.)  Head h reads group g = h / heads_per_group:
 *     s_t = scale * (q_nope . K_g,t + RoPE(q_rope, p) . k^R_t),   t <= p
 *     out = sum_t softmax(s)_t V_g,t
 * Arguments as mla_decode_absorbed, with expanded_cache from gqla_expand_cache and
 * latent_cache supplying the shared RoPE key k^R.
 */
MLA_API mla_status gqla_decode_grouped(const mla_dims *dims, const void *q, const void *expanded_cache,
                               const void *latent_cache, const int32_t *page_table,
                               const int32_t *seq_lens, const int32_t *seq_lens_host,
                               int32_t batch, int32_t s_q, int32_t max_pages,
                               int32_t n_pages_total, void *out, void *workspace,
                               size_t workspace_bytes, mla_stream_t stream);

/*
 * mla_get_device_status — synchronise `stream`, then read and clear the current device's
 * error word.  Returns MLA_OK, MLA_ERR_DEVICE_BOUNDS, MLA_ERR_TIMEOUT, MLA_ERR_INVALID_ARG
 * (device seq_lens disagreed with the host copy) or MLA_ERR_CUDA.
 */
MLA_API mla_status mla_get_device_status(mla_stream_t stream);

/*
 * mla_decode_absorbed_noalloc — mla_decode_absorbed for callers that cannot allocate device
 * memory.  The pages have no counterpart to this entry point; it changes where scratch lives,
 * not what is computed.
 *
 * Some callers have no way to obtain a workspace: an engine whose memory manager has already
 * reserved the whole device for its KV-cache pool and forbids ad-hoc cudaMalloc, or a
 * latency-critical loop where cudaMalloc/cudaFree would stall on an implicit device
 * synchronisation.  This variant takes the same inputs and output as mla_decode_absorbed but no
 * workspace: its scratch is a static device array of MLA_NOALLOC_SCRATCH_BYTES compiled into
 * the library, which every GPU that loads the library holds until the process exits.
 *   - Returns MLA_ERR_WORKSPACE (nothing enqueued) when the batch needs more scratch than that;
 *     mla_decode_workspace_size() tells how much a batch needs.
 *   - The first call on a device looks up that device's address of the array (no allocation);
 *     make the first call on each device before any stream capture.
 *   - All calls share the one array, and every call rewrites what it reads from it, so nothing
 *     needs clearing; but two calls that overlap on the GPU (different streams, or different
 *     host threads, without ordering between them) race on it and corrupt each other.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define MLA_NOALLOC_SCRATCH_BYTES (32u << 20)
MLA_API mla_status mla_decode_absorbed_noalloc(const mla_dims *dims, const void *q, const void *W_uk,
                                               const void *W_uv, const void *latent_cache,
                                               const int32_t *page_table, const int32_t *seq_lens,
                                               const int32_t *seq_lens_host, int32_t batch,
                                               int32_t s_q, int32_t max_pages,
                                               int32_t n_pages_total, void *out,
                                               mla_stream_t stream);

/*
 * mla_set_profile_events — measurement hook.  When both are non-NULL, every later
 * mla_decode_absorbed / gqla_decode_grouped call on the calling thread records `start_event`
 * on its stream immediately before launching its main attention kernel and `stop_event`
 * immediately after, so cudaEventElapsedTime gives that kernel's duration.  Both are
 * cudaEvent_t handles owned by the caller; NULL, NULL turns the hook off.  No computation
 * changes.
 */
MLA_API mla_status mla_set_profile_events(void *start_event, void *stop_event);

/*
 * mla_prefill_workspace_size / mla_prefill_expanded — head-expanded causal attention of the last
 * n_q tokens of every request: a prefill chunk, or a batch of n_q draft tokens to verify.
 * ("GQLA ..." abstract: MLA offers absorbed and head-expanded forms; the expanded form attends
 *  with keys and values up-projected per head, "MLA and GRPO architecture", "The Mathematics
 *  of MLA": k^C = W_UK c, v^C = W_UV c.)  For head h in group g = h / heads_per_group and query
 * j at position p_j = seq_lens[b] - n_q + j:
 *     s_t = scale * ([q_nope | RoPE(q_rope, p_j)] . [K_g,t | k^R_t]),  t <= p_j
 *     out = sum_t softmax(s)_t V_g,t
 * with K_g, V_g the expanded cache of gqla_expand_cache (pass dims with heads_per_group = 1
 * there for per-head MLA weights).  Same math as gqla_decode_grouped, for any n_q.
 *
 *   q             device [batch, n_q, H, d_nope + d_rope]; RoPE part NOT yet rotated.
 *   expanded_cache device [n_pages_total, H / heads_per_group, page_size, d_nope + d_v].
 *   latent_cache  device [n_pages_total, page_size, d_c + d_rope] (source of k^R).
 *   page_table, seq_lens, seq_lens_host as for the decode calls, with n_q <= seq_lens[b].
 *   out           device [batch, n_q, H, d_v].
 *   workspace     >= mla_prefill_workspace_size() bytes, 256-byte aligned (scratch).
 * Needs bf16, d_nope = d_v = 128, d_rope = 64, d_c = 512, page_size = 64
 * (MLA_ERR_UNSUPPORTED otherwise).
 */
MLA_API mla_status mla_prefill_workspace_size(const mla_dims *dims, int32_t batch, int32_t n_q,
                                              const int32_t *seq_lens_host, size_t *bytes);
MLA_API mla_status mla_prefill_expanded(const mla_dims *dims, const void *q, const void *expanded_cache,
                                        const void *latent_cache, const int32_t *page_table, const int32_t *seq_lens,
                                        const int32_t *seq_lens_host, int32_t batch, int32_t n_q, int32_t max_pages,
                                        int32_t n_pages_total, void *out, void *workspace, size_t workspace_bytes,
                                        mla_stream_t stream);

/*
 * mla_select_path — runtime choice between the two decoding paths of the same weights.
 * ("GQLA ..." abstract: the runtime picks the path that matches the target hardware; the
 *  MQA-absorb path trades memory traffic for computation and replicates the latent on every
 *  rank, the GQA path shards its KV groups over up to 8 ranks.)  Pure host arithmetic: no
 * CUDA call, no device pointer.
 *
 * Roofline model of one decode call on one rank (tp ranks share the heads):
 *   visible  = sum_b sum_j (seq_lens[b] - s_q + j + 1)        (query-token pairs)
 *   tokens   = sum_b seq_lens[b]
 *   absorbed: bytes = tokens*(d_c + d_rope)*e            (the latent, replicated on every rank)
 *                     + (G/tp)*(d_nope + d_v)*d_c*e           (this rank's W_UK and W_UV)
 *             flops = visible*2*(H/tp)*(2*d_c + d_rope)
 *                     + batch*s_q*(H/tp)*2*d_c*(d_nope + d_v)    (q absorption, W_UV)
 *   grouped:  bytes = tokens*((G/tp)*(d_nope + d_v) + d_rope)*e
 *             flops = visible*2*(H/tp)*(d_nope + d_rope + d_v)
 *   time     = max(bytes / hbm_bytes_per_s, flops / flops_per_s) for each path
 * with e the element size, G = H / heads_per_group, and q / out traffic left out (equal on
 * both paths).  The grouped path's expanded cache must exist (gqla_expand_cache); its upkeep
 * is per appended page and is not counted.
 *
 *   dims              as for the decode calls (heads_per_group = 8 for GQLA weights)
 *   batch, s_q        > 0; 1 <= s_q <= 4
 *   seq_lens_host     host [batch], each >= s_q
 *   hbm_bytes_per_s   target memory bandwidth (> 0)
 *   flops_per_s       target dense tensor throughput for dims->dtype (> 0)
 *   tp                ranks that shard the heads / KV groups: 1 for one GPU; must divide
 *                     H / heads_per_group
 *   path              out: MLA_PATH_ABSORBED or MLA_PATH_GROUPED (the smaller time; absorbed
 *                     on a tie)
 *   t_absorbed_s, t_grouped_s   out (may be NULL): the two modelled times, seconds
 */
typedef enum { MLA_PATH_ABSORBED = 0, MLA_PATH_GROUPED = 1 } mla_path;
MLA_API mla_status mla_select_path(const mla_dims *dims, int32_t batch, int32_t s_q, const int32_t *seq_lens_host,
                                   double hbm_bytes_per_s, double flops_per_s, int32_t tp, mla_path *path,
                                   double *t_absorbed_s, double *t_grouped_s);

/*
 * mla_debug_decode_fault — test hook of the bounded device waits (failure detection).  The
 * pages have no counterpart to it.  After a call with withhold_step >= 0, every tensor-core
 * absorbed decode launched from the calling thread skips the completion signal of pipeline
 * step `withhold_step` (the PV product of that 128-token step) in every CTA pair, so the waits
 * on it run out: the kernel records MLA_ERR_TIMEOUT in the device error word, stops issuing
 * work, frees its tensor memory and returns without faulting; the call's output is garbage and
 * mla_get_device_status() reports MLA_ERR_TIMEOUT.  wait_us (1..2000000) replaces the 2 s limit
 * of every device wait, so the test ends in milliseconds; 0 keeps the default.
 * mla_debug_decode_fault(-1, 0) restores normal operation.  Returns MLA_ERR_INVALID_ARG for
 * withhold_step < -1 or wait_us > 2000000.  Not for production use.
 */
MLA_API mla_status mla_debug_decode_fault(int32_t withhold_step, uint32_t wait_us);

/* Text of the last error on the calling thread ("" if none).  Valid until the next call. */
MLA_API const char *mla_last_error_string(void);

/* Library version as major*10000 + minor*100 + patch. */
MLA_API int32_t mla_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MLA_H_ */
