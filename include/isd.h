/*
 * isd.h - C ABI of the B200 (sm_100a) Introspective Strided Decoding library.
 *
 * One ISD step: every request of a batch runs one strictly causal forward of
 * a Qwen3-shaped decoder over a block [x* | N-1 pending drafts | N-1 MASK]
 * against its paged KV prefix; the drafts are verified left to right with
 * u < min(1, p/q) (p: this forward's anchor, q: the previous forward's
 * proposal), the first rejected slot is refilled from norm(max(0, p - q)),
 * and the MASK rows propose the next drafts.
 *   Sources: Bud's Wiki "Introspective Diffusion Language Models" (TL;DR,
 *   Key claims, Method); Agentic Commons blog of the same title ("How
 *   Introspective Strided Decoding Works"); GeekNews (hi/pt) summaries
 *   ("Inference & ISD", "Lossless R-ISD", "Speedup Factor Explorer").
 *
 * Block layout (rows r = 0..2N-2 at positions L..L+2N-2, L = committed length):
 *   full step (n = N-1 drafts):  [x*, d_1..d_{N-1}, MASK x (N-1)]
 *   restart step (n = 0):        [x*, MASK x (N-1), MASK padding x (N-1)]
 * Row t scores the token at position t+1 (logit shift). Draft d_j is tested
 * on row j-1; the new final token comes from row A (A = accepted drafts);
 * rows n+1..n+N-1 propose the next drafts when no draft was rejected.
 * Uniform slots per request (2N-1 floats in [0,1)): [0, N-1) accept tests,
 * [N-1] the new token, [N, 2N-1) sampled proposals.
 *
 * Conventions for every entry point:
 *  - Pointers named *_dev are device memory owned by the caller; the library
 *    never frees or reallocates them. Host arrays of device pointers are
 *    copied during the call that receives them.
 *  - Matrices are row-major. "nn.Linear layout" means [out_features][in_features].
 *  - bf16 means IEEE bfloat16 (torch.bfloat16).
 *  - Functions return ISD_OK (0) or a negative ISD_E_* code; the text of the
 *    last error of the calling thread is returned by isd_last_error().
 *  - Work is enqueued on the given cudaStream_t (passed as void*); nothing
 *    synchronises the stream. Faults found on the device (pool exhausted,
 *    token or page id out of range, a bounded wait that ran out) are OR-ed
 *    into the caller's int32 status word as ISD_DEV_* bits; read it after
 *    synchronising. No kernel traps or asserts.
 */
#ifndef ISD_H_
#define ISD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ------------------------------------------------------ */
#define ISD_OK             0
#define ISD_E_INVALID     -1  /* null pointer, size or flag out of range            */
#define ISD_E_UNSUPPORTED -2  /* a shape the kernels do not implement               */
#define ISD_E_CUDA        -3  /* a CUDA runtime call failed                         */
#define ISD_E_NOMEM       -4  /* workspace allocation failed (isd_init only)        */

/* ---- device status bits (OR-ed into *status_dev) ----------------------- */
#define ISD_DEV_POOL_EXHAUSTED 0x01 /* free list too short: no page handed out  */
#define ISD_DEV_TABLE_FULL     0x02 /* a request outgrew max_pages_per_req      */
#define ISD_DEV_BAD_TOKEN      0x04 /* token id outside [0, vocab)              */
#define ISD_DEV_BAD_PAGE       0x08 /* page id outside [0, num_pages)           */
#define ISD_DEV_TIMEOUT        0x10 /* a bounded device wait ran out            */
#define ISD_DEV_BAD_STATE      0x20 /* n_draft not 0 or N-1, or length < 0      */

/* ---- step mode flags ---------------------------------------------------- */
#define ISD_PROPOSE_ARGMAX 0x0  /* MASK rows propose by argmax (lowest index on ties) */
#define ISD_PROPOSE_SAMPLE 0x1  /* MASK rows sample; q rows stored in q_cache         */
#define ISD_VERIFY_SAMPLE  0x0  /* u*q(d) < p(d) test, residual / bonus sampling      */
#define ISD_VERIFY_GREEDY  0x2  /* temperature 0: accept iff d == argmax p            */
#define ISD_USE_LORA       0x4  /* add the loaded gated LoRA on MASK rows only        */

/* ---- model ------------------------------------------------------------- */
typedef struct {
  int32_t n_layers, hidden, n_q_heads, n_kv_heads, head_dim, intermediate, vocab;
  float rope_theta;      /* NeoX rotate-half RoPE base (1e6 for Qwen3)            */
  float rms_eps;         /* RMSNorm epsilon                                       */
  int32_t mask_token_id; /* token fed to MASK rows                                */
  int32_t page_size;     /* KV positions per page: 16, 32 or 64                   */
  int32_t max_batch;     /* most requests one call may carry (workspace size)      */
  int32_t max_rows;      /* most block rows one call may process (workspace size) */
  int32_t max_position;  /* positions must stay below this (RoPE table size, and
                            max_pages_per_req * page_size <= max_position)         */
} isd_model_cfg;
/* Supported: head_dim 64 or 128; hidden, n_q_heads*head_dim, intermediate
 * multiples of 128 (intermediate of 64); n_q_heads/n_kv_heads in {1,2,4,8};
 * vocab a multiple of 128. */

typedef struct {
  const void *embed_dev;        /* [vocab][hidden] bf16                                  */
  const void *lm_head_dev;      /* [vocab][hidden] bf16 (nn.Linear layout, untied)       */
  const float *final_norm_dev;  /* [hidden] fp32                                         */
  /* host arrays of n_layers device pointers each:                                      */
  const void *const *w_qkv;     /* [(nq+2nkv)*head_dim][hidden] bf16: q rows, k rows, v rows */
  const void *const *w_o;       /* [hidden][nq*head_dim] bf16                            */
  const void *const *w_gate_up; /* [2*intermediate][hidden] bf16; row block b of 32 holds
                                   gate rows 16b..16b+15 then up rows 16b..16b+15       */
  const void *const *w_down;    /* [hidden][intermediate] bf16                           */
  const float *const *attn_norm;/* [hidden] fp32 (pre-attention RMSNorm weight)          */
  const float *const *mlp_norm; /* [hidden] fp32 (pre-MLP RMSNorm weight)                */
  const float *const *q_norm;   /* [head_dim] fp32 (per-head RMSNorm of q)               */
  const float *const *k_norm;   /* [head_dim] fp32 (per-head RMSNorm of k)               */
} isd_weights;

/* Gated LoRA of R-ISD (Bud's Wiki, Key claims and Method: rank 128, active
 * only at MASK positions, verify positions on base weights). Targets in
 * order q, k, v, o, gate, up, down; each a host array of n_layers device
 * pointers. A_t: [rank][in_t] bf16, B_t: [out_t][rank] bf16 (the two
 * nn.Linear weights); delta = scale * (x A_t^T) B_t^T on MASK rows only. */
typedef struct {
  int32_t rank;     /* 128, the rank the pages give (others: ISD_E_UNSUPPORTED) */
  float scale;
  const void *const *A[7];
  const void *const *B[7];
} isd_lora;

/* ---- per-call state (all device memory, caller-owned) ------------------ */
typedef struct {
  int32_t batch;       /* B requests, 1..1024                                   */
  int32_t stride_n;    /* N, 1..8                                               */
  int32_t flags;       /* ISD_PROPOSE_* | ISD_VERIFY_* | ISD_USE_LORA            */
  int32_t *seq_len_dev;/* [B] committed length L_b (updated: L_b += 1 + A_b)     */
  int32_t *n_draft_dev;/* [B] pending drafts, 0 or N-1 (updated)                 */
  float *logits_out_dev; /* optional [B*(2N-1)][vocab] fp32 block logits, or NULL */
} isd_batch;

typedef struct {
  void *k_pool_dev;    /* [n_layers][num_pages][n_kv_heads][page_size][head_dim] bf16;
                          must be initialised to finite values (e.g. zeros)       */
  void *v_pool_dev;    /* same layout as k_pool_dev                              */
  int32_t *page_table_dev; /* [B][max_pages_per_req] physical page ids (updated) */
  const int32_t *free_list_dev; /* [free_count] page ids handed out in order     */
  int32_t *free_head_dev;       /* [1] next unused free_list entry (updated)      */
  int32_t num_pages, max_pages_per_req, free_count;
} isd_kv;
/* Invariant at entry of isd_step: request b holds valid pages for positions
 * [0, seq_len[b] + 2N - 1). The step keeps it for the updated lengths. */

typedef struct isd_ctx isd_ctx;

/* Create a context: copies cfg and the weight pointer arrays (the weights
 * stay caller-owned and must outlive the context), builds TMA descriptors,
 * the RoPE table and the workspace (the library's only allocation).
 * Returns ISD_E_UNSUPPORTED for shapes outside the list above. */
int isd_init(const isd_model_cfg *cfg, const isd_weights *w, isd_ctx **out);

/* Attach a gated LoRA (copies the pointer arrays; the tensors stay
 * caller-owned). Steps use it when flags has ISD_USE_LORA. The library packs
 * the adapters into fused matrices it owns (freed by isd_destroy).
 * Errors: ISD_E_UNSUPPORTED for a rank other than 128; ISD_E_INVALID for a
 * null ctx or lora or a missing pointer; ISD_E_NOMEM when the packed
 * matrices cannot be allocated; ISD_E_CUDA when packing fails. */
int isd_load_gated_lora(isd_ctx *ctx, const isd_lora *lora);

/* One ISD step for the whole batch (enqueue only; CUDA-graph capturable).
 *  pending_dev   [B][N] int32: x* then the n drafts (in); next x* then the
 *                next drafts (out).
 *  q_cache_dev   [B][N-1][vocab] fp32 proposal distributions of the pending
 *                drafts (read) and of the next drafts (written); used only
 *                with ISD_PROPOSE_SAMPLE, may be NULL otherwise.
 *  uniforms_dev  [B][2N-1] fp32 in [0,1), slot map above.
 *  out_accepted_dev  [B] int32: A_b in [0, n_b].
 *  out_committed_dev [B][N] int32: the A_b accepted drafts then the new
 *                final token (A_b + 1 valid entries), or NULL.
 *  status_dev    [1] int32 device status word (bits OR-ed in).
 *  stream        cudaStream_t.
 * Errors (nothing is enqueued): ISD_E_INVALID for a null argument, a batch
 * outside [1, min(1024, cfg.max_batch)], N outside [1, 8], unknown flag
 * bits, ISD_USE_LORA without an adapter, SAMPLE proposals without q_cache,
 * batch * (2N-1) above cfg.max_rows, or an inconsistent isd_kv;
 * ISD_E_UNSUPPORTED when (2N-1) * n_q_heads / n_kv_heads exceeds 64, the
 * KV pool holds 2^31 or more rows (layers x pages x KV heads x page_size)
 * or the block rows exceed the logits workspace (pass logits_out_dev);
 * ISD_E_CUDA
 * when a launch fails (the work enqueued before it stays enqueued). */
int isd_step(isd_ctx *ctx, const isd_batch *batch, const isd_kv *kv, int32_t *pending_dev,
             float *q_cache_dev, const float *uniforms_dev, int32_t *out_accepted_dev,
             int32_t *out_committed_dev, int32_t *status_dev, void *stream);

/* Prefill prompts into the paged KV cache and set the starting state:
 * KV of positions [0, len_b - 1), seq_len = len_b - 1, pending[b][0] =
 * last prompt token, n_draft = 0 (so the first step is a restart step).
 *  tokens_dev [B][max_len] int32; lens_host [B] host int32, 1 <= len <= max_len.
 * Pages for positions [0, len_b - 1 + 2N - 1) must already be in the page
 * table. Rows are processed in chunks through the same kernels as a step.
 * Errors: ISD_E_INVALID for a null argument, batch outside [1,
 * cfg.max_batch], stride_n outside [1, 8], a length outside [1, max_len] or
 * an inconsistent isd_kv (nothing enqueued); ISD_E_UNSUPPORTED for a KV
 * pool of 2^31 or more rows; ISD_E_CUDA when a launch fails. */
int isd_prefill(isd_ctx *ctx, const isd_kv *kv, const int32_t *tokens_dev, int32_t max_len,
                const int32_t *lens_host, int32_t batch, int32_t stride_n,
                int32_t *seq_len_dev, int32_t *n_draft_dev, int32_t *pending_dev,
                int32_t *status_dev, void *stream);

/* Number of kernel launches the last isd_step / isd_prefill enqueued. */
int isd_last_launch_count(const isd_ctx *ctx);

/* Per-kernel-class timing with CUDA events recorded around each launch on
 * the step's stream (for measurement; off by default, not for use inside a
 * CUDA graph capture). isd_profile_read synchronises on the last recorded
 * event, writes the summed milliseconds and launch counts of each class
 * (ISD_PROF_CLASSES entries, host arrays) and clears the record.
 * isd_profile_class_name gives a class's name ("" outside the range).
 * Errors: ISD_E_INVALID for a null argument; ISD_E_CUDA when an event
 * query fails. */
#define ISD_PROF_CLASSES 16
int isd_profile_enable(isd_ctx *ctx, int enable);
int isd_profile_read(isd_ctx *ctx, double *total_ms, int32_t *counts);
const char *isd_profile_class_name(int cls);

/* Text of the calling thread's last error (owned by the library, valid
 * until that thread's next failing call). */
const char *isd_last_error(void);
/* Free the context, its workspace and any packed adapter (NULL is a no-op).
 * The caller first makes sure no work it enqueued with the context is still
 * running. Caller-owned buffers are untouched. */
void isd_destroy(isd_ctx *ctx);

/* Cycle limit of every bounded device wait (an mbarrier phase, a stream-K
 * partner's flag) on the current device; 0 restores the default of 4e9
 * cycles (about 2 s). A wait that runs out sets ISD_DEV_TIMEOUT and its
 * kernel returns without writing the affected results, so a context stays
 * usable. For tests of failure handling: a short limit lets a test make a
 * wait run out quickly. Synchronous (not during stream capture); affects
 * every context on the device. No counterpart on the pages: the status word
 * is this library's own failure reporting. Returns ISD_E_INVALID for a limit
 * below 1000 cycles, ISD_E_CUDA if the copy fails. */
int isd_set_wait_limit(long long cycles);

/* ---- component entry points (used by the tests; same kernels as a step) -- */

/* Y = X W^T on the tcgen05 tensor cores, fp32 accumulate.
 *  w_dev [n][k] bf16 (nn.Linear layout), x_dev [m][k] bf16,
 *  y_dev [split_k][m][n] fp32: split s holds the partial sum over its share
 *  of k (the caller adds the splits). n % 128 == 0, k % 64 == 0,
 *  1 <= m <= 4096, 1 <= split_k <= 16.
 * Errors: ISD_E_INVALID for a null operand or a pointer TMA cannot address
 * (16-byte alignment); ISD_E_UNSUPPORTED outside the limits above or when
 * split_k leaves a split without K-blocks; ISD_E_CUDA when the launch
 * fails. */
int isd_gemm_bf16(const void *w_dev, const void *x_dev, float *y_dev, int32_t m, int32_t n,
                  int32_t k, int32_t split_k, int32_t *status_dev, void *stream);

/* Y = X W^T as one fp32 slice, planned as a step plans its single-slice
 * projections (the MLP gate/up, the LM head): when the 128-row weight tiles
 * overfill one wave of SMs it runs as stream-K, CTAs sharing the (tile,
 * K-block) iterations, and a tile cut between two CTAs is completed by the
 * one that finishes second from the other's fp32 partial, parked in the
 * workspace. Same operand layouts and limits as isd_gemm_bf16.
 *  workspace_dev: isd_gemm_workspace_bytes(m, n, k) bytes (0: none needed,
 *  may be NULL). Its first 4096 bytes must be zero before the first call;
 *  each call leaves them zero, so a workspace serves any number of calls
 *  in stream order (not two calls running at once).
 * isd_gemm_workspace_bytes returns 0 for shapes outside the limits too.
 * Errors of isd_gemm_bf16_single: as isd_gemm_bf16, and ISD_E_INVALID for a
 * missing or short workspace. */
size_t isd_gemm_workspace_bytes(int32_t m, int32_t n, int32_t k);

/* The tile plan the library would use for Y = X W^T with m rows, n outputs
 * and k inputs on a GPU with num_sms SMs (host computation only; no device
 * access). single != 0: one output slice (stream-K when the tiles overfill a
 * wave), else up to max_splits K-splits. out[ISD_GEMM_PLAN_FIELDS] receives
 * n_pad (token columns per CTA), token chunks, splits, K-blocks per split,
 * MMAs per k-step, MMA N, TMA box rows, boxes, pipeline stages, 2-SM pair
 * (0/1), stream-K (0/1), stream-K units, TMEM columns, dynamic shared
 * memory bytes. Returns ISD_E_UNSUPPORTED when no plan exists (n not a
 * multiple of 128, k not of 64), ISD_E_INVALID for m, max_splits or num_sms
 * below 1 or a null out. */
#define ISD_GEMM_PLAN_FIELDS 14
int isd_gemm_plan(int32_t m, int32_t n, int32_t k, int32_t single, int32_t max_splits,
                  int32_t num_sms, int32_t *out);
int isd_gemm_bf16_single(const void *w_dev, const void *x_dev, float *y_dev, int32_t m,
                         int32_t n, int32_t k, void *workspace_dev, size_t workspace_bytes,
                         int32_t *status_dev, void *stream);

/* Paged causal GQA attention for one layer.
 *  q_dev [B*R][n_q_heads][head_dim] bf16 (already QK-normed and rotated)
 *  row_pos_dev [B*R] int32: position of each row; a row sees keys t <= pos
 *  (pos < 0: no keys, output 0). Keys live in the pools at layer `layer`.
 *  out_dev [B*R][n_q_heads*head_dim] bf16.
 *  workspace_dev: isd_attention_workspace_bytes(...) bytes of device memory.
 * Errors: ISD_E_INVALID for a null argument, head counts that do not
 * divide, sizes or layer out of range, or a short workspace;
 * ISD_E_UNSUPPORTED for head_dim other than 64 / 128, a group size other
 * than 1, 2, 4, 8, rows_per_req * group above 64, a page size other than
 * 16, 32, 64, or a pool of 2^31 or more rows; ISD_E_CUDA when a launch
 * fails. A page id outside [0, num_pages) read on the device sets
 * ISD_DEV_BAD_PAGE and reads zeros. */
size_t isd_attention_workspace_bytes(int32_t batch, int32_t rows_per_req, int32_t n_q_heads,
                                     int32_t n_kv_heads, int32_t head_dim,
                                     int32_t max_pages_per_req, int32_t page_size);
int isd_paged_attention(const void *q_dev, const int32_t *row_pos_dev, const void *k_pool_dev,
                        const void *v_pool_dev, const int32_t *page_table_dev, int32_t batch,
                        int32_t rows_per_req, int32_t n_q_heads, int32_t n_kv_heads,
                        int32_t head_dim, int32_t page_size, int32_t num_pages,
                        int32_t max_pages_per_req, int32_t n_layers, int32_t layer,
                        void *out_dev, void *workspace_dev, size_t workspace_bytes,
                        int32_t *status_dev, void *stream);

/* Host-only query of the work split of the tcgen05 attention kernel (head_dim
 * 128, 64-key pages, at most 64 query rows per KV head): no GPU work. The
 * kernel runs one CTA per SM over the (request, KV head, 128-key tile)
 * sequence; each CTA takes a contiguous range in which every (request, KV
 * head) pair costs a fixed 3 tiles besides its own tiles (5 above 32 query
 * rows per KV head: starting and finishing a pair), and a pair cut
 * between CTAs leaves one partial per CTA, merged in CTA order (paged
 * attention on tensor cores, a block's queries against its request's paged
 * prefix; Bud's Wiki "Introspective Diffusion Language Models", Method).
 *  kend_host [batch]: keys visible to each request's last row (its largest
 *  row position + 1; clipped to max_pages_per_req * page_size as the kernel
 *  does). num_sms: CTAs of the launch.
 *  seg_out [seg_capacity][ISD_ATTN_SEG_FIELDS]: per segment, in CTA order:
 *  CTA, request, KV head, first tile, tiles, partial slot ((request * n_kv +
 *  head) * max_parts + part; -1 if part >= max_parts, which a valid split
 *  never produces). *n_segments: the segments (also when capacity is short);
 *  *max_parts: the partial slots per (request, KV head).
 * Returns ISD_OK, ISD_E_UNSUPPORTED for shapes the tcgen05 kernel does not
 * serve, ISD_E_INVALID for bad arguments or a short seg_capacity. */
#define ISD_ATTN_SEG_FIELDS 6
int isd_attention_split(int32_t batch, int32_t rows_per_req, int32_t n_q_heads,
                        int32_t n_kv_heads, int32_t head_dim, int32_t max_pages_per_req,
                        int32_t page_size, const int32_t *kend_host, int32_t num_sms,
                        int32_t *seg_out, int32_t seg_capacity, int32_t *n_segments,
                        int32_t *max_parts);

/* Verify / resample / propose from given block logits, then the length and
 * page bookkeeping: the tail of isd_step without the forward.
 *  logits_dev [B*(2N-1)][vocab] fp32; other arguments as in isd_step (kv
 *  supplies page_table / free list / num_pages / max_pages_per_req / page_size).
 *  workspace_dev: isd_accept_workspace_bytes(B, N, vocab) bytes.
 * Errors: ISD_E_INVALID for a null argument, batch outside [1, 1024], N
 * outside [1, 8], page_size below 1, SAMPLE proposals without q_cache, or a
 * short workspace; ISD_E_UNSUPPORTED for a vocab that is not a multiple of
 * 4 in [4, 524288]; ISD_E_CUDA when a launch fails. */
size_t isd_accept_workspace_bytes(int32_t batch, int32_t stride_n, int32_t vocab);
int isd_accept_propose(const float *logits_dev, const isd_batch *batch, const isd_kv *kv,
                       int32_t page_size, int32_t vocab, int32_t *pending_dev,
                       float *q_cache_dev, const float *uniforms_dev,
                       int32_t *out_accepted_dev, int32_t *out_committed_dev,
                       void *workspace_dev, size_t workspace_bytes, int32_t *status_dev,
                       void *stream);

/* The same verify / resample / propose and bookkeeping as
 * isd_accept_propose, for callers that cannot allocate device memory (a host
 * program that hands out all GPU memory from its own fixed pool, a serving
 * loop that must never enter the allocator, a plugin with no allocator of
 * its own). The paper has no counterpart: this is a deployment variant.
 * Scratch comes from a 4 MiB array compiled into the library, present on
 * every GPU that loads it until the process exits; a call needs
 * isd_accept_workspace_bytes(batch, N, vocab) bytes of it (the chunk
 * statistics, batch * (2N-1) * ceil(vocab/8192) * 16 bytes, then 4 bytes
 * per request; at most 4 MiB, e.g. batch <= 1024 at N = 4 and vocab 151936)
 * and returns ISD_E_UNSUPPORTED above that. The first call on each device looks up the array's device
 * address with that device current. Under CUDA's lazy module loading (the
 * default) that lookup is also what loads this part of the library onto the
 * device and places the array there, so the first call on a device does
 * allocate (the array and the module's code) and can fail with ISD_E_CUDA
 * when the device is out of memory: make that first call at start-up,
 * before a pool takes the GPU's memory and before any stream capture.
 * Later calls allocate nothing. All calls share the array: calls that
 * overlap on the GPU race and must be serialised by the caller. No scratch
 * needs clearing. */
int isd_accept_propose_noalloc(const float *logits_dev, const isd_batch *batch, const isd_kv *kv,
                               int32_t page_size, int32_t vocab, int32_t *pending_dev,
                               float *q_cache_dev, const float *uniforms_dev,
                               int32_t *out_accepted_dev, int32_t *out_committed_dev,
                               int32_t *status_dev, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* ISD_H_ */
