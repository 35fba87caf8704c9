// Host-side launchers of the ISD kernels (internal to libisd.so).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

namespace isd {

// Record msg as the calling thread's last error (see isd_last_error); returns code.
int set_error(int code, const char* msg);

// Cycle limit of the bounded device waits of the GEMM and attention kernels
// on the current device (synchronous copies to each file's limit).
cudaError_t set_wait_limit_gemm(long long cycles);
cudaError_t set_wait_limit_attention(long long cycles);

// --------------------------------------------------------------- tensor maps
// 2-D bf16 tensor map over a row-major [rows][cols] matrix, box
// {64 columns (128 B), box_rows}, 128-byte swizzle, zero fill out of bounds.
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows, std::string* err);
// 3-D bf16 tensor map over a dense [d2][d1][d0] array (d0 innermost), box
// {b0, b1, b2}, 128-byte swizzle (b0 * 2 must be 128), zero fill out of bounds.
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint32_t b0, uint32_t b1, uint32_t b2, std::string* err);

// ---------------------------------------------------------------------- GEMM
enum GemmEpilogue : int32_t { kEpiF32 = 0, kEpiSiluMul = 1 };

struct GemmPlan {
  int32_t n_pad = 0, n_mma = 0, mma_n = 0, box_rows = 0, n_boxes = 0;
  int32_t n_chunks = 0, splits = 0, kb_per_split = 0, stages = 0;
  int32_t pair = 0;     // 1: clusters of two CTAs issue 2-SM (cta_group::2) MMAs
  int32_t streamk = 0;  // 1: persistent ranges of (tile, K-block) iterations
  int32_t units = 0;    // stream-K: CTAs (pairs) sharing the iterations
  uint32_t tmem_cols = 0;
  size_t smem_bytes = 0;
};

// Tile plan for Y[m][n_out] = X[m][k] W[n_out][k]^T. force_splits > 0 pins
// the split-K factor; max_splits bounds the automatic choice; allow_streamk
// lets a single-split plan with more tiles than one wave run as stream-K
// (its output is one slice; it needs gemm_streamk_workspace_bytes of
// workspace whose first gemm_streamk_sync_bytes() bytes, the sync words,
// start at zero; every launch leaves them at zero).
GemmPlan plan_gemm(int32_t m, int32_t n_out, int32_t k, int32_t force_splits, int32_t max_splits,
                   int32_t num_sms, bool allow_streamk = false);
size_t gemm_streamk_workspace_bytes(const GemmPlan& plan);
size_t gemm_streamk_sync_bytes();

// A second operand pair whose product is added to the result: the last
// split (under stream-K, the segment that ends a tile's base K-blocks) runs
// k / 64 more K-blocks with W2 (box rows 128, the same n_out rows) and X2
// (box rows = plan.box_rows, the same m rows). Stream-K ranges are cut on the
// base K-blocks alone, so the base part of every result is summed exactly as
// without the second pair.
struct GemmAugment {
  const CUtensorMap* tmap_w;
  const CUtensorMap* tmap_x;
  int32_t k;
};

// tmap_w: W with box_rows 128; tmap_x: X with rows = m and box_rows = plan.box_rows.
// kEpiF32: out_f32[split][m][n_out]; kEpiSiluMul: out_act[m][n_out / 2] bf16
// with W's rows interleaved in blocks of 16 (gate rows then up rows).
// row_stats (kEpiF32, one slice): [m][n_out / 32] of {max, sum of
// exp(y - max), max again, first argmax as int bits} over each 32 outputs.
// pdl: launch with programmatic stream serialisation (the first ring of
// weight tiles loads while the kernel ahead in the stream finishes).
cudaError_t launch_gemm(const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const GemmPlan& plan,
                        int32_t m, int32_t n_out, int32_t k, GemmEpilogue epi, float* out_f32,
                        __nv_bfloat16* out_act, int32_t* status, cudaStream_t stream,
                        void* sk_workspace = nullptr, size_t sk_workspace_bytes = 0,
                        const GemmAugment* augment = nullptr, float4* row_stats = nullptr,
                        bool pdl = false);

// ----------------------------------------------------------------- attention
struct AttnShape {
  int32_t batch, rows_per_req, n_q_heads, n_kv_heads, head_dim, page_size, num_pages,
      max_pages_per_req, n_layers;
};
size_t attention_workspace_bytes(const AttnShape& s);
// Host mirror of the tcgen05 attention kernel's work split over num_sms CTAs,
// from the per-request key counts kend[batch]: one record {CTA, request, KV
// head, first 128-key tile, tiles, partial slot} per segment, in CTA order.
// Returns 0; -1 when the tcgen05 kernel does not serve the shape; -2 when
// seg_capacity records are too few (n_segments holds the count needed).
int attention_split(const AttnShape& s, const int32_t* kend, int num_sms, int32_t* seg,
                    int seg_capacity, int* n_segments, int* max_parts);
// k_map / v_map: tensor maps over the pools as [n_layers*num_pages*n_kv*page_size][head_dim]
// with box_rows = page_size.
// qkv (optional): this layer's QKV split-K reduction, which produces q and
// the block's K/V rows; it is launched first, as its own kernel.
struct QkvReduceArgs;
cudaError_t launch_attention(const CUtensorMap& k_map, const CUtensorMap& v_map, const AttnShape& s,
                             int32_t layer, const __nv_bfloat16* q, const int32_t* row_pos,
                             const int32_t* page_table, __nv_bfloat16* out, void* workspace,
                             int32_t* status, cudaStream_t stream, int* launches,
                             cudaEvent_t between = nullptr, const QkvReduceArgs* qkv = nullptr,
                             bool prefix_early = false, bool pdl = false);
// (prefix_early: each request's rows are one block at consecutive positions,
// a decode step, so K/V tiles below a request's first row do not depend on
// the QKV reduction and may be loaded before waiting for it. pdl: the
// tcgen05 kernel is launched with programmatic stream serialisation right
// after the QKV reduction this call launches.)

// ------------------------------------------------------------------ row ops
struct RowMeta {
  int32_t* tok;     // [rows] input token
  int32_t* pos;     // [rows] absolute position (-1: none)
  int32_t* flags;   // [rows] bit0: write KV, bit1: MASK row (gated LoRA)
};
constexpr int32_t kRowWriteKV = 1;
constexpr int32_t kRowMask = 2;

cudaError_t launch_assemble_step(const int32_t* pending, const int32_t* n_draft,
                                 const int32_t* seq_len, int32_t batch, int32_t stride_n,
                                 int32_t mask_token, RowMeta meta, int32_t* status,
                                 cudaStream_t stream);
// rows of `batch` requests, request order[i] (or i when order is null) in
// block i of `chunk` rows
cudaError_t launch_assemble_prefill(const int32_t* tokens, int32_t max_len, const int32_t* lens,
                                    const int32_t* order, int32_t batch, int32_t chunk,
                                    int32_t start, RowMeta meta, cudaStream_t stream);
// dst row (i * repeat + j) = src row order[i] for i < rows, j < repeat (int rows of row_len).
cudaError_t launch_gather_rows(const int32_t* src, const int32_t* order, int32_t rows,
                               int32_t row_len, int32_t repeat, int32_t* dst, cudaStream_t stream);
cudaError_t launch_embed_norm(const __nv_bfloat16* embed, const float* norm_w, RowMeta meta,
                              int32_t rows, int32_t hidden, int32_t vocab, float eps, float* x,
                              __nv_bfloat16* hn, int32_t* status, cudaStream_t stream);

struct QkvReduceArgs {
  const float* part;        // [splits][rows][qkv_dim]
  int32_t splits, rows, rows_per_req;
  int32_t n_q, n_kv, head_dim;
  const float* q_norm;      // [head_dim]
  const float* k_norm;
  float eps;
  const float2* rope;       // [max_position][head_dim/2] (cos, sin)
  int32_t max_position;
  RowMeta meta;
  const int32_t* page_table;
  int32_t max_pages_per_req, page_size, num_pages, layer;
  __nv_bfloat16* k_pool;
  __nv_bfloat16* v_pool;
  __nv_bfloat16* q_out;     // [rows][n_q][head_dim]
  int32_t* status;
};
cudaError_t launch_qkv_reduce(const QkvReduceArgs& a, cudaStream_t stream);

// x[row] += sum_s part[s][row] (splits in order); hn[row] = bf16(RMSNorm(x[row]) * norm_w).
cudaError_t launch_residual_norm(const float* part, int32_t splits, int32_t rows, int32_t hidden,
                                 const float* norm_w, float eps, float* x, __nv_bfloat16* hn,
                                 cudaStream_t stream);

// ---------------------------------------------------------------- gated LoRA
cudaError_t launch_pack_rows(const __nv_bfloat16* src, int rows, int cols, __nv_bfloat16* dst,
                             int dst_ld, int row0, int col0, int interleave_off,
                             cudaStream_t stream);
// out = bf16(scale * sum of the splits) on MASK rows (row_flags), 0 elsewhere.
cudaError_t launch_sum_cast(const float* part, int splits, int rows, int n, const int32_t* row_flags,
                            float scale, __nv_bfloat16* out, cudaStream_t stream);


// ---------------------------------------------------------- accept / propose
struct AcceptArgs {
  const float* logits;      // [B*R][V]
  int32_t batch, stride_n, vocab, flags, page_size;
  int32_t* pending;         // [B][N]
  int32_t* n_draft;         // [B]
  int32_t* seq_len;         // [B]
  float* q_cache;           // [B][N-1][V] or null
  const float* uniforms;    // [B][R]
  int32_t* accepted;        // [B]
  int32_t* committed;       // [B][N] or null
  int32_t* page_table;      // [B][max_pages]
  const int32_t* free_list;
  int32_t* free_head;
  int32_t num_pages, max_pages_per_req, free_count;
  int32_t* status;
  // per (row, 32-token slab) statistics of the logits from the LM head's
  // epilogue (launch_gemm row_stats); null: computed from the logits
  const float4* slab_stats = nullptr;
};
size_t accept_workspace_bytes(int32_t batch, int32_t stride_n, int32_t vocab);
// between[0] / between[1]: optional events recorded after the first and second kernel.
cudaError_t launch_accept(const AcceptArgs& a, void* workspace, cudaStream_t stream, int* launches,
                          cudaEvent_t between0 = nullptr, cudaEvent_t between1 = nullptr);

}  // namespace isd
