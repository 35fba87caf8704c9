// Host engine and C ABI of the ISD library: context creation (TMA
// descriptors, RoPE table, workspace), the kernel sequence of one ISD step,
// chunked prefill and the component entry points. Host code only enqueues
// work on the caller's stream; it never synchronises it, so a step can be
// captured into a CUDA graph.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/isd.h"
#include "kernels.h"

namespace {

thread_local std::string g_err;

int fail(int code, const std::string& msg) {
  g_err = msg;
  return code;
}

#define ISD_CUDA(call)                                                                  \
  do {                                                                                  \
    cudaError_t e_ = (call);                                                            \
    if (e_ != cudaSuccess)                                                              \
      return fail(ISD_E_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_));      \
  } while (0)

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool load_encode(std::string* err) {
  if (g_encode) return true;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
    if (err) *err = "cuTensorMapEncodeTiled unavailable";
    return false;
  }
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

namespace isd {

// Lets other translation units of the library report an error through
// isd_last_error().
int set_error(int code, const char* msg) { return fail(code, msg); }

bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows, std::string* err) {
  if (!load_encode(err)) return false;
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0 || (cols * 2) % 16 != 0) {
    if (err) *err = "tensor map base or row pitch not 16-byte aligned";
    return false;
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (err) *err = "cuTensorMapEncodeTiled failed (" + std::to_string(static_cast<int>(r)) + ")";
    return false;
  }
  return true;
}

bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint32_t b0, uint32_t b1, uint32_t b2, std::string* err) {
  if (!load_encode(err)) return false;
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0 || (d0 * 2) % 16 != 0) {
    if (err) *err = "tensor map base or row pitch not 16-byte aligned";
    return false;
  }
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (err) *err = "cuTensorMapEncodeTiled (3-D) failed (" + std::to_string(static_cast<int>(r)) + ")";
    return false;
  }
  return true;
}

}  // namespace isd

using isd::GemmPlan;

// K-splits allowed for the adapter's thin x A^T products
constexpr int kLoraSplits = 16;

struct isd_ctx {
  isd_model_cfg cfg{};
  const void* embed = nullptr;
  const void* lm_head = nullptr;
  const float* final_norm = nullptr;
  std::vector<const void*> w_qkv, w_o, w_gu, w_down;
  std::vector<const float*> attn_norm, mlp_norm, q_norm, k_norm;
  std::vector<CUtensorMap> tm_qkv, tm_o, tm_gu, tm_down;
  CUtensorMap tm_lm{};
  int32_t qkv_dim = 0, q_dim = 0;
  int32_t max_splits = 8;
  // GEMMs (and the tcgen05 attention) launched with programmatic stream
  // serialisation: each loads what does not depend on the kernel ahead of
  // it (weight tiles; K/V tiles of earlier steps) while that kernel finishes
  bool pdl = true;

  // workspace (the library's only allocation)
  void* ws = nullptr;
  float* x = nullptr;               // [max_rows][hidden] residual stream
  __nv_bfloat16* hn = nullptr;      // [max_rows][hidden] normalised GEMM input
  float* part = nullptr;            // [max_splits][max_rows][max(qkv_dim, hidden)]
  size_t part_elems = 0;
  size_t logit_rows = 0;            // rows the logits buffer holds (steps only)
  int prefill_sub_max = 1;          // attention sub-requests per request in a prefill chunk
  int32_t* prefill_table = nullptr; // [max_batch * prefill_sub_max][max pages] repeated page rows
  __nv_bfloat16* qbuf = nullptr;    // [max_rows][q_dim]
  __nv_bfloat16* attn = nullptr;    // [max_rows][q_dim]
  __nv_bfloat16* act = nullptr;     // [max_rows][intermediate]
  float* logits = nullptr;          // [logit_rows][vocab]
  float4* slab_stats = nullptr;     // [logit_rows][vocab / 32] from the LM head's epilogue
  int32_t* meta_tok = nullptr;
  int32_t* meta_pos = nullptr;
  int32_t* meta_flags = nullptr;
  float2* rope = nullptr;           // [max_position][head_dim/2]
  void* attn_ws = nullptr;
  size_t attn_ws_bytes = 0;
  void* acc_ws = nullptr;
  size_t acc_ws_bytes = 0;
  int32_t* prefill_lens = nullptr;  // [max_batch]
  int32_t* prefill_order = nullptr; // [max_batch] requests by descending prompt length
  int32_t* prefill_ptab = nullptr;  // [max_batch][max pages] page table rows in that order

  std::map<std::tuple<const void*, int, int, int>, CUtensorMap> act_maps;
  std::map<std::tuple<int, int, int, int>, GemmPlan> plans;
  void* sk_ws = nullptr;            // stream-K partials + sync words (sync words zeroed)
  size_t sk_ws_bytes = 0;
  int launches = 0;

  // gated LoRA (R-ISD): packed adapters per layer + their workspace
  bool has_lora = false;
  int32_t lora_rank = 0;
  float lora_scale = 1.f;
  void* lora_mem = nullptr;
  struct LoraLayer {
    __nv_bfloat16 *a_qkv, *b_qkv, *a_o, *b_o, *a_gu, *b_gu, *a_d, *b_d;
    CUtensorMap ta_qkv, tb_qkv, ta_o, tb_o, ta_gu, tb_gu, ta_d, tb_d;
  };
  std::vector<LoraLayer> lora;
  float* lora_xa_part = nullptr;         // [kLoraSplits][max_rows][3r]
  __nv_bfloat16* lora_xa = nullptr;      // [max_rows][3r]

  // per-kernel-class event timing (isd_profile_enable)
  bool prof_on = false;
  std::vector<cudaEvent_t> prof_pool;
  size_t prof_next = 0;
  std::vector<std::tuple<int, cudaEvent_t, cudaEvent_t>> prof_recs;
};

namespace {

enum ProfClass {
  kPAssemble = 0, kPEmbed, kPGemmQkv, kPQkvReduce, kPAttnSplit, kPAttnCombine, kPGemmO,
  kPResNorm, kPGemmGateUp, kPGemmDown, kPGemmLmHead, kPAcceptStats, kPAcceptDecide,
  kPBookkeep, kPOther, kPCount
};
const char* kProfNames[ISD_PROF_CLASSES] = {
    "assemble", "embed_norm", "gemm_qkv", "qkv_reduce_rope_kvwrite", "attention",
    "attention_combine", "gemm_o", "residual_norm", "gemm_gate_up_silu", "gemm_down",
    "gemm_lm_head", "accept_stats", "accept_decide", "bookkeep", "lora", "unused"};

cudaEvent_t prof_event(isd_ctx* c) {
  if (!c->prof_on) return nullptr;
  if (c->prof_next == c->prof_pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    c->prof_pool.push_back(e);
  }
  return c->prof_pool[c->prof_next++];
}

// Record an event on the stream (when profiling) and return it.
cudaEvent_t prof_mark(isd_ctx* c, cudaStream_t st) {
  cudaEvent_t e = prof_event(c);
  if (e) cudaEventRecord(e, st);
  return e;
}

void prof_add(isd_ctx* c, int cls, cudaEvent_t a, cudaEvent_t b) {
  if (a && b) c->prof_recs.emplace_back(cls, a, b);
}

int tmap_for(isd_ctx* c, const void* base, int rows, int cols, int box_rows, CUtensorMap** out) {
  auto key = std::make_tuple(base, rows, cols, box_rows);
  auto it = c->act_maps.find(key);
  if (it == c->act_maps.end()) {
    CUtensorMap m;
    std::string err;
    if (!isd::make_tmap_bf16(&m, base, rows, cols, box_rows, &err))
      return fail(ISD_E_CUDA, "activation tensor map: " + err);
    it = c->act_maps.emplace(key, m).first;
  }
  *out = &it->second;
  return ISD_OK;
}

// single: one output slice (the SiLU epilogue, the LM head); such plans may
// run as stream-K when the tiles overfill one wave. Otherwise up to
// max_splits K-splits.
const GemmPlan& plan_for(isd_ctx* c, int m, int n, int k, bool single, int max_splits) {
  auto key = std::make_tuple(m, n, k, single ? 1 : max_splits);
  auto it = c->plans.find(key);
  if (it == c->plans.end()) {
    const GemmPlan p = single ? isd::plan_gemm(m, n, k, 0, 1, num_sms(), true)
                              : isd::plan_gemm(m, n, k, 0, max_splits, num_sms());
    it = c->plans.emplace(key, p).first;
  }
  return it->second;
}

// One projection: X [m][k] (bf16 workspace buffer) times W^T. kEpiF32
// writes `splits` partial slices of m x n floats, so the output must hold
// out_elems >= splits * m * n; max_splits = 1 asks for the plain product.
// A second operand pair for the last split of a split-K GEMM (the gated
// adapter's B with xa, see lora_xa): W2 [n][k2], X2 [m][k2].
struct AugSpec {
  const CUtensorMap* tw2;
  const __nv_bfloat16* x2;
  int k2;
};

// The residual add + RMSNorm that produces a GEMM's input (c->hn) from the
// previous projection's split-K slices, launched right before that GEMM.
// (Run as the GEMM's own prologue, behind a barrier over its grid, it cost
// more per step than the separate launch.)
struct PendingNorm {
  const float* part = nullptr;
  int splits = 0;
  const float* norm_w = nullptr;
};

int gemm(isd_ctx* c, int cls, const CUtensorMap& tw, const __nv_bfloat16* x, int m, int n, int k,
         isd::GemmEpilogue epi, float* out, size_t out_elems, int max_splits,
         __nv_bfloat16* act, int* splits_used, int32_t* status, cudaStream_t st,
         const AugSpec* aug = nullptr, const PendingNorm* pn = nullptr,
         float4* row_stats = nullptr) {
  if (epi == isd::kEpiF32 && out_elems > 0) {
    // large prefill chunks: no more splits than the partial buffer holds
    const size_t fit = out_elems / (static_cast<size_t>(m) * static_cast<size_t>(n));
    max_splits = static_cast<int>(std::max<size_t>(1, std::min<size_t>(max_splits, fit)));
  }
  const GemmPlan& plan =
      plan_for(c, m, n, k, epi != isd::kEpiF32 || max_splits == 1, std::min(max_splits, kLoraSplits));
  if (plan.n_pad == 0) return fail(ISD_E_UNSUPPORTED, "no GEMM plan");
  if (isd::gemm_streamk_workspace_bytes(plan) > c->sk_ws_bytes)
    return fail(ISD_E_UNSUPPORTED, "stream-K workspace too small for the GEMM plan");
  if (plan.splits > max_splits) return fail(ISD_E_UNSUPPORTED, "GEMM plan exceeds the split limit");
  if (epi == isd::kEpiF32 &&
      static_cast<size_t>(plan.splits) * static_cast<size_t>(m) * static_cast<size_t>(n) > out_elems)
    return fail(ISD_E_UNSUPPORTED, "GEMM output buffer too small for its split-K partials");
  CUtensorMap* tx = nullptr;
  int rc = tmap_for(c, x, m, k, plan.box_rows, &tx);
  if (rc) return rc;
  isd::GemmAugment ga{nullptr, nullptr, 0};
  if (aug) {
    CUtensorMap* tx2 = nullptr;
    rc = tmap_for(c, aug->x2, m, aug->k2, plan.box_rows, &tx2);
    if (rc) return rc;
    ga = isd::GemmAugment{aug->tw2, tx2, aug->k2};
  }
  if (pn) {
    const isd_model_cfg& g = c->cfg;
    cudaEvent_t r0 = prof_mark(c, st);
    ISD_CUDA(isd::launch_residual_norm(pn->part, pn->splits, m, g.hidden, pn->norm_w, g.rms_eps,
                                       c->x, c->hn, st));
    prof_add(c, kPResNorm, r0, prof_mark(c, st));
    c->launches += 1;
  }
  cudaEvent_t e0 = prof_mark(c, st);
  ISD_CUDA(isd::launch_gemm(tw, *tx, plan, m, n, k, epi, out, act, status, st, c->sk_ws,
                            c->sk_ws_bytes, aug ? &ga : nullptr, row_stats, c->pdl));
  prof_add(c, cls, e0, prof_mark(c, st));
  if (splits_used) *splits_used = plan.splits;
  c->launches += 1;
  return ISD_OK;
}

int check_shapes(const isd_model_cfg& c) {
  if (c.n_layers < 0 || c.hidden <= 0 || c.n_q_heads <= 0 || c.n_kv_heads <= 0 || c.vocab <= 0 ||
      c.intermediate <= 0 || c.max_rows <= 0 || c.max_batch <= 0 || c.max_position <= 0)
    return fail(ISD_E_INVALID, "model config has a non-positive size");
  if (c.head_dim != 64 && c.head_dim != 128)
    return fail(ISD_E_UNSUPPORTED, "head_dim must be 64 or 128");
  const int G = c.n_q_heads / c.n_kv_heads;
  if (c.n_q_heads % c.n_kv_heads || (G != 1 && G != 2 && G != 4 && G != 8))
    return fail(ISD_E_UNSUPPORTED, "n_q_heads / n_kv_heads must be 1, 2, 4 or 8");
  if (c.hidden % 128 || (c.n_q_heads * c.head_dim) % 128 || c.intermediate % 64 ||
      c.vocab % 128 || ((c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim) % 128)
    return fail(ISD_E_UNSUPPORTED, "hidden, q/kv widths and vocab must be multiples of 128, "
                                   "intermediate of 64");
  if (c.page_size != 16 && c.page_size != 32 && c.page_size != 64)
    return fail(ISD_E_UNSUPPORTED, "page_size must be 16, 32 or 64");
  if (c.max_rows > 4096) return fail(ISD_E_UNSUPPORTED, "max_rows above 4096");
  if (c.vocab > 64 * 8192) return fail(ISD_E_UNSUPPORTED, "vocab above 524288");
  if (c.max_batch > 1024) return fail(ISD_E_UNSUPPORTED, "max_batch above 1024");
  if (c.mask_token_id < 0 || c.mask_token_id >= c.vocab)
    return fail(ISD_E_INVALID, "mask_token_id outside the vocabulary");
  return ISD_OK;
}

int check_kv(const isd_ctx* c, const isd_kv* kv, int batch) {
  if (!kv || !kv->k_pool_dev || !kv->v_pool_dev || !kv->page_table_dev)
    return fail(ISD_E_INVALID, "kv pools and page table are required");
  if (kv->num_pages <= 0 || kv->max_pages_per_req <= 0)
    return fail(ISD_E_INVALID, "num_pages and max_pages_per_req must be positive");
  if (static_cast<int64_t>(kv->max_pages_per_req) * c->cfg.page_size > c->cfg.max_position)
    return fail(ISD_E_INVALID, "max_pages_per_req * page_size exceeds max_position");
  const int64_t rows = static_cast<int64_t>(std::max(c->cfg.n_layers, 1)) * kv->num_pages *
                       c->cfg.n_kv_heads * c->cfg.page_size;
  if (rows >= (1LL << 31) - 1) return fail(ISD_E_UNSUPPORTED, "KV pool above 2^31 rows");
  if (batch > c->cfg.max_batch) return fail(ISD_E_INVALID, "batch above cfg.max_batch");
  return ISD_OK;
}

isd::AttnShape attn_shape(const isd_ctx* c, const isd_kv* kv, int batch, int rows_per_req) {
  isd::AttnShape s;
  s.batch = batch;
  s.rows_per_req = rows_per_req;
  s.n_q_heads = c->cfg.n_q_heads;
  s.n_kv_heads = c->cfg.n_kv_heads;
  s.head_dim = c->cfg.head_dim;
  s.page_size = c->cfg.page_size;
  s.num_pages = kv->num_pages;
  s.max_pages_per_req = kv->max_pages_per_req;
  s.n_layers = std::max(c->cfg.n_layers, 1);
  return s;
}

// xa = bf16(scale * x A^T) on MASK rows, 0 on the others, into c->lora_xa
// ([M][n_a]): split-K GEMM, fixed-order sum. Multiplied by B inside the base
// GEMM, it adds the gated delta on MASK rows and exact zeros on verify rows.
int lora_xa(isd_ctx* c, const CUtensorMap& ta, const __nv_bfloat16* x, int M, int in, int n_a,
            int32_t* status, cudaStream_t st) {
  int s = 1;
  // a thin product (1-3 tiles of 128 outputs): many K-splits keep the SMs busy
  int rc = gemm(c, kPOther, ta, x, M, n_a, in, isd::kEpiF32, c->lora_xa_part,
                static_cast<size_t>(kLoraSplits) *
                    std::min<size_t>(c->cfg.max_rows, static_cast<size_t>(c->cfg.max_batch) * 15) *
                    3 * c->lora_rank,
                kLoraSplits, nullptr, &s, status, st);
  if (rc) return rc;
  cudaEvent_t e0 = prof_mark(c, st);
  ISD_CUDA(isd::launch_sum_cast(c->lora_xa_part, s, M, n_a, c->meta_flags, c->lora_scale,
                                c->lora_xa, st));
  prof_add(c, kPOther, e0, prof_mark(c, st));
  c->launches += 1;
  return ISD_OK;
}

// The decoder layers over the rows described by the row metadata; leaves
// bf16(final RMSNorm(x)) in c->hn. attn_sub > 1 (prefill): the attention sees
// each request's rows_per_req rows as attn_sub consecutive sub-requests of
// rows_per_req / attn_sub rows that share the request's pages (attn_table:
// the page table with each row repeated attn_sub times); attention is
// read-only on the cache, so this is the same computation in query tiles the
// attention kernel holds.
// tail: the residual add + RMSNorm (final norm) after the last layer, left
// for the next GEMM (the LM head) to run; null when no GEMM follows.
int forward_layers(isd_ctx* c, const isd_kv* kv, int batch, int rows_per_req, int32_t* status,
                   cudaStream_t st, bool use_lora = false, int attn_sub = 1,
                   const int32_t* attn_table = nullptr, PendingNorm* tail = nullptr) {
  const isd_model_cfg& g = c->cfg;
  const int M = batch * rows_per_req;
  const int H = g.hidden;
  isd::RowMeta meta{c->meta_tok, c->meta_pos, c->meta_flags};
  cudaEvent_t e0 = prof_mark(c, st);
  ISD_CUDA(isd::launch_embed_norm(static_cast<const __nv_bfloat16*>(c->embed),
                                  g.n_layers > 0 ? c->attn_norm[0] : c->final_norm, meta, M, H,
                                  g.vocab, g.rms_eps, c->x, c->hn, status, st));
  prof_add(c, kPEmbed, e0, prof_mark(c, st));
  c->launches += 1;
  if (g.n_layers == 0) return ISD_OK;
  CUtensorMap kmap, vmap;
  std::string err;
  const uint64_t pool_rows =
      static_cast<uint64_t>(g.n_layers) * kv->num_pages * g.n_kv_heads * g.page_size;
  if (!isd::make_tmap_bf16(&kmap, kv->k_pool_dev, pool_rows, g.head_dim, g.page_size, &err) ||
      !isd::make_tmap_bf16(&vmap, kv->v_pool_dev, pool_rows, g.head_dim, g.page_size, &err))
    return fail(ISD_E_INVALID, "KV pool tensor map: " + err);
  if (attn_sub < 1 || rows_per_req % attn_sub || (attn_sub > 1 && attn_table == nullptr))
    return fail(ISD_E_INVALID, "attention sub-requests must split the rows evenly");
  const isd::AttnShape ash = attn_shape(c, kv, batch * attn_sub, rows_per_req / attn_sub);
  const int32_t* ash_table = attn_sub > 1 ? attn_table : kv->page_table_dev;
  if (isd::attention_workspace_bytes(ash) > c->attn_ws_bytes)
    return fail(ISD_E_UNSUPPORTED, "attention workspace too small for this batch shape");

  PendingNorm pending;            // layer l's input norm, from layer l - 1's down slices
  bool have_pending = false;
  for (int l = 0; l < g.n_layers; ++l) {
    int s = 1;
    int rc = ISD_OK;
    const int r = c->lora_rank;
    const isd_ctx::LoraLayer* ll = use_lora ? &c->lora[l] : nullptr;
    // gated adapter on q/k/v: xa first, then B rides on the base GEMM's last split
    AugSpec aug_qkv{ll ? &ll->tb_qkv : nullptr, c->lora_xa, 3 * r};
    if (ll) {
      if (have_pending) {
        // the adapter's x A^T reads the normalised input first
        cudaEvent_t r0 = prof_mark(c, st);
        ISD_CUDA(isd::launch_residual_norm(pending.part, pending.splits, M, H, pending.norm_w,
                                           g.rms_eps, c->x, c->hn, st));
        prof_add(c, kPResNorm, r0, prof_mark(c, st));
        c->launches += 1;
        have_pending = false;
      }
      rc = lora_xa(c, ll->ta_qkv, c->hn, M, H, 3 * r, status, st);
      if (rc) return rc;
    }
    rc = gemm(c, kPGemmQkv, c->tm_qkv[l], c->hn, M, c->qkv_dim, H, isd::kEpiF32, c->part,
              c->part_elems, c->max_splits, nullptr, &s, status, st, ll ? &aug_qkv : nullptr,
              have_pending ? &pending : nullptr);
    if (rc) return rc;
    isd::QkvReduceArgs qa;
    qa.part = c->part;
    qa.splits = s;
    qa.rows = M;
    qa.rows_per_req = rows_per_req;
    qa.n_q = g.n_q_heads;
    qa.n_kv = g.n_kv_heads;
    qa.head_dim = g.head_dim;
    qa.q_norm = c->q_norm[l];
    qa.k_norm = c->k_norm[l];
    qa.eps = g.rms_eps;
    qa.rope = c->rope;
    qa.max_position = g.max_position;
    qa.meta = meta;
    qa.page_table = kv->page_table_dev;
    qa.max_pages_per_req = kv->max_pages_per_req;
    qa.page_size = g.page_size;
    qa.num_pages = kv->num_pages;
    qa.layer = l;
    qa.k_pool = static_cast<__nv_bfloat16*>(kv->k_pool_dev);
    qa.v_pool = static_cast<__nv_bfloat16*>(kv->v_pool_dev);
    qa.q_out = c->qbuf;
    qa.status = status;
    // the QKV reduction, then the attention (both in launch_attention)
    cudaEvent_t a1 = prof_mark(c, st);
    cudaEvent_t amid = prof_event(c);
    ISD_CUDA(isd::launch_attention(kmap, vmap, ash, l, c->qbuf, c->meta_pos, ash_table,
                                   c->attn, c->attn_ws, status, st, &c->launches, amid, &qa,
                                   attn_sub == 1 && ash_table == kv->page_table_dev &&
                                                        rows_per_req == ash.rows_per_req,
                                   c->pdl));
    cudaEvent_t a2 = prof_mark(c, st);
    prof_add(c, kPAttnSplit, a1, amid);
    prof_add(c, kPAttnCombine, amid, a2);
    AugSpec aug_o{ll ? &ll->tb_o : nullptr, c->lora_xa, r};
    if (ll) {
      rc = lora_xa(c, ll->ta_o, c->attn, M, c->q_dim, r, status, st);
      if (rc) return rc;
    }
    rc = gemm(c, kPGemmO, c->tm_o[l], c->attn, M, H, c->q_dim, isd::kEpiF32, c->part, c->part_elems,
              c->max_splits, nullptr, &s, status, st, ll ? &aug_o : nullptr);
    if (rc) return rc;
    // the MLP's input norm, launched before the gate/up GEMM
    PendingNorm mlp_in{c->part, s, c->mlp_norm[l]};
    if (ll) {
      cudaEvent_t r0 = prof_mark(c, st);
      ISD_CUDA(isd::launch_residual_norm(c->part, s, M, H, c->mlp_norm[l], g.rms_eps, c->x, c->hn, st));
      prof_add(c, kPResNorm, r0, prof_mark(c, st));
      c->launches += 1;
    }
    // gate/up with the fused SiLU epilogue; with the adapter, its (xa, B)
    // K-blocks follow each tile's base K-blocks (stream-K cuts unchanged)
    AugSpec aug_gu{ll ? &ll->tb_gu : nullptr, c->lora_xa, 2 * r};
    if (ll) {
      rc = lora_xa(c, ll->ta_gu, c->hn, M, H, 2 * r, status, st);
      if (rc) return rc;
    }
    rc = gemm(c, kPGemmGateUp, c->tm_gu[l], c->hn, M, 2 * g.intermediate, H, isd::kEpiSiluMul,
              nullptr, 0, 1, c->act, nullptr, status, st, ll ? &aug_gu : nullptr,
              ll ? nullptr : &mlp_in);
    if (rc) return rc;
    AugSpec aug_d{ll ? &ll->tb_d : nullptr, c->lora_xa, r};
    if (ll) {
      rc = lora_xa(c, ll->ta_d, c->act, M, g.intermediate, r, status, st);
      if (rc) return rc;
    }
    rc = gemm(c, kPGemmDown, c->tm_down[l], c->act, M, H, g.intermediate, isd::kEpiF32, c->part,
              c->part_elems, c->max_splits, nullptr, &s, status, st, ll ? &aug_d : nullptr);
    if (rc) return rc;
    // the next layer's input norm (the final norm after the last layer),
    // launched before the next GEMM
    pending = PendingNorm{c->part, s, l + 1 < g.n_layers ? c->attn_norm[l + 1] : c->final_norm};
    have_pending = true;
  }
  if (have_pending) {
    if (tail) {
      *tail = pending;
    } else {
      cudaEvent_t r1 = prof_mark(c, st);
      ISD_CUDA(isd::launch_residual_norm(pending.part, pending.splits, M, H, pending.norm_w,
                                         g.rms_eps, c->x, c->hn, st));
      prof_add(c, kPResNorm, r1, prof_mark(c, st));
      c->launches += 1;
    }
  } else if (tail) {
    tail->part = nullptr;
  }
  return ISD_OK;
}

int alloc_workspace(isd_ctx* c) {
  const isd_model_cfg& g = c->cfg;
  const size_t R = g.max_rows;
  const size_t wide = std::max(c->qkv_dim, g.hidden);
  // a step has at most batch x (2N - 1) <= max_batch x 15 rows; only steps
  // need logits and many K-splits, prefill chunks may use all max_rows
  const size_t step_rows = std::min(R, static_cast<size_t>(g.max_batch) * 15);
  const size_t part_rows = std::max(static_cast<size_t>(c->max_splits) * step_rows, R);
  const int G = g.n_q_heads / g.n_kv_heads;
  const int att_rows = std::max(1, 64 / G);   // rows per request in one attention query tile
  c->prefill_sub_max = static_cast<int>(std::max<size_t>(
      1, std::min<size_t>(G, R / (static_cast<size_t>(g.max_batch) * att_rows))));
  const size_t max_pages = (g.max_position + g.page_size - 1) / g.page_size;
  // attention workspace: the largest query tile (64 rows) at max_batch, longest requests
  isd::AttnShape a;
  a.batch = g.max_batch;
  a.rows_per_req = 64 / (g.n_q_heads / g.n_kv_heads);
  a.n_q_heads = g.n_q_heads;
  a.n_kv_heads = g.n_kv_heads;
  a.head_dim = g.head_dim;
  a.page_size = g.page_size;
  a.num_pages = 1;
  a.max_pages_per_req = (g.max_position + g.page_size - 1) / g.page_size;
  a.n_layers = 1;
  c->attn_ws_bytes = isd::attention_workspace_bytes(a);
  // decode blocks of up to 32 query rows per KV head take the tcgen05 path,
  // whose work split differs: size for both
  isd::AttnShape a_dec = a;
  a_dec.rows_per_req = std::max(1, 32 / (g.n_q_heads / g.n_kv_heads));
  c->attn_ws_bytes = std::max(c->attn_ws_bytes, isd::attention_workspace_bytes(a_dec));
  // prefill chunks: up to prefill_sub_max query tiles per request
  isd::AttnShape a_pre = a;
  a_pre.batch = g.max_batch * c->prefill_sub_max;
  c->attn_ws_bytes = std::max(c->attn_ws_bytes, isd::attention_workspace_bytes(a_pre));
  const int maxN = 8;
  c->acc_ws_bytes = isd::accept_workspace_bytes(g.max_batch, maxN, g.vocab);
  // stream-K: one slot per SM of fp32 partials of up to 512 tokens x 128 rows
  c->sk_ws_bytes = isd::gemm_streamk_sync_bytes() +
                   static_cast<size_t>(num_sms()) * 512 * 128 * sizeof(float);
  size_t sizes[] = {
      R * g.hidden * sizeof(float),                       // x
      R * g.hidden * 2,                                   // hn
      part_rows * wide * sizeof(float),                   // part
      R * c->q_dim * 2,                                   // qbuf
      R * c->q_dim * 2,                                   // attn
      R * g.intermediate * 2,                             // act
      step_rows * static_cast<size_t>(g.vocab) * sizeof(float),  // logits
      R * 4, R * 4, R * 4,                                // meta
      static_cast<size_t>(g.max_position) * (g.head_dim / 2) * sizeof(float2),  // rope
      c->attn_ws_bytes, c->acc_ws_bytes,
      static_cast<size_t>(g.max_batch) * 4,
      c->sk_ws_bytes,
      static_cast<size_t>(g.max_batch) * c->prefill_sub_max * max_pages * 4,   // prefill table
      static_cast<size_t>(g.max_batch) * 4,                                    // prefill order
      static_cast<size_t>(g.max_batch) * max_pages * 4,                        // prefill page rows
      step_rows * static_cast<size_t>(g.vocab / 32) * sizeof(float4),          // slab statistics
  };
  size_t total = 0;
  std::vector<size_t> off;
  for (size_t s : sizes) {
    off.push_back(total);
    total += (s + 1023) & ~static_cast<size_t>(1023);
  }
  if (cudaMalloc(&c->ws, total) != cudaSuccess)
    return fail(ISD_E_NOMEM, "workspace allocation of " + std::to_string(total) + " bytes failed");
  char* b = static_cast<char*>(c->ws);
  int i = 0;
  c->x = reinterpret_cast<float*>(b + off[i++]);
  c->hn = reinterpret_cast<__nv_bfloat16*>(b + off[i++]);
  c->part = reinterpret_cast<float*>(b + off[i++]);
  c->part_elems = part_rows * wide;
  c->logit_rows = step_rows;
  c->qbuf = reinterpret_cast<__nv_bfloat16*>(b + off[i++]);
  c->attn = reinterpret_cast<__nv_bfloat16*>(b + off[i++]);
  c->act = reinterpret_cast<__nv_bfloat16*>(b + off[i++]);
  c->logits = reinterpret_cast<float*>(b + off[i++]);
  c->meta_tok = reinterpret_cast<int32_t*>(b + off[i++]);
  c->meta_pos = reinterpret_cast<int32_t*>(b + off[i++]);
  c->meta_flags = reinterpret_cast<int32_t*>(b + off[i++]);
  c->rope = reinterpret_cast<float2*>(b + off[i++]);
  c->attn_ws = b + off[i++];
  c->acc_ws = b + off[i++];
  c->prefill_lens = reinterpret_cast<int32_t*>(b + off[i++]);
  c->sk_ws = b + off[i++];
  c->prefill_table = reinterpret_cast<int32_t*>(b + off[i++]);
  c->prefill_order = reinterpret_cast<int32_t*>(b + off[i++]);
  c->prefill_ptab = reinterpret_cast<int32_t*>(b + off[i++]);
  c->slab_stats = reinterpret_cast<float4*>(b + off[i++]);
  if (cudaMemset(c->sk_ws, 0, isd::gemm_streamk_sync_bytes()) != cudaSuccess)
    return fail(ISD_E_CUDA, "GEMM synchronisation words clear failed");
  // RoPE table in double precision: angle = pos * theta^(-2i/d)
  const int half = g.head_dim / 2;
  std::vector<float2> tab(static_cast<size_t>(g.max_position) * half);
  for (int p = 0; p < g.max_position; ++p)
    for (int k = 0; k < half; ++k) {
      const double inv = std::pow(static_cast<double>(g.rope_theta), -2.0 * k / g.head_dim);
      const double ang = static_cast<double>(p) * inv;
      tab[static_cast<size_t>(p) * half + k] =
          make_float2(static_cast<float>(std::cos(ang)), static_cast<float>(std::sin(ang)));
    }
  ISD_CUDA(cudaMemcpy(c->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice));
  return ISD_OK;
}

}  // namespace

extern "C" {

const char* isd_last_error(void) { return g_err.c_str(); }

int isd_last_launch_count(const isd_ctx* ctx) { return ctx ? ctx->launches : 0; }

int isd_init(const isd_model_cfg* cfg, const isd_weights* w, isd_ctx** out) {
  if (!cfg || !out) return fail(ISD_E_INVALID, "cfg and out are required");
  *out = nullptr;
  int rc = check_shapes(*cfg);
  if (rc) return rc;
  std::string err;
  if (!load_encode(&err)) return fail(ISD_E_CUDA, err);
  isd_ctx* c = new isd_ctx();
  c->cfg = *cfg;
  c->q_dim = cfg->n_q_heads * cfg->head_dim;
  c->qkv_dim = (cfg->n_q_heads + 2 * cfg->n_kv_heads) * cfg->head_dim;
  const int L = cfg->n_layers;
  if (w) {
    if (!w->embed_dev || !w->lm_head_dev || !w->final_norm_dev ||
        (L > 0 && (!w->w_qkv || !w->w_o || !w->w_gate_up || !w->w_down || !w->attn_norm ||
                   !w->mlp_norm || !w->q_norm || !w->k_norm))) {
      delete c;
      return fail(ISD_E_INVALID, "missing weight pointer");
    }
    c->embed = w->embed_dev;
    c->lm_head = w->lm_head_dev;
    c->final_norm = w->final_norm_dev;
    for (int l = 0; l < L; ++l) {
      if (!w->w_qkv[l] || !w->w_o[l] || !w->w_gate_up[l] || !w->w_down[l] || !w->attn_norm[l] ||
          !w->mlp_norm[l] || !w->q_norm[l] || !w->k_norm[l]) {
        delete c;
        return fail(ISD_E_INVALID, "missing weight pointer in layer " + std::to_string(l));
      }
      c->w_qkv.push_back(w->w_qkv[l]);
      c->w_o.push_back(w->w_o[l]);
      c->w_gu.push_back(w->w_gate_up[l]);
      c->w_down.push_back(w->w_down[l]);
      c->attn_norm.push_back(w->attn_norm[l]);
      c->mlp_norm.push_back(w->mlp_norm[l]);
      c->q_norm.push_back(w->q_norm[l]);
      c->k_norm.push_back(w->k_norm[l]);
      CUtensorMap a, b, d, e;
      const int I = cfg->intermediate;
      if (!isd::make_tmap_bf16(&a, w->w_qkv[l], c->qkv_dim, cfg->hidden, 128, &err) ||
          !isd::make_tmap_bf16(&b, w->w_o[l], cfg->hidden, c->q_dim, 128, &err) ||
          !isd::make_tmap_bf16(&d, w->w_gate_up[l], 2 * I, cfg->hidden, 128, &err) ||
          !isd::make_tmap_bf16(&e, w->w_down[l], cfg->hidden, I, 128, &err)) {
        delete c;
        return fail(ISD_E_INVALID, "weight tensor map: " + err);
      }
      c->tm_qkv.push_back(a);
      c->tm_o.push_back(b);
      c->tm_gu.push_back(d);
      c->tm_down.push_back(e);
    }
    if (!isd::make_tmap_bf16(&c->tm_lm, w->lm_head_dev, cfg->vocab, cfg->hidden, 128, &err)) {
      delete c;
      return fail(ISD_E_INVALID, "lm_head tensor map: " + err);
    }
  }
  rc = alloc_workspace(c);
  if (rc) {
    if (c->ws) cudaFree(c->ws);
    delete c;
    return rc;
  }
  *out = c;
  return ISD_OK;
}

void isd_destroy(isd_ctx* ctx) {
  if (!ctx) return;
  for (cudaEvent_t e : ctx->prof_pool) cudaEventDestroy(e);
  if (ctx->lora_mem) cudaFree(ctx->lora_mem);
  if (ctx->ws) cudaFree(ctx->ws);
  delete ctx;
}

int isd_load_gated_lora(isd_ctx* ctx, const isd_lora* lora) {
  if (!ctx || !lora) return fail(ISD_E_INVALID, "ctx and lora are required");
  const isd_model_cfg& g = ctx->cfg;
  const int r = lora->rank, L = g.n_layers;
  if (r != 128) return fail(ISD_E_UNSUPPORTED, "gated LoRA rank must be 128");
  if (L < 1) return fail(ISD_E_INVALID, "the model has no layers");
  for (int t = 0; t < 7; ++t) {
    if (!lora->A[t] || !lora->B[t]) return fail(ISD_E_INVALID, "missing LoRA pointer array");
    for (int l = 0; l < L; ++l)
      if (!lora->A[t][l] || !lora->B[t][l]) return fail(ISD_E_INVALID, "missing LoRA weight");
  }
  const int H = g.hidden, I = g.intermediate, Q = ctx->q_dim, KV = g.n_kv_heads * g.head_dim;
  // packed per layer: A_qkv [3r][H], B_qkv [qkv][3r] (block diagonal), A_o [r][Q], B_o [H][r],
  // A_gu [2r][H], B_gu [2I][2r] (block diagonal, 16-row gate/up interleave), A_d [r][I], B_d [H][r]
  const size_t e_aqkv = 3ull * r * H, e_bqkv = 3ull * r * ctx->qkv_dim, e_ao = 1ull * r * Q,
               e_bo = 1ull * H * r, e_agu = 2ull * r * H, e_bgu = 2ull * I * 2 * r, e_ad = 1ull * r * I,
               e_bd = 1ull * H * r;
  const size_t per_layer = e_aqkv + e_bqkv + e_ao + e_bo + e_agu + e_bgu + e_ad + e_bd;
  const size_t R = g.max_rows;
  // x A^T split slices, xa (bf16); the adapter runs in steps only
  const size_t Rs = std::min(R, static_cast<size_t>(ctx->cfg.max_batch) * 15);
  const size_t ws_bytes = kLoraSplits * Rs * 3 * r * 4 + ((Rs * 3 * r * 2 + 255) / 256) * 256;
  if (ctx->lora_mem) {
    cudaFree(ctx->lora_mem);
    ctx->lora_mem = nullptr;
    ctx->has_lora = false;
  }
  char* mem = nullptr;
  const size_t w_bytes = per_layer * L * 2;
  if (cudaMalloc(&mem, w_bytes + ws_bytes + 4096) != cudaSuccess)
    return fail(ISD_E_NOMEM, "gated LoRA allocation failed");
  ctx->lora_mem = mem;
  ISD_CUDA(cudaMemset(mem, 0, w_bytes));   // block-diagonal zeros
  cudaStream_t st;
  ISD_CUDA(cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking));
  ctx->lora.assign(L, isd_ctx::LoraLayer{});
  auto bf = [](const void* p) { return static_cast<const __nv_bfloat16*>(p); };
  std::string err;
  __nv_bfloat16* cur = reinterpret_cast<__nv_bfloat16*>(mem);
  int rc = ISD_OK;
  for (int l = 0; l < L && rc == ISD_OK; ++l) {
    isd_ctx::LoraLayer& x = ctx->lora[l];
    x.a_qkv = cur; cur += e_aqkv;
    x.b_qkv = cur; cur += e_bqkv;
    x.a_o = cur; cur += e_ao;
    x.b_o = cur; cur += e_bo;
    x.a_gu = cur; cur += e_agu;
    x.b_gu = cur; cur += e_bgu;
    x.a_d = cur; cur += e_ad;
    x.b_d = cur; cur += e_bd;
    // targets: 0 q, 1 k, 2 v, 3 o, 4 gate, 5 up, 6 down
    cudaError_t e = cudaSuccess;
    auto chk = [&](cudaError_t v) { if (e == cudaSuccess) e = v; };
    chk(isd::launch_pack_rows(bf(lora->A[0][l]), r, H, x.a_qkv, H, 0, 0, -1, st));
    chk(isd::launch_pack_rows(bf(lora->A[1][l]), r, H, x.a_qkv, H, r, 0, -1, st));
    chk(isd::launch_pack_rows(bf(lora->A[2][l]), r, H, x.a_qkv, H, 2 * r, 0, -1, st));
    chk(isd::launch_pack_rows(bf(lora->B[0][l]), Q, r, x.b_qkv, 3 * r, 0, 0, -1, st));
    chk(isd::launch_pack_rows(bf(lora->B[1][l]), KV, r, x.b_qkv, 3 * r, Q, r, -1, st));
    chk(isd::launch_pack_rows(bf(lora->B[2][l]), KV, r, x.b_qkv, 3 * r, Q + KV, 2 * r, -1, st));
    chk(isd::launch_pack_rows(bf(lora->A[3][l]), r, Q, x.a_o, Q, 0, 0, -1, st));
    chk(isd::launch_pack_rows(bf(lora->B[3][l]), H, r, x.b_o, r, 0, 0, -1, st));
    chk(isd::launch_pack_rows(bf(lora->A[4][l]), r, H, x.a_gu, H, 0, 0, -1, st));
    chk(isd::launch_pack_rows(bf(lora->A[5][l]), r, H, x.a_gu, H, r, 0, -1, st));
    chk(isd::launch_pack_rows(bf(lora->B[4][l]), I, r, x.b_gu, 2 * r, 0, 0, 0, st));
    chk(isd::launch_pack_rows(bf(lora->B[5][l]), I, r, x.b_gu, 2 * r, 0, r, 16, st));
    chk(isd::launch_pack_rows(bf(lora->A[6][l]), r, I, x.a_d, I, 0, 0, -1, st));
    chk(isd::launch_pack_rows(bf(lora->B[6][l]), H, r, x.b_d, r, 0, 0, -1, st));
    if (e != cudaSuccess) {
      rc = fail(ISD_E_CUDA, std::string("LoRA packing: ") + cudaGetErrorString(e));
      break;
    }
    if (!isd::make_tmap_bf16(&x.ta_qkv, x.a_qkv, 3 * r, H, 128, &err) ||
        !isd::make_tmap_bf16(&x.tb_qkv, x.b_qkv, ctx->qkv_dim, 3 * r, 128, &err) ||
        !isd::make_tmap_bf16(&x.ta_o, x.a_o, r, Q, 128, &err) ||
        !isd::make_tmap_bf16(&x.tb_o, x.b_o, H, r, 128, &err) ||
        !isd::make_tmap_bf16(&x.ta_gu, x.a_gu, 2 * r, H, 128, &err) ||
        !isd::make_tmap_bf16(&x.tb_gu, x.b_gu, 2 * I, 2 * r, 128, &err) ||
        !isd::make_tmap_bf16(&x.ta_d, x.a_d, r, I, 128, &err) ||
        !isd::make_tmap_bf16(&x.tb_d, x.b_d, H, r, 128, &err))
      rc = fail(ISD_E_INVALID, "LoRA tensor map: " + err);
  }
  const cudaError_t se = cudaStreamSynchronize(st);
  cudaStreamDestroy(st);
  if (rc == ISD_OK && se != cudaSuccess) rc = fail(ISD_E_CUDA, cudaGetErrorString(se));
  if (rc != ISD_OK) {
    cudaFree(ctx->lora_mem);
    ctx->lora_mem = nullptr;
    ctx->lora.clear();
    return rc;
  }
  char* w = mem + ((w_bytes + 1023) & ~static_cast<size_t>(1023));
  ctx->lora_xa_part = reinterpret_cast<float*>(w);
  w += kLoraSplits * Rs * 3 * r * 4;
  ctx->lora_xa = reinterpret_cast<__nv_bfloat16*>(w);
  ctx->lora_rank = r;
  ctx->lora_scale = lora->scale;
  ctx->has_lora = true;
  return ISD_OK;
}

int isd_step(isd_ctx* ctx, const isd_batch* batch, const isd_kv* kv, int32_t* pending_dev,
             float* q_cache_dev, const float* uniforms_dev, int32_t* out_accepted_dev,
             int32_t* out_committed_dev, int32_t* status_dev, void* stream) {
  if (!ctx || !batch || !pending_dev || !uniforms_dev || !out_accepted_dev || !status_dev)
    return fail(ISD_E_INVALID, "null argument");
  if (!ctx->embed) return fail(ISD_E_INVALID, "context has no model weights");
  const isd_model_cfg& g = ctx->cfg;
  const int B = batch->batch, N = batch->stride_n;
  if (B < 1 || B > 1024) return fail(ISD_E_INVALID, "batch must be in [1, 1024]");
  if (N < 1 || N > 8) return fail(ISD_E_INVALID, "stride_n must be in [1, 8]");
  if (!batch->seq_len_dev || !batch->n_draft_dev)
    return fail(ISD_E_INVALID, "seq_len and n_draft are required");
  if (batch->flags & ~(ISD_PROPOSE_SAMPLE | ISD_VERIFY_GREEDY | ISD_USE_LORA))
    return fail(ISD_E_INVALID, "unknown flag bits");
  const bool use_lora = (batch->flags & ISD_USE_LORA) != 0;
  if (use_lora && !ctx->has_lora) return fail(ISD_E_INVALID, "ISD_USE_LORA without a loaded gated LoRA");
  if ((batch->flags & ISD_PROPOSE_SAMPLE) && N > 1 && !q_cache_dev)
    return fail(ISD_E_INVALID, "SAMPLE proposals need q_cache");
  const int R = 2 * N - 1;
  if (B * R > g.max_rows) return fail(ISD_E_INVALID, "batch * (2N-1) exceeds cfg.max_rows");
  if (R * (g.n_q_heads / g.n_kv_heads) > 64)
    return fail(ISD_E_UNSUPPORTED, "(2N-1) * (n_q_heads/n_kv_heads) above 64");
  int rc = check_kv(ctx, kv, B);
  if (rc) return rc;
  if (!kv->free_list_dev || !kv->free_head_dev) return fail(ISD_E_INVALID, "free list is required");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ctx->launches = 0;
  isd::RowMeta meta{ctx->meta_tok, ctx->meta_pos, ctx->meta_flags};
  cudaEvent_t e0 = prof_mark(ctx, st);
  ISD_CUDA(isd::launch_assemble_step(pending_dev, batch->n_draft_dev, batch->seq_len_dev, B, N,
                                     g.mask_token_id, meta, status_dev, st));
  prof_add(ctx, kPAssemble, e0, prof_mark(ctx, st));
  ctx->launches += 1;
  PendingNorm tail;
  rc = forward_layers(ctx, kv, B, R, status_dev, st, use_lora, 1, nullptr, &tail);
  if (rc) return rc;
  const int M = B * R;
  if (!batch->logits_out_dev && static_cast<size_t>(M) > ctx->logit_rows)
    return fail(ISD_E_UNSUPPORTED, "more block rows than the logits workspace holds");
  float* logits = batch->logits_out_dev ? batch->logits_out_dev : ctx->logits;
  // the LM head writes the logits themselves: never split-K; the final norm
  // is launched before it. Its epilogue also writes the max, sum of exp and
  // first argmax of every 32 logits, which the accept step merges instead
  // of reading the logits once more.
  float4* slab = static_cast<size_t>(M) <= ctx->logit_rows ? ctx->slab_stats : nullptr;
  rc = gemm(ctx, kPGemmLmHead, ctx->tm_lm, ctx->hn, M, g.vocab, g.hidden, isd::kEpiF32, logits,
            static_cast<size_t>(M) * g.vocab, 1, nullptr, nullptr, status_dev, st, nullptr,
            tail.part ? &tail : nullptr, slab);
  if (rc) return rc;
  isd::AcceptArgs a;
  a.logits = logits;
  a.batch = B;
  a.stride_n = N;
  a.vocab = g.vocab;
  a.flags = batch->flags;
  a.page_size = g.page_size;
  a.pending = pending_dev;
  a.n_draft = batch->n_draft_dev;
  a.seq_len = batch->seq_len_dev;
  a.q_cache = q_cache_dev;
  a.uniforms = uniforms_dev;
  a.accepted = out_accepted_dev;
  a.committed = out_committed_dev;
  a.page_table = kv->page_table_dev;
  a.free_list = kv->free_list_dev;
  a.free_head = kv->free_head_dev;
  a.num_pages = kv->num_pages;
  a.max_pages_per_req = kv->max_pages_per_req;
  a.free_count = kv->free_count;
  a.status = status_dev;
  a.slab_stats = slab;
  cudaEvent_t c0 = prof_mark(ctx, st);
  cudaEvent_t c1 = prof_event(ctx), c2 = prof_event(ctx);
  ISD_CUDA(isd::launch_accept(a, ctx->acc_ws, st, &ctx->launches, c1, c2));
  cudaEvent_t c3 = prof_mark(ctx, st);
  prof_add(ctx, kPAcceptStats, c0, c1);
  prof_add(ctx, kPAcceptDecide, c1, c2);
  prof_add(ctx, kPBookkeep, c2, c3);
  return ISD_OK;
}

int isd_profile_enable(isd_ctx* ctx, int enable) {
  if (!ctx) return fail(ISD_E_INVALID, "ctx is required");
  ctx->prof_on = enable != 0;
  ctx->prof_next = 0;
  ctx->prof_recs.clear();
  return ISD_OK;
}

int isd_profile_read(isd_ctx* ctx, double* total_ms, int32_t* counts) {
  if (!ctx || !total_ms || !counts) return fail(ISD_E_INVALID, "null argument");
  for (int i = 0; i < ISD_PROF_CLASSES; ++i) {
    total_ms[i] = 0.0;
    counts[i] = 0;
  }
  if (!ctx->prof_recs.empty()) {
    ISD_CUDA(cudaEventSynchronize(std::get<2>(ctx->prof_recs.back())));
    for (auto& r : ctx->prof_recs) {
      float ms = 0.f;
      ISD_CUDA(cudaEventElapsedTime(&ms, std::get<1>(r), std::get<2>(r)));
      total_ms[std::get<0>(r)] += ms;
      counts[std::get<0>(r)] += 1;
    }
  }
  ctx->prof_recs.clear();
  ctx->prof_next = 0;
  return ISD_OK;
}

const char* isd_profile_class_name(int cls) {
  return (cls >= 0 && cls < ISD_PROF_CLASSES) ? kProfNames[cls] : "";
}

int isd_prefill(isd_ctx* ctx, const isd_kv* kv, const int32_t* tokens_dev, int32_t max_len,
                const int32_t* lens_host, int32_t batch, int32_t stride_n, int32_t* seq_len_dev,
                int32_t* n_draft_dev, int32_t* pending_dev, int32_t* status_dev, void* stream) {
  if (!ctx || !tokens_dev || !lens_host || !seq_len_dev || !n_draft_dev || !pending_dev ||
      !status_dev)
    return fail(ISD_E_INVALID, "null argument");
  if (!ctx->embed) return fail(ISD_E_INVALID, "context has no model weights");
  if (batch < 1 || batch > ctx->cfg.max_batch) return fail(ISD_E_INVALID, "batch out of range");
  if (stride_n < 1 || stride_n > 8) return fail(ISD_E_INVALID, "stride_n must be in [1, 8]");
  int longest = 0;
  for (int b = 0; b < batch; ++b) {
    if (lens_host[b] < 1 || lens_host[b] > max_len)
      return fail(ISD_E_INVALID, "prompt length outside [1, max_len]");
    longest = std::max(longest, lens_host[b]);
  }
  int rc = check_kv(ctx, kv, batch);
  if (rc) return rc;
  const isd_model_cfg& g = ctx->cfg;
  const int G = g.n_q_heads / g.n_kv_heads;
  // rows per request and pass: up to prefill_sub_max attention query tiles
  // (each 64 / G rows of one request), as far as max_rows allows
  const int att_rows = std::max(1, 64 / G);
  int chunk = std::max(1, std::min(att_rows * ctx->prefill_sub_max, g.max_rows / batch));
  int sub = 1;
  if (chunk > att_rows) {
    sub = chunk / att_rows;
    chunk = sub * att_rows;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ctx->launches = 0;
  // requests by descending prompt length: the requests a pass still has rows
  // for are then a prefix of this order, and a pass runs only those
  std::vector<int32_t> order(batch);
  for (int b = 0; b < batch; ++b) order[b] = b;
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int b) { return lens_host[a] > lens_host[b]; });
  ISD_CUDA(cudaMemcpyAsync(ctx->prefill_lens, lens_host, sizeof(int32_t) * batch,
                           cudaMemcpyHostToDevice, st));
  ISD_CUDA(cudaMemcpyAsync(ctx->prefill_order, order.data(), sizeof(int32_t) * batch,
                           cudaMemcpyHostToDevice, st));
  // the page table in that order, and again with every row repeated once per
  // attention sub-request
  ISD_CUDA(isd::launch_gather_rows(kv->page_table_dev, ctx->prefill_order, batch,
                                   kv->max_pages_per_req, 1, ctx->prefill_ptab, st));
  ISD_CUDA(isd::launch_gather_rows(kv->page_table_dev, ctx->prefill_order, batch,
                                   kv->max_pages_per_req, sub, ctx->prefill_table, st));
  ctx->launches += 2;
  isd_kv kv_sorted = *kv;
  kv_sorted.page_table_dev = ctx->prefill_ptab;
  isd::RowMeta meta{ctx->meta_tok, ctx->meta_pos, ctx->meta_flags};
  int active = batch;
  for (int start = 0; start < longest - 1; start += chunk) {
    while (active > 0 && lens_host[order[active - 1]] - 1 <= start) --active;
    ISD_CUDA(isd::launch_assemble_prefill(tokens_dev, max_len, ctx->prefill_lens, ctx->prefill_order,
                                          active, chunk, start, meta, st));
    ctx->launches += 1;
    rc = forward_layers(ctx, &kv_sorted, active, chunk, status_dev, st, false, sub,
                        ctx->prefill_table);
    if (rc) return rc;
  }
  // starting state: L = len - 1, x* = last prompt token, no drafts
  std::vector<int32_t> L(batch), nd(batch, 0);
  for (int b = 0; b < batch; ++b) L[b] = lens_host[b] - 1;
  ISD_CUDA(cudaMemcpyAsync(seq_len_dev, L.data(), sizeof(int32_t) * batch, cudaMemcpyHostToDevice, st));
  ISD_CUDA(cudaMemcpyAsync(n_draft_dev, nd.data(), sizeof(int32_t) * batch, cudaMemcpyHostToDevice, st));
  for (int b = 0; b < batch; ++b)
    ISD_CUDA(cudaMemcpyAsync(pending_dev + static_cast<int64_t>(b) * stride_n,
                             tokens_dev + static_cast<int64_t>(b) * max_len + lens_host[b] - 1,
                             sizeof(int32_t), cudaMemcpyDeviceToDevice, st));
  // the host vectors above must outlive the copies
  ISD_CUDA(cudaStreamSynchronize(st));
  return ISD_OK;
}

int isd_gemm_bf16(const void* w_dev, const void* x_dev, float* y_dev, int32_t m, int32_t n,
                  int32_t k, int32_t split_k, int32_t* status_dev, void* stream) {
  if (!w_dev || !x_dev || !y_dev) return fail(ISD_E_INVALID, "null argument");
  if (m < 1 || m > 4096 || n < 128 || n % 128 || k < 64 || k % 64 || split_k < 1 || split_k > 16 ||
      split_k > k / 64)
    return fail(ISD_E_UNSUPPORTED, "need 1<=m<=4096, n%128==0, k%64==0, 1<=split_k<=min(16,k/64)");
  GemmPlan plan = isd::plan_gemm(m, n, k, split_k, split_k, num_sms());
  if (plan.n_pad == 0 || plan.splits != split_k)
    return fail(ISD_E_UNSUPPORTED, "split_k leaves an empty split");
  std::string err;
  CUtensorMap tw, tx;
  if (!isd::make_tmap_bf16(&tw, w_dev, n, k, 128, &err) ||
      !isd::make_tmap_bf16(&tx, x_dev, m, k, plan.box_rows, &err))
    return fail(ISD_E_INVALID, "tensor map: " + err);
  ISD_CUDA(isd::launch_gemm(tw, tx, plan, m, n, k, isd::kEpiF32, y_dev, nullptr, status_dev,
                            static_cast<cudaStream_t>(stream)));
  return ISD_OK;
}

int isd_gemm_plan(int32_t m, int32_t n, int32_t k, int32_t single, int32_t max_splits,
                  int32_t num_sms_hint, int32_t* out) {
  if (!out) return fail(ISD_E_INVALID, "null argument");
  if (m < 1 || max_splits < 1 || num_sms_hint < 1)
    return fail(ISD_E_INVALID, "need m >= 1, max_splits >= 1, sms >= 1");
  if (n < 128 || n % 128 || k < 64 || k % 64)
    return fail(ISD_E_UNSUPPORTED, "need n % 128 == 0 and k % 64 == 0");
  const GemmPlan p = single ? isd::plan_gemm(m, n, k, 0, 1, num_sms_hint, true)
                            : isd::plan_gemm(m, n, k, 0, max_splits, num_sms_hint);
  const int32_t v[ISD_GEMM_PLAN_FIELDS] = {p.n_pad,  p.n_chunks, p.splits,  p.kb_per_split,
                                           p.n_mma,  p.mma_n,    p.box_rows, p.n_boxes,
                                           p.stages, p.pair,     p.streamk, p.units,
                                           static_cast<int32_t>(p.tmem_cols),
                                           static_cast<int32_t>(p.smem_bytes)};
  for (int i = 0; i < ISD_GEMM_PLAN_FIELDS; ++i) out[i] = v[i];
  return p.n_pad > 0 ? ISD_OK : fail(ISD_E_UNSUPPORTED, "no GEMM plan");
}

int isd_attention_split(int32_t batch, int32_t rows_per_req, int32_t n_q_heads,
                        int32_t n_kv_heads, int32_t head_dim, int32_t max_pages_per_req,
                        int32_t page_size, const int32_t* kend_host, int32_t num_sms,
                        int32_t* seg_out, int32_t seg_capacity, int32_t* n_segments,
                        int32_t* max_parts) {
  if (!kend_host || !n_segments || !max_parts || (seg_capacity > 0 && !seg_out))
    return fail(ISD_E_INVALID, "null argument");
  if (batch < 1 || batch > 1024 || rows_per_req < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads ||
      head_dim < 1 || max_pages_per_req < 1 || page_size < 1 || num_sms < 1 || seg_capacity < 0)
    return fail(ISD_E_INVALID, "bad shape");
  isd::AttnShape s{batch, rows_per_req, n_q_heads, n_kv_heads, head_dim, page_size, 1,
                   max_pages_per_req, 1};
  int n = 0, mp = 0;
  const int rc = isd::attention_split(s, kend_host, num_sms, seg_out, seg_capacity, &n, &mp);
  if (rc == -1) return fail(ISD_E_UNSUPPORTED, "shape not served by the tcgen05 attention kernel");
  *n_segments = n;
  *max_parts = mp;
  return rc == 0 ? ISD_OK : fail(ISD_E_INVALID, "seg_capacity too small");
}

size_t isd_gemm_workspace_bytes(int32_t m, int32_t n, int32_t k) {
  if (m < 1 || m > 4096 || n < 128 || n % 128 || k < 64 || k % 64) return 0;
  return isd::gemm_streamk_workspace_bytes(isd::plan_gemm(m, n, k, 0, 1, num_sms(), true));
}

int isd_gemm_bf16_single(const void* w_dev, const void* x_dev, float* y_dev, int32_t m, int32_t n,
                         int32_t k, void* workspace_dev, size_t workspace_bytes,
                         int32_t* status_dev, void* stream) {
  if (!w_dev || !x_dev || !y_dev) return fail(ISD_E_INVALID, "null argument");
  if (m < 1 || m > 4096 || n < 128 || n % 128 || k < 64 || k % 64)
    return fail(ISD_E_UNSUPPORTED, "need 1<=m<=4096, n%128==0, k%64==0");
  GemmPlan plan = isd::plan_gemm(m, n, k, 0, 1, num_sms(), true);
  if (plan.n_pad == 0) return fail(ISD_E_UNSUPPORTED, "no GEMM plan");
  const size_t need = isd::gemm_streamk_workspace_bytes(plan);
  if (need > 0 && (workspace_dev == nullptr || workspace_bytes < need))
    return fail(ISD_E_INVALID, "workspace smaller than isd_gemm_workspace_bytes");
  std::string err;
  CUtensorMap tw, tx;
  if (!isd::make_tmap_bf16(&tw, w_dev, n, k, 128, &err) ||
      !isd::make_tmap_bf16(&tx, x_dev, m, k, plan.box_rows, &err))
    return fail(ISD_E_INVALID, "tensor map: " + err);
  ISD_CUDA(isd::launch_gemm(tw, tx, plan, m, n, k, isd::kEpiF32, y_dev, nullptr, status_dev,
                            static_cast<cudaStream_t>(stream), workspace_dev, workspace_bytes));
  return ISD_OK;
}

size_t isd_attention_workspace_bytes(int32_t batch, int32_t rows_per_req, int32_t n_q_heads,
                                     int32_t n_kv_heads, int32_t head_dim,
                                     int32_t max_pages_per_req, int32_t page_size) {
  isd::AttnShape s{batch, rows_per_req, n_q_heads, n_kv_heads, head_dim, page_size, 1,
                   max_pages_per_req, 1};
  return isd::attention_workspace_bytes(s);
}

int isd_paged_attention(const void* q_dev, const int32_t* row_pos_dev, const void* k_pool_dev,
                        const void* v_pool_dev, const int32_t* page_table_dev, int32_t batch,
                        int32_t rows_per_req, int32_t n_q_heads, int32_t n_kv_heads,
                        int32_t head_dim, int32_t page_size, int32_t num_pages,
                        int32_t max_pages_per_req, int32_t n_layers, int32_t layer, void* out_dev,
                        void* workspace_dev, size_t workspace_bytes, int32_t* status_dev,
                        void* stream) {
  if (!q_dev || !row_pos_dev || !k_pool_dev || !v_pool_dev || !page_table_dev || !out_dev ||
      !workspace_dev)
    return fail(ISD_E_INVALID, "null argument");
  if (head_dim != 64 && head_dim != 128) return fail(ISD_E_UNSUPPORTED, "head_dim must be 64 or 128");
  if (n_kv_heads <= 0 || n_q_heads % n_kv_heads) return fail(ISD_E_INVALID, "bad head counts");
  const int G = n_q_heads / n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(ISD_E_UNSUPPORTED, "group size");
  if (rows_per_req < 1 || rows_per_req * G > 64) return fail(ISD_E_UNSUPPORTED, "rows_per_req * G > 64");
  if (page_size != 16 && page_size != 32 && page_size != 64) return fail(ISD_E_UNSUPPORTED, "page size");
  if (batch < 1 || num_pages < 1 || max_pages_per_req < 1 || layer < 0 || layer >= n_layers)
    return fail(ISD_E_INVALID, "size out of range");
  isd::AttnShape s{batch, rows_per_req, n_q_heads, n_kv_heads, head_dim, page_size, num_pages,
                   max_pages_per_req, n_layers};
  if (isd::attention_workspace_bytes(s) > workspace_bytes) return fail(ISD_E_INVALID, "workspace too small");
  const uint64_t rows = static_cast<uint64_t>(n_layers) * num_pages * n_kv_heads * page_size;
  if (rows >= (1ULL << 31) - 1) return fail(ISD_E_UNSUPPORTED, "pool above 2^31 rows");
  std::string err;
  CUtensorMap km, vm;
  if (!isd::make_tmap_bf16(&km, k_pool_dev, rows, head_dim, page_size, &err) ||
      !isd::make_tmap_bf16(&vm, v_pool_dev, rows, head_dim, page_size, &err))
    return fail(ISD_E_INVALID, "tensor map: " + err);
  ISD_CUDA(isd::launch_attention(km, vm, s, layer, static_cast<const __nv_bfloat16*>(q_dev),
                                 row_pos_dev, page_table_dev, static_cast<__nv_bfloat16*>(out_dev),
                                 workspace_dev, status_dev, static_cast<cudaStream_t>(stream),
                                 nullptr));
  return ISD_OK;
}

int isd_set_wait_limit(long long cycles) {
  if (cycles != 0 && cycles < 1000) return fail(ISD_E_INVALID, "wait limit below 1000 cycles");
  const long long c = cycles == 0 ? 4000000000LL : cycles;
  ISD_CUDA(isd::set_wait_limit_gemm(c));
  ISD_CUDA(isd::set_wait_limit_attention(c));
  return ISD_OK;
}

size_t isd_accept_workspace_bytes(int32_t batch, int32_t stride_n, int32_t vocab) {
  return isd::accept_workspace_bytes(batch, stride_n, vocab);
}

int isd_accept_propose(const float* logits_dev, const isd_batch* batch, const isd_kv* kv,
                       int32_t page_size, int32_t vocab, int32_t* pending_dev, float* q_cache_dev,
                       const float* uniforms_dev, int32_t* out_accepted_dev,
                       int32_t* out_committed_dev, void* workspace_dev, size_t workspace_bytes,
                       int32_t* status_dev, void* stream) {
  if (!logits_dev || !batch || !kv || !pending_dev || !uniforms_dev || !out_accepted_dev ||
      !workspace_dev || !status_dev || !batch->seq_len_dev || !batch->n_draft_dev ||
      !kv->page_table_dev || !kv->free_list_dev || !kv->free_head_dev)
    return fail(ISD_E_INVALID, "null argument");
  const int B = batch->batch, N = batch->stride_n;
  if (B < 1 || B > 1024 || N < 1 || N > 8) return fail(ISD_E_INVALID, "batch or stride_n out of range");
  if (vocab < 4 || vocab % 4 || vocab > 64 * 8192) return fail(ISD_E_UNSUPPORTED, "vocab");
  if (page_size < 1) return fail(ISD_E_INVALID, "page_size");
  if ((batch->flags & ISD_PROPOSE_SAMPLE) && N > 1 && !q_cache_dev)
    return fail(ISD_E_INVALID, "SAMPLE proposals need q_cache");
  if (isd::accept_workspace_bytes(B, N, vocab) > workspace_bytes)
    return fail(ISD_E_INVALID, "workspace too small");
  isd::AcceptArgs a;
  a.logits = logits_dev;
  a.batch = B;
  a.stride_n = N;
  a.vocab = vocab;
  a.flags = batch->flags;
  a.page_size = page_size;
  a.pending = pending_dev;
  a.n_draft = batch->n_draft_dev;
  a.seq_len = batch->seq_len_dev;
  a.q_cache = q_cache_dev;
  a.uniforms = uniforms_dev;
  a.accepted = out_accepted_dev;
  a.committed = out_committed_dev;
  a.page_table = kv->page_table_dev;
  a.free_list = kv->free_list_dev;
  a.free_head = kv->free_head_dev;
  a.num_pages = kv->num_pages;
  a.max_pages_per_req = kv->max_pages_per_req;
  a.free_count = kv->free_count;
  a.status = status_dev;
  ISD_CUDA(isd::launch_accept(a, workspace_dev, static_cast<cudaStream_t>(stream), nullptr));
  return ISD_OK;
}

}  // extern "C"
