// One (row, head) of the QKV projection's split-K reduction (one warp per
// item in qkv_reduce_kernel): the splits summed in ascending order; for q and
// k heads RMSNorm over head_dim and NeoX rotary embedding (pairs (i, i +
// d/2)) at the row's absolute position; q to the attention input, k and v
// into the row's page slot. Lane l holds elements l + 32 j of the head.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace isd {

template <int HD>
__device__ __forceinline__ void qkv_head_sum(const QkvReduceArgs& a, int row, int hd, int lane,
                                             float (&v)[HD / 32]) {
  constexpr int J = HD / 32;
  const int qkv_dim = (a.n_q + 2 * a.n_kv) * HD;
  const int64_t split_stride = static_cast<int64_t>(a.rows) * qkv_dim;
  const float* pr = a.part + static_cast<int64_t>(row) * qkv_dim + hd * HD + lane;
#pragma unroll
  for (int j = 0; j < J; ++j) v[j] = 0.f;
  // unrolled to the most splits a projection uses, so every load is in flight
#pragma unroll
  for (int sp = 0; sp < 8; ++sp) {
    if (sp < a.splits) {
#pragma unroll
      for (int j = 0; j < J; ++j) v[j] += __ldcg(pr + sp * split_stride + 32 * j);
    }
  }
}

template <int HD>
__device__ __forceinline__ void qkv_head_finish(const QkvReduceArgs& a, int row, int hd, int lane,
                                                float (&v)[HD / 32]) {
  constexpr int J = HD / 32;       // values per lane
  constexpr int JH = J / 2;        // partner offset (d + HD/2)
  const int flags = a.meta.flags[row];
  int pos = a.meta.pos[row];
  const bool write_kv = (flags & kRowWriteKV) && pos >= 0;
  if (pos >= a.max_position) {
    if (lane == 0 && hd == 0) flag(a.status, ISD_DEV_BAD_STATE);
    pos = a.max_position - 1;
  }
  const int rpos = pos < 0 ? 0 : pos;
  if (hd < a.n_q + a.n_kv) {
    const float* nw = hd < a.n_q ? a.q_norm : a.k_norm;
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < J; ++j) ss += v[j] * v[j];
    ss = warp_sum(ss);
    const float rstd = rsqrtf(ss / HD + a.eps);
#pragma unroll
    for (int j = 0; j < J; ++j) v[j] *= rstd * nw[lane + 32 * j];
    const float2* cs = a.rope + static_cast<int64_t>(rpos) * (HD / 2);
#pragma unroll
    for (int j = 0; j < JH; ++j) {
      const float2 c = cs[lane + 32 * j];
      const float x1 = v[j], x2 = v[j + JH];
      v[j] = x1 * c.x - x2 * c.y;
      v[j + JH] = x2 * c.x + x1 * c.y;
    }
  }
  if (hd < a.n_q) {
    __nv_bfloat16* qo = a.q_out + (static_cast<int64_t>(row) * a.n_q + hd) * HD;
#pragma unroll
    for (int j = 0; j < J; ++j) qo[lane + 32 * j] = __float2bfloat16_rn(v[j]);
  } else if (write_kv) {
    const int b = row / a.rows_per_req;
    const int pidx = pos / a.page_size;
    const int page = pidx < a.max_pages_per_req
                         ? a.page_table[static_cast<int64_t>(b) * a.max_pages_per_req + pidx]
                         : -1;
    if (page < 0 || page >= a.num_pages) {
      if (lane == 0) flag(a.status, ISD_DEV_BAD_PAGE);
      return;
    }
    const int64_t slot_base = (static_cast<int64_t>(a.layer) * a.num_pages + page) * a.n_kv;
    const bool is_k = hd < a.n_q + a.n_kv;
    const int g = is_k ? hd - a.n_q : hd - a.n_q - a.n_kv;
    __nv_bfloat16* dst = (is_k ? a.k_pool : a.v_pool) +
                         (((slot_base + g) * a.page_size) + pos % a.page_size) * HD;
#pragma unroll
    for (int j = 0; j < J; ++j) dst[lane + 32 * j] = __float2bfloat16_rn(v[j]);
  }
}

}  // namespace isd
