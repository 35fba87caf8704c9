// Row-wise kernels of the ISD forward (sm_100a): block assembly, embedding
// + RMSNorm, the split-K reduction of the QKV projection fused with QK-norm,
// rotary embedding and the KV page write, and residual add + RMSNorm.
//
// One CTA per block row; every row is computed independently of the others
// (rows only meet inside causal attention), which keeps verify rows bitwise
// independent of what happens on MASK rows.
#include "common.cuh"
#include "kernels.h"
#include "qkv_row.cuh"

namespace isd {

namespace {

template <int NT>
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  if (threadIdx.x < 32) {
    t = threadIdx.x < NT / 32 ? red[threadIdx.x] : 0.f;
    t = warp_sum(t);
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  t = red[0];
  __syncthreads();
  return t;
}

// Block layout of one ISD step: rows [x*, d_1..d_n, MASK...] at positions
// L..L+2N-2 (Bud's Wiki, Method: verify the previous drafts and propose at
// MASK positions in the same forward).
__global__ void assemble_step_kernel(const int32_t* pending, const int32_t* n_draft,
                                     const int32_t* seq_len, int32_t stride_n, int32_t mask_token,
                                     RowMeta meta, int32_t* status) {
  const int b = blockIdx.x, r = threadIdx.x;
  const int R = 2 * stride_n - 1;
  if (r >= R) return;
  int n = n_draft[b];
  const int L = seq_len[b];
  if (n != 0 && n != stride_n - 1) {
    if (r == 0) flag(status, ISD_DEV_BAD_STATE);
    n = 0;
  }
  if (L < 0 && r == 0) flag(status, ISD_DEV_BAD_STATE);
  const int row = b * R + r;
  int tok = mask_token;
  if (r == 0) tok = pending[b * stride_n];
  else if (r <= n) tok = pending[b * stride_n + r];
  meta.tok[row] = tok;
  meta.pos[row] = L < 0 ? -1 : L + r;
  meta.flags[row] = (L < 0 ? 0 : kRowWriteKV) | (r > n ? kRowMask : 0);
}

// Prefill chunk: rows [start, start+chunk) of the prompt of request
// order[i] (i = block); positions past len-2 are padding rows that see the
// prompt's keys but write nothing.
__global__ void assemble_prefill_kernel(const int32_t* tokens, int32_t max_len, const int32_t* lens,
                                        const int32_t* order, int32_t chunk, int32_t start,
                                        RowMeta meta) {
  const int i = blockIdx.x, r = threadIdx.x;
  if (r >= chunk) return;
  const int b = order ? order[i] : i;
  const int row = i * chunk + r;
  const int len = lens[b];
  const int q = start + r;
  if (q < len - 1) {
    meta.tok[row] = tokens[static_cast<int64_t>(b) * max_len + q];
    meta.pos[row] = q;
    meta.flags[row] = kRowWriteKV;
  } else {
    meta.tok[row] = tokens[static_cast<int64_t>(b) * max_len];
    meta.pos[row] = len >= 2 ? min(start, len - 2) : -1;
    meta.flags[row] = 0;
  }
}

// x = embed[tok] (fp32 residual stream); hn = bf16(RMSNorm(x) * w).
__global__ void __launch_bounds__(256)
    embed_norm_kernel(const __nv_bfloat16* embed, const float* norm_w, RowMeta meta, int32_t hidden,
                      int32_t vocab, float eps, float* x, __nv_bfloat16* hn, int32_t* status) {
  __shared__ float red[32];
  griddep_launch_dependents();   // the next GEMM may load its weights meanwhile
  const int row = blockIdx.x;
  int tok = meta.tok[row];
  if (tok < 0 || tok >= vocab) {
    if (threadIdx.x == 0) flag(status, ISD_DEV_BAD_TOKEN);
    tok = 0;
  }
  const __nv_bfloat16* e = embed + static_cast<int64_t>(tok) * hidden;
  float* xr = x + static_cast<int64_t>(row) * hidden;
  float ss = 0.f;
  for (int i = threadIdx.x * 8; i < hidden; i += 256 * 8) {
    const uint4 raw = *reinterpret_cast<const uint4*>(e + i);
    const __nv_bfloat16* h8 = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float v = __bfloat162float(h8[k]);
      xr[i + k] = v;
      ss += v * v;
    }
  }
  const float tot = block_sum<256>(ss, red);
  const float rstd = rsqrtf(tot / hidden + eps);
  __nv_bfloat16* hr = hn + static_cast<int64_t>(row) * hidden;
  for (int i = threadIdx.x * 8; i < hidden; i += 256 * 8) {
    const uint4 raw = *reinterpret_cast<const uint4*>(e + i);
    const __nv_bfloat16* h8 = reinterpret_cast<const __nv_bfloat16*>(&raw);
    __align__(16) __nv_bfloat16 o8[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) o8[k] = __float2bfloat16_rn(__bfloat162float(h8[k]) * rstd * norm_w[i + k]);
    *reinterpret_cast<uint4*>(hr + i) = *reinterpret_cast<const uint4*>(o8);
  }
}

// x[row] += sum_s part[s][row] (fixed order); hn[row] = bf16(RMSNorm(x[row]) * w).
// Each thread holds up to kResIters float4 of the row and loads kBatch
// splits of them at once (one memory round trip per kBatch splits, not per
// split); the sum order (x, then splits ascending) is fixed. kIters float4
// per thread cover hidden <= kIters * 1024; kMinCtas CTAs of 256 threads
// share an SM, so a thread has 256 / kMinCtas registers: 4 CTAs when the
// rows need them all for one wave, else 2 and a deeper batch.
constexpr int kResThreads = 256;
constexpr int kResIters = 8;        // hidden <= 8192
constexpr int kResMaxSplits = 8;

template <int kIters, int kBatch, int kMinCtas>
__global__ void __launch_bounds__(kResThreads, kMinCtas)
    residual_norm_kernel(const float* part, int32_t splits, int64_t split_stride, int32_t hidden,
                         const float* norm_w, float eps, float* x, __nv_bfloat16* hn) {
  __shared__ float red[32];
  griddep_launch_dependents();   // the next GEMM may load its weights meanwhile
  const int row = blockIdx.x;
  float* xr = x + static_cast<int64_t>(row) * hidden;
  const float* pr = part + static_cast<int64_t>(row) * hidden;
  float4 v[kIters];
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int i = (it * kResThreads + threadIdx.x) * 4;
    v[it] = i < hidden ? *reinterpret_cast<const float4*>(xr + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int s0 = 0; s0 < kResMaxSplits; s0 += kBatch) {
    if (s0 < splits) {
      float4 d[kBatch][kIters];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
#pragma unroll
        for (int it = 0; it < kIters; ++it) {
          const int i = (it * kResThreads + threadIdx.x) * 4;
          d[u][it] = s0 + u < splits && i < hidden
                         ? *reinterpret_cast<const float4*>(pr + (s0 + u) * split_stride + i)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        if (s0 + u < splits) {
#pragma unroll
          for (int it = 0; it < kIters; ++it) {
            v[it].x += d[u][it].x;
            v[it].y += d[u][it].y;
            v[it].z += d[u][it].z;
            v[it].w += d[u][it].w;
          }
        }
      }
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int i = (it * kResThreads + threadIdx.x) * 4;
    if (i < hidden) {
      *reinterpret_cast<float4*>(xr + i) = v[it];
      ss += v[it].x * v[it].x + v[it].y * v[it].y + v[it].z * v[it].z + v[it].w * v[it].w;
    }
  }
  const float tot = block_sum<kResThreads>(ss, red);
  const float rstd = rsqrtf(tot / hidden + eps);
  __nv_bfloat16* hr = hn + static_cast<int64_t>(row) * hidden;
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int i = (it * kResThreads + threadIdx.x) * 4;
    if (i < hidden) {
      const float4 w = *reinterpret_cast<const float4*>(norm_w + i);
      __align__(8) __nv_bfloat16 o4[4] = {
          __float2bfloat16_rn(v[it].x * rstd * w.x), __float2bfloat16_rn(v[it].y * rstd * w.y),
          __float2bfloat16_rn(v[it].z * rstd * w.z), __float2bfloat16_rn(v[it].w * rstd * w.w)};
      *reinterpret_cast<uint2*>(hr + i) = *reinterpret_cast<const uint2*>(o4);
    }
  }
}

// QKV split-K reduction, then per head: RMSNorm over head_dim for q and k,
// NeoX rotary embedding (pairs (i, i + d/2)) at the row's absolute position,
// q to the attention input, k and v into the row's page slot.
// Grid (rows, ceil(heads / kQkvWarps)): one warp per (row, head), so every
// warp has all of its split loads in flight at once.
constexpr int kQkvWarps = 16;
constexpr int kQkvMaxSplits = 8;

template <int HD>
// (4 CTAs of 512 threads per SM: at most 32 registers per thread)
__global__ void __launch_bounds__(kQkvWarps * 32, 4) qkv_reduce_kernel(const QkvReduceArgs a) {
  griddep_launch_dependents();   // the attention may load earlier steps' K/V meanwhile
  const int row = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hd = blockIdx.y * kQkvWarps + warp;
  if (hd >= a.n_q + 2 * a.n_kv) return;
  float v[HD / 32];
  qkv_head_sum<HD>(a, row, hd, lane, v);
  qkv_head_finish<HD>(a, row, hd, lane, v);
}

}  // namespace

cudaError_t launch_assemble_step(const int32_t* pending, const int32_t* n_draft,
                                 const int32_t* seq_len, int32_t batch, int32_t stride_n,
                                 int32_t mask_token, RowMeta meta, int32_t* status,
                                 cudaStream_t stream) {
  assemble_step_kernel<<<batch, 32, 0, stream>>>(pending, n_draft, seq_len, stride_n, mask_token,
                                                 meta, status);
  return cudaGetLastError();
}

cudaError_t launch_assemble_prefill(const int32_t* tokens, int32_t max_len, const int32_t* lens,
                                    const int32_t* order, int32_t batch, int32_t chunk,
                                    int32_t start, RowMeta meta, cudaStream_t stream) {
  if (batch < 1) return cudaSuccess;
  assemble_prefill_kernel<<<batch, 64, 0, stream>>>(tokens, max_len, lens, order, chunk, start,
                                                    meta);
  return cudaGetLastError();
}

// dst row (i * repeat + j) = src row order[i], rows of row_len ints.
__global__ void gather_rows_kernel(const int32_t* src, const int32_t* order, int32_t row_len,
                                   int32_t repeat, int32_t* dst) {
  const int i = blockIdx.x;
  const int32_t* s = src + static_cast<int64_t>(order[i]) * row_len;
  for (int j = 0; j < repeat; ++j) {
    int32_t* d = dst + (static_cast<int64_t>(i) * repeat + j) * row_len;
    for (int k = threadIdx.x; k < row_len; k += blockDim.x) d[k] = s[k];
  }
}

cudaError_t launch_gather_rows(const int32_t* src, const int32_t* order, int32_t rows,
                               int32_t row_len, int32_t repeat, int32_t* dst, cudaStream_t stream) {
  if (rows < 1) return cudaSuccess;
  gather_rows_kernel<<<rows, 128, 0, stream>>>(src, order, row_len, repeat, dst);
  return cudaGetLastError();
}

cudaError_t launch_embed_norm(const __nv_bfloat16* embed, const float* norm_w, RowMeta meta,
                              int32_t rows, int32_t hidden, int32_t vocab, float eps, float* x,
                              __nv_bfloat16* hn, int32_t* status, cudaStream_t stream) {
  embed_norm_kernel<<<rows, 256, 0, stream>>>(embed, norm_w, meta, hidden, vocab, eps, x, hn,
                                              status);
  return cudaGetLastError();
}

cudaError_t launch_qkv_reduce(const QkvReduceArgs& a, cudaStream_t stream) {
  if (a.splits < 1 || a.splits > kQkvMaxSplits) return cudaErrorInvalidValue;
  const dim3 grid(a.rows, (a.n_q + 2 * a.n_kv + kQkvWarps - 1) / kQkvWarps);
  if (a.head_dim == 128)
    qkv_reduce_kernel<128><<<grid, kQkvWarps * 32, 0, stream>>>(a);
  else
    qkv_reduce_kernel<64><<<grid, kQkvWarps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_residual_norm(const float* part, int32_t splits, int32_t rows, int32_t hidden,
                                 const float* norm_w, float eps, float* x, __nv_bfloat16* hn,
                                 cudaStream_t stream) {
  if (hidden % 4 || hidden > kResThreads * 4 * kResIters || splits < 0 || splits > kResMaxSplits)
    return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const bool deep = rows <= 2 * sms;   // one wave at 2 CTAs per SM
  const int64_t stride = static_cast<int64_t>(rows) * hidden;
  if (hidden <= kResThreads * 4 * 4) {
    if (deep)
      residual_norm_kernel<4, 4, 2><<<rows, kResThreads, 0, stream>>>(part, splits, stride, hidden,
                                                                      norm_w, eps, x, hn);
    else
      residual_norm_kernel<4, 2, 4><<<rows, kResThreads, 0, stream>>>(part, splits, stride, hidden,
                                                                      norm_w, eps, x, hn);
  } else if (hidden <= kResThreads * 4 * 5) {
    if (deep)
      residual_norm_kernel<5, 4, 2><<<rows, kResThreads, 0, stream>>>(part, splits, stride, hidden,
                                                                      norm_w, eps, x, hn);
    else
      residual_norm_kernel<5, 1, 4><<<rows, kResThreads, 0, stream>>>(part, splits, stride, hidden,
                                                                      norm_w, eps, x, hn);
  } else {
    if (deep)
      residual_norm_kernel<kResIters, 2, 2><<<rows, kResThreads, 0, stream>>>(
          part, splits, stride, hidden, norm_w, eps, x, hn);
    else
      residual_norm_kernel<kResIters, 1, 4><<<rows, kResThreads, 0, stream>>>(
          part, splits, stride, hidden, norm_w, eps, x, hn);
  }
  return cudaGetLastError();
}

}  // namespace isd
