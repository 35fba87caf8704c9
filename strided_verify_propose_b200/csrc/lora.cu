// Gated LoRA of R-ISD (sm_100a): a rank-r update active only on MASK rows
// (Bud's Wiki "Introspective Diffusion Language Models", Key claims and
// Method: verify positions stay on base weights, so their outputs equal the
// base model's bit for bit).
//
// The deltas themselves come from the tcgen05 GEMM (x A^T, then (x A^T) B^T);
// this file holds the small kernels around them: packing the adapters into
// GEMM-ready fused matrices, the fixed-order split-K sum of x A^T cast to
// bf16, and the SwiGLU of the LoRA path (base gate/up in fp32 plus the delta
// on MASK rows). Verify rows never read a delta.
#include "common.cuh"
#include "kernels.h"

namespace isd {

namespace {

// dst[map(i)][col0 + c] = src[i][c] for i < rows, c < cols (bf16).
// map: identity + row0, or the gate/up interleave (16 rows of a block of 32,
// gate at offset 0, up at offset 16).
__global__ void pack_rows_kernel(const __nv_bfloat16* src, int rows, int cols, __nv_bfloat16* dst,
                                 int dst_ld, int row0, int col0, int interleave_off) {
  const int i = blockIdx.x;
  if (i >= rows) return;
  int r = row0 + i;
  if (interleave_off >= 0) r = (i / 16) * 32 + interleave_off + (i % 16);
  const __nv_bfloat16* s = src + static_cast<int64_t>(i) * cols;
  __nv_bfloat16* d = dst + static_cast<int64_t>(r) * dst_ld + col0;
  for (int c = threadIdx.x; c < cols; c += blockDim.x) d[c] = s[c];
}

// out[row][c] = bf16(sum_s part[s][row][c]) in split order.
__global__ void sum_cast_kernel(const float* part, int splits, int64_t split_stride, int n,
                                __nv_bfloat16* out) {
  const int row = blockIdx.x;
  for (int c = threadIdx.x; c < n; c += blockDim.x) {
    float v = 0.f;
    for (int s = 0; s < splits; ++s) v += part[s * split_stride + static_cast<int64_t>(row) * n + c];
    out[static_cast<int64_t>(row) * n + c] = __float2bfloat16_rn(v);
  }
}

// act[row][f] = bf16(SiLU(g) * u), g and u read from the base gate/up
// output (16-row interleave), plus scale * delta on MASK rows only. silu_mul
// is the expression the fused GEMM epilogue evaluates, so verify rows get the
// same bits as a step without the adapter.
__global__ void lora_silu_kernel(const float* gu, const float* delta, float scale,
                                 const int32_t* row_flags, int inter, __nv_bfloat16* act) {
  const int row = blockIdx.x;
  const bool mask_row = row_flags[row] & kRowMask;
  const float* gr = gu + static_cast<int64_t>(row) * 2 * inter;
  const float* dr = delta + static_cast<int64_t>(row) * 2 * inter;
  for (int f = threadIdx.x; f < inter; f += blockDim.x) {
    const int gc = (f / 16) * 32 + (f % 16);
    float g = gr[gc], u = gr[gc + 16];
    if (mask_row) {
      g += scale * dr[gc];
      u += scale * dr[gc + 16];
    }
    act[static_cast<int64_t>(row) * inter + f] = __float2bfloat16_rn(silu_mul(g, u));
  }
}

}  // namespace

cudaError_t launch_pack_rows(const __nv_bfloat16* src, int rows, int cols, __nv_bfloat16* dst,
                             int dst_ld, int row0, int col0, int interleave_off,
                             cudaStream_t stream) {
  pack_rows_kernel<<<rows, 128, 0, stream>>>(src, rows, cols, dst, dst_ld, row0, col0,
                                             interleave_off);
  return cudaGetLastError();
}

cudaError_t launch_sum_cast(const float* part, int splits, int rows, int n, __nv_bfloat16* out,
                            cudaStream_t stream) {
  sum_cast_kernel<<<rows, 128, 0, stream>>>(part, splits, static_cast<int64_t>(rows) * n, n, out);
  return cudaGetLastError();
}

cudaError_t launch_lora_silu(const float* gu, const float* delta, float scale,
                             const int32_t* row_flags, int rows, int inter, __nv_bfloat16* act,
                             cudaStream_t stream) {
  lora_silu_kernel<<<rows, 256, 0, stream>>>(gu, delta, scale, row_flags, inter, act);
  return cudaGetLastError();
}

}  // namespace isd
