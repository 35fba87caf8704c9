// Gated LoRA of R-ISD (sm_100a): a rank-r update active only on MASK rows
// (Bud's Wiki "Introspective Diffusion Language Models", Key claims and
// Method: verify positions stay on base weights, so their outputs equal the
// base model's bit for bit).
//
// The deltas themselves come from the tcgen05 GEMM (x A^T, then (x A^T) B^T;
// for the MLP gate/up the second GEMM's epilogue adds the delta to the base
// product on MASK rows and forms the SwiGLU); this file holds the small
// kernels around them: packing the adapters into GEMM-ready fused matrices
// and the fixed-order split-K sum of x A^T cast to bf16. Verify rows never
// read a delta.
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

// out[row][c] = bf16(scale * sum_s part[s][row][c]) (splits in order) on
// MASK rows, exactly 0 on every other row: x A^T of the gated adapter, ready
// to be multiplied by B, contributing nothing to verify rows.
__global__ void sum_cast_kernel(const float* part, int splits, int64_t split_stride, int n,
                                const int32_t* row_flags, float scale, __nv_bfloat16* out) {
  const int row = blockIdx.x;
  const bool mask_row = row_flags[row] & kRowMask;
  for (int c = threadIdx.x; c < n; c += blockDim.x) {
    float v = 0.f;
    if (mask_row) {
      const float* pc = part + static_cast<int64_t>(row) * n + c;
#pragma unroll 8
      for (int s = 0; s < splits; ++s) v += pc[s * split_stride];   // loads ahead, adds in order
    }
    out[static_cast<int64_t>(row) * n + c] = __float2bfloat16_rn(mask_row ? scale * v : 0.f);
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

cudaError_t launch_sum_cast(const float* part, int splits, int rows, int n, const int32_t* row_flags,
                            float scale, __nv_bfloat16* out, cudaStream_t stream) {
  sum_cast_kernel<<<rows, 128, 0, stream>>>(part, splits, static_cast<int64_t>(rows) * n, n, row_flags,
                                            scale, out);
  return cudaGetLastError();
}

}  // namespace isd
