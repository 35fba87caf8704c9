// Paged causal GQA attention for the ISD block (sm_100a).
//
// Every request's block rows attend to its paged KV prefix plus the earlier
// rows of the same block (strict causal attention over [prefix | block]:
// Bud's Wiki "Introspective Diffusion Language Models", TL;DR and Method;
// the block's own K/V are written to their page slots before this kernel
// runs, so one causal mask over positions covers both parts).
//
// Work unit = (request b, KV head g, key split s). The R rows x G query heads
// that share KV head g form one query tile of R*G rows (28 at stride 4 with
// Qwen3-8B's 4:1 grouping), so each K/V byte is read once per request. A
// producer warp streams 64-key tiles of K and V page by page with TMA
// (128-byte swizzled boxes of one page x 64 dims, zero-filled past the
// request's end) into a ring of stages; four consumer warps run QK^T and PV
// on mma.sync bf16 tensor cores with an fp32 online softmax. Warps split the
// query rows into 16-row tiles and the 64 keys of a tile into key groups;
// key groups are merged through shared memory, splits by a second kernel.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace isd {

namespace {

constexpr int kKeysPerTile = 64;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;

struct AttnParams {
  const __nv_bfloat16* q;      // [B*R][nq][HD]
  const int32_t* row_pos;      // [B*R]
  const int32_t* page_table;   // [B][maxp]
  int32_t R, nq, nkv, G, page_size, num_pages, maxp, layer;
  int32_t RG, MT, KG, stages;
  int32_t split_keys, max_splits;
  int32_t oob_row;             // a row coordinate past the pool: zero fill
  float scale_log2;            // log2(e) / sqrt(HD)
  float* part_o;               // [B][nkv][max_splits][MT*16][HD]
  float2* part_ml;             // [B][nkv][max_splits][MT*16]  (max (log2 units), sum)
  int32_t* status;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of element (key, dim) in a TMA 128B-swizzled tile stored as
// [dim / 64][key][64 dims].
__device__ __forceinline__ uint32_t sw_off(int key, int dim) {
  return static_cast<uint32_t>((dim >> 6) * (kKeysPerTile * 128) + key * 128 +
                               ((((dim & 63) >> 3) ^ (key & 7)) << 4) + (dim & 7) * 2);
}

template <int HD>
__global__ void __launch_bounds__(kThreads)
    attn_split_kernel(const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const AttnParams p) {
  constexpr int kTileBytes = kKeysPerTile * HD * 2;   // one of K or V
  constexpr int kQStride = HD + 8;                    // padded Q row (bf16 elements)
  constexpr int kNT = HD / 8;                         // output n-tiles per warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // rows of this request and the key range they need
  __shared__ int s_pos[64];
  __shared__ int s_kend;
  if (threadIdx.x == 0) s_kend = 0;
  __syncthreads();
  if (threadIdx.x < p.R) {
    const int ps = p.row_pos[b * p.R + threadIdx.x];
    s_pos[threadIdx.x] = ps;
    atomicMax(&s_kend, ps + 1);
  }
  __syncthreads();
  const int kend = min(s_kend, p.maxp * p.page_size);   // keys past the page table do not exist
  const int k_lo = split * p.split_keys;
  if (k_lo >= kend) return;                 // the combine kernel skips this split too
  const int k_hi = min(kend, k_lo + p.split_keys);
  const int n_tiles = (k_hi - k_lo + kKeysPerTile - 1) / kKeysPerTile;

  uint8_t* kv_base = smem;                                       // stages x (K, V)
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(smem + p.stages * 2 * kTileBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(qs + p.MT * 16 * kQStride);
  uint64_t* empty = full + p.stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_barrier_init();
  }
  // Q tile: row qi = r * G + h  <->  token row b*R + r, query head g*G + h
  const int qrows = p.MT * 16;
  for (int i = threadIdx.x; i < qrows * (HD / 8); i += blockDim.x) {
    const int qi = i / (HD / 8), c = i % (HD / 8);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (qi < p.RG) {
      const int r = qi / p.G, h = qi % p.G;
      const __nv_bfloat16* src = p.q + (static_cast<int64_t>(b * p.R + r) * p.nq + g * p.G + h) * HD;
      v = reinterpret_cast<const uint4*>(src)[c];
    }
    *reinterpret_cast<uint4*>(qs + qi * kQStride + c * 8) = v;
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int per_tile = kKeysPerTile / p.page_size;
      const int32_t* pt = p.page_table + static_cast<int64_t>(b) * p.maxp;
      for (int t = 0; t < n_tiles; ++t) {
        const int st = t % p.stages;
        if (!mbar_wait(&empty[st], ((t / p.stages) & 1) ^ 1)) {
          flag(p.status, ISD_DEV_TIMEOUT);
          break;
        }
        uint8_t* ks = kv_base + st * 2 * kTileBytes;
        uint8_t* vs = ks + kTileBytes;
        mbar_arrive_expect_tx(&full[st], 2 * kTileBytes);
        for (int j = 0; j < per_tile; ++j) {
          const int key0 = k_lo + t * kKeysPerTile + j * p.page_size;
          int row = p.oob_row;
          if (key0 < k_hi) {
            const int page = pt[key0 / p.page_size];
            if (page >= 0 && page < p.num_pages) {
              row = ((p.layer * p.num_pages + page) * p.nkv + g) * p.page_size;
            } else {
              flag(p.status, ISD_DEV_BAD_PAGE);
            }
          }
#pragma unroll
          for (int hh = 0; hh < HD / 64; ++hh) {
            const int off = hh * kKeysPerTile * 128 + j * p.page_size * 128;
            tma_load_2d(ks + off, &kmap, &full[st], hh * 64, row);
            tma_load_2d(vs + off, &vmap, &full[st], hh * 64, row);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int mt = warp % p.MT;
    const int kg = warp / p.MT;
    const int KW = kKeysPerTile / p.KG;         // keys per warp in a tile (16, 32 or 64)
    const int kw0 = kg * KW;
    const bool active = kg < p.KG;
    const int row_a = mt * 16 + (lane >> 2);
    const int row_b = row_a + 8;
    const int pos_a = row_a < p.RG ? s_pos[row_a / p.G] : -1;
    const int pos_b = row_b < p.RG ? s_pos[row_b / p.G] : -1;

    // Q fragments for the whole head dim
    uint32_t qf[HD / 16][4];
    {
      const uint32_t qbase = smem_u32(qs);
      const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const int row = mt * 16 + rr + ((mi & 1) << 3);
        const int col = kk * 16 + ((mi >> 1) << 3);
        ldsm_x4(qbase + (row * kQStride + col) * 2, qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    float o[kNT][4];
#pragma unroll
    for (int i = 0; i < kNT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

    for (int t = 0; t < n_tiles; ++t) {
      const int st = t % p.stages;
      if (!mbar_wait(&full[st], (t / p.stages) & 1)) {
        flag(p.status, ISD_DEV_TIMEOUT);
        break;
      }
      if (active) {
        const uint32_t kbase = smem_u32(kv_base + st * 2 * kTileBytes);
        const uint32_t vbase = kbase + kTileBytes;
        const int mi = lane >> 3, rr = lane & 7;
        float s[8][4];   // up to 64 keys per warp = 8 n-tiles
        const int nkt = KW / 8;
#pragma unroll
        for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            if (qq * 2 < nkt) {
              const int key = kw0 + qq * 16 + rr + ((mi >> 1) << 3);
              const int dim = kk * 16 + ((mi & 1) << 3);
              uint32_t b0, b1, b2, b3;
              ldsm_x4(kbase + sw_off(key, dim), b0, b1, b2, b3);
              mma_bf16(s[2 * qq], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
              mma_bf16(s[2 * qq + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
            }
          }
        }
        // mask + online softmax (base 2)
        const int key_base = k_lo + t * kKeysPerTile + kw0 + 2 * (lane & 3);
        float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          if (n < nkt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int key = key_base + n * 8 + (e & 1);
              const int lim = e < 2 ? pos_a : pos_b;
              const bool ok = key < k_hi && key <= lim;
              s[n][e] = ok ? s[n][e] * p.scale_log2 : -INFINITY;
            }
            mx_a = fmaxf(mx_a, fmaxf(s[n][0], s[n][1]));
            mx_b = fmaxf(mx_b, fmaxf(s[n][2], s[n][3]));
          }
        }
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
        const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
        const float ref_a = mn_a == -INFINITY ? 0.f : mn_a;
        const float ref_b = mn_b == -INFINITY ? 0.f : mn_b;
        const float c_a = exp2f(m_a - ref_a), c_b = exp2f(m_b - ref_b);
        m_a = mn_a;
        m_b = mn_b;
        l_a *= c_a;
        l_b *= c_b;
#pragma unroll
        for (int i = 0; i < kNT; ++i) {
          o[i][0] *= c_a;
          o[i][1] *= c_a;
          o[i][2] *= c_b;
          o[i][3] *= c_b;
        }
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          if (n < nkt) {
            s[n][0] = exp2f(s[n][0] - ref_a);
            s[n][1] = exp2f(s[n][1] - ref_a);
            s[n][2] = exp2f(s[n][2] - ref_b);
            s[n][3] = exp2f(s[n][3] - ref_b);
            l_a += s[n][0] + s[n][1];
            l_b += s[n][2] + s[n][3];
          }
        }
        // O += P V, 16 keys per k-step
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          if (ks * 2 < nkt) {
            const uint32_t a0 = pack_bf16(s[2 * ks][0], s[2 * ks][1]);
            const uint32_t a1 = pack_bf16(s[2 * ks][2], s[2 * ks][3]);
            const uint32_t a2 = pack_bf16(s[2 * ks + 1][0], s[2 * ks + 1][1]);
            const uint32_t a3 = pack_bf16(s[2 * ks + 1][2], s[2 * ks + 1][3]);
            const int key = kw0 + ks * 16 + rr + ((mi & 1) << 3);
#pragma unroll
            for (int dq = 0; dq < HD / 16; ++dq) {
              const int dim = dq * 16 + ((mi >> 1) << 3);
              uint32_t b0, b1, b2, b3;
              ldsm_x4_t(vbase + sw_off(key, dim), b0, b1, b2, b3);
              mma_bf16(o[2 * dq], a0, a1, a2, a3, b0, b1);
              mma_bf16(o[2 * dq + 1], a0, a1, a2, a3, b2, b3);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);

    // merge key groups through shared memory (the stage ring is idle after this barrier)
    asm volatile("bar.sync 1, 128;" ::: "memory");
    float* xo = reinterpret_cast<float*>(kv_base);               // [4 warps][32][kNT*4]
    float* xm = xo + kConsumerWarps * 32 * kNT * 4;              // [4 warps][32][4]
    if (active && kg > 0) {
      float* dst = xo + (warp * 32 + lane) * kNT * 4;
#pragma unroll
      for (int i = 0; i < kNT; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[i * 4 + e] = o[i][e];
      float* dm = xm + (warp * 32 + lane) * 4;
      dm[0] = m_a;
      dm[1] = m_b;
      dm[2] = l_a;
      dm[3] = l_b;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (active && kg == 0) {
      float M_a = m_a, M_b = m_b;
      for (int k2 = 1; k2 < p.KG; ++k2) {
        const float* dm = xm + ((k2 * p.MT + mt) * 32 + lane) * 4;
        M_a = fmaxf(M_a, dm[0]);
        M_b = fmaxf(M_b, dm[1]);
      }
      const float R_a = M_a == -INFINITY ? 0.f : M_a, R_b = M_b == -INFINITY ? 0.f : M_b;
      float f_a = exp2f(m_a - R_a), f_b = exp2f(m_b - R_b);
      float L_a = l_a * f_a, L_b = l_b * f_b;
#pragma unroll
      for (int i = 0; i < kNT; ++i) {
        o[i][0] *= f_a;
        o[i][1] *= f_a;
        o[i][2] *= f_b;
        o[i][3] *= f_b;
      }
      for (int k2 = 1; k2 < p.KG; ++k2) {
        const int w2 = k2 * p.MT + mt;
        const float* dm = xm + (w2 * 32 + lane) * 4;
        const float g_a = exp2f(dm[0] - R_a), g_b = exp2f(dm[1] - R_b);
        L_a += dm[2] * g_a;
        L_b += dm[3] * g_b;
        const float* src = xo + (w2 * 32 + lane) * kNT * 4;
#pragma unroll
        for (int i = 0; i < kNT; ++i) {
          o[i][0] += src[i * 4 + 0] * g_a;
          o[i][1] += src[i * 4 + 1] * g_a;
          o[i][2] += src[i * 4 + 2] * g_b;
          o[i][3] += src[i * 4 + 3] * g_b;
        }
      }
      const int64_t unit = (static_cast<int64_t>(b) * p.nkv + g) * p.max_splits + split;
      const int rows16 = p.MT * 16;
      const float inv_a = L_a > 0.f ? 1.f / L_a : 0.f;
      const float inv_b = L_b > 0.f ? 1.f / L_b : 0.f;
      float* po = p.part_o + unit * rows16 * HD;
      const int col0 = 2 * (lane & 3);
#pragma unroll
      for (int i = 0; i < kNT; ++i) {
        *reinterpret_cast<float2*>(po + row_a * HD + i * 8 + col0) =
            make_float2(o[i][0] * inv_a, o[i][1] * inv_a);
        *reinterpret_cast<float2*>(po + row_b * HD + i * 8 + col0) =
            make_float2(o[i][2] * inv_b, o[i][3] * inv_b);
      }
      if ((lane & 3) == 0) {
        p.part_ml[unit * rows16 + row_a] = make_float2(M_a, L_a);
        p.part_ml[unit * rows16 + row_b] = make_float2(M_b, L_b);
      }
    }
  }
}

// out[b*R + r][(g*G + h)*HD + d] = sum over splits, weighted by each split's softmax mass.
template <int HD>
__global__ void attn_combine_kernel(const AttnParams p, __nv_bfloat16* out) {
  const int g = blockIdx.x, b = blockIdx.y;
  __shared__ int s_kend;
  if (threadIdx.x == 0) s_kend = 0;
  __syncthreads();
  if (threadIdx.x < p.R) atomicMax(&s_kend, p.row_pos[b * p.R + threadIdx.x] + 1);
  __syncthreads();
  const int kend = min(s_kend, p.maxp * p.page_size);
  const int n_splits = min(p.max_splits, kend > 0 ? (kend + p.split_keys - 1) / p.split_keys : 0);
  const int rows16 = p.MT * 16;
  const int64_t unit0 = (static_cast<int64_t>(b) * p.nkv + g) * p.max_splits;
  for (int i = threadIdx.x; i < p.RG * HD; i += blockDim.x) {
    const int qi = i / HD, d = i % HD;
    float M = -INFINITY;
    for (int s = 0; s < n_splits; ++s) M = fmaxf(M, p.part_ml[(unit0 + s) * rows16 + qi].x);
    const float Rm = M == -INFINITY ? 0.f : M;
    float L = 0.f, acc = 0.f;
    for (int s = 0; s < n_splits; ++s) {
      const float2 ml = p.part_ml[(unit0 + s) * rows16 + qi];
      const float w = ml.y * exp2f(ml.x - Rm);
      L += w;
      acc += w * p.part_o[((unit0 + s) * rows16 + qi) * HD + d];
    }
    const float v = L > 0.f ? acc / L : 0.f;
    const int r = qi / p.G, h = qi % p.G;
    out[(static_cast<int64_t>(b * p.R + r) * p.nq + g * p.G + h) * HD + d] = __float2bfloat16_rn(v);
  }
}

struct Derived {
  int RG, MT, KG, split_keys, max_splits, stages;
  size_t smem;
};

Derived derive(const AttnShape& s) {
  Derived d;
  const int G = s.n_q_heads / s.n_kv_heads;
  d.RG = s.rows_per_req * G;
  d.MT = (d.RG + 15) / 16;
  if (d.MT == 3) d.MT = 4;
  d.KG = kConsumerWarps / d.MT;
  const int64_t max_keys = static_cast<int64_t>(s.max_pages_per_req) * s.page_size;
  int64_t sk = (static_cast<int64_t>(s.batch) * s.n_kv_heads * max_keys) / (148 * 8);
  sk = ((sk + 63) / 64) * 64;
  sk = std::max<int64_t>(128, std::min<int64_t>(1024, sk));
  d.split_keys = static_cast<int>(sk);
  d.max_splits = static_cast<int>((max_keys + sk - 1) / sk);
  d.stages = s.head_dim == 128 ? 3 : 4;
  const size_t tile = static_cast<size_t>(kKeysPerTile) * s.head_dim * 2;
  d.smem = 1024 + d.stages * 2 * tile + static_cast<size_t>(d.MT) * 16 * (s.head_dim + 8) * 2 +
           2 * d.stages * 8 + 64;
  return d;
}

}  // namespace

size_t attention_workspace_bytes(const AttnShape& s) {
  const Derived d = derive(s);
  const size_t units = static_cast<size_t>(s.batch) * s.n_kv_heads * d.max_splits;
  const size_t rows = static_cast<size_t>(d.MT) * 16;
  return units * rows * (s.head_dim * sizeof(float) + sizeof(float2)) + 256;
}

cudaError_t launch_attention(const CUtensorMap& k_map, const CUtensorMap& v_map, const AttnShape& s,
                             int32_t layer, const __nv_bfloat16* q, const int32_t* row_pos,
                             const int32_t* page_table, __nv_bfloat16* out, void* workspace,
                             int32_t* status, cudaStream_t stream, int* launches,
                             cudaEvent_t between) {
  const Derived d = derive(s);
  AttnParams p;
  p.q = q;
  p.row_pos = row_pos;
  p.page_table = page_table;
  p.R = s.rows_per_req;
  p.nq = s.n_q_heads;
  p.nkv = s.n_kv_heads;
  p.G = s.n_q_heads / s.n_kv_heads;
  p.page_size = s.page_size;
  p.num_pages = s.num_pages;
  p.maxp = s.max_pages_per_req;
  p.layer = layer;
  p.RG = d.RG;
  p.MT = d.MT;
  p.KG = d.KG;
  p.stages = d.stages;
  p.split_keys = d.split_keys;
  p.max_splits = d.max_splits;
  p.oob_row = s.n_layers * s.num_pages * s.n_kv_heads * s.page_size;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(s.head_dim));
  const size_t units = static_cast<size_t>(s.batch) * s.n_kv_heads * d.max_splits;
  const size_t rows = static_cast<size_t>(d.MT) * 16;
  p.part_o = static_cast<float*>(workspace);
  p.part_ml = reinterpret_cast<float2*>(p.part_o + units * rows * s.head_dim);
  p.status = status;
  dim3 grid(d.max_splits, s.n_kv_heads, s.batch);
  static bool attr_set = false;
  if (!attr_set) {
    // the largest configuration: head_dim 128, 64 query rows, 3 stages
    cudaError_t e = cudaFuncSetAttribute(attn_split_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 120 * 1024);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_split_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               120 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  if (s.head_dim == 128) {
    attn_split_kernel<128><<<grid, kThreads, d.smem, stream>>>(k_map, v_map, p);
    if (between) cudaEventRecord(between, stream);
    attn_combine_kernel<128><<<dim3(s.n_kv_heads, s.batch), 256, 0, stream>>>(p, out);
  } else {
    attn_split_kernel<64><<<grid, kThreads, d.smem, stream>>>(k_map, v_map, p);
    if (between) cudaEventRecord(between, stream);
    attn_combine_kernel<64><<<dim3(s.n_kv_heads, s.batch), 256, 0, stream>>>(p, out);
  }
  if (launches) *launches += 2;
  return cudaGetLastError();
}

}  // namespace isd
