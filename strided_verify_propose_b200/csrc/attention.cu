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
#include <cstdlib>
#include <string>

#include "common.cuh"
#include "kernels.h"

namespace isd {

namespace {

constexpr int kKeysPerTile = 64;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kCtasPerSm = 2;
constexpr int kMaxSplits = 64;
constexpr int kMaxBatch = 1024;

struct AttnParams {
  const int32_t* row_pos;      // [B*R]
  const int32_t* page_table;   // [B][maxp]
  int32_t B, R, nq, nkv, G, page_size, num_pages, maxp, layer;
  int32_t RG, MT, stages;
  int32_t split_keys;
  int32_t max_items;           // workspace capacity in work items
  int32_t oob_row;             // a row coordinate past the pool: zero fill
  float scale_log2;            // log2(e) / sqrt(HD)
  float* part_o;               // [item][MT*16][HD]
  float2* part_ml;             // [item][MT*16]  (max (log2 units), sum)
  int32_t* item_base;          // [B+1] first split index of each request (written by CTA 0)
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

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Byte offset of element (row, dim) in a TMA 128B-swizzled tile stored as
// [dim / 64][row][64 dims], with half_bytes between the two 64-dim halves.
__device__ __forceinline__ uint32_t sw_off(int row, int dim, int half_bytes) {
  return static_cast<uint32_t>((dim >> 6) * half_bytes + row * 128 +
                               ((((dim & 63) >> 3) ^ (row & 7)) << 4) + (dim & 7) * 2);
}

// Shared state every CTA derives from the row positions: per request the
// key count, its number of key splits and the first item index.
struct ItemTable {
  int kend[kMaxBatch];
  int base[kMaxBatch + 1];   // exclusive prefix of the split counts
};

__device__ void build_items(const AttnParams& p, ItemTable& t) {
  for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
    int ke = 0;
    for (int r = 0; r < p.R; ++r) ke = max(ke, p.row_pos[b * p.R + r] + 1);
    ke = min(ke, p.maxp * p.page_size);
    t.kend[b] = ke;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    // one warp scans the split counts: lane l owns a contiguous run of requests
    const int lane = threadIdx.x;
    const int per = (p.B + 31) / 32;
    const int b0 = lane * per, b1 = min(p.B, b0 + per);
    int local = 0;
    for (int b = b0; b < b1; ++b) local += t.kend[b] > 0 ? (t.kend[b] + p.split_keys - 1) / p.split_keys : 0;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int b = b0; b < b1; ++b) {
      t.base[b] = run;
      run += t.kend[b] > 0 ? (t.kend[b] + p.split_keys - 1) / p.split_keys : 0;
    }
    if (lane == 31) t.base[p.B] = incl;
  }
  __syncthreads();
}

// item -> (b, g, split): items are ordered request-major, then KV head, then split.
__device__ __forceinline__ void decode_item(const AttnParams& p, const ItemTable& t, int item,
                                            int& b, int& g, int& sp) {
  int lo = 0, hi = p.B;   // find b with base[b]*nkv <= item < base[b+1]*nkv
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (t.base[mid] * p.nkv <= item) lo = mid; else hi = mid;
  }
  b = lo;
  const int ns = t.base[b + 1] - t.base[b];
  const int rem = item - t.base[b] * p.nkv;
  g = rem / ns;
  sp = rem % ns;
}

// Persistent paged attention. HD: head dim; NG: tile groups. Warp w works on
// query tile w % MTS and tile group w / MTS (MTS = 8 / NG): tile number tc of
// the CTA's stream belongs to group tc % NG, so NG tiles are in flight in
// the consumers at once and every warp owns all 64 keys of its tiles.
template <int HD, int NG>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    attn_persistent_kernel(const __grid_constant__ CUtensorMap kmap,
                           const __grid_constant__ CUtensorMap vmap,
                           const __grid_constant__ CUtensorMap qmap, const AttnParams p) {
  constexpr int kTileBytes = kKeysPerTile * HD * 2;   // one of K or V
  constexpr int kHalfTile = kKeysPerTile * 128;       // one 64-dim half of a K or V tile
  constexpr int kNT = HD / 8;                         // output n-tiles per warp
  constexpr int MTS = kConsumerWarps / NG;            // query-tile slots per group
  constexpr int NKT = kKeysPerTile / 8;               // key n-tiles per warp (all 64 keys)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ ItemTable items;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows16 = p.MT * 16;
  const int q_half = rows16 * 128;                    // bytes of one 64-dim half of Q
  const int q_buf = (HD / 64) * q_half;

  uint8_t* ring = smem;                                           // stages x (K, V)
  uint8_t* qs = smem + p.stages * 2 * kTileBytes;                 // 2 x Q buffers
  // merge area: one slot per warp of tile groups 1..NG-1
  float* xo = reinterpret_cast<float*>(qs + 2 * q_buf);
  float* xm = xo + (kConsumerWarps - MTS) * 32 * kNT * 4;
  uint64_t* bars = reinterpret_cast<uint64_t*>(xm + (kConsumerWarps - MTS) * 32 * 4);
  uint64_t* full = bars;
  uint64_t* empty = full + p.stages;
  uint64_t* q_full = empty + p.stages;
  uint64_t* q_empty = q_full + 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], MTS);     // the warps of the tile's group release it
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], kConsumerWarps);
    }
    fence_barrier_init();
  }
  build_items(p, items);     // ends with __syncthreads
  const int total = items.base[p.B] * p.nkv;
  if (blockIdx.x == 0)
    for (int b = threadIdx.x; b <= p.B; b += blockDim.x) p.item_base[b] = items.base[b];
  if (total > p.max_items) {
    if (threadIdx.x == 0) flag(p.status, ISD_DEV_BAD_STATE);
    return;
  }

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int per_tile = kKeysPerTile / p.page_size;
      int tc = 0, it = 0;
      for (int item = blockIdx.x; item < total; item += gridDim.x, ++it) {
        int b, g, sp;
        decode_item(p, items, item, b, g, sp);
        const int k_lo = sp * p.split_keys;
        const int k_hi = min(items.kend[b], k_lo + p.split_keys);
        const int n_tiles = (k_hi - k_lo + kKeysPerTile - 1) / kKeysPerTile;
        const int qb = it & 1;
        if (!mbar_wait(&q_empty[qb], ((it >> 1) & 1) ^ 1)) {
          flag(p.status, ISD_DEV_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(&q_full[qb], (HD / 64) * p.RG * 128);
#pragma unroll
        for (int hh = 0; hh < HD / 64; ++hh)
          tma_load_3d(qs + qb * q_buf + hh * q_half, &qmap, &q_full[qb], hh * 64, g * p.G, b * p.R);
        const int32_t* pt = p.page_table + static_cast<int64_t>(b) * p.maxp;
        for (int t = 0; t < n_tiles; ++t, ++tc) {
          const int st = tc % p.stages;
          if (!mbar_wait(&empty[st], ((tc / p.stages) & 1) ^ 1)) {
            flag(p.status, ISD_DEV_TIMEOUT);
            it = -1;
            break;
          }
          uint8_t* ks = ring + st * 2 * kTileBytes;
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
              const int off = hh * kHalfTile + j * p.page_size * 128;
              tma_load_2d(ks + off, &kmap, &full[st], hh * 64, row);
              tma_load_2d(vs + off, &vmap, &full[st], hh * 64, row);
            }
          }
        }
        if (it < 0) break;
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int mt = warp % MTS;
  const int grp = warp / MTS;
  const bool active = mt < p.MT;
  const int row_a = mt * 16 + (lane >> 2);
  const int row_b = row_a + 8;
  const int mi = lane >> 3, rr = lane & 7;
  const int q_row = mt * 16 + rr + ((mi & 1) << 3);
  int tc = 0, it = 0;
  bool failed = false;
  for (int item = blockIdx.x; item < total && !failed; item += gridDim.x, ++it) {
    int b, g, sp;
    decode_item(p, items, item, b, g, sp);
    const int k_lo = sp * p.split_keys;
    const int k_hi = min(items.kend[b], k_lo + p.split_keys);
    const int n_tiles = (k_hi - k_lo + kKeysPerTile - 1) / kKeysPerTile;
    const int pos_a = row_a < p.RG ? p.row_pos[b * p.R + row_a / p.G] : -1;
    const int pos_b = row_b < p.RG ? p.row_pos[b * p.R + row_b / p.G] : -1;
    const int qb = it & 1;
    if (!mbar_wait(&q_full[qb], (it >> 1) & 1)) {
      flag(p.status, ISD_DEV_TIMEOUT);
      break;
    }
    const uint32_t qbase = smem_u32(qs + qb * q_buf);

    float o[kNT][4];
#pragma unroll
    for (int i = 0; i < kNT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

    for (int t = 0; t < n_tiles; ++t, ++tc) {
      if (tc % NG != grp) continue;          // another group's tile
      const int st = tc % p.stages;
      if (!mbar_wait(&full[st], (tc / p.stages) & 1)) {
        flag(p.status, ISD_DEV_TIMEOUT);
        failed = true;
        break;
      }
      if (active) {
        const uint32_t kbase = smem_u32(ring + st * 2 * kTileBytes);
        const uint32_t vbase = kbase + kTileBytes;
        float s[NKT][4];
#pragma unroll
        for (int n = 0; n < NKT; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(qbase + sw_off(q_row, kk * 16 + ((mi >> 1) << 3), q_half), a0, a1, a2, a3);
#pragma unroll
          for (int qq = 0; qq < NKT / 2; ++qq) {
            const int key = qq * 16 + rr + ((mi >> 1) << 3);
            const int dim = kk * 16 + ((mi & 1) << 3);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kbase + sw_off(key, dim, kHalfTile), b0, b1, b2, b3);
            mma_bf16(s[2 * qq], a0, a1, a2, a3, b0, b1);
            mma_bf16(s[2 * qq + 1], a0, a1, a2, a3, b2, b3);
          }
        }
        // mask + online softmax (base 2)
        const int key_base = k_lo + t * kKeysPerTile + 2 * (lane & 3);
        float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
        for (int n = 0; n < NKT; ++n) {
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
        for (int n = 0; n < NKT; ++n) {
          s[n][0] = exp2f(s[n][0] - ref_a);
          s[n][1] = exp2f(s[n][1] - ref_a);
          s[n][2] = exp2f(s[n][2] - ref_b);
          s[n][3] = exp2f(s[n][3] - ref_b);
          l_a += s[n][0] + s[n][1];
          l_b += s[n][2] + s[n][3];
        }
        // O += P V, 16 keys per k-step
#pragma unroll
        for (int ks = 0; ks < NKT / 2; ++ks) {
          const uint32_t a0 = pack_bf16(s[2 * ks][0], s[2 * ks][1]);
          const uint32_t a1 = pack_bf16(s[2 * ks][2], s[2 * ks][3]);
          const uint32_t a2 = pack_bf16(s[2 * ks + 1][0], s[2 * ks + 1][1]);
          const uint32_t a3 = pack_bf16(s[2 * ks + 1][2], s[2 * ks + 1][3]);
          const int key = ks * 16 + rr + ((mi & 1) << 3);
#pragma unroll
          for (int dq = 0; dq < HD / 16; ++dq) {
            const int dim = dq * 16 + ((mi >> 1) << 3);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vbase + sw_off(key, dim, kHalfTile), b0, b1, b2, b3);
            mma_bf16(o[2 * dq], a0, a1, a2, a3, b0, b1);
            mma_bf16(o[2 * dq + 1], a0, a1, a2, a3, b2, b3);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    // Q buffer no longer needed by this warp
    __syncwarp();
    if (lane == 0) mbar_arrive(&q_empty[qb]);
    if (failed) break;
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);

    // merge the tile groups of each query tile through the merge area
    if (NG > 1) {
      asm volatile("bar.sync 1, %0;" ::"r"(kConsumerWarps * 32) : "memory");
      if (active && grp > 0) {
        float* dst = xo + ((warp - MTS) * 32 + lane) * kNT * 4;
#pragma unroll
        for (int i = 0; i < kNT; ++i)
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[i * 4 + e] = o[i][e];
        float* dm = xm + ((warp - MTS) * 32 + lane) * 4;
        dm[0] = m_a;
        dm[1] = m_b;
        dm[2] = l_a;
        dm[3] = l_b;
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kConsumerWarps * 32) : "memory");
    }
    if (active && grp == 0) {
      float M_a = m_a, M_b = m_b;
#pragma unroll
      for (int k2 = 1; k2 < NG; ++k2) {
        const float* dm = xm + (((k2 - 1) * MTS + mt) * 32 + lane) * 4;
        M_a = fmaxf(M_a, dm[0]);
        M_b = fmaxf(M_b, dm[1]);
      }
      const float R_a = M_a == -INFINITY ? 0.f : M_a, R_b = M_b == -INFINITY ? 0.f : M_b;
      const float f_a = exp2f(m_a - R_a), f_b = exp2f(m_b - R_b);
      float L_a = l_a * f_a, L_b = l_b * f_b;
#pragma unroll
      for (int i = 0; i < kNT; ++i) {
        o[i][0] *= f_a;
        o[i][1] *= f_a;
        o[i][2] *= f_b;
        o[i][3] *= f_b;
      }
#pragma unroll
      for (int k2 = 1; k2 < NG; ++k2) {
        const int w2 = (k2 - 1) * MTS + mt;   // merge slot of group k2's warp
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
      const float inv_a = L_a > 0.f ? 1.f / L_a : 0.f;
      const float inv_b = L_b > 0.f ? 1.f / L_b : 0.f;
      float* po = p.part_o + static_cast<int64_t>(item) * rows16 * HD;
      const int col0 = 2 * (lane & 3);
#pragma unroll
      for (int i = 0; i < kNT; ++i) {
        *reinterpret_cast<float2*>(po + row_a * HD + i * 8 + col0) =
            make_float2(o[i][0] * inv_a, o[i][1] * inv_a);
        *reinterpret_cast<float2*>(po + row_b * HD + i * 8 + col0) =
            make_float2(o[i][2] * inv_b, o[i][3] * inv_b);
      }
      if ((lane & 3) == 0) {
        p.part_ml[static_cast<int64_t>(item) * rows16 + row_a] = make_float2(M_a, L_a);
        p.part_ml[static_cast<int64_t>(item) * rows16 + row_b] = make_float2(M_b, L_b);
      }
    }
  }
}

// out[b*R + r][(g*G + h)*HD + d] = sum over the request's key splits,
// weighted by each split's softmax mass: per-(row, split) weights once in
// shared memory, then float4 accumulation.
template <int HD>
__global__ void __launch_bounds__(128) attn_combine_kernel(const AttnParams p, __nv_bfloat16* out) {
  const int g = blockIdx.x, b = blockIdx.y;
  __shared__ float w[64][kMaxSplits];
  const int base = p.item_base[b], ns = p.item_base[b + 1] - base;
  const int first = base * p.nkv + g * ns;   // the request's splits for KV head g
  const int rows16 = p.MT * 16;
  if (base < 0 || ns < 0 || ns > kMaxSplits || first + ns > p.max_items) {
    if (threadIdx.x == 0) flag(p.status, ISD_DEV_BAD_STATE);
    return;
  }
  for (int qi = threadIdx.x; qi < p.RG; qi += blockDim.x) {
    float M = -INFINITY;
    for (int s = 0; s < ns; ++s) M = fmaxf(M, p.part_ml[static_cast<int64_t>(first + s) * rows16 + qi].x);
    const float Rm = M == -INFINITY ? 0.f : M;
    float L = 0.f;
    for (int s = 0; s < ns; ++s) {
      const float2 ml = p.part_ml[static_cast<int64_t>(first + s) * rows16 + qi];
      const float ws = ml.y * exp2f(ml.x - Rm);
      w[qi][s] = ws;
      L += ws;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    for (int s = 0; s < ns; ++s) w[qi][s] *= inv;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < p.RG * (HD / 4); i += blockDim.x) {
    const int qi = i / (HD / 4), d = (i % (HD / 4)) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < ns; ++s) {
      const float ws = w[qi][s];
      const float4 v = *reinterpret_cast<const float4*>(
          p.part_o + (static_cast<int64_t>(first + s) * rows16 + qi) * HD + d);
      acc.x += ws * v.x;
      acc.y += ws * v.y;
      acc.z += ws * v.z;
      acc.w += ws * v.w;
    }
    const int r = qi / p.G, h = qi % p.G;
    __align__(8) __nv_bfloat16 o4[4] = {__float2bfloat16_rn(acc.x), __float2bfloat16_rn(acc.y),
                                        __float2bfloat16_rn(acc.z), __float2bfloat16_rn(acc.w)};
    *reinterpret_cast<uint2*>(out + (static_cast<int64_t>(b * p.R + r) * p.nq + g * p.G + h) * HD + d) =
        *reinterpret_cast<const uint2*>(o4);
  }
}

struct Derived {
  int RG, MT, NG, split_keys, max_splits, stages, max_items;
  size_t smem;
};

Derived derive(const AttnShape& s) {
  Derived d;
  const int G = s.n_q_heads / s.n_kv_heads;
  d.RG = s.rows_per_req * G;
  d.MT = (d.RG + 15) / 16;
  if (d.MT == 3) d.MT = 4;
  d.NG = kConsumerWarps / d.MT;               // consumer warps = MT query tiles x NG groups
  if (d.NG < 1) d.NG = 1;
  const int64_t max_keys = static_cast<int64_t>(s.max_pages_per_req) * s.page_size;
  // About 4 work items per CTA over the whole batch at the longest lengths;
  // each split at least 64 and at most 4096 keys, at most kMaxSplits per request.
  int64_t sk = (static_cast<int64_t>(s.batch) * s.n_kv_heads * max_keys) / (148 * kCtasPerSm * 4);
  sk = ((sk + 63) / 64) * 64;
  sk = std::max<int64_t>(64, std::min<int64_t>(4096, sk));
  sk = std::max<int64_t>(sk, ((max_keys + kMaxSplits - 1) / kMaxSplits + 63) / 64 * 64);
  d.split_keys = static_cast<int>(sk);
  d.max_splits = static_cast<int>((max_keys + sk - 1) / sk);
  d.max_items = s.batch * s.n_kv_heads * d.max_splits;
  const size_t tile = static_cast<size_t>(kKeysPerTile) * s.head_dim * 2;
  const size_t q_bufs = 2 * static_cast<size_t>(s.head_dim / 64) * d.MT * 16 * 128;
  const size_t budget = (228 * 1024) / kCtasPerSm - 1024 - 64;   // per CTA, with the 1 KB reserve
  // fewer tile groups when their stages do not fit (a stage always serves one group)
  size_t fixed = 0;
  for (;;) {
    const int mts = kConsumerWarps / d.NG;
    const size_t merge = static_cast<size_t>(kConsumerWarps - mts) * 32 * (s.head_dim / 8 * 4 + 4) * 4;
    fixed = 1024 + q_bufs + merge + 256 + sizeof(ItemTable);
    const int fit = budget > fixed ? static_cast<int>((budget - fixed) / (2 * tile)) : 0;
    d.stages = std::min(6, fit);
    d.stages -= d.stages % d.NG;
    if (d.stages >= d.NG || d.NG == 1) break;
    d.NG /= 2;
  }
  if (d.stages < 1) d.stages = 1;   // cannot happen for head_dim <= 128; the launch check catches it
  d.smem = fixed - sizeof(ItemTable) + d.stages * 2 * tile;
  return d;
}

}  // namespace

size_t attention_workspace_bytes(const AttnShape& s) {
  const Derived d = derive(s);
  const size_t rows = static_cast<size_t>(d.MT) * 16;
  return static_cast<size_t>(d.max_items) * rows * (s.head_dim * sizeof(float) + sizeof(float2)) +
         (static_cast<size_t>(s.batch) + 1) * sizeof(int32_t) + 512;
}

cudaError_t launch_attention(const CUtensorMap& k_map, const CUtensorMap& v_map, const AttnShape& s,
                             int32_t layer, const __nv_bfloat16* q, const int32_t* row_pos,
                             const int32_t* page_table, __nv_bfloat16* out, void* workspace,
                             int32_t* status, cudaStream_t stream, int* launches,
                             cudaEvent_t between) {
  if (s.batch > kMaxBatch) return cudaErrorInvalidValue;
  const Derived d = derive(s);
  const int G = s.n_q_heads / s.n_kv_heads;
  // Q as [rows][n_q][head_dim]: a 3-D box {64 dims, G heads, R rows} holds the
  // R*G query rows that share one KV head, row qi = r * G + h.
  CUtensorMap qmap;
  {
    std::string err;
    if (!make_tmap_bf16_3d(&qmap, q, s.head_dim, s.n_q_heads,
                           static_cast<uint64_t>(s.batch) * s.rows_per_req, 64, G, s.rows_per_req,
                           &err))
      return cudaErrorInvalidResourceHandle;   // the query tensor map could not be built
  }
  AttnParams p;
  p.row_pos = row_pos;
  p.page_table = page_table;
  p.B = s.batch;
  p.R = s.rows_per_req;
  p.nq = s.n_q_heads;
  p.nkv = s.n_kv_heads;
  p.G = G;
  p.page_size = s.page_size;
  p.num_pages = s.num_pages;
  p.maxp = s.max_pages_per_req;
  p.layer = layer;
  p.RG = d.RG;
  p.MT = d.MT;
  p.stages = d.stages;
  p.split_keys = d.split_keys;
  p.max_items = d.max_items;
  p.oob_row = s.n_layers * s.num_pages * s.n_kv_heads * s.page_size;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(s.head_dim));
  const size_t rows = static_cast<size_t>(d.MT) * 16;
  p.part_o = static_cast<float*>(workspace);
  p.part_ml = reinterpret_cast<float2*>(p.part_o + static_cast<size_t>(d.max_items) * rows * s.head_dim);
  p.item_base = reinterpret_cast<int32_t*>(p.part_ml + static_cast<size_t>(d.max_items) * rows);
  p.status = status;
  static bool attr_set = false;
  if (!attr_set) {
    // dynamic + static shared memory of each CTA within its share of the SM
    const int mx = (228 * 1024) / kCtasPerSm - 1024 - static_cast<int>(sizeof(ItemTable)) - 64;
    cudaError_t e = cudaSuccess;
    auto set = [&](const void* f) {
      if (e == cudaSuccess) e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    };
    set(reinterpret_cast<const void*>(attn_persistent_kernel<128, 4>));
    set(reinterpret_cast<const void*>(attn_persistent_kernel<128, 2>));
    set(reinterpret_cast<const void*>(attn_persistent_kernel<128, 1>));
    set(reinterpret_cast<const void*>(attn_persistent_kernel<64, 4>));
    set(reinterpret_cast<const void*>(attn_persistent_kernel<64, 2>));
    set(reinterpret_cast<const void*>(attn_persistent_kernel<64, 1>));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const dim3 grid(sms * kCtasPerSm);
  if (s.head_dim == 128) {
    if (d.NG == 4)
      attn_persistent_kernel<128, 4><<<grid, kThreads, d.smem, stream>>>(k_map, v_map, qmap, p);
    else if (d.NG == 2)
      attn_persistent_kernel<128, 2><<<grid, kThreads, d.smem, stream>>>(k_map, v_map, qmap, p);
    else
      attn_persistent_kernel<128, 1><<<grid, kThreads, d.smem, stream>>>(k_map, v_map, qmap, p);
    const cudaError_t le = cudaGetLastError();
    if (le != cudaSuccess) return le;   // the combine reads what this kernel writes
    if (between) cudaEventRecord(between, stream);
    attn_combine_kernel<128><<<dim3(s.n_kv_heads, s.batch), 128, 0, stream>>>(p, out);
  } else {
    if (d.NG == 4)
      attn_persistent_kernel<64, 4><<<grid, kThreads, d.smem, stream>>>(k_map, v_map, qmap, p);
    else if (d.NG == 2)
      attn_persistent_kernel<64, 2><<<grid, kThreads, d.smem, stream>>>(k_map, v_map, qmap, p);
    else
      attn_persistent_kernel<64, 1><<<grid, kThreads, d.smem, stream>>>(k_map, v_map, qmap, p);
    const cudaError_t le = cudaGetLastError();
    if (le != cudaSuccess) return le;   // the combine reads what this kernel writes
    if (between) cudaEventRecord(between, stream);
    attn_combine_kernel<64><<<dim3(s.n_kv_heads, s.batch), 128, 0, stream>>>(p, out);
  }
  if (launches) *launches += 2;
  return cudaGetLastError();
}

}  // namespace isd
