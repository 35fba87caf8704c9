// Paged causal GQA attention for the ISD block (sm_100a).
//
// Every request's block rows attend to its paged KV prefix plus the earlier
// rows of the same block (strict causal attention over [prefix | block]:
// Bud's Wiki "Introspective Diffusion Language Models", TL;DR and Method;
// the block's own K/V are written to their page slots before this kernel
// runs, so one causal mask over positions covers both parts).
//
// The R rows x G query heads that share KV head g form one query tile of
// R*G rows (28 at stride 4 with Qwen3-8B's 4:1 grouping, 56 with
// Qwen3-32B's 8:1), so each K/V byte is read once per request. Two kernels:
//
// * attn_tc_kernel (head_dim 128, 64-key pages, up to 64 query rows): the
//   decode path. tcgen05 MMAs with TMEM accumulators: S^T = K Q^T and
//   O_t^T = V^T P^T, K and V streamed by TMA through separate rings, one warp
//   issuing the S MMAs and one the PV MMAs, eight softmax warps. One CTA per
//   SM takes a contiguous range of the (request, KV head, 128-key tile)
//   sequence, balanced by tiles plus a fixed cost per segment; the pairs cut
//   between CTAs are merged by attn_combine_tc_kernel. Launched right after
//   the QKV reduction with programmatic stream serialisation, so its first
//   tiles of earlier steps' K/V load before it waits for that reduction.
// * attn_persistent_kernel (the other shapes): work unit = (request, KV
//   head, key split); a producer warp streams 64-key tiles with TMA into a
//   ring; four consumer warps run QK^T and PV on mma.sync bf16 tensor cores
//   with an fp32 online softmax; key groups are merged through shared
//   memory, splits by attn_combine_kernel.
#include <algorithm>
#include <cstdlib>
#include <string>
#include <vector>

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
  // tcgen05 kernel: balanced contiguous tile ranges
  int32_t max_parts;           // partial slots per (request, KV head)
  int32_t min_tiles;           // fewest tiles per CTA (fewer CTAs for small work)
  int32_t kstages, vstages;    // K and V ring slots
  int32_t* status;
  // rows of a request hold one block at consecutive positions (a decode
  // step): K/V tiles of keys below its first row are not written by the
  // QKV reduction and may be loaded before waiting for it
  int32_t prefix_early;
  // launched with programmatic stream serialisation right after the QKV
  // reduction that writes q and the block's K/V rows: nothing it writes is
  // read before griddep_wait()
  int32_t pdl;
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

// kend[b]: keys request b attends to; base[b]: exclusive prefix of the
// per-request split counts (base[B] = total). Ends with __syncthreads.
__device__ void build_items(const AttnParams& p, int* kend, int* base) {
  for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
    int ke = 0;
    for (int r = 0; r < p.R; ++r) ke = max(ke, p.row_pos[b * p.R + r] + 1);
    ke = min(ke, p.maxp * p.page_size);
    kend[b] = ke;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    // one warp scans the split counts: lane l owns a contiguous run of requests
    const int lane = threadIdx.x;
    const int per = (p.B + 31) / 32;
    const int b0 = lane * per, b1 = min(p.B, b0 + per);
    int local = 0;
    for (int b = b0; b < b1; ++b) local += kend[b] > 0 ? (kend[b] + p.split_keys - 1) / p.split_keys : 0;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int b = b0; b < b1; ++b) {
      base[b] = run;
      run += kend[b] > 0 ? (kend[b] + p.split_keys - 1) / p.split_keys : 0;
    }
    if (lane == 31) base[p.B] = incl;
  }
  __syncthreads();
}

__device__ __forceinline__ void build_items(const AttnParams& p, ItemTable& t) {
  build_items(p, t.kend, t.base);
}

// item -> (b, g, split): items are ordered request-major, then KV head, then split.
__device__ __forceinline__ void decode_item(const AttnParams& p, const int* base, int item, int& b,
                                            int& g, int& sp) {
  int lo = 0, hi = p.B;   // find b with base[b]*nkv <= item < base[b+1]*nkv
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (base[mid] * p.nkv <= item) lo = mid; else hi = mid;
  }
  b = lo;
  const int ns = base[b + 1] - base[b];
  const int rem = item - base[b] * p.nkv;
  g = rem / ns;
  sp = rem % ns;
}

__device__ __forceinline__ void decode_item(const AttnParams& p, const ItemTable& t, int item,
                                            int& b, int& g, int& sp) {
  decode_item(p, t.base, item, b, g, sp);
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

// ---------------------------------------------------------------------------
// tcgen05 variant (head_dim 128, 64-key pages, at most 64 query rows per KV
// head, in tiles of NP = 32 or 64 rows): the contractions run on the
// 5th-generation tensor cores with fp32 accumulators in tensor memory, so the
// tile math no longer competes with the HBM stream. At NP = 64 (Qwen3-32B's
// 56 rows; prefill passes) S and O take all 512 TMEM columns, P^T rows are
// 128 bytes (128-byte swizzle) and the V ring is one slot shorter.
//
// Per 128-key tile (two pages) of a work item:
//   S^T[key][row] = K Q^T     UMMA M = 128 keys, N = 32 rows, K = 128 dims
//   P = exp2(S * scale - m)   softmax warps: TMEM lane = key, column = row
//   O_t^T[dim][row] = V^T P^T UMMA M = 128 dims (V read MN-major), N = 32,
//                             K = 128 keys; P^T staged in shared memory as
//                             [key][row] (MN-major B, 64-byte swizzle), so
//                             a thread's 16 rows of one key are two 16-byte
//                             stores
//   O = O * alpha + O_t       softmax warps, registers (lane = dim)
// Warps 0-7 (two per TMEM lane quadrant) run the softmax and accumulate O;
// warp 8 is the TMA producer, warp 9 issues the S MMAs and warp 10 the PV
// MMAs, so neither kind waits behind the other. S and O_t tiles are
// double-buffered in tensor memory: the S MMA of tile t+1 runs while the
// softmax warps work on tile t. K and V tiles sit in separate rings: a K
// slot is free again as soon as S has been computed from it, and only the V
// slot is held through the softmax, which keeps more of the ring's bytes in
// flight from HBM. Each contraction accumulates into two column blocks (S:
// dims 0-63 and 64-127; PV: keys 0-63 and 64-127) issued alternately: one
// chain of dependent small MMAs is latency-bound, two interleaved chains are
// not, and the softmax warps add the two halves as they read them. The row
// positions of the next work segment are loaded while the current one runs.
// The work split and the partial-sum format are shared with the mma.sync
// kernel; the same combine kernel finishes.
constexpr int kTcKeys = 128;                 // keys per tile (two 64-key pages)
constexpr int kTcMaxNP = 64;                 // most query rows per tile (UMMA N: 32 or 64)
constexpr int kTcSoftWarps = 8;              // two per TMEM lane quadrant
constexpr int kTcThreads = (kTcSoftWarps + 3) * 32;
constexpr int kTcSlot = kTcKeys * 128 * 2;        // one K or V tile, 32 KB
constexpr int kTcHalf = 64 * 128;                 // one [64 keys][64 dims] box, 8 KB
constexpr int kTcBars = 256;
constexpr int kTcMinTiles = 2;                    // fewest tiles per working CTA
constexpr int kTcMaxStages = 3;                   // slots per ring (barriers: 2 per slot + 16)
// Per NP (query rows of a tile: 32, or 64 for groups of up to 64 rows):
// Q: two 64-dim halves of NP rows; P^T: [128 keys][NP rows] bf16; reduction
// scratch and row state
__host__ __device__ constexpr int tc_qbuf(int np) { return 2 * np * 128; }
__host__ __device__ constexpr int tc_pbuf(int np) { return kTcKeys * np * 2; }
__host__ __device__ constexpr int tc_misc(int np) { return np <= 32 ? 2048 : 3072; }

// Max or sum of v[0..15] over the 32 lanes, reduce-scatter style: after 16
// shuffles lanes 2i and 2i+1 both hold the reduction of value i.
template <bool kMax>
__device__ __forceinline__ float lane_reduce16(float (&v)[16], int lane) {
#pragma unroll
  for (int off = 16; off >= 2; off >>= 1) {
    const int h = off / 2;               // values kept this step
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = upper ? v[i] : v[i + h];
      const float keep = upper ? v[i + h] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, off);
      v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  const float other = __shfl_xor_sync(0xffffffffu, v[0], 1);
  return kMax ? fmaxf(v[0], other) : v[0] + other;
}

// 2^x with the hardware approximation (flushes denormal results to zero;
// 2^-126 is far below what a softmax weight needs).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_ld_32x32_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Max of v over the 32 lanes of the warp, returned to every lane.
__device__ __forceinline__ float warp_redux_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// MN-major, 64-byte swizzle: 32 MN elements per 64-byte row, rows along K
// 64 B apart, 8-row groups 512 B apart (SBO); one 32-element MN block.
__device__ __forceinline__ uint64_t sw64_desc_mn(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(8192 >> 4) << 16;
  d |= static_cast<uint64_t>(512 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(4) << 61;
  return d;
}

__device__ __forceinline__ uint64_t sw128_desc_mn(uint32_t addr, uint32_t lbo_bytes) {
  // MN-major, 128-byte swizzle: 64 MN elements per 128-byte row, rows along
  // K 128 B apart, 8-row groups 1024 B apart (SBO), 64-element MN blocks
  // lbo_bytes apart (LBO).
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Work of the tcgen05 kernel: the (request, KV head) pairs in one sequence,
// request-major, then head. Pair (b, g) occupies nt_b + tc_seg_cost(p) units:
// the first tc_seg_cost(p) stand for the fixed cost of starting and finishing
// a segment (row state, partial-output write, the pipeline drain at its end),
// then one unit per 128-key tile. CTA c of the C working CTAs takes units
// [c U / C, (c+1) U / C), so a CTA whose range crosses many short pairs gets
// fewer tiles. A maximal run of one pair's tiles inside a CTA's range is a
// segment; it leaves its partial output in slot (b * nkv + g) * max_parts +
// (c - the CTA of the pair's first tile).

struct TcSeg {
  int b, g, t0, len, slot;
};

struct TcRange {
  int64_t x, hi, U;
  int C, c;   // working CTAs; this CTA
};

// The split functions serve the kernel and, unchanged, the host-side query
// isd_attention_split.
__host__ __device__ __forceinline__ int64_t i64min(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t i64max(int64_t a, int64_t b) { return a > b ? a : b; }

__host__ __device__ __forceinline__ int tc_cta_of(int64_t x, int64_t U, int C) {
  return static_cast<int>(((x + 1) * C - 1) / U);
}

// A segment's fixed cost in tile units: 3 at 32 query rows, 5 at 64 (the
// row state and the partial write double; measured best at each size:
// attention 4.44 vs 4.54 ms per step at 2 and 4.52 at 5 for Qwen3-8B widths,
// batch 64; 16.46 vs 17.12 ms at 3 for Qwen3-32B widths).
__host__ __device__ __forceinline__ int tc_seg_cost(const AttnParams& p) { return p.RG > 32 ? 5 : 3; }

// First unit of request b (base[b] = 128-key tiles of the requests before b).
__host__ __device__ __forceinline__ int64_t tc_ubase(const AttnParams& p, const int* base, int b) {
  return static_cast<int64_t>(p.nkv) * (base[b] + static_cast<int64_t>(tc_seg_cost(p)) * b);
}

// Working CTAs: each takes at least min_tiles units.
__host__ __device__ __forceinline__ int tc_ctas(const AttnParams& p, int64_t U, int grid) {
  return static_cast<int>(i64max(1, i64min(grid, U / p.min_tiles)));
}

// The unit range of CTA c of a grid of `grid` CTAs.
__host__ __device__ __forceinline__ TcRange tc_range(const AttnParams& p, const int* base, int grid,
                                                     int c) {
  TcRange r;
  r.U = tc_ubase(p, base, p.B);
  r.C = tc_ctas(p, r.U, grid);
  r.c = c;
  r.x = c < r.C ? c * r.U / r.C : 0;
  r.hi = c < r.C ? (c + 1) * r.U / r.C : 0;
  return r;
}

__host__ __device__ __forceinline__ bool tc_next(const AttnParams& p, const int* base, TcRange& r,
                                                 TcSeg& sg) {
  while (r.x < r.hi) {
    int lo = 0, hi = p.B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (tc_ubase(p, base, mid) <= r.x) lo = mid; else hi = mid;
    }
    const int b = lo;
    const int nt = base[b + 1] - base[b];
    const int sc = tc_seg_cost(p);
    const int w = nt + sc;
    const int64_t x0b = tc_ubase(p, base, b);
    const int rem = static_cast<int>(r.x - x0b);
    const int g = rem / w, off = rem % w;
    const int64_t first = x0b + static_cast<int64_t>(g) * w + sc;   // the pair's first tile
    if (off < sc) {
      r.x = first;   // start of the pair's tiles (of the next pair when nt = 0)
      continue;
    }
    sg.b = b;
    sg.g = g;
    sg.t0 = off - sc;
    sg.len = static_cast<int>(i64min(r.hi - r.x, nt - sg.t0));
    const int part = r.c - tc_cta_of(first, r.U, r.C);
    sg.slot = part < p.max_parts ? (b * p.nkv + sg.g) * p.max_parts + part : -1;
    r.x += sg.len;
    return true;
  }
  return false;
}

// Combine for the tcgen05 kernel's balanced ranges: (request b, KV head g)
// has parts from CTAs c(first tile) .. c(last tile), in slots
// (b * nkv + g) * max_parts + 0 .. parts - 1. One CTA of 128 threads takes
// kCombRows query rows q0 .. q0 + 7 of the pair: per row the parts' softmax
// masses give weights (16 lanes per row, each over parts lane, lane + 16,
// ...), then each output is the weighted sum of the parts in part order,
// with kCombBatch parts' loads in flight per round trip.
constexpr int kCombRows = 8;
constexpr int kCombBatch = 4;
template <int NP>
__device__ __forceinline__ void combine_rows_tc(const AttnParams& p, const int* base, int C_grid,
                                                int b, int g, int q0, float (*w)[kMaxSplits],
                                                __nv_bfloat16* out) {
  constexpr int HD = 128, NT = 128;
  static_assert(NT == kCombRows * 16 && kMaxSplits == 16 * 4, "16 lanes x 4 parts per row");
  const int tid = threadIdx.x;
  const int64_t U = tc_ubase(p, base, p.B);
  const int nt = base[b + 1] - base[b];
  int parts = 0;
  if (nt > 0) {
    const int C = tc_ctas(p, U, C_grid);
    const int sc = tc_seg_cost(p);
    const int64_t first = tc_ubase(p, base, b) + static_cast<int64_t>(g) * (nt + sc) + sc;
    parts = tc_cta_of(first + nt - 1, U, C) - tc_cta_of(first, U, C) + 1;
  }
  if (parts > p.max_parts || parts > kMaxSplits) {
    if (tid == 0) flag(p.status, ISD_DEV_BAD_STATE);
    parts = 0;
  }
  const int64_t slot0 = static_cast<int64_t>(b * p.nkv + g) * p.max_parts;
  {
    const int r = tid >> 4, k = tid & 15;
    const int qi = q0 + r;
    float2 ml[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int sp = k + 16 * u;
      ml[u] = sp < parts && qi < p.RG ? __ldcg(&p.part_ml[(slot0 + sp) * NP + qi])
                                      : make_float2(-INFINITY, 0.f);
    }
    float M = fmaxf(fmaxf(ml[0].x, ml[1].x), fmaxf(ml[2].x, ml[3].x));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float Rm = M == -INFINITY ? 0.f : M;
    float ws[4], L = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      ws[u] = k + 16 * u < parts ? ml[u].y * exp2f(ml[u].x - Rm) : 0.f;
      L += ws[u];
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (k + 16 * u < parts) w[r][k + 16 * u] = ws[u] * inv;
  }
  __syncthreads();
  constexpr int kVec = kCombRows * (HD / 4) / NT;   // float4 outputs per thread
  float4 acc[kVec];
#pragma unroll
  for (int j = 0; j < kVec; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < parts; s0 += kCombBatch) {
    float4 v[kCombBatch][kVec];
#pragma unroll
    for (int u = 0; u < kCombBatch; ++u) {
#pragma unroll
      for (int j = 0; j < kVec; ++j) {
        const int i = tid + j * NT;
        const int qi = q0 + i / (HD / 4), d = (i % (HD / 4)) * 4;
        v[u][j] = s0 + u < parts && qi < p.RG
                      ? __ldcg(reinterpret_cast<const float4*>(p.part_o + ((slot0 + s0 + u) * NP + qi) * HD + d))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int u = 0; u < kCombBatch; ++u) {
      if (s0 + u < parts) {
#pragma unroll
        for (int j = 0; j < kVec; ++j) {
          const float wsu = w[(tid + j * NT) / (HD / 4)][s0 + u];
          acc[j].x += wsu * v[u][j].x;
          acc[j].y += wsu * v[u][j].y;
          acc[j].z += wsu * v[u][j].z;
          acc[j].w += wsu * v[u][j].w;
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kVec; ++j) {
    const int i = tid + j * NT;
    const int qi = q0 + i / (HD / 4), d = (i % (HD / 4)) * 4;
    if (qi < p.RG) {
      const int r = qi / p.G, h = qi % p.G;
      __align__(8) __nv_bfloat16 o4[4] = {__float2bfloat16_rn(acc[j].x), __float2bfloat16_rn(acc[j].y),
                                          __float2bfloat16_rn(acc[j].z), __float2bfloat16_rn(acc[j].w)};
      *reinterpret_cast<uint2*>(out + (static_cast<int64_t>(b * p.R + r) * p.nq + g * p.G + h) * HD + d) =
          *reinterpret_cast<const uint2*>(o4);
    }
  }
}

template <int NP>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                   const __grid_constant__ CUtensorMap qmap, const AttnParams p) {
  constexpr int NR = NP / 2;                 // query rows per softmax warp
  constexpr int kQBuf = tc_qbuf(NP);
  constexpr int kPBuf = tc_pbuf(NP);
  constexpr int kRowWarps = NP / 32;         // warps that keep the per-row state
  constexpr int kSoftThreads = kTcSoftWarps * 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KS = p.kstages, VS = p.vstages;
  uint8_t* ring_k = smem;                                 // KS x K tile
  uint8_t* ring_v = ring_k + KS * kTcSlot;                // VS x V tile
  uint8_t* qs = ring_v + VS * kTcSlot;                    // 2 x Q
  uint8_t* ps = qs + 2 * kQBuf;                           // P^T
  float* red = reinterpret_cast<float*>(ps + kPBuf);      // [4 quadrants][NP]
  float* m_sh = red + 4 * NP;                             // running max per row (log2 units)
  float* alpha_sh = m_sh + NP;                            // [2][NP] per-tile rescale
  float* l_sh = alpha_sh + 2 * NP;                        // 1 / row sum at item end
  float* mu_sh = l_sh + NP;                               // exponent offset (m, 0 while m = -inf)
  int* pos_sh = reinterpret_cast<int*>(mu_sh + NP);       // row positions of the item
  int* minpos_sh = pos_sh + NP;                           // [kRowWarps]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(red) + tc_misc(NP));
  uint64_t* full_k = bars;                 // [KS] each
  uint64_t* empty_k = full_k + KS;
  uint64_t* full_v = empty_k + KS;         // [VS] each
  uint64_t* empty_v = full_v + VS;
  uint64_t* q_full = empty_v + VS;         // [2]
  uint64_t* q_empty = q_full + 2;          // [2]
  uint64_t* s_full = q_empty + 2;          // [2]
  uint64_t* s_empty = s_full + 2;          // [2]
  uint64_t* o_full = s_empty + 2;          // [2]
  uint64_t* o_empty = o_full + 2;          // [2]
  uint64_t* p_full = o_empty + 2;
  uint64_t* p_empty = p_full + 1;
  uint64_t* drain = p_empty + 1;           // [2]: S issuer, PV issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(bars) + kTcBars);
  int* kend = reinterpret_cast<int*>(tmem_slot + 4);
  int* base = kend + p.B;

  if (threadIdx.x == 0) {
    for (int i = 0; i < KS; ++i) {
      mbar_init(&full_k[i], 1);
      mbar_init(&empty_k[i], 1);
    }
    for (int i = 0; i < VS; ++i) {
      mbar_init(&full_v[i], 1);
      mbar_init(&empty_v[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], kTcSoftWarps);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], kTcSoftWarps);
    }
    mbar_init(p_full, kTcSoftWarps);
    mbar_init(p_empty, 1);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    fence_barrier_init();
  }
  // query rows past the tile's RG rows are never loaded: keep them zero
  for (int i = threadIdx.x; i < 2 * kQBuf / 16; i += blockDim.x)
    reinterpret_cast<int4*>(qs)[i] = make_int4(0, 0, 0, 0);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (warp == 0) {
    tmem_alloc(tmem_slot, 8 * NP);
    tmem_relinquish();
    tc_fence_before();
  }
  build_items(p, kend, base);     // ends with __syncthreads
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // base[b]: tiles of the requests before b (128-key tiles, split_keys = 128)
  if (blockIdx.x == 0)
    for (int b = threadIdx.x; b <= p.B; b += blockDim.x) p.item_base[b] = base[b];
  const bool fits = true;

  if (warp == kTcSoftWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && fits) {
      int tc = 0, it = 0, q_issued = 0, nk = 0;
      bool ok = true;
      // K and V of tile t of a (request b, KV head g) run whose keys start
      // at k_lo and end before k_hi, as ring slot tc
      auto load_kv = [&](int b, int g, int k_lo, int k_hi, int t) -> bool {
        const int32_t* pt = p.page_table + static_cast<int64_t>(b) * p.maxp;
        const int st = tc % KS, sv = tc % VS;
        const uint32_t ph = ((tc / KS) & 1) ^ 1, phv = ((tc / VS) & 1) ^ 1;
        int rows[2];
        for (int j = 0; j < 2; ++j) {
          const int key0 = k_lo + t * kTcKeys + j * 64;
          rows[j] = p.oob_row;
          if (key0 < k_hi) {
            const int page = pt[key0 / 64];
            if (page >= 0 && page < p.num_pages)
              rows[j] = ((p.layer * p.num_pages + page) * p.nkv + g) * 64;
            else
              flag(p.status, ISD_DEV_BAD_PAGE);
          }
        }
        // K as [dim half][page][64 keys][64 dims]: the 128 keys of a dim
        // half are one K-major operand
        if (!mbar_wait(&empty_k[st], ph)) return false;
        uint8_t* ks = ring_k + st * kTcSlot;
        mbar_arrive_expect_tx(&full_k[st], kTcSlot);
        for (int j = 0; j < 2; ++j)
          for (int hh = 0; hh < 2; ++hh)
            tma_load_2d(ks + hh * 2 * kTcHalf + j * kTcHalf, &kmap, &full_k[st], hh * 64, rows[j]);
        ++nk;
        // V as [page][dim half]: each page is 16 keys per MMA k-step, dim
        // halves LBO apart
        if (!mbar_wait(&empty_v[sv], phv)) return false;
        uint8_t* vs = ring_v + sv * kTcSlot;
        mbar_arrive_expect_tx(&full_v[sv], kTcSlot);
        for (int j = 0; j < 2; ++j)
          for (int hh = 0; hh < 2; ++hh)
            tma_load_2d(vs + j * 2 * kTcHalf + hh * kTcHalf, &vmap, &full_v[sv], hh * 64, rows[j]);
        ++tc;
        return true;
      };
      TcRange rg = tc_range(p, base, gridDim.x, blockIdx.x);
      TcSeg sg;
      bool have = tc_next(p, base, rg, sg);
      int pre = 0;   // tiles of the first segment loaded before the wait for q and K/V
      if (p.pdl) {
        if (have && p.prefix_early) {
          // prefix keys only: the block's own rows are the QKV reduction's output
          const int k_lo = sg.t0 * kTcKeys;
          const int k_hi = min(kend[sg.b], k_lo + sg.len * kTcKeys);
          const int prefix_end = kend[sg.b] - p.R;
          while (ok && pre < sg.len && pre < KS && pre < VS &&
                 k_lo + (pre + 1) * kTcKeys <= prefix_end) {
            ok = load_kv(sg.b, sg.g, k_lo, k_hi, pre);
            ++pre;
          }
        }
        griddep_wait();   // the QKV reduction ahead in the stream has finished
      }
      for (; ok && have; have = tc_next(p, base, rg, sg), ++it) {
        const int b = sg.b, g = sg.g;
        const int k_lo = sg.t0 * kTcKeys;
        const int k_hi = min(kend[b], k_lo + sg.len * kTcKeys);
        const int n_tiles = sg.len;
        const int qb = it & 1;
        if (!mbar_wait(&q_empty[qb], ((it >> 1) & 1) ^ 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&q_full[qb], 2 * p.RG * 128);
        for (int hh = 0; hh < 2; ++hh)
          tma_load_3d(qs + qb * kQBuf + hh * (NP * 128), &qmap, &q_full[qb], hh * 64, g * p.G,
                      b * p.R);
        ++q_issued;
        for (int t = it == 0 ? pre : 0; t < n_tiles; ++t) {
          if (!load_kv(b, g, k_lo, k_hi, t)) {
            ok = false;
            break;
          }
        }
      }
      if (!ok) flag(p.status, ISD_DEV_TIMEOUT);
      // copies in flight land before the CTA exits (after a timeout the last
      // K load may have no V load beside it)
      for (int j = max(0, nk - KS); j < nk; ++j)
        if (!mbar_wait(&full_k[j % KS], (j / KS) & 1)) break;
      for (int j = max(0, tc - VS); j < tc; ++j)
        if (!mbar_wait(&full_v[j % VS], (j / VS) & 1)) break;
      if (q_issued > 0) mbar_wait(&q_full[(q_issued - 1) & 1], ((q_issued - 1) >> 1) & 1);
    }
  } else if (warp == kTcSoftWarps + 1) {
    // ------------------------------------------------------------ S issuer
    if (lane == 0 && fits) {
      const uint32_t idesc_s = idesc_bf16(128, NP);
      const uint32_t rk_a = smem_u32(ring_k), q_a = smem_u32(qs);
      int tc = 0, it = 0;
      bool ok = true;
      TcRange rg = tc_range(p, base, gridDim.x, blockIdx.x);
      TcSeg sg;
      for (; ok && tc_next(p, base, rg, sg); ++it) {
        const int n_tiles = sg.len;
        const int qb = it & 1;
        if (!mbar_wait(&q_full[qb], (it >> 1) & 1)) {
          ok = false;
          break;
        }
        const uint64_t b0 = sw128_desc(q_a + qb * kQBuf);
        for (int t = 0; t < n_tiles; ++t, ++tc) {
          const int st = tc % KS;
          if (!mbar_wait(&full_k[st], (tc / KS) & 1) ||
              !mbar_wait(&s_empty[tc & 1], ((tc >> 1) & 1) ^ 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // dims 0-63 and 64-127 accumulate into two column blocks, issued
          // alternately so that consecutive MMAs do not depend on each other
          const uint32_t d = tmem + (tc & 1) * 2 * NP;
          const uint64_t a0 = sw128_desc(rk_a + st * kTcSlot);
          // descriptor start addresses count 16-byte units
#pragma unroll
          for (int i = 0; i < 128 / 16; ++i) {
            const int hh = i & 1, kk = i >> 1;
            umma_bf16(d + hh * NP, a0 + ((hh * 2 * kTcHalf + kk * 32) >> 4),
                      b0 + ((hh * (NP * 128) + kk * 32) >> 4), idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[tc & 1]);
          umma_commit(&empty_k[st]);
        }
        if (!ok) break;
        umma_commit(&q_empty[qb]);   // this item's S MMAs are the last readers of Q
      }
      if (!ok) flag(p.status, ISD_DEV_TIMEOUT);
      // every MMA has finished before tensor memory is freed
      umma_commit(&drain[0]);
      mbar_wait(&drain[0], 0);
    }
  } else if (warp == kTcSoftWarps + 2) {
    // ------------------------------------------------------------ PV issuer
    if (lane == 0 && fits) {
      // A (V^T) and B (P^T) both MN-major
      const uint32_t idesc_o = idesc_bf16(128, NP) | (1u << 15) | (1u << 16);
      const uint32_t rv_a = smem_u32(ring_v);
      // P^T rows of NP bf16: 64 bytes (64-byte swizzle) or 128 bytes (128-byte swizzle)
      const uint64_t b0 = NP == 32 ? sw64_desc_mn(smem_u32(ps)) : sw128_desc_mn(smem_u32(ps), 8192);
      int n_total = 0;
      {
        TcRange rg = tc_range(p, base, gridDim.x, blockIdx.x);
        TcSeg sg;
        while (tc_next(p, base, rg, sg)) n_total += sg.len;
      }
      bool ok = true;
      for (int j = 0; j < n_total; ++j) {
        const int st = j % VS;
        if (!mbar_wait(p_full, j & 1) || !mbar_wait(&o_empty[j & 1], ((j >> 1) & 1) ^ 1) ||
            !mbar_wait(&full_v[st], (j / VS) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // keys 0-63 and 64-127 accumulate into two column blocks, alternately
        const uint32_t d = tmem + 4 * NP + (j & 1) * 2 * NP;
        const uint64_t a0 = sw128_desc_mn(rv_a + st * kTcSlot, kTcHalf);
#pragma unroll
        for (int i = 0; i < kTcKeys / 16; ++i) {
          const int jj = i & 1, kk = i >> 1;   // page jj, 16-key step kk in it
          umma_bf16(d + jj * NP, a0 + ((jj * 2 * kTcHalf + kk * 2048) >> 4),
                    b0 + (((jj * 4 + kk) * 16 * (NP * 2)) >> 4), idesc_o, kk > 0 ? 1u : 0u);
        }
        umma_commit(&o_full[j & 1]);
        umma_commit(&empty_v[st]);
        umma_commit(p_empty);
      }
      if (!ok) flag(p.status, ISD_DEV_TIMEOUT);
      umma_commit(&drain[1]);
      mbar_wait(&drain[1], 0);
    }
  } else if (fits) {
    // ------------------------ softmax / accumulate warps (0 .. kTcSoftWarps - 1)
    // warp w: TMEM lane quadrant w % 4 (keys of S, dims of O) and query
    // rows r0 .. r0 + 15 (TMEM columns), r0 = 16 * (w / 4)
    const int quad = warp & 3;
    const int r0 = (warp >> 2) * NR;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const int kl = quad * 32 + lane;           // key within the tile; dim for O
    // P^T row of this thread's key: NP bf16 (64 or 128 bytes), 16-byte chunks
    // swizzled by key (64- or 128-byte swizzle)
    uint8_t* p_row = ps + kl * (NP * 2);
    const int p_sw = NP == 32 ? (kl >> 1) & 3 : kl & 7;
    const int my_row = warp * 32 + lane;       // the row whose state this thread keeps (warps < kRowWarps)
    float o[NR];
    float ls[NR];
    int tc = 0;
    bool fine = true;
    TcRange rg = tc_range(p, base, gridDim.x, blockIdx.x);
    TcSeg sg;
    bool have = tc_next(p, base, rg, sg);
    // row positions are loaded one segment ahead (warps < kRowWarps, one row per thread)
    int pr_cur = warp < kRowWarps && have && my_row < p.RG ? p.row_pos[sg.b * p.R + my_row / p.G] : -1;
    while (have) {
      TcSeg nx;
      const bool have_nx = tc_next(p, base, rg, nx);
      const int pr_nx =
          warp < kRowWarps && have_nx && my_row < p.RG ? p.row_pos[nx.b * p.R + my_row / p.G] : -1;
      const int b = sg.b;
      const int k_lo = sg.t0 * kTcKeys;
      const int k_hi = min(kend[b], k_lo + sg.len * kTcKeys);
      const int n_tiles = sg.len;
      if (warp < kRowWarps) {
        const int pr = pr_cur;
        pos_sh[my_row] = pr;
        m_sh[my_row] = -INFINITY;
        int mn = my_row < p.RG ? pr : INT_MAX;
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o2));
        if (lane == 0) minpos_sh[warp] = mn;
      }
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        o[r] = 0.f;
        ls[r] = 0.f;
      }
      named_bar_sync(2, kSoftThreads);
      int minpos = minpos_sh[0];
#pragma unroll
      for (int w2 = 1; w2 < kRowWarps; ++w2) minpos = min(minpos, minpos_sh[w2]);
      for (int t = 0; t < n_tiles; ++t, ++tc) {
        const int sb = tc & 1;
        // ---- S tile -> registers
        fine = fine && mbar_wait(&s_full[sb], (tc >> 1) & 1);
        tc_fence_after();
        float x[NR];
#pragma unroll
        for (int gq = 0; gq < NR / 16; ++gq) {
          uint32_t ra[16], rb[16];
          tmem_ld_32x32_x16(lane_base + sb * 2 * NP + r0 + gq * 16, ra);
          tmem_ld_32x32_x16(lane_base + sb * 2 * NP + NP + r0 + gq * 16, rb);
          tmem_ld_wait();
#pragma unroll
          for (int r = 0; r < 16; ++r)
            x[gq * 16 + r] = __uint_as_float(ra[r]) + __uint_as_float(rb[r]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[sb]);
        const int key = k_lo + t * kTcKeys + kl;
        const int last = k_lo + t * kTcKeys + kTcKeys - 1;
        if (!(last < k_hi && last <= minpos)) {
#pragma unroll
          for (int r = 0; r < NR; ++r)
            if (!(key < k_hi && key <= pos_sh[r0 + r])) x[r] = -INFINITY;
        }
        // ---- row max over the tile's 128 keys (raw scores: the scale is
        // positive, so it is applied to the max)
        {
          float mx[NR];
#pragma unroll
          for (int r = 0; r < NR; ++r) mx[r] = warp_redux_max(x[r]);
          if (lane == 0) {
#pragma unroll
            for (int r = 0; r < NR; r += 4)
              *reinterpret_cast<float4*>(red + quad * NP + r0 + r) =
                  make_float4(mx[r], mx[r + 1], mx[r + 2], mx[r + 3]);
          }
        }
        // all softmax warps agree on going on (they share named barriers)
        if (!named_bar_and(2, kSoftThreads, fine)) {
          fine = false;
          break;
        }
        if (warp < kRowWarps) {
          const int q = my_row;
          const float m_old = m_sh[q];
          const float mt = fmaxf(fmaxf(red[q], red[NP + q]), fmaxf(red[2 * NP + q], red[3 * NP + q]));
          const float m_new = fmaxf(m_old, mt * p.scale_log2);
          alpha_sh[sb * NP + q] = m_new == -INFINITY ? 1.f : ex2(m_old - m_new);
          m_sh[q] = m_new;
          // a row with no key yet: every x is -inf and 2^(x - 0) = 0
          mu_sh[q] = m_new == -INFINITY ? 0.f : m_new;
        }
        named_bar_sync(2, kSoftThreads);
        // ---- P = 2^(x scale - m), partial row sums, P^T to shared memory
        // (all shared-memory reads first: a store between them would
        // serialise every row on the possible aliasing)
#pragma unroll
        for (int r = 0; r < NR; r += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(mu_sh + r0 + r);
          const float4 a4 = *reinterpret_cast<const float4*>(alpha_sh + sb * NP + r0 + r);
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
          const float aa[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float e = ex2(fmaf(x[r + i], p.scale_log2, -mm[i]));
            ls[r + i] = ls[r + i] * aa[i] + e;
            x[r + i] = e;
          }
        }
        fine = fine && mbar_wait(p_empty, (tc & 1) ^ 1);
        {
          // rows r0 + 8 cc .. r0 + 8 cc + 7: 16-byte chunk r0 / 8 + cc of the key's row
          const int ch = r0 >> 3;
#pragma unroll
          for (int cc = 0; cc < NR / 8; ++cc) {
            const uint4 cv = make_uint4(pack_bf16(x[8 * cc], x[8 * cc + 1]),
                                        pack_bf16(x[8 * cc + 2], x[8 * cc + 3]),
                                        pack_bf16(x[8 * cc + 4], x[8 * cc + 5]),
                                        pack_bf16(x[8 * cc + 6], x[8 * cc + 7]));
            *reinterpret_cast<uint4*>(p_row + (((ch + cc) ^ p_sw) << 4)) = cv;
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        // ---- O += previous tile's O_t (its PV ran while this tile's S did)
        if (t > 0) {
          const int j = tc - 1;
          fine = fine && mbar_wait(&o_full[j & 1], (j >> 1) & 1);
          tc_fence_after();
#pragma unroll
          for (int gq = 0; gq < NR / 16; ++gq) {
            uint32_t ra[16], rb[16];
            tmem_ld_32x32_x16(lane_base + 4 * NP + (j & 1) * 2 * NP + r0 + gq * 16, ra);
            tmem_ld_32x32_x16(lane_base + 4 * NP + (j & 1) * 2 * NP + NP + r0 + gq * 16, rb);
            tmem_ld_wait();
#pragma unroll
            for (int r = 0; r < 16; ++r)
              o[gq * 16 + r] = o[gq * 16 + r] * alpha_sh[(j & 1) * NP + r0 + gq * 16 + r] +
                               (__uint_as_float(ra[r]) + __uint_as_float(rb[r]));
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&o_empty[j & 1]);
        }
      }
      if (!fine) break;
      if (n_tiles > 0) {
        const int j = tc - 1;
        fine = mbar_wait(&o_full[j & 1], (j >> 1) & 1);
        tc_fence_after();
#pragma unroll
        for (int gq = 0; gq < NR / 16; ++gq) {
          uint32_t ra[16], rb[16];
          tmem_ld_32x32_x16(lane_base + 4 * NP + (j & 1) * 2 * NP + r0 + gq * 16, ra);
          tmem_ld_32x32_x16(lane_base + 4 * NP + (j & 1) * 2 * NP + NP + r0 + gq * 16, rb);
          tmem_ld_wait();
#pragma unroll
          for (int r = 0; r < 16; ++r)
            o[gq * 16 + r] = o[gq * 16 + r] * alpha_sh[(j & 1) * NP + r0 + gq * 16 + r] +
                             (__uint_as_float(ra[r]) + __uint_as_float(rb[r]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_empty[j & 1]);
      }
      // ---- row sums over the 128 key lanes, then the partial output
#pragma unroll
      for (int gq = 0; gq < NR / 16; ++gq) {
        float l16[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) l16[r] = ls[gq * 16 + r];
        const float sm = lane_reduce16<false>(l16, lane);
        if ((lane & 1) == 0) red[quad * NP + r0 + gq * 16 + (lane >> 1)] = sm;
      }
      if (!named_bar_and(2, kSoftThreads, fine)) {
        fine = false;
        break;
      }
      if (warp < kRowWarps) {
        const int q = my_row;
        const float L = (red[q] + red[NP + q]) + (red[2 * NP + q] + red[3 * NP + q]);
        l_sh[q] = L > 0.f ? 1.f / L : 0.f;   // one reciprocal per row
        if (sg.slot >= 0)
          p.part_ml[static_cast<int64_t>(sg.slot) * NP + q] = make_float2(m_sh[q], L);
        else if (q == 0)
          flag(p.status, ISD_DEV_BAD_STATE);
      }
      named_bar_sync(2, kSoftThreads);
      if (sg.slot >= 0) {
        float* po = p.part_o + (static_cast<int64_t>(sg.slot) * NP + r0) * 128 + kl;
#pragma unroll
        for (int r = 0; r < NR; ++r) po[r * 128] = o[r] * l_sh[r0 + r];
      }
      named_bar_sync(2, kSoftThreads);   // row state is rewritten by the next segment
      sg = nx;
      have = have_nx;
      pr_cur = pr_nx;
    }
    if (!fine && lane == 0) flag(p.status, ISD_DEV_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 8 * NP);
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

// The tcgen05 kernel's (request, KV head) pairs: grid (KV head, request,
// groups of kCombRows query rows). (Merging them at the end of the
// attention kernel itself, after a barrier over its grid, measured 0.19 ms
// per step slower: 148 CTAs merged 512 pairs.)
template <int NP>
__global__ void __launch_bounds__(128) attn_combine_tc_kernel(const AttnParams p, int C_grid,
                                                              __nv_bfloat16* out) {
  __shared__ float w[kCombRows][kMaxSplits];
  griddep_launch_dependents();   // the O projection may load its weights meanwhile
  combine_rows_tc<NP>(p, p.item_base, C_grid, blockIdx.y, blockIdx.x, blockIdx.z * kCombRows, w, out);
}

struct Derived {
  int RG, MT, NG, split_keys, max_splits, stages, max_items;
  int min_tiles = 1;
  bool tc;        // the tcgen05 kernel serves this shape
  int np = 32;    // its query rows per tile
  int kstages = 0, vstages = 0;
  size_t smem;
};

// Shared memory of the tcgen05 kernel for a batch of B requests.
size_t tc_smem(int np, int kstages, int vstages, int B) {
  return 1024 + static_cast<size_t>(kstages + vstages) * kTcSlot + 2 * tc_qbuf(np) + tc_pbuf(np) +
         tc_misc(np) + kTcBars +
         16 + (2 * static_cast<size_t>(B) + 1) * sizeof(int);
}

Derived derive(const AttnShape& s) {
  Derived d;
  const int G = s.n_q_heads / s.n_kv_heads;
  d.RG = s.rows_per_req * G;
  d.np = d.RG <= 32 ? 32 : 64;
  d.tc = s.head_dim == 128 && s.page_size == 64 && d.RG <= kTcMaxNP &&
         tc_smem(d.np, 2, 2, s.batch) <= 232448;
  if (d.tc) {
    // one CTA per SM, equal contiguous tile ranges of at least kTcMinTiles
    // tiles; a (request, head) run of n tiles then spans at most
    // ceil(n / kTcMinTiles) + 1 CTAs
    const int64_t max_tiles =
        (static_cast<int64_t>(s.max_pages_per_req) * s.page_size + kTcKeys - 1) / kTcKeys;
    d.split_keys = kTcKeys;
    d.min_tiles = static_cast<int>(
        std::max<int64_t>(kTcMinTiles, (max_tiles + kMaxSplits - 2) / (kMaxSplits - 1)));
    d.max_splits = static_cast<int>((max_tiles + d.min_tiles - 1) / d.min_tiles + 1);
    d.max_items = s.batch * s.n_kv_heads * d.max_splits;
    d.MT = d.np / 16;
    d.NG = 1;
    // the deepest rings that fit, the K ring first (a K slot frees as soon as
    // S is computed, a V slot only after the softmax and PV)
    d.kstages = kTcMaxStages;
    d.vstages = kTcMaxStages;
    while (d.kstages > 2 && tc_smem(d.np, d.kstages, d.vstages, s.batch) > 232448) --d.kstages;
    while (d.vstages > 2 && tc_smem(d.np, d.kstages, d.vstages, s.batch) > 232448) --d.vstages;
    d.stages = d.kstages;
    d.smem = tc_smem(d.np, d.kstages, d.vstages, s.batch);
    return d;
  }
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

int attention_split(const AttnShape& s, const int32_t* kend, int num_sms, int32_t* seg,
                    int seg_capacity, int* n_segments, int* max_parts) {
  const Derived d = derive(s);
  if (!d.tc) return -1;
  AttnParams p{};
  p.B = s.batch;
  p.nkv = s.n_kv_heads;
  p.RG = d.RG;                  // the tile height sets the segment cost
  p.min_tiles = d.min_tiles;
  p.max_parts = d.max_splits;
  // 128-key tile prefix, as the kernel builds it from the row positions
  std::vector<int> base(static_cast<size_t>(s.batch) + 1, 0);
  const int cap = s.max_pages_per_req * s.page_size;
  for (int b = 0; b < s.batch; ++b) {
    const int ke = std::min(std::max(kend[b], 0), cap);
    base[b + 1] = base[b] + (ke + kTcKeys - 1) / kTcKeys;
  }
  int n = 0;
  for (int c = 0; c < num_sms; ++c) {
    TcRange r = tc_range(p, base.data(), num_sms, c);
    TcSeg sg;
    while (tc_next(p, base.data(), r, sg)) {
      if (n < seg_capacity) {
        int32_t* o = seg + static_cast<size_t>(n) * 6;
        o[0] = c;
        o[1] = sg.b;
        o[2] = sg.g;
        o[3] = sg.t0;
        o[4] = sg.len;
        o[5] = sg.slot;
      }
      ++n;
    }
  }
  *n_segments = n;
  *max_parts = d.max_splits;
  return n <= seg_capacity ? 0 : -2;
}

cudaError_t set_wait_limit_attention(long long cycles) { return set_wait_limit_here(cycles); }

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
                             cudaEvent_t between, const QkvReduceArgs* qkv, bool prefix_early,
                             bool pdl) {
  if (s.batch > kMaxBatch) return cudaErrorInvalidValue;
  const Derived d = derive(s);
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  // The layer's QKV reduction (QK-norm, RoPE, q and the block's K/V rows)
  // runs first, as its own kernel. (Run instead as this kernel's prologue,
  // every warp taking (row, head) items before a barrier over the grid, it
  // measured 0.38 ms per step slower at 448 rows and, once the kernel loaded
  // earlier steps' K/V before waiting for the reduction, 0.08 ms slower at
  // 7 rows too.)
  if (qkv != nullptr) {
    const cudaError_t e = launch_qkv_reduce(*qkv, stream);
    if (e != cudaSuccess) return e;
    if (launches) *launches += 1;
  }
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
  p.prefix_early = prefix_early ? 1 : 0;
  // programmatic launch only right after the QKV reduction launched above
  p.pdl = pdl && qkv != nullptr && d.tc ? 1 : 0;
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
  const dim3 grid(sms * kCtasPerSm);
  if (d.tc) {
    static bool tc_attr = false;
    if (!tc_attr) {
      cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(attn_tc_kernel<32>),
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(reinterpret_cast<const void*>(attn_tc_kernel<64>),
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
      if (e != cudaSuccess) return e;
      tc_attr = true;
    }
    p.max_parts = d.max_splits;
    p.min_tiles = d.min_tiles;
    p.kstages = d.kstages;
    p.vstages = d.vstages;
    // cudaLaunchKernelEx returns this launch's own status
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms, 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = d.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.pdl ? 1 : 0;
    const cudaError_t le = d.np == 32 ? cudaLaunchKernelEx(&cfg, attn_tc_kernel<32>, k_map, v_map, qmap, p)
                                      : cudaLaunchKernelEx(&cfg, attn_tc_kernel<64>, k_map, v_map, qmap, p);
    if (le != cudaSuccess) return le;   // the combine reads what this kernel writes
    if (between) cudaEventRecord(between, stream);
    const dim3 cgrid(s.n_kv_heads, s.batch, (d.RG + kCombRows - 1) / kCombRows);
    if (d.np == 32)
      attn_combine_tc_kernel<32><<<cgrid, 128, 0, stream>>>(p, sms, out);
    else
      attn_combine_tc_kernel<64><<<cgrid, 128, 0, stream>>>(p, sms, out);
    if (launches) *launches += 2;
    return cudaGetLastError();
  }
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
