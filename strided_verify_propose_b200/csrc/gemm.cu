// Dense bf16 projection GEMMs on the tcgen05 tensor cores (sm_100a).
//
// Y[m][n_out] = X[m][k] * W[n_out][k]^T, with W a weight matrix in
// nn.Linear layout and X the block's activations. Decode blocks are short
// (m = B * (2N-1) rows, 7..448 at stride 4), so the kernel swaps the roles:
// 128 weight rows form the UMMA M side and all of a CTA's token rows (up to
// 512) form N, so every weight byte is read from HBM once and the fp32
// accumulators of the whole token range sit in tensor memory (<= 512 columns).
//
// Warp roles: warp 0 (one lane) issues TMA loads of a 128x64 weight tile and
// the token tile per K-block into a ring of shared-memory stages; warp 1
// (one lane) issues tcgen05.mma and releases each stage with tcgen05.commit;
// warps 2..9 read the accumulators back with tcgen05.ld (a warp reads the 32
// TMEM lanes of its quadrant, warp % 4; two warps share a quadrant and split
// its columns) and run the epilogue.
//
// Work split, two modes:
// * split-K: one (tile, token chunk, K-split) per CTA; split s writes its
//   partial sums to slice s, which a row-wise kernel adds in a fixed order;
// * stream-K (when there are more tiles than SMs): a persistent grid where
//   each CTA, or 2-SM pair, owns a contiguous range of the (tile, K-block)
//   iterations. Ranges are at least one tile long, so a tile is cut at most
//   once; of its two parts the first to finish parks its fp32 partial in a
//   workspace slot and the second adds it to its own and runs the epilogue.
//   Two addends commute exactly, so results do not depend on which part
//   finishes first, and no CTA ever waits for one that has not started.
// Both are bitwise reproducible run to run.
#include <algorithm>
#include <cmath>
#include <cstring>

#include "common.cuh"
#include "kernels.h"


namespace isd {

namespace {

constexpr int kTileM = 128;                 // weight rows per CTA
constexpr int kTileK = 64;                  // K elements per stage (128 bytes)
constexpr int kStageA = kTileM * kTileK * 2;  // 16 KB
constexpr size_t kMaxSmem = 231424;         // 226 KB dynamic (+ a few static bytes <= 227 KB)
constexpr int kEpiWarps = 8;                // epilogue warps (two per TMEM quadrant)
constexpr int kMaxChunksPerWarp = 8;        // 32-token chunks per epilogue warp (512 tokens / 32 / 2)
constexpr int kRedRows = 2;                 // rows per warp per round of the in-kernel split-K sum
constexpr int kRedSplits = 4;               // splits whose loads are unrolled (more take a loop)
constexpr int kThreads = 64 + 32 * kEpiWarps;

struct GemmParams {
  int32_t m, n_out, kb_total, kb_per_split;
  int32_t n_pad, n_mma, mma_n, box_rows, n_boxes, stages;
  uint32_t tmem_cols;
  int32_t epi;
  float* out;
  __nv_bfloat16* out_act;
  int64_t split_stride;
  int32_t* status;
  // stream-K: `units` CTAs or pairs share the iterations of all tiles
  int32_t streamk, units;
  int64_t iters;      // unit tiles (256-row pair tiles or 128-row tiles) x kb_total
  float* sk_part;     // [units * (pair ? 2 : 1)][n_pad rounded up to 32][128] fp32 partials
  int32_t* sk_sync;   // [units * (pair ? 2 : 1)][2]: arrival count, ready flag
  // the last split (stream-K: the segment ending the tile's base K-blocks)
  // continues over aug_kb K-blocks of a second operand pair (tmap_w2,
  // tmap_x2), accumulating into the same result
  int32_t aug_kb;
  // split-K reduced in the kernel: every split parks its fp32 partial in
  // red[(tile * n_chunks + chunk) * splits + split][tokens][128], then each
  // split sums its share of the tile's token chunks over all splits in split
  // order and writes one output slice; red_cnt[2 * (tile * n_chunks + chunk)]
  // counts arrivals, [.. + 1] departures (the last departure zeroes both)
  int32_t reduce;
  float* red;
  int32_t* red_cnt;
  // reduce == 2: the reduced output is the fused QKV projection; instead of
  // writing it, apply QK-norm and RoPE and write q and the K/V page slots
  QkvReduceArgs qkv;
  // reduce == 3: the reduced output is added to the residual stream and the
  // next RMSNorm follows (after a barrier over the whole grid)
  ResNormArgs rn;
};

// QK-norm + NeoX RoPE + q / KV-page writes for one token row of one
// 128-feature tile of the fused QKV projection, reduced over the splits:
// lane l holds features 4l..4l+3 of the tile (heads of a.head_dim features,
// 128 / head_dim per tile). Per head: RMSNorm over head_dim for q and k,
// rotate-half pairs (i, i + head_dim/2) at the row's absolute position, q to
// the attention input, k and v into the row's page slot.
__device__ __forceinline__ void qkv_row_epilogue(const QkvReduceArgs& a, float4 v, int row, int mt,
                                                 int lane) {
  const int HD = a.head_dim;
  const int f = mt * kTileM + lane * 4;          // first feature of this lane
  const int hd = f / HD, d = f % HD;             // head and its first dim
  const int flags = a.meta.flags[row];
  int pos = a.meta.pos[row];
  const bool write_kv = (flags & kRowWriteKV) && pos >= 0;
  if (pos >= a.max_position) {
    if (lane == 0 && mt == 0) flag(a.status, ISD_DEV_BAD_STATE);
    pos = a.max_position - 1;
  }
  const int rpos = pos < 0 ? 0 : pos;
  float x[4] = {v.x, v.y, v.z, v.w};
  if (hd < a.n_q + a.n_kv) {
    // every lane of the warp holds the same head kind (a tile never mixes
    // q / k with v: q and k widths are multiples of 128)
    const float* nw = hd < a.n_q ? a.q_norm : a.k_norm;
    float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
    // sum over the head's lanes: head_dim / 4 lanes (32 or 16)
    for (int o = HD / 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rstd = rsqrtf(ss / HD + a.eps);
    const float4 w4 = *reinterpret_cast<const float4*>(nw + d);
    x[0] *= rstd * w4.x;
    x[1] *= rstd * w4.y;
    x[2] *= rstd * w4.z;
    x[3] *= rstd * w4.w;
    // the partner dims d +- head_dim/2 sit head_dim/8 lanes away
    float y[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) y[j] = __shfl_xor_sync(0xffffffffu, x[j], HD / 8);
    const bool lower = d < HD / 2;
    const int i0 = lower ? d : d - HD / 2;
    const float2* cs = a.rope + static_cast<int64_t>(rpos) * (HD / 2) + i0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 c = cs[j];
      x[j] = lower ? x[j] * c.x - y[j] * c.y : x[j] * c.x + y[j] * c.y;
    }
  }
  __align__(8) __nv_bfloat16 o4[4] = {__float2bfloat16_rn(x[0]), __float2bfloat16_rn(x[1]),
                                       __float2bfloat16_rn(x[2]), __float2bfloat16_rn(x[3])};
  if (hd < a.n_q) {
    __nv_bfloat16* qo = a.q_out + (static_cast<int64_t>(row) * a.n_q + hd) * HD + d;
    *reinterpret_cast<uint2*>(qo) = *reinterpret_cast<const uint2*>(o4);
  } else if (write_kv) {
    const int b = row / a.rows_per_req;
    const int pidx = pos / a.page_size;
    const int page = pidx < a.max_pages_per_req
                         ? a.page_table[static_cast<int64_t>(b) * a.max_pages_per_req + pidx]
                         : -1;
    if (page < 0 || page >= a.num_pages) {
      if ((lane & (HD / 4 - 1)) == 0) flag(a.status, ISD_DEV_BAD_PAGE);
      return;
    }
    const int64_t slot_base = (static_cast<int64_t>(a.layer) * a.num_pages + page) * a.n_kv;
    const bool is_k = hd < a.n_q + a.n_kv;
    const int g = is_k ? hd - a.n_q : hd - a.n_q - a.n_kv;
    __nv_bfloat16* dst = (is_k ? a.k_pool : a.v_pool) +
                         (((slot_base + g) * a.page_size) + pos % a.page_size) * HD + d;
    *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(o4);
  }
}

// One contiguous run of K-blocks of one tile, processed by one CTA (pair).
struct Segment {
  int ut;          // unit tile (pair tile for pairs)
  int kb_lo, kb_hi;
  int aug;         // K-blocks of the second operand pair after kb_hi (the last split, or
                   // the stream-K segment that holds the tile's last base K-block)
  bool whole;      // covers every K-block of the tile (or split-K mode)
  int slot;        // stream-K workspace slot of a cut tile (per unit boundary)
};

// The idx-th segment of this CTA's work; false past the last one.
template <bool kPair>
__device__ __forceinline__ bool get_segment(const GemmParams& p, int idx, Segment& sg) {
  if (!p.streamk) {
    if (idx > 0) return false;
    const int kb0 = blockIdx.z * p.kb_per_split;
    sg.ut = kPair ? (blockIdx.x >> 1) : blockIdx.x;
    sg.kb_lo = kb0;
    sg.kb_hi = min(p.kb_total, kb0 + p.kb_per_split);
    sg.aug = blockIdx.z == gridDim.z - 1 ? p.aug_kb : 0;
    sg.whole = true;
    sg.slot = -1;
    return true;
  }
  const int u = kPair ? (blockIdx.x >> 1) : blockIdx.x;
  const int64_t b = static_cast<int64_t>(u) * p.iters / p.units;
  const int64_t e = static_cast<int64_t>(u + 1) * p.iters / p.units;
  const int64_t kbt = p.kb_total;
  const int64_t tile = b / kbt + idx;
  const int64_t lo = max(b, tile * kbt), hi = min(e, (tile + 1) * kbt);
  if (lo >= hi) return false;
  sg.ut = static_cast<int>(tile);
  sg.kb_lo = static_cast<int>(lo - tile * kbt);
  sg.kb_hi = static_cast<int>(hi - tile * kbt);
  sg.whole = sg.kb_lo == 0 && sg.kb_hi == p.kb_total;
  // the second operand pair follows a tile's last base K-block; the ranges
  // are cut on base K-blocks only, so the cut points do not depend on it
  sg.aug = sg.kb_hi == p.kb_total ? p.aug_kb : 0;
  // a cut tile straddles the boundary between units s and s + 1: the head
  // part ends unit s's range (slot s = u), the tail part starts unit s + 1's
  // (slot s = u - 1)
  sg.slot = sg.whole ? -1 : (sg.kb_lo == 0 ? u : u - 1);
  return true;
}

// kPair: a cluster of two CTAs (adjacent 128-row weight tiles) runs as one
// 2-SM MMA group (tcgen05 cta_group::2, M = 256). Each CTA stages its own
// 128 weight rows and half of every MMA's token columns, so a pair reads
// the token tile once per 256 weight rows instead of once per 128. The
// leader CTA (rank 0) issues the MMAs; both CTAs' loads complete on the
// leader's full barrier; each commit arrives on the barrier of both CTAs;
// the epilogue warps of both CTAs release the accumulator on the leader's
// tmem_empty barrier. Each CTA's tensor memory holds its own 128 rows x all
// tokens, so the epilogue is the same as for a single CTA.
template <bool kPair, int kNmma>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_bf16_tcgen05(const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ CUtensorMap tmap_x,
                      const __grid_constant__ CUtensorMap tmap_w2,
                      const __grid_constant__ CUtensorMap tmap_x2, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ int epi_mode;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tok0 = blockIdx.y * p.n_pad;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  // token rows this CTA stages per K-block
  const uint32_t b_rows = static_cast<uint32_t>(p.n_boxes * p.box_rows);
  const uint32_t stage_bytes = kStageA + b_rows * 128u;

  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.stages * stage_bytes);
  uint64_t* empty = full + p.stages;
  uint64_t* tmem_full = empty + p.stages;
  uint64_t* tmem_empty = tmem_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tmem_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, kEpiWarps * (kPair ? 2 : 1));
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmap_w);
    prefetch_tensormap(&tmap_x);
    if (p.aug_kb > 0) {
      prefetch_tensormap(&tmap_w2);
      prefetch_tensormap(&tmap_x2);
    }
  }
  if (warp == 0) {
    if (kPair) {
      tmem_alloc_pair(tmem_slot, p.tmem_cols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, p.tmem_cols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  // the peer's barriers are initialised and its tensor memory allocated
  // before any load, MMA or arrive of the pair touches them
  if (kPair) cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer (both CTAs of a pair)
    const uint64_t pol_w = policy_evict_first();
    const uint64_t pol_x = policy_evict_last();
    const uint32_t tx = (kPair ? 2u : 1u) * stage_bytes;
    int s = 0;
    uint32_t ph = 0;
    int issued = 0;
    bool ok = true;
    Segment sg;
    for (int idx = 0; ok && get_segment<kPair>(p, idx, sg); ++idx) {
      const int mt = kPair ? sg.ut * 2 + static_cast<int>(rank) : sg.ut;
      const int n_base = sg.kb_hi - sg.kb_lo;
      for (int i = 0; i < n_base + sg.aug; ++i) {
        if (!mbar_wait(&empty[s], ph ^ 1) || *abort_flag) {
          flag(p.status, ISD_DEV_TIMEOUT);
          *abort_flag = 1;
          ok = false;
          break;
        }
        uint8_t* sa = smem + s * stage_bytes;
        uint8_t* sb = sa + kStageA;
        const bool aug = i >= n_base;
        const int kc = (aug ? i - n_base : sg.kb_lo + i) * kTileK;
        const CUtensorMap* mw = aug ? &tmap_w2 : &tmap_w;
        const CUtensorMap* mx = aug ? &tmap_x2 : &tmap_x;
        if (kPair) {
          const uint32_t bar = map_to_rank(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&full[s], tx);
          tma_load_2d_pair(sa, mw, bar, kc, mt * kTileM, pol_w);
          for (int bx = 0; bx < p.n_boxes; ++bx)
            tma_load_2d_pair(sb + bx * p.box_rows * 128, mx, bar, kc,
                             tok0 + bx * p.mma_n + static_cast<int>(rank) * p.box_rows, pol_x);
        } else {
          mbar_arrive_expect_tx(&full[s], tx);
          tma_load_2d_hint(sa, mw, &full[s], kc, mt * kTileM, pol_w);
          for (int bx = 0; bx < p.n_boxes; ++bx)
            tma_load_2d_hint(sb + bx * p.box_rows * 128, mx, &full[s], kc,
                             tok0 + bx * p.box_rows, pol_x);
        }
        ++issued;
        if (++s == p.stages) {
          s = 0;
          ph ^= 1;
        }
      }
    }
    if (ok) {
      // Drain: the last commits still arrive on this CTA's empty barriers;
      // wait for them so none lands after the CTA has exited.
      for (int j = max(0, issued - p.stages); j < issued; ++j) {
        if (!mbar_wait(&empty[j % p.stages], (j / p.stages) & 1)) {
          flag(p.status, ISD_DEV_TIMEOUT);
          *abort_flag = 1;
          break;
        }
      }
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ---------------- MMA issuer (the leader of a pair)
    // One thread issues every MMA, so its loop is kept to the bare
    // instructions: descriptors advance by adding the byte offset >> 4 to
    // precomputed bases (smem addresses stay below 2^18, inside the 14-bit
    // address field), and the k-steps and MMAs of a stage are unrolled.
    const uint32_t idesc = idesc_bf16(kPair ? 256u : 128u, static_cast<uint32_t>(p.mma_n));
    const uint32_t base = smem_u32(smem);
    const uint64_t da0 = sw128_desc(base);
    const uint64_t db0 = sw128_desc(base + kStageA);
    const uint64_t d_stage = stage_bytes >> 4;
    // offset between consecutive MMAs' token tiles in this CTA, >> 4
    const uint64_t d_mma = (static_cast<uint64_t>(kPair ? p.box_rows : p.mma_n) * 128u) >> 4;
    const uint32_t tmem1 = tmem + static_cast<uint32_t>(p.mma_n);
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    Segment sg;
    for (int idx = 0; ok && get_segment<kPair>(p, idx, sg); ++idx) {
      // the epilogue has read the previous segment's accumulators
      if (!mbar_wait(tmem_empty, (idx & 1) ^ 1)) {
        flag(p.status, ISD_DEV_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int n_kb = sg.kb_hi - sg.kb_lo + sg.aug;
      for (int i = 0; i < n_kb; ++i) {
        if (!mbar_wait(&full[s], ph)) {
          flag(p.status, ISD_DEV_TIMEOUT);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t da = da0 + static_cast<uint64_t>(s) * d_stage;
        const uint64_t db = db0 + static_cast<uint64_t>(s) * d_stage;
#pragma unroll
        for (int kk = 0; kk < kTileK / 16; ++kk) {
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          if (kPair) {
            umma_bf16_pair(tmem, da + 2 * kk, db + 2 * kk, idesc, acc);
            if (kNmma == 2) umma_bf16_pair(tmem1, da + 2 * kk, db + d_mma + 2 * kk, idesc, acc);
          } else {
            umma_bf16(tmem, da + 2 * kk, db + 2 * kk, idesc, acc);
            if (kNmma == 2) umma_bf16(tmem1, da + 2 * kk, db + d_mma + 2 * kk, idesc, acc);
          }
        }
        if (kPair)
          umma_commit_pair(&empty[s]);
        else
          umma_commit(&empty[s]);
        if (++s == p.stages) {
          s = 0;
          ph ^= 1;
        }
      }
      if (!ok) break;
      if (kPair)
        umma_commit_pair(tmem_full);
      else
        umma_commit(tmem_full);
    }
  } else if (warp >= 2) {
    // ---------------- epilogue: TMEM -> registers -> global
    const int ew = warp - 2;
    const int quad = warp & 3;             // TMEM lanes 32 * quad .. + 31
    const int half = ew >> 2;              // which of the quadrant's two warps
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const int nchunk = (p.n_pad + 31) / 32;  // tmem_cols >= 32 * nchunk
    const uint32_t empty_addr = kPair ? map_to_rank(smem_u32(tmem_empty), 0) : 0u;
    const int split = p.streamk ? 0 : static_cast<int>(blockIdx.z);
    Segment sg;
    for (int idx = 0; get_segment<kPair>(p, idx, sg); ++idx) {
      // every epilogue warp takes the same branch (they share named barriers)
      const bool ok =
          named_bar_and(1, 32 * kEpiWarps, mbar_wait(tmem_full, idx & 1) && !*abort_flag);
      if (!ok) {
        if (lane == 0) flag(p.status, ISD_DEV_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int mt = kPair ? sg.ut * 2 + static_cast<int>(rank) : sg.ut;
      // cut tile: 1 = first part to finish (park the partial), 2 = second
      // (add the parked partial, then the normal epilogue), 3 = second after
      // a timeout (status flagged, nothing written); 4 = a split of an
      // in-kernel reduced split-K tile (park the partial, then reduce)
      int mode = 0;
      float* part = nullptr;
      int32_t* sync = nullptr;
      const int red_tile = mt * static_cast<int>(gridDim.y) + static_cast<int>(blockIdx.y);
      if (p.reduce) {
        mode = 4;
        part = p.red + (static_cast<int64_t>(red_tile) * gridDim.z + split) * nchunk * 32 * kTileM;
      } else if (!sg.whole) {
        const int slot = sg.slot * (kPair ? 2 : 1) + static_cast<int>(rank);
        part = p.sk_part + static_cast<int64_t>(slot) * nchunk * 32 * kTileM;
        sync = p.sk_sync + 2 * slot;
        if (ew == 0 && lane == 0) {
          int m_ = atomicAdd(&sync[0], 1) == 0 ? 1 : 2;
          if (m_ == 2) {
            // the first part's CTA is in its epilogue: wait for its flag
            const long long t0 = clock64();
            const long long limit = *const_cast<volatile long long*>(&g_wait_limit);
            while (ld_acquire_gpu(&sync[1]) == 0) {
              if (clock64() - t0 > limit) {
                flag(p.status, ISD_DEV_TIMEOUT);
                m_ = 3;
                break;
              }
            }
          }
          epi_mode = m_;
        }
        named_bar_sync(1, 32 * kEpiWarps);
        mode = epi_mode;
      }
      // TMEM loads run one chunk ahead of the chunk being written out
      uint32_t r[32];
      if (half < nchunk) tmem_ld_32x32_async(lane_addr + half * 32, r);
      // SwiGLU tiles: the bf16 results stay in registers until every chunk is
      // read, then the accumulator is released and the stores follow, so the
      // next tile's MMAs run while this tile's results leave
      const bool staged = p.epi == kEpiSiluMul && (mode == 0 || mode == 2);
      bool released = false;
      if (staged) {
        const bool hi = lane >= 16;
        uint32_t ov[kMaxChunksPerWarp * 8];   // [chunk][8]: token pairs (2k, 2k + 1) of 16 results
#pragma unroll
        for (int ci = 0; ci < kMaxChunksPerWarp; ++ci) {
          const int c = half + 2 * ci;
          if (c < nchunk) {
            float v[32];
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
            if (c + 2 < nchunk) tmem_ld_32x32_async(lane_addr + (c + 2) * 32, r);
            if (mode == 2) {
              const float* pp = part + static_cast<int64_t>(c * 32) * kTileM + quad * 32 + lane;
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] += __ldcg(pp + j * kTileM);
            }
            // gate and up rows of a feature sit 16 lanes apart: low lanes
            // finish even tokens, high lanes odd ones
#pragma unroll
            for (int k = 0; k < 16; k += 2) {
              float o2[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int j = 2 * (k + e);
                const float x_j = __shfl_xor_sync(0xffffffffu, v[j], 16);
                const float x_j1 = __shfl_xor_sync(0xffffffffu, v[j + 1], 16);
                const float g = hi ? x_j1 : v[j];
                const float u = hi ? v[j + 1] : x_j;
                o2[e] = silu_mul(g, u);
              }
              __nv_bfloat162 pk = __floats2bfloat162_rn(o2[0], o2[1]);
              ov[ci * 8 + k / 2] = *reinterpret_cast<uint32_t*>(&pk);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (kPair)
            mbar_arrive_cluster(empty_addr);
          else
            mbar_arrive(tmem_empty);
        }
        released = true;
        const int half_n = p.n_out / 2;
        const int f = mt * 64 + quad * 16 + (lane & 15);
#pragma unroll
        for (int ci = 0; ci < kMaxChunksPerWarp; ++ci) {
          const int c = half + 2 * ci;
          if (c < nchunk) {
            const int t0 = tok0 + c * 32;
            const bool full_chunk = c * 32 + 32 <= p.n_pad && t0 + 32 <= p.m;
            __nv_bfloat16* rowp =
                p.out_act + static_cast<int64_t>(t0 + (hi ? 1 : 0)) * half_n + f;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const int jj = 2 * k + (hi ? 1 : 0);
              const uint32_t w = ov[ci * 8 + k / 2];
              const uint16_t bits = (k & 1) ? static_cast<uint16_t>(w >> 16) : static_cast<uint16_t>(w);
              if (full_chunk || (c * 32 + jj < p.n_pad && t0 + jj < p.m))
                *reinterpret_cast<uint16_t*>(rowp) = bits;
              rowp += 2 * half_n;
            }
          }
        }
      }
      for (int c = half; !staged && c < nchunk; c += 2) {
        float v[32];
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (c + 2 < nchunk) tmem_ld_32x32_async(lane_addr + (c + 2) * 32, r);
        const int t0 = tok0 + c * 32;
        // partial slot: rows of 128 fp32, tokens 0 .. 32 * nchunk - 1
        if (mode == 1 || mode == 4) {
          float* pp = part + static_cast<int64_t>(c * 32) * kTileM + quad * 32 + lane;
#pragma unroll
          for (int j = 0; j < 32; ++j) pp[j * kTileM] = v[j];
          continue;
        }
        if (mode == 3) continue;
        if (mode == 2) {
          const float* pp = part + static_cast<int64_t>(c * 32) * kTileM + quad * 32 + lane;
          // L2 loads: another SM wrote the slot
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] += __ldcg(pp + j * kTileM);
        }
        // a chunk whose 32 tokens all exist needs no per-store bounds check
        const bool full_chunk = c * 32 + 32 <= p.n_pad && t0 + 32 <= p.m;
        if (p.epi == kEpiF32) {
          const int f = mt * kTileM + quad * 32 + lane;
          float* rowp = p.out + split * p.split_stride + static_cast<int64_t>(t0) * p.n_out + f;
          if (full_chunk) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              *rowp = v[j];
              rowp += p.n_out;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (c * 32 + j < p.n_pad && t0 + j < p.m) *rowp = v[j];
              rowp += p.n_out;
            }
          }
        } else {
          // Each quadrant's 32 TMEM lanes hold 16 gate rows then the 16 up
          // rows of the same features (see the gate/up layout in isd.h). A
          // lane pairs with lane ^ 16: low lanes finish even tokens, high
          // lanes odd ones.
          const int half_n = p.n_out / 2;
          const bool hi = lane >= 16;
          const int f = mt * 64 + quad * 16 + (lane & 15);
          __nv_bfloat16* rowp =
              p.out_act + static_cast<int64_t>(t0 + (hi ? 1 : 0)) * half_n + f;
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float x_j = __shfl_xor_sync(0xffffffffu, v[j], 16);
            const float x_j1 = __shfl_xor_sync(0xffffffffu, v[j + 1], 16);
            const float g = hi ? x_j1 : v[j];
            const float u = hi ? v[j + 1] : x_j;
            const int jj = j + (hi ? 1 : 0);
            if (full_chunk || (c * 32 + jj < p.n_pad && t0 + jj < p.m))
              *rowp = __float2bfloat16_rn(silu_mul(g, u));
            rowp += 2 * half_n;
          }
        }
      }
      // accumulators read: release them to the MMA issuer (of the pair)
      if (!released) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (kPair)
            mbar_arrive_cluster(empty_addr);
          else
            mbar_arrive(tmem_empty);
        }
      }
      if (mode == 1) {
        // partial parked: publish it
        __threadfence();
        named_bar_sync(1, 32 * kEpiWarps);
        if (ew == 0 && lane == 0) st_release_gpu(&sync[1], 1);
      } else if (mode == 4) {
        // every split of the tile parks its partial; then this split sums
        // its share of the token chunks over the splits, in split order
        __threadfence();
        named_bar_sync(1, 32 * kEpiWarps);
        const int S = static_cast<int>(gridDim.z);
        int32_t* cnt = p.red_cnt + 2 * red_tile;
        if (ew == 0 && lane == 0) {
          atomicAdd(&cnt[0], 1);
          int ok_ = 1;
          const long long t0 = clock64();
          const long long limit = *const_cast<volatile long long*>(&g_wait_limit);
          while (ld_acquire_gpu(&cnt[0]) < S) {
            if (clock64() - t0 > limit) {
              flag(p.status, ISD_DEV_TIMEOUT);
              ok_ = 0;
              break;
            }
          }
          epi_mode = ok_;
        }
        named_bar_sync(1, 32 * kEpiWarps);
        if (epi_mode) {
          const int c_lo = split * nchunk / S, c_hi = (split + 1) * nchunk / S;
          const int t_lo = c_lo * 32, t_hi = min(c_hi * 32, p.n_pad);
          const int64_t sstride = static_cast<int64_t>(nchunk) * 32 * kTileM;
          const float* base = p.red + static_cast<int64_t>(red_tile) * S * sstride;
          // warp ew takes token rows t_lo + ew, + 8, ...; lane l features
          // 4l..4l+3. Rows go kRedRows at a time with every split's load of
          // them (and the residual's) in flight together; the sum still runs
          // in split order.
          const int t_end = min(t_hi, p.m - tok0);
          for (int t = t_lo + ew; t < t_end; t += kEpiWarps * kRedRows) {
            float4 part4[kRedSplits][kRedRows];
            float4 xo[kRedRows];
#pragma unroll
            for (int rr = 0; rr < kRedRows; ++rr) {
              const int tr = t + rr * kEpiWarps;
              const float* q = base + static_cast<int64_t>(tr) * kTileM + lane * 4;
#pragma unroll
              for (int s2 = 0; s2 < kRedSplits; ++s2)
                part4[s2][rr] = (tr < t_end && s2 < S)
                                    ? __ldcg(reinterpret_cast<const float4*>(q + s2 * sstride))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
              xo[rr] = (p.reduce == 3 && tr < t_end)
                           ? *reinterpret_cast<const float4*>(
                                 p.rn.x + static_cast<int64_t>(tok0 + tr) * p.n_out + mt * kTileM + lane * 4)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int rr = 0; rr < kRedRows; ++rr) {
              const int tr = t + rr * kEpiWarps;
              if (tr >= t_end) continue;   // uniform across the warp
              float4 acc = part4[0][rr];
#pragma unroll
              for (int s2 = 1; s2 < kRedSplits; ++s2) {
                if (s2 < S) {
                  acc.x += part4[s2][rr].x;
                  acc.y += part4[s2][rr].y;
                  acc.z += part4[s2][rr].z;
                  acc.w += part4[s2][rr].w;
                }
              }
              // more splits than the unrolled loads cover
              for (int s2 = kRedSplits; s2 < S; ++s2) {
                const float4 d = __ldcg(reinterpret_cast<const float4*>(
                    base + s2 * sstride + static_cast<int64_t>(tr) * kTileM + lane * 4));
                acc.x += d.x;
                acc.y += d.y;
                acc.z += d.z;
                acc.w += d.w;
              }
              if (p.reduce == 2) {
                qkv_row_epilogue(p.qkv, acc, tok0 + tr, mt, lane);
              } else if (p.reduce == 3) {
                // x += the projection; this tile's share of the row's sum of squares
                float4 x4 = xo[rr];
                x4.x += acc.x;
                x4.y += acc.y;
                x4.z += acc.z;
                x4.w += acc.w;
                *reinterpret_cast<float4*>(p.rn.x + static_cast<int64_t>(tok0 + tr) * p.n_out +
                                           mt * kTileM + lane * 4) = x4;
                const float ss = warp_sum(x4.x * x4.x + x4.y * x4.y + x4.z * x4.z + x4.w * x4.w);
                if (lane == 0) p.rn.ss[static_cast<int64_t>(mt) * p.rn.ss_stride + tok0 + tr] = ss;
              } else {
                *reinterpret_cast<float4*>(p.out + static_cast<int64_t>(tok0 + tr) * p.n_out +
                                           mt * kTileM + lane * 4) = acc;
              }
            }
          }
        }
        if (p.reduce == 3) {
          // every row's residual and tile sums are written once every CTA of
          // the grid has passed here; then this split normalises its rows
          const int total = static_cast<int>(gridDim.x * gridDim.y * gridDim.z);
          __threadfence();
          named_bar_sync(1, 32 * kEpiWarps);
          if (ew == 0 && lane == 0) {
            atomicAdd(&p.rn.grid_cnt[0], 1);
            int ok_ = epi_mode;
            const long long t0 = clock64();
            const long long limit = *const_cast<volatile long long*>(&g_wait_limit);
            while (ld_acquire_gpu(&p.rn.grid_cnt[0]) < total) {
              if (clock64() - t0 > limit) {
                flag(p.status, ISD_DEV_TIMEOUT);
                ok_ = 0;
                break;
              }
            }
            epi_mode = ok_;
          }
          named_bar_sync(1, 32 * kEpiWarps);
          if (epi_mode) {
            const int c_lo = split * nchunk / S, c_hi = (split + 1) * nchunk / S;
            const int t_lo = c_lo * 32, t_end = min(min(c_hi * 32, p.n_pad), p.m - tok0);
            const int tiles = p.n_out / kTileM;
            const float4 w4 = *reinterpret_cast<const float4*>(p.rn.norm_w + mt * kTileM + lane * 4);
            // kRedRows rows per round, their loads in flight together; the
            // tile sums of a row are added lane by lane in tile order, then
            // across lanes by the fixed butterfly
            for (int t = t_lo + ew; t < t_end; t += kEpiWarps * kRedRows) {
              float tot[kRedRows];
              float4 xo[kRedRows];
#pragma unroll
              for (int rr = 0; rr < kRedRows; ++rr) {
                const int tr = t + rr * kEpiWarps;
                tot[rr] = 0.f;
                xo[rr] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (tr < t_end) {
                  const int row = tok0 + tr;
                  for (int i = lane; i < tiles; i += 32)
                    tot[rr] += __ldcg(p.rn.ss + static_cast<int64_t>(i) * p.rn.ss_stride + row);
                  xo[rr] = *reinterpret_cast<const float4*>(
                      p.rn.x + static_cast<int64_t>(row) * p.n_out + mt * kTileM + lane * 4);
                }
              }
#pragma unroll
              for (int rr = 0; rr < kRedRows; ++rr) {
                const int tr = t + rr * kEpiWarps;
                if (tr >= t_end) continue;   // uniform across the warp
                const int row = tok0 + tr;
                const float rstd = rsqrtf(warp_sum(tot[rr]) / p.n_out + p.rn.eps);
                __align__(8) __nv_bfloat16 o4[4] = {
                    __float2bfloat16_rn(xo[rr].x * rstd * w4.x), __float2bfloat16_rn(xo[rr].y * rstd * w4.y),
                    __float2bfloat16_rn(xo[rr].z * rstd * w4.z), __float2bfloat16_rn(xo[rr].w * rstd * w4.w)};
                *reinterpret_cast<uint2*>(p.rn.hn + static_cast<int64_t>(row) * p.n_out + mt * kTileM +
                                          lane * 4) = *reinterpret_cast<const uint2*>(o4);
              }
            }
          }
          named_bar_sync(1, 32 * kEpiWarps);
          if (ew == 0 && lane == 0 && atomicAdd(&p.rn.grid_cnt[1], 1) == total - 1) {
            p.rn.grid_cnt[0] = 0;
            p.rn.grid_cnt[1] = 0;
          }
        }
        named_bar_sync(1, 32 * kEpiWarps);
        if (ew == 0 && lane == 0 && atomicAdd(&cnt[1], 1) == S - 1) {
          cnt[0] = 0;
          cnt[1] = 0;
        }
      } else if (mode >= 2) {
        // every read of the parked partial is done: reset the slot
        named_bar_sync(1, 32 * kEpiWarps);
        if (ew == 0 && lane == 0) {
          sync[1] = 0;
          sync[0] = 0;
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  // neither CTA of a pair frees its tensor memory or exits while the other
  // may still read it or signal its barriers
  if (kPair) cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    if (kPair)
      tmem_dealloc_pair(tmem, p.tmem_cols);
    else
      tmem_dealloc(tmem, p.tmem_cols);
  }
}

uint32_t pow2_at_least(uint32_t v) {
  uint32_t r = 32;
  while (r < v) r <<= 1;
  return r;
}

}  // namespace

GemmPlan plan_gemm(int32_t m, int32_t n_out, int32_t k, int32_t force_splits, int32_t max_splits,
                   int32_t num_sms, bool allow_streamk) {
  GemmPlan best;
  const int kb_total = k / kTileK;
  const int m_tiles = n_out / kTileM;
  const int min_chunks = (m + 511) / 512;
  double best_t = 1e30;
  // Measured on B200 (m = 448): one token chunk (all tokens of a CTA in
  // TMEM, two N = 224 MMAs per k-step) beats finer chunks for every
  // projection, and split-K that fills the SMs in one wave beats two waves.
  // So: the fewest chunks that fit TMEM, then the split count whose waves
  // cost least, counting each split's partial-sum traffic.
  const int nch = min_chunks;
  {
    const int tok = (m + nch - 1) / nch;
    const int n_pad = tok <= 256 ? ((tok + 15) / 16) * 16 : ((tok + 31) / 32) * 32;
    const int s_lo = force_splits > 0 ? force_splits : 1;
    const int s_hi = force_splits > 0 ? force_splits : std::min(max_splits, kb_total);
    for (int s = s_lo; s <= s_hi && n_pad <= 512; ++s) {
      const int kbs = (kb_total + s - 1) / s;
      if ((s - 1) * kbs >= kb_total) continue;  // an empty split
      const long units = static_cast<long>(m_tiles) * nch * s;
      const long waves = (units + num_sms - 1) / num_sms;
      // per K-block: ~2 cycles per token column of MMA, or weight streaming
      // when the token count is small
      const double t_kb = std::max(2.0 * n_pad, 700.0) + 250.0;
      const double t_partial = s > 1 ? 0.5 * s * m * (double)n_out * 4.0 / 3400.0 : 0.0;
      const double t = waves * (kbs * t_kb + 5.0 * n_pad + 2000.0) + t_partial;
      if (t < best_t * 0.999) {
        best_t = t;
        best.n_pad = n_pad;
        best.n_chunks = nch;
        best.splits = s;
        best.kb_per_split = kbs;
      }
    }
  }
  if (best.n_pad == 0) return best;
  best.n_mma = best.n_pad > 256 ? 2 : 1;
  best.mma_n = best.n_pad / best.n_mma;
  // 2-SM pairs need an even number of 128-row tiles; mma_n is a multiple of
  // 16 (n_pad is padded to 16, or to 32 when split over two MMAs), so each
  // CTA's half of an MMA's tokens is a whole number of 8-row swizzle atoms.
  best.pair = (m_tiles % 2 == 0 && best.mma_n % 16 == 0) ? 1 : 0;
  if (best.pair) {
    best.box_rows = best.mma_n / 2;
    best.n_boxes = best.n_mma;
  } else {
    best.box_rows = best.n_pad > 256 ? best.n_pad / 2 : best.n_pad;
    best.n_boxes = best.n_pad / best.box_rows;
  }
  // Stream-K when one chunk and one split leave more tiles than one wave
  // holds, and the last wave would be partly idle. Every range spans at
  // least one tile (unit_tiles > cap), so a tile is cut at most once.
  const int per_unit = best.pair ? 2 : 1;
  const int unit_tiles = m_tiles / per_unit;
  const int cap = std::max(1, num_sms / per_unit);
  if (allow_streamk && force_splits <= 0 && best.n_chunks == 1 && best.splits == 1 &&
      unit_tiles > cap && unit_tiles % cap != 0) {
    best.streamk = 1;
    best.units = cap;
  }
  const size_t stage =
      kStageA + static_cast<size_t>(best.n_boxes) * static_cast<size_t>(best.box_rows) * 128;
  const size_t extra = 1024 + 256;
  int stages = static_cast<int>((kMaxSmem - extra) / stage);
  stages = std::min(stages, 8);
  if (!best.streamk) stages = std::min(stages, std::max(best.kb_per_split, 2));
  best.stages = std::max(stages, 2);
  best.tmem_cols = pow2_at_least(static_cast<uint32_t>(best.n_pad));
  best.smem_bytes = best.stages * stage + extra;
  return best;
}

// Workspace layout: the sync words of up to kSkMaxSlots slots at offset 0
// (the same place for every plan, so a plan's partials never overwrite
// another plan's sync words), then the fp32 partials.
constexpr size_t kSkMaxSlots = 512;
constexpr size_t kSkSyncBytes = kSkMaxSlots * 2 * sizeof(int32_t);

size_t gemm_streamk_workspace_bytes(const GemmPlan& plan) {
  if (!plan.streamk) return 0;
  const size_t slots = static_cast<size_t>(plan.units) * (plan.pair ? 2 : 1);
  const size_t rows = (static_cast<size_t>(plan.n_pad) + 31) / 32 * 32;
  return kSkSyncBytes + slots * rows * kTileM * sizeof(float);
}

size_t gemm_streamk_sync_bytes() { return kSkSyncBytes; }

cudaError_t set_wait_limit_gemm(long long cycles) { return set_wait_limit_here(cycles); }

size_t gemm_reduce_floats(const GemmPlan& plan, int32_t n_out) {
  if (plan.splits < 2 || plan.streamk) return 0;
  const size_t rows = (static_cast<size_t>(plan.n_pad) + 31) / 32 * 32;
  return static_cast<size_t>(n_out) * plan.n_chunks * plan.splits * rows;
}

int gemm_reduce_counters(const GemmPlan& plan, int32_t n_out) {
  return 2 * (n_out / kTileM) * plan.n_chunks;
}

int gemm_coresident_ctas(const GemmPlan& plan) {
  auto kernel = plan.pair
                    ? (plan.n_mma == 2 ? gemm_bf16_tcgen05<true, 2> : gemm_bf16_tcgen05<true, 1>)
                    : (plan.n_mma == 2 ? gemm_bf16_tcgen05<false, 2> : gemm_bf16_tcgen05<false, 1>);
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kMaxSmem)) != cudaSuccess)
    return 0;
  if (!plan.pair) {
    int per_sm = 0, dev = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads,
                                                      plan.smem_bytes) != cudaSuccess ||
        cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return 0;
    return per_sm * sms;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem_bytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg) != cudaSuccess) return 0;
  return 2 * clusters;
}

cudaError_t launch_gemm(const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const GemmPlan& plan,
                        int32_t m, int32_t n_out, int32_t k, GemmEpilogue epi, float* out_f32,
                        __nv_bfloat16* out_act, int32_t* status, cudaStream_t stream,
                        void* sk_workspace, size_t sk_workspace_bytes,
                        const GemmAugment* augment, const GemmReduce* reduce,
                        const QkvReduceArgs* qkv, const ResNormArgs* rn) {
  auto kernel = plan.pair
                    ? (plan.n_mma == 2 ? gemm_bf16_tcgen05<true, 2> : gemm_bf16_tcgen05<true, 1>)
                    : (plan.n_mma == 2 ? gemm_bf16_tcgen05<false, 2> : gemm_bf16_tcgen05<false, 1>);
  static bool attr_set = false;
  if (!attr_set) {
    for (auto fn : {gemm_bf16_tcgen05<false, 1>, gemm_bf16_tcgen05<false, 2>,
                    gemm_bf16_tcgen05<true, 1>, gemm_bf16_tcgen05<true, 2>}) {
      cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(kMaxSmem));
      if (e != cudaSuccess) return e;
    }
    attr_set = true;
  }
  if (plan.n_mma != 1 && plan.n_mma != 2) return cudaErrorInvalidValue;
  GemmParams p;
  p.m = m;
  p.n_out = n_out;
  p.kb_total = k / kTileK;
  p.kb_per_split = plan.kb_per_split;
  p.n_pad = plan.n_pad;
  p.n_mma = plan.n_mma;
  p.mma_n = plan.mma_n;
  p.box_rows = plan.box_rows;
  p.n_boxes = plan.n_boxes;
  p.stages = plan.stages;
  p.tmem_cols = plan.tmem_cols;
  p.epi = epi;
  p.out = out_f32;
  p.out_act = out_act;
  p.split_stride = static_cast<int64_t>(m) * n_out;
  p.status = status;
  p.streamk = plan.streamk;
  p.units = plan.units;
  p.iters = 0;
  p.sk_part = nullptr;
  p.sk_sync = nullptr;
  p.aug_kb = 0;
  p.reduce = 0;
  p.red = nullptr;
  p.red_cnt = nullptr;
  if (reduce != nullptr) {
    // every CTA of the grid must be resident at once (the splits of a tile
    // wait for each other), one slice of fp32 output, partials and counters
    // in the caller's buffers
    const int64_t ctas = static_cast<int64_t>(n_out / kTileM) * plan.n_chunks * plan.splits;
    if (epi != kEpiF32 || plan.streamk || plan.splits < 2 || reduce->red == nullptr ||
        reduce->counters == nullptr || reduce->red_floats < gemm_reduce_floats(plan, n_out) ||
        reduce->n_counters < gemm_reduce_counters(plan, n_out) || ctas > reduce->coresident)
      return cudaErrorInvalidValue;
    p.reduce = 1;
    p.red = reduce->red;
    p.red_cnt = reduce->counters;
    if (qkv != nullptr) {
      // q / k widths are whole tiles, so a tile never mixes v with q or k
      const int hd = qkv->head_dim;
      if ((hd != 64 && hd != 128) || (qkv->n_q * hd) % kTileM || (qkv->n_kv * hd) % kTileM ||
          (qkv->n_q + 2 * qkv->n_kv) * hd != n_out || qkv->rows_per_req < 1)
        return cudaErrorInvalidValue;
      p.reduce = 2;
      p.qkv = *qkv;
    } else if (rn != nullptr) {
      if (rn->x == nullptr || rn->norm_w == nullptr || rn->hn == nullptr || rn->ss == nullptr ||
          rn->grid_cnt == nullptr || rn->ss_stride < m)
        return cudaErrorInvalidValue;
      p.reduce = 3;
      p.rn = *rn;
    }
  }
  const CUtensorMap* tw2 = &tmap_w;
  const CUtensorMap* tx2 = &tmap_x;
  if (augment != nullptr && augment->k > 0) {
    if (augment->k % kTileK != 0 || augment->tmap_w == nullptr || augment->tmap_x == nullptr)
      return cudaErrorInvalidValue;
    p.aug_kb = augment->k / kTileK;
    tw2 = augment->tmap_w;
    tx2 = augment->tmap_x;
  }
  const int per_unit = plan.pair ? 2 : 1;
  dim3 grid(n_out / kTileM, plan.n_chunks, plan.splits);
  if (plan.streamk) {
    const size_t need = gemm_streamk_workspace_bytes(plan);
    if (sk_workspace == nullptr || sk_workspace_bytes < need || plan.n_chunks != 1 ||
        plan.splits != 1 || plan.units < 1 ||
        static_cast<size_t>(plan.units) * per_unit > kSkMaxSlots)
      return cudaErrorInvalidValue;
    const int64_t unit_tiles = n_out / kTileM / per_unit;
    p.iters = unit_tiles * p.kb_total;
    if (p.iters / plan.units < p.kb_total) return cudaErrorInvalidValue;  // a range < one tile
    p.sk_sync = static_cast<int32_t*>(sk_workspace);
    p.sk_part = reinterpret_cast<float*>(static_cast<uint8_t*>(sk_workspace) + kSkSyncBytes);
    grid = dim3(plan.units * per_unit, 1, 1);
  }
  if (!plan.pair) {
    kernel<<<grid, kThreads, plan.smem_bytes, stream>>>(tmap_w, tmap_x, *tw2, *tx2, p);
    return cudaGetLastError();
  }
  if (grid.x % 2 != 0) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, tmap_w, tmap_x, *tw2, *tx2, p);
}

}  // namespace isd
