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
//
// Plans with more than 32 token columns run even tile counts as 2-SM pairs
// (tcgen05 cta_group::2, M = 256). Launched with programmatic stream
// serialisation, the producer loads the first ring of weight tiles before
// it waits for the kernel ahead. The fp32 epilogue can also write, per 32
// output rows, the max, the sum of exp and the first argmax of each token's
// results (the LM head's accept statistics).
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
  // kEpiF32 with one slice: per (token, 32-row slab) max, sum of exp(y - max)
  // and first argmax of the finished result, [m][n_out / 32]
  float4* row_stats;
  // launched with programmatic stream serialisation: the producer loads the
  // first ring of weight tiles, then waits for the kernel ahead of it
  int32_t pdl;
};

// For each of the 32 values a lane holds (value j of every lane is token j;
// lane L holds output row f0 + L): the max over the warp's 32 rows, the sum
// of exp(y - max) over them and the first row reaching the max. A butterfly:
// at offset o a lane keeps half of its 2o entries and merges the partner's
// copy of that half into them (31 merges per lane), so that lane L ends with
// token L's result. In a merge one of the two rescale factors is exp(0) = 1,
// so each merge takes one exponential, of minus the gap between the maxima.
__device__ __forceinline__ void slab_stats32(const float (&v)[32], int f, int lane, float& m_out,
                                             float& s_out, int& i_out) {
  float m[16], s[16];
  int id[16];
  {
    const bool lo = (lane & 16) == 0;
    const int fb = f ^ 16;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float a = lo ? v[k] : v[k + 16];
      const float b = __shfl_xor_sync(0xffffffffu, lo ? v[k + 16] : v[k], 16);
      s[k] = 1.f + __expf(-fabsf(a - b));
      m[k] = fmaxf(a, b);
      id[k] = (b > a || (b == a && fb < f)) ? fb : f;
    }
  }
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) {
    const bool lo = (lane & o) == 0;
#pragma unroll
    for (int k = 0; k < o; ++k) {
      const float am = lo ? m[k] : m[k + o], as = lo ? s[k] : s[k + o];
      const int ai = lo ? id[k] : id[k + o];
      const float bm = __shfl_xor_sync(0xffffffffu, lo ? m[k + o] : m[k], o);
      const float bs = __shfl_xor_sync(0xffffffffu, lo ? s[k + o] : s[k], o);
      const int bi = __shfl_xor_sync(0xffffffffu, lo ? id[k + o] : id[k], o);
      const float gap = am - bm;
      const float e = __expf(-fabsf(gap));
      s[k] = gap >= 0.f ? fmaf(bs, e, as) : fmaf(as, e, bs);
      m[k] = fmaxf(am, bm);
      id[k] = (bm > am || (bm == am && bi < ai)) ? bi : ai;
    }
  }
  m_out = m[0];
  s_out = s[0];
  i_out = id[0];
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
    // With programmatic launch, the weight tiles of the first p.stages
    // iterations are loaded before the wait for the kernel ahead (they do
    // not depend on it; the fresh ring needs no empty wait); the main pass
    // then adds only their token tiles. `pre` counts those iterations.
    int pre = 0;
    if (p.pdl) {
      int s0 = 0;
      for (int idx = 0; pre < p.stages && get_segment<kPair>(p, idx, sg); ++idx) {
        const int mt = kPair ? sg.ut * 2 + static_cast<int>(rank) : sg.ut;
        const int n_base = sg.kb_hi - sg.kb_lo;
        for (int i = 0; i < n_base + sg.aug && pre < p.stages; ++i, ++pre, ++s0) {
          uint8_t* sa = smem + s0 * stage_bytes;
          const bool aug = i >= n_base;
          const int kc = (aug ? i - n_base : sg.kb_lo + i) * kTileK;
          const CUtensorMap* mw = aug ? &tmap_w2 : &tmap_w;
          if (kPair) {
            const uint32_t bar = map_to_rank(smem_u32(&full[s0]), 0);
            if (leader) mbar_arrive_expect_tx(&full[s0], tx);
            tma_load_2d_pair(sa, mw, bar, kc, mt * kTileM, pol_w);
          } else {
            mbar_arrive_expect_tx(&full[s0], tx);
            tma_load_2d_hint(sa, mw, &full[s0], kc, mt * kTileM, pol_w);
          }
        }
      }
      griddep_wait();
    }
    for (int idx = 0; ok && get_segment<kPair>(p, idx, sg); ++idx) {
      const int mt = kPair ? sg.ut * 2 + static_cast<int>(rank) : sg.ut;
      const int n_base = sg.kb_hi - sg.kb_lo;
      for (int i = 0; i < n_base + sg.aug; ++i) {
        const bool w_done = issued < pre;   // weights already on their way
        if (!w_done && (!mbar_wait(&empty[s], ph ^ 1) || *abort_flag)) {
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
          if (!w_done) {
            if (leader) mbar_arrive_expect_tx(&full[s], tx);
            tma_load_2d_pair(sa, mw, bar, kc, mt * kTileM, pol_w);
          }
          for (int bx = 0; bx < p.n_boxes; ++bx)
            tma_load_2d_pair(sb + bx * p.box_rows * 128, mx, bar, kc,
                             tok0 + bx * p.mma_n + static_cast<int>(rank) * p.box_rows, pol_x);
        } else {
          if (!w_done) {
            mbar_arrive_expect_tx(&full[s], tx);
            tma_load_2d_hint(sa, mw, &full[s], kc, mt * kTileM, pol_w);
          }
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
      // a timeout (status flagged, nothing written)
      int mode = 0;
      float* part = nullptr;
      int32_t* sync = nullptr;
      if (!sg.whole) {
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
      for (int c = half; c < nchunk; c += 2) {
        float v[32];
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (c + 2 < nchunk) tmem_ld_32x32_async(lane_addr + (c + 2) * 32, r);
        const int t0 = tok0 + c * 32;
        // partial slot: rows of 128 fp32, tokens 0 .. 32 * nchunk - 1
        if (mode == 1) {
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
          if (p.row_stats != nullptr) {
            // lane L: token t0 + L over this quadrant's 32 output rows
            float sm, ss;
            int si;
            slab_stats32(v, f, lane, sm, ss, si);
            if (c * 32 + lane < p.n_pad && t0 + lane < p.m)
              p.row_stats[static_cast<int64_t>(t0 + lane) * (p.n_out / 32) + (f >> 5)] =
                  make_float4(sm, ss, sm, __int_as_float(si));
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (kPair)
          mbar_arrive_cluster(empty_addr);
        else
          mbar_arrive(tmem_empty);
      }
      if (mode == 1) {
        // partial parked: publish it
        __threadfence();
        named_bar_sync(1, 32 * kEpiWarps);
        if (ew == 0 && lane == 0) st_release_gpu(&sync[1], 1);
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
  // With at most 32 token columns a pair shares almost nothing (a few KB of
  // tokens per K-block) and its cluster set-up and barriers are pure cost:
  // single CTAs there (batch 1: 4.40 -> 4.28 ms per step).
  best.pair = (m_tiles % 2 == 0 && best.mma_n % 16 == 0 && best.n_pad > 32) ? 1 : 0;
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
  // (12 slots for the few-token plans of batch-1 decode measured the same
  // step time as 8)
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

cudaError_t launch_gemm(const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const GemmPlan& plan,
                        int32_t m, int32_t n_out, int32_t k, GemmEpilogue epi, float* out_f32,
                        __nv_bfloat16* out_act, int32_t* status, cudaStream_t stream,
                        void* sk_workspace, size_t sk_workspace_bytes,
                        const GemmAugment* augment, float4* row_stats, bool pdl) {
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
  p.row_stats = row_stats;
  p.pdl = pdl ? 1 : 0;
  if (row_stats != nullptr && (epi != kEpiF32 || plan.splits != 1 || n_out % 32 != 0))
    return cudaErrorInvalidValue;
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
  // cudaLaunchKernelEx returns this launch's own status (never an error
  // left behind by an earlier call)
  if (plan.pair && grid.x % 2 != 0) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (plan.pair) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 2;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, tmap_w, tmap_x, *tw2, *tx2, p);
}

}  // namespace isd
