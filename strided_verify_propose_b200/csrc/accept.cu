// Verify, resample and propose from the block logits, then the length and
// KV-page bookkeeping (sm_100a).
//
// The rule is the pages' min(1, p/q) acceptance with the anchor p of this
// forward and the proposal q of the previous one, tested left to right; at
// the first rejection the slot is refilled from norm(max(0, p - q)) and the
// block restarts there (Bud's Wiki "Introspective Diffusion Language
// Models", Key claims and Method; Agentic Commons blog, "How Introspective
// Strided Decoding Works": the rule is speculative sampling's and keeps the
// AR distribution). Proposals at MASK rows are by argmax (the serving
// default, Bud's Wiki Key claims) or sampled. No probability row is written
// back to HBM except the q rows that SAMPLE mode must keep for the next step.
//
// Kernels:
//  1. accept_stats: one CTA per (row, 8192-token chunk): max, sum of
//     exp(z - max) and the first argmax of the chunk, from the logits, or
//     (accept_slab_stats) from the statistics of 32-token slabs that the
//     LM head's epilogue wrote beside the logits.
//  2. accept_decide: one CTA per request: combines the chunk statistics,
//     runs the sequential accept tests, draws the new token by inverse CDF
//     (chunk totals first, then a block scan inside one chunk) and reads or
//     samples the proposals; in SAMPLE mode write_q_rows then stores the
//     proposals' q rows with one CTA per 8192-token chunk.
//  3. bookkeep: one CTA: lengths += 1 + A; pages for the next block from
//     the free list by an exclusive prefix sum in request order.
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace isd {

namespace {

constexpr int kChunk = 8192;
constexpr int kThreads = 256;
constexpr int kItems = 8;                      // elements per thread per scan tile
constexpr int kTile = kThreads * kItems;       // 2048

struct ChunkStat {
  float m;     // max of the chunk
  float s;     // sum of exp(z - m)
  float amax;  // value of the first maximum
  int idx;     // its index
};

__device__ __forceinline__ void merge_ms(float& m, float& s, float m2, float s2) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) {
    m = m2;
    s = s2;
    return;
  }
  const float mn = fmaxf(m, m2);
  s = s * expf(m - mn) + s2 * expf(m2 - mn);
  m = mn;
}

__device__ __forceinline__ void merge_arg(float& v, int& i, float v2, int i2) {
  if (v2 > v || (v2 == v && i2 < i)) {
    v = v2;
    i = i2;
  }
}

__global__ void __launch_bounds__(kThreads)
    accept_stats_kernel(const float* logits, int32_t vocab, int32_t n_chunks, ChunkStat* stats) {
  // every load of the thread is issued before any arithmetic (vocab is a
  // multiple of 4, so a float4 is either wholly inside the chunk or outside)
  constexpr int kVec = kChunk / (kThreads * 4);
  const int c = blockIdx.x, row = blockIdx.y;
  const int lo = c * kChunk, hi = min(vocab, lo + kChunk);
  const float* z = logits + static_cast<int64_t>(row) * vocab;
  float4 v4[kVec];
#pragma unroll
  for (int j = 0; j < kVec; ++j) {
    const int i = lo + (j * kThreads + threadIdx.x) * 4;
    v4[j] = i < hi ? *reinterpret_cast<const float4*>(z + i)
                   : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
  }
  // the thread's max with its first index, then the sum of exp(z - max)
  float av = -INFINITY;
  int ai = INT_MAX;
#pragma unroll
  for (int j = 0; j < kVec; ++j) {
    const int i = lo + (j * kThreads + threadIdx.x) * 4;
    if (i < hi) {
      merge_arg(av, ai, v4[j].x, i);
      merge_arg(av, ai, v4[j].y, i + 1);
      merge_arg(av, ai, v4[j].z, i + 2);
      merge_arg(av, ai, v4[j].w, i + 3);
    }
  }
  float m = av, s = 0.f;
  if (m != -INFINITY) {
#pragma unroll
    for (int j = 0; j < kVec; ++j)
      s += (expf(v4[j].x - m) + expf(v4[j].y - m)) + (expf(v4[j].z - m) + expf(v4[j].w - m));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    const float v2 = __shfl_xor_sync(0xffffffffu, av, o);
    const int i2 = __shfl_xor_sync(0xffffffffu, ai, o);
    merge_ms(m, s, m2, s2);
    merge_arg(av, ai, v2, i2);
  }
  __shared__ ChunkStat part[kThreads / 32];
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) part[w] = ChunkStat{m, s, av, ai};
  __syncthreads();
  if (threadIdx.x == 0) {
    ChunkStat r = part[0];
    for (int k = 1; k < kThreads / 32; ++k) {
      merge_ms(r.m, r.s, part[k].m, part[k].s);
      merge_arg(r.amax, r.idx, part[k].amax, part[k].idx);
    }
    stats[static_cast<int64_t>(row) * n_chunks + c] = r;
  }
}

// The same chunk statistics from the LM head's per-(row, 32-token slab)
// statistics: thread t merges slab c * 256 + t, then the warps and the
// block merge as above (max and argmax are exact; the sums differ from the
// logits pass only in the order of the additions).
__global__ void __launch_bounds__(kThreads)
    accept_slab_stats_kernel(const float4* slab, int32_t vocab, int32_t n_chunks, ChunkStat* stats) {
  static_assert(kChunk == 32 * kThreads, "one slab per thread");
  const int c = blockIdx.x, row = blockIdx.y;
  const int n_slabs = vocab / 32;
  const int sl = c * kThreads + threadIdx.x;
  float m = -INFINITY, s = 0.f, av = -INFINITY;
  int ai = INT_MAX;
  if (sl < n_slabs) {
    const float4 t = slab[static_cast<int64_t>(row) * n_slabs + sl];
    m = t.x;
    s = t.y;
    av = t.z;
    ai = __float_as_int(t.w);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    const float v2 = __shfl_xor_sync(0xffffffffu, av, o);
    const int i2 = __shfl_xor_sync(0xffffffffu, ai, o);
    merge_ms(m, s, m2, s2);
    merge_arg(av, ai, v2, i2);
  }
  __shared__ ChunkStat part[kThreads / 32];
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) part[w] = ChunkStat{m, s, av, ai};
  __syncthreads();
  if (threadIdx.x == 0) {
    ChunkStat r = part[0];
    for (int k = 1; k < kThreads / 32; ++k) {
      merge_ms(r.m, r.s, part[k].m, part[k].s);
      merge_arg(r.amax, r.idx, part[k].amax, part[k].idx);
    }
    stats[static_cast<int64_t>(row) * n_chunks + c] = r;
  }
}

// One row's max, sum of exp(z - max) and first argmax from its chunk
// statistics, by one warp (lane-strided, then a butterfly); every caller
// merges in this order, so all of them get the same bits.
__device__ __forceinline__ void row_stats(const ChunkStat* st, int n_chunks, int lane, float& m,
                                          float& s, int& ai) {
  m = -INFINITY;
  s = 0.f;
  float av = -INFINITY;
  ai = INT_MAX;
  for (int c = lane; c < n_chunks; c += 32) {
    merge_ms(m, s, st[c].m, st[c].s);
    merge_arg(av, ai, st[c].amax, st[c].idx);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    const float v2 = __shfl_xor_sync(0xffffffffu, av, o);
    const int i2 = __shfl_xor_sync(0xffffffffu, ai, o);
    merge_ms(m, s, m2, s2);
    merge_arg(av, ai, v2, i2);
  }
}

// Block-wide inclusive scan of one float per thread (kThreads threads).
__device__ float block_incl_scan(float v, float* warp_tot) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) warp_tot[w] = v;
  __syncthreads();
  float base = 0.f;
  for (int k = 0; k < w; ++k) base += warp_tot[k];
  __syncthreads();
  return v + base;
}

struct DecideShared {
  float M[16], S[16];
  int amax[16];
  float W[64];           // per-chunk weights of the row being sampled (n_chunks <= 64)
  float warp_tot[kThreads / 32];
  float red[kThreads / 32];
  int found, last_pos;
  int A, new_tok;
  int props[8];
};

// Weight of token i in the row being sampled (mode decides the formula):
//  bonus:          exp(z_i - M)
//  residual argmax: exp(z_i - M), 0 at the rejected draft
//  residual sample: max(0, exp(z_i - M) / S - q_i)
struct Weights {
  const float* z;
  const float* q;   // residual-sample only
  float M, inv_S;
  int excluded;     // residual argmax: the rejected draft, else -1
  __device__ __forceinline__ float operator()(int i) const {
    if (q) return fmaxf(0.f, expf(z[i] - M) * inv_S - q[i]);
    return i == excluded ? 0.f : expf(z[i] - M);
  }
};

// Inverse-CDF draw: smallest i with running sum > u * total, scanning in
// token order; chunk totals W[] locate the chunk, a block scan the token.
// Falls back to the last token with positive weight when rounding leaves
// no crossing. Block-uniform result.
__device__ int sample_row(const Weights& wf, int vocab, int n_chunks, float u, DecideShared& sh) {
  float total = 0.f;
  for (int c = 0; c < n_chunks; ++c) total += sh.W[c];
  const float target = u * total;
  int cstar = -1;
  float base = 0.f;
  {
    float run = 0.f;
    for (int c = 0; c < n_chunks; ++c) {
      if (run + sh.W[c] > target) {
        cstar = c;
        base = run;
        break;
      }
      run += sh.W[c];
    }
    if (cstar < 0) {
      for (int c = n_chunks - 1; c >= 0; --c)
        if (sh.W[c] > 0.f) {
          cstar = c;
          base = run - sh.W[c];
          break;
        }
      if (cstar < 0) return 0;
    }
  }
  const int lo = cstar * kChunk, hi = min(vocab, lo + kChunk);
  if (threadIdx.x == 0) {
    sh.found = INT_MAX;
    sh.last_pos = -1;
  }
  __syncthreads();
  float run = base;
  for (int t0 = lo; t0 < hi; t0 += kTile) {
    float w[kItems];
    float local = 0.f;
    int lastk = -1;
    const int i0 = t0 + threadIdx.x * kItems;
#pragma unroll
    for (int k = 0; k < kItems; ++k) {
      w[k] = (i0 + k < hi) ? wf(i0 + k) : 0.f;
      local += w[k];
      if (w[k] > 0.f) lastk = i0 + k;
    }
    if (lastk >= 0) atomicMax(&sh.last_pos, lastk);
    const float incl = block_incl_scan(local, sh.warp_tot);
    const float excl = incl - local;
    if (local > 0.f && run + excl <= target && target < run + incl) {
      float acc = run + excl;
      int hit = -1, lastpos = -1;
#pragma unroll
      for (int k = 0; k < kItems; ++k) {
        acc += w[k];
        if (w[k] > 0.f) lastpos = i0 + k;
        if (hit < 0 && acc > target) hit = i0 + k;
      }
      // rounding can let two neighbours both claim the crossing: the lower index wins
      atomicMin(&sh.found, hit >= 0 ? hit : lastpos);
    }
    if (threadIdx.x == kThreads - 1) sh.red[0] = incl;
    __syncthreads();
    run += sh.red[0];
    const int f = sh.found;
    __syncthreads();
    if (f != INT_MAX) return f;
  }
  return sh.last_pos >= 0 ? sh.last_pos : lo;
}

__global__ void __launch_bounds__(kThreads) accept_decide_kernel(const AcceptArgs a,
                                                                 const ChunkStat* stats,
                                                                 int32_t n_chunks, int32_t* qsrc) {
  __shared__ DecideShared sh;
  const int b = blockIdx.x;
  const int N = a.stride_n, R = 2 * N - 1;
  const int V = a.vocab;
  const bool propose_sample = a.flags & ISD_PROPOSE_SAMPLE;
  const bool greedy = a.flags & ISD_VERIFY_GREEDY;
  int n = a.n_draft[b];
  if (n != 0 && n != N - 1) n = 0;   // flagged by the assembly kernel
  const float* u = a.uniforms + static_cast<int64_t>(b) * R;
  const int32_t* pend = a.pending + static_cast<int64_t>(b) * N;

  // combine chunk statistics: one warp per row
  {
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int r = w; r < R; r += kThreads / 32) {
      float m, s;
      int ai;
      row_stats(stats + (static_cast<int64_t>(b) * R + r) * n_chunks, n_chunks, lane, m, s, ai);
      if (lane == 0) {
        sh.M[r] = m;
        sh.S[r] = s;
        sh.amax[r] = ai;
      }
    }
  }
  __syncthreads();

  // sequential accept tests, left to right
  if (threadIdx.x == 0) {
    int A = n;
    for (int j = 1; j <= n; ++j) {
      const int row = b * R + j - 1;
      int d = pend[j];
      if (d < 0 || d >= V) {
        flag(a.status, ISD_DEV_BAD_TOKEN);
        A = j - 1;
        break;
      }
      bool ok;
      if (greedy) {
        ok = d == sh.amax[j - 1];
      } else {
        const float p = expf(a.logits[static_cast<int64_t>(row) * V + d] - sh.M[j - 1]) / sh.S[j - 1];
        const float qd =
            propose_sample ? a.q_cache[(static_cast<int64_t>(b) * (N - 1) + j - 1) * V + d] : 1.f;
        ok = u[j - 1] * qd < p;
      }
      if (!ok) {
        A = j - 1;
        break;
      }
    }
    sh.A = A;
  }
  __syncthreads();
  const int A = sh.A;

  // the new final token from row A
  int new_tok;
  {
    const int row = b * R + A;
    const float* z = a.logits + static_cast<int64_t>(row) * V;
    if (greedy) {
      new_tok = sh.amax[A];
    } else {
      Weights wf{z, nullptr, sh.M[A], 1.f / sh.S[A], -1};
      const ChunkStat* st = stats + static_cast<int64_t>(row) * n_chunks;
      if (A < n && propose_sample) {
        wf.q = a.q_cache + (static_cast<int64_t>(b) * (N - 1) + A) * V;
        for (int c = 0; c < n_chunks; ++c) {
          const int lo = c * kChunk, hi = min(V, lo + kChunk);
          float part = 0.f;
          for (int i = lo + threadIdx.x; i < hi; i += kThreads) part += wf(i);
          part = warp_sum(part);
          if ((threadIdx.x & 31) == 0) sh.red[threadIdx.x >> 5] = part;
          __syncthreads();
          if (threadIdx.x == 0) {
            float t = 0.f;
            for (int k = 0; k < kThreads / 32; ++k) t += sh.red[k];
            sh.W[c] = t;
          }
          __syncthreads();
        }
        float tot = 0.f;
        for (int c = 0; c < n_chunks; ++c) tot += sh.W[c];
        __syncthreads();
        if (!(tot > 0.f)) {         // p == q exactly: the residual is empty, draw from p
          wf.q = nullptr;
          if (threadIdx.x < n_chunks) sh.W[threadIdx.x] = st[threadIdx.x].s * expf(st[threadIdx.x].m - wf.M);
        }
      } else {
        if (A < n) {
          const int d = pend[A + 1];
          wf.excluded = (d >= 0 && d < V) ? d : -1;   // an out-of-range draft was flagged already
        }
        if (threadIdx.x < n_chunks) {
          float wc = st[threadIdx.x].s * expf(st[threadIdx.x].m - wf.M);
          if (wf.excluded >= 0 && wf.excluded / kChunk == static_cast<int>(threadIdx.x))
            wc = fmaxf(0.f, wc - expf(z[wf.excluded] - wf.M));
          sh.W[threadIdx.x] = wc;
        }
      }
      __syncthreads();
      new_tok = sample_row(wf, V, n_chunks, u[N - 1], sh);
    }
  }
  __syncthreads();

  // proposals from MASK rows n+1..n+N-1 when nothing was rejected
  if (A == n) {
    for (int i = 1; i < N; ++i) {
      const int r = n + i;
      if (!propose_sample) {
        if (threadIdx.x == 0) sh.props[i] = sh.amax[r];
      } else {
        // (the q row itself is written by write_q_rows_kernel, over the
        // whole device, once this kernel has read the previous q rows)
        const int row = b * R + r;
        const float* z = a.logits + static_cast<int64_t>(row) * V;
        const float M = sh.M[r], inv_S = 1.f / sh.S[r];
        const ChunkStat* st = stats + static_cast<int64_t>(row) * n_chunks;
        if (threadIdx.x < n_chunks) sh.W[threadIdx.x] = st[threadIdx.x].s * expf(st[threadIdx.x].m - M);
        __syncthreads();
        Weights wf{z, nullptr, M, inv_S, -1};
        const int d = sample_row(wf, V, n_chunks, u[N + i - 1], sh);
        if (threadIdx.x == 0) sh.props[i] = d;
        __syncthreads();
      }
    }
  }
  __syncthreads();

  if (threadIdx.x == 0) {
    if (propose_sample) qsrc[b] = A == n ? n : -1;
    a.accepted[b] = A;
    if (a.committed) {
      int32_t* cm = a.committed + static_cast<int64_t>(b) * N;
      for (int j = 0; j < N; ++j) cm[j] = j < A ? pend[j + 1] : (j == A ? new_tok : -1);
    }
    int32_t* pw = a.pending + static_cast<int64_t>(b) * N;
    pw[0] = new_tok;
    for (int i = 1; i < N; ++i) pw[i] = (A == n) ? sh.props[i] : -1;
    a.n_draft[b] = (A == n) ? N - 1 : 0;
  }
}

// SAMPLE mode: the proposal rows' q' = softmax(z), one CTA per (8192-token
// chunk, request, proposal i), for the requests whose proposals stand
// (qsrc[b] = n >= 0: rows n + 1 .. n + N - 1). q = exp(z - M) * (1 / S)
// with the row's M and S merged exactly as the decide kernel merges them.
// Every load of a thread is issued before its arithmetic.
__global__ void __launch_bounds__(kThreads)
    write_q_rows_kernel(const AcceptArgs a, const ChunkStat* stats, int32_t n_chunks,
                        const int32_t* qsrc) {
  constexpr int kVec = kChunk / (kThreads * 4);
  __shared__ float ms[2];
  const int c = blockIdx.x, b = blockIdx.y, i = blockIdx.z + 1;
  const int N = a.stride_n, R = 2 * N - 1, V = a.vocab;
  const int n = qsrc[b];
  if (n < 0) return;
  const int row = b * R + n + i;
  if (threadIdx.x < 32) {
    float m, s;
    int ai;
    row_stats(stats + static_cast<int64_t>(row) * n_chunks, n_chunks, threadIdx.x, m, s, ai);
    if (threadIdx.x == 0) {
      ms[0] = m;
      ms[1] = s;
    }
  }
  __syncthreads();
  const float M = ms[0], inv_S = 1.f / ms[1];
  const float* z = a.logits + static_cast<int64_t>(row) * V;
  float* qo = a.q_cache + (static_cast<int64_t>(b) * (N - 1) + i - 1) * V;
  const int lo = c * kChunk, hi = min(V, lo + kChunk);
  float4 v4[kVec];
#pragma unroll
  for (int j = 0; j < kVec; ++j) {
    const int t = lo + (j * kThreads + threadIdx.x) * 4;
    v4[j] = t < hi ? *reinterpret_cast<const float4*>(z + t) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int j = 0; j < kVec; ++j) {
    const int t = lo + (j * kThreads + threadIdx.x) * 4;
    if (t < hi)
      *reinterpret_cast<float4*>(qo + t) =
          make_float4(expf(v4[j].x - M) * inv_S, expf(v4[j].y - M) * inv_S,
                      expf(v4[j].z - M) * inv_S, expf(v4[j].w - M) * inv_S);
  }
}

// seq_len += 1 + A; request b receives the pages that cover its next block,
// taken from the free list at head + (exclusive prefix sum of the counts of
// requests 0..b-1). Nothing is handed out if the list cannot cover all.
__global__ void __launch_bounds__(1024) bookkeep_kernel(const AcceptArgs a) {
  __shared__ int warp_tot[32];
  __shared__ int s_total, s_ok;
  const int b = threadIdx.x;
  const int R = 2 * a.stride_n - 1, P = a.page_size;
  int have = 0, want = 0, L1 = 0;
  bool full = false;
  if (b < a.batch) {
    const int L = a.seq_len[b];
    L1 = L + 1 + a.accepted[b];
    have = (L + R + P - 1) / P;
    want = (L1 + R + P - 1) / P;
    if (want > a.max_pages_per_req) full = true;
  }
  int cnt = want - have;
  // block exclusive scan of cnt
  int v = cnt;
  const int lane = b & 31, w = b >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) warp_tot[w] = v;
  if (b == 0) s_ok = 1;
  __syncthreads();
  int base = 0;
  for (int k = 0; k < w; ++k) base += warp_tot[k];
  const int excl = base + v - cnt;
  if (b == blockDim.x - 1) s_total = base + v;
  if (full) atomicAnd(&s_ok, 0);
  __syncthreads();
  const int head = *a.free_head;
  const bool ok = s_ok && head + s_total <= a.free_count;
  if (b < a.batch) {
    a.seq_len[b] = L1;
    if (ok) {
      int32_t* pt = a.page_table + static_cast<int64_t>(b) * a.max_pages_per_req;
      for (int j = 0; j < cnt; ++j) pt[have + j] = a.free_list[head + excl + j];
    }
  }
  __syncthreads();
  if (b == 0) {
    if (ok) {
      *a.free_head = head + s_total;
    } else {
      flag(a.status, s_ok ? ISD_DEV_POOL_EXHAUSTED : ISD_DEV_TABLE_FULL);
    }
  }
}

}  // namespace

// Workspace: the chunk statistics, then (256-byte aligned) qsrc[batch].
static size_t stats_bytes(int32_t batch, int32_t stride_n, int32_t vocab) {
  const int n_chunks = (vocab + kChunk - 1) / kChunk;
  const size_t b = static_cast<size_t>(batch) * (2 * stride_n - 1) * n_chunks * sizeof(ChunkStat);
  return (b + 255) & ~static_cast<size_t>(255);
}

size_t accept_workspace_bytes(int32_t batch, int32_t stride_n, int32_t vocab) {
  return stats_bytes(batch, stride_n, vocab) + static_cast<size_t>(batch) * sizeof(int32_t) + 256;
}

cudaError_t launch_accept(const AcceptArgs& a, void* workspace, cudaStream_t stream, int* launches,
                          cudaEvent_t between0, cudaEvent_t between1) {
  const int R = 2 * a.stride_n - 1;
  const int n_chunks = (a.vocab + kChunk - 1) / kChunk;
  ChunkStat* stats = static_cast<ChunkStat*>(workspace);
  if (a.slab_stats != nullptr) {
    if (a.vocab % 32 != 0) return cudaErrorInvalidValue;
    accept_slab_stats_kernel<<<dim3(n_chunks, a.batch * R), kThreads, 0, stream>>>(
        a.slab_stats, a.vocab, n_chunks, stats);
  } else {
    accept_stats_kernel<<<dim3(n_chunks, a.batch * R), kThreads, 0, stream>>>(a.logits, a.vocab,
                                                                             n_chunks, stats);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;   // each kernel reads what the previous one wrote
  if (between0) cudaEventRecord(between0, stream);
  int32_t* qsrc = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) +
                                             stats_bytes(a.batch, a.stride_n, a.vocab));
  accept_decide_kernel<<<a.batch, kThreads, 0, stream>>>(a, stats, n_chunks, qsrc);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const bool q_rows = (a.flags & ISD_PROPOSE_SAMPLE) && a.q_cache != nullptr && a.stride_n > 1;
  if (q_rows) {
    write_q_rows_kernel<<<dim3(n_chunks, a.batch, a.stride_n - 1), kThreads, 0, stream>>>(
        a, stats, n_chunks, qsrc);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (between1) cudaEventRecord(between1, stream);
  bookkeep_kernel<<<1, 1024, 0, stream>>>(a);
  if (launches) *launches += q_rows ? 4 : 3;
  return cudaGetLastError();
}

}  // namespace isd
