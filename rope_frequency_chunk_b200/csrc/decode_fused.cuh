// Single-launch decode for bf16 caches: one thread-block cluster per
// (batch, KV head) row scores, selects and attends without a round trip
// through global memory.
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2): TIP scores from the dominant FCs only, the critical set T_t = the k
// highest-scoring tokens (ties to the lower index, k_eff = min(k, L)), then
// full softmax attention of every query head of the group over exactly those
// rows at their original positions.
//
// Grid C x rows, cluster C x 1 x 1 (C <= 16); CTA r of a cluster owns the
// tokens [r*n_loc, (r+1)*n_loc) of its row. Three phases in one launch:
//  1. score: warp 15 streams the CTA's sketch rows through a ring of
//     shared-memory stages with 1-D bulk copies (no multicast); warps 0-14
//     compute the float64 TIP scores (the score kernel's arithmetic), keep
//     the order-preserving 32-bit keys in shared memory and count the top 12
//     key bits in a 4096-bin histogram.
//  2. select: each CTA counts the top 8 bits of its keys (256 bins) while
//     scoring and writes that histogram into every CTA of the cluster
//     (distributed shared memory). After a cluster barrier every CTA knows
//     the row's histogram, hence the bin B holding the k_eff-th key; the same
//     exchange for B's 16 sub-bins (key bits 20..23) gives the 12-bit bin
//     b12 holding it, the count above, and every CTA's count inside b12. The
//     CTAs write their tokens of b12, compacted in rank order, into every
//     CTA, and after a third barrier each CTA resolves the exact k_eff-th
//     key of the row and its ties (lower token index first) from that union
//     alone. A union too large for shared memory (heavy ties) sends all CTAs
//     to an exact distributed radix select over the keys of b12 instead.
//  3. attend: each CTA attends its own kept rows on tensor cores
//     (mma.sync m16n8k16, Q split into three bf16 terms and P into two, as in
//     the split-K attention kernel) and merges its warps pairwise; the CTAs
//     write their partials straight into the CTA that owns each output
//     element, and after one more cluster barrier each CTA finishes its share
//     of the outputs from local memory, in rank order (deterministic). A last
//     cluster barrier keeps every CTA resident until all are done.
#pragma once

#include "attend_mma.cuh"
#include "score.cuh"
#include "select_attend.cuh"

namespace fasa {

constexpr int kFuThreads = kSAThreads;  // 512: the radix and histogram helpers' block size
constexpr int kFuWarps = kFuThreads / 32;
constexpr int kFuScoreWarps = kFuWarps - 1;  // + one producer warp
constexpr int kFuMaxStages = 16;
constexpr int kFuMinRing = kFuWarps * kAttStageBytes;  // 128 KB: one K+V chunk per warp
constexpr int kFuMaxLoc = 16384;                        // tokens per CTA
constexpr int kFuMaxCluster = 16;
constexpr int kFuSlot = 68 * 32;  // floats of one warp's (o, m, l) fragments in the warp merge
constexpr int kFuPartOff = 98304; // byte offset of the CTA partial inside the ring
constexpr int kFuPStride = 132;   // floats per head row of the CTA partial
constexpr int kFuRecvO = 16 * kD + kFuMaxCluster;  // floats: every rank's part of this CTA's outputs
constexpr int kFuRadixBytes = (kSAWarps * 256 + 264) * 4;
static_assert(kFuSlot * 4 * (kFuWarps / 2) <= kFuPartOff, "warp-merge slots overlap the CTA partial");
static_assert(kFuPartOff + (32 + 16 * kFuPStride) * 4 + (kFuMaxCluster * 16 + 16) * 4 <= kFuMinRing,
              "CTA partial exceeds the ring");

// Stage of the score stream: one warp step of every scoring warp.
template <int LPT>
__host__ __device__ constexpr int fu_stage_bytes() {
  return kFuScoreWarps * ScoreShape<__nv_bfloat16, LPT>::TPW * ScoreShape<__nv_bfloat16, LPT>::ROWB;
}

// exchange words, one row of kFuMaxCluster per kind, written by rank r at [kind][r]
enum FuXch { kXTies = 0, kXKept = 1, kXRows = 2 };

struct FusedParams {
  const __nv_bfloat16* sketch;  // [rows][max_len][stride]
  const float* scores;          // [rows][sld] TIP scores (the from-scores variant), else unused
  int64_t sld;                  // their row stride
  const __nv_bfloat16* k;       // [rows][max_len][128], rotated
  const __nv_bfloat16* v;
  const __nv_bfloat16* q;       // [B][Hq][128], pre-RoPE
  const int32_t* dom_idx;       // [Hkv][n_dom]
  __nv_bfloat16* out;           // [B][Hq][128]
  int32_t* idx_out;             // [rows][n_keep] kept indices, ascending, or null
  int64_t max_len;
  int32_t len;
  int32_t stride;
  int32_t n_kv_heads;
  int32_t group;
  int32_t n_dom;
  int32_t n_keep;    // k_eff >= 1
  int32_t n_loc;     // tokens per CTA, a multiple of 32, <= kFuMaxLoc
  int32_t ring;      // ring bytes: n_stages score stages, >= kFuMinRing
  int32_t n_stages;  // <= kFuMaxStages
  int32_t ucap;      // union capacity (entries): (ring - kFuRadixBytes) / 8
  double cosv[kNFC];
  double sinv[kNFC];
};

struct FuLayout {
  int ring, keys, bm, hloc, hall, hfine, qt, sq, qraw, dom, bars, chist, xch, scan, rml, ro, total;
};
__host__ __device__ inline FuLayout fu_layout(int n_loc, int ring) {
  FuLayout L;
  int o = 0;
  L.ring = o;  // score stages; then the union and the radix scratch; then attention
  o += ring;
  L.keys = o;  // keys, later the kept list (local indices)
  o += n_loc * 4;
  L.bm = o;
  o += sa_align(n_loc / 32 * 4, 16);
  L.hloc = o;  // this CTA's 256-bin histogram of the top 8 key bits, then the row's
  o += 256 * 4;
  L.hall = o;  // every rank's histogram [kFuMaxCluster][256]
  o += kFuMaxCluster * 256 * 4;
  L.hfine = o;  // every rank's 16 sub-bins of the boundary bin [kFuMaxCluster][16], then this CTA's own
  o += (kFuMaxCluster + 1) * 16 * 4;
  L.qt = o;  // attention Q: 3 bf16 terms x 16 heads x 128, rows of 256 B, 16-B chunks swizzled
  o += 3 * 16 * kD * 2;
  L.sq = o;
  o += kD * 8;
  L.qraw = o;
  o += FASA_MAX_GROUP * kD * 2;
  L.dom = o;
  o += kNFC * 4;
  L.bars = o;
  o += 2 * kFuMaxStages * 8;
  L.chist = o;  // per-digit cluster histograms of the exact fallback (the leader's copy is used)
  o += 4 * 256 * 4;
  L.xch = o;
  o += kXRows * kFuMaxCluster * 4;
  o = sa_align(o, 16);
  L.scan = o;
  o += 64 * 4;
  L.rml = o;  // partials received: (m[16], l[16]) per rank
  o += kFuMaxCluster * 32 * 4;
  L.ro = o;  // and each rank's o values of this CTA's share
  o += kFuRecvO * 4;
  L.total = o;
  return L;
}

// One warp: the bin of a 256-bin histogram (bin = key >> 24) holding the
// k-th largest key, and the count in higher bins (k <= total); lane l owns
// bins 255 - 8l .. 248 - 8l. Every lane gets the result.
__device__ __forceinline__ uint2 warp_bin256(const uint32_t* h, int k, int lane) {
  uint32_t c[8], sum = 0u;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    c[u] = h[255 - 8 * lane - u];
    sum += c[u];
  }
  uint32_t incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += v;
  }
  const uint32_t excl = incl - sum;
  const bool here = excl < (uint32_t)k && (uint32_t)k <= incl;
  uint32_t bin = 0u, above = 0u;
  if (here) {
    uint32_t acc = excl;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (acc + c[u] >= (uint32_t)k) {
        bin = 255u - (uint32_t)(8 * lane + u);
        above = acc;
        break;
      }
      acc += c[u];
    }
  }
  const unsigned who = __ballot_sync(0xFFFFFFFFu, here);
  const int src = who ? __ffs(who) - 1 : 0;
  return make_uint2(__shfl_sync(0xFFFFFFFFu, bin, src), __shfl_sync(0xFFFFFFFFu, above, src));
}

// The bin of a 1024-bin histogram holding the k-th largest entry (counting
// from bin 1023 down) and the count in higher bins (k <= total). All
// threads; thread t owns bins 1023 - 2t and 1022 - 2t; uses sc[0, 20).
__device__ __forceinline__ void bins1024_threshold(const uint32_t* h, int k, uint32_t* sc, uint32_t& bin,
                                                   uint32_t& above) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t ca = h[1023 - 2 * tid], cb = h[1022 - 2 * tid];
  const uint32_t sum = ca + cb;
  uint32_t incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) sc[warp] = incl;
  if (tid == 0) sc[16] = sc[17] = 0u;  // (only reached when k exceeds the total)
  __syncthreads();
  uint32_t before = 0u;
  for (int w = 0; w < warp; ++w) before += sc[w];
  incl += before;
  const uint32_t excl = incl - sum;
  if (excl < (uint32_t)k && (uint32_t)k <= excl + ca) {
    sc[16] = 1023u - 2u * (uint32_t)tid;
    sc[17] = excl;
  } else if (excl + ca < (uint32_t)k && (uint32_t)k <= incl) {
    sc[16] = 1022u - 2u * (uint32_t)tid;
    sc[17] = excl + ca;
  }
  __syncthreads();
  bin = sc[16] & 1023u;
  above = sc[17];
  __syncthreads();
}

// Exact k-th largest of n keys that share their top 12 bits (`prefix`):
// two passes over the remaining 20 bits, 10-bit digits counted with shared
// memory atomics into cnt[1024]. Returns the key and how many keys equal to
// it must still be taken. All threads.
__device__ __forceinline__ void select_low20(const uint32_t* key, int n, int k, uint32_t prefix, uint32_t* cnt,
                                             uint32_t* sc, uint32_t& thr, int& quota) {
  const int tid = threadIdx.x;
  uint32_t d1, d2, above;
  for (int i = tid; i < 1024; i += kFuThreads) cnt[i] = 0u;
  __syncthreads();
  for (int e = tid; e < n; e += kFuThreads) atomicAdd(&cnt[(key[e] >> 10) & 1023u], 1u);
  __syncthreads();
  bins1024_threshold(cnt, k, sc, d1, above);
  k -= (int)above;
  for (int i = tid; i < 1024; i += kFuThreads) cnt[i] = 0u;
  __syncthreads();
  for (int e = tid; e < n; e += kFuThreads) {
    const uint32_t x = key[e];
    if (((x >> 10) & 1023u) == d1) atomicAdd(&cnt[x & 1023u], 1u);
  }
  __syncthreads();
  bins1024_threshold(cnt, k, sc, d2, above);
  thr = prefix | (d1 << 10) | d2;
  quota = k - (int)above;
}

// Per-warp contiguous ranges of 32-token words of n tokens.
__device__ __forceinline__ void fu_words(int n, int& w0, int& w1) {
  const int warp = threadIdx.x >> 5;
  const int words = (n + 31) / 32;
  const int wseg = (words + kFuWarps - 1) / kFuWarps;
  w0 = min(words, warp * wseg);
  w1 = min(words, w0 + wseg);
}

// Tokens of [0, n) satisfying pred(i), counted per warp over its word range;
// returns (count in lower warps' ranges, total). All threads; uses scan[0, 16).
template <typename Pred>
__device__ __forceinline__ uint2 fu_count(int n, uint32_t* scan, Pred&& pred) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int w0, w1;
  fu_words(n, w0, w1);
  uint32_t c = 0u;
  for (int w = w0; w < w1; ++w) {
    const int i = w * 32 + lane;
    c += __popc(__ballot_sync(0xFFFFFFFFu, i < n && pred(i)));
  }
  if (lane == 0) scan[warp] = c;
  __syncthreads();
  uint32_t before = 0u, total = 0u;
#pragma unroll
  for (int w = 0; w < kFuWarps; ++w) {
    before += (w < warp) ? scan[w] : 0u;
    total += scan[w];
  }
  __syncthreads();
  return make_uint2(before, total);
}

// Visits, lane-parallel, the tokens satisfying pred(i) in ascending order:
// fn(position, i); `before` from fu_count with the same predicate.
template <typename Pred, typename Fn>
__device__ __forceinline__ void fu_visit(int n, uint32_t before, Pred&& pred, Fn&& fn) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  int w0, w1;
  fu_words(n, w0, w1);
  uint32_t pos = before;
  for (int w = w0; w < w1; ++w) {
    const int i = w * 32 + lane;
    const bool v = i < n && pred(i);
    const unsigned m = __ballot_sync(0xFFFFFFFFu, v);
    if (v) fn((int)(pos + __popc(m & lt)), i);
    pos += __popc(m);
  }
}

// kFromScores: phase 1 reads the TIP scores a score-kernel launch wrote
// (L2-resident) instead of streaming and scoring the sketch; LPT is unused.
template <int LPT, bool kFromScores>
__global__ void __launch_bounds__(kFuThreads, 1) decode_fused_kernel(const FusedParams p) {
  using T = __nv_bfloat16;
  using S = ScoreShape<T, LPT>;
  constexpr int kStage = fu_stage_bytes<LPT>();
  constexpr int TPS = kStage / S::ROWB;  // tokens per stage
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int cr = (int)cluster.block_rank();
  const FuLayout Ly = fu_layout(p.n_loc, p.ring);
  unsigned char* ring = smem + Ly.ring;
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + Ly.keys);
  int32_t* kept = reinterpret_cast<int32_t*>(smem + Ly.keys);
  uint32_t* bm = reinterpret_cast<uint32_t*>(smem + Ly.bm);
  uint32_t* hloc = reinterpret_cast<uint32_t*>(smem + Ly.hloc);
  uint32_t* hall = reinterpret_cast<uint32_t*>(smem + Ly.hall);
  uint32_t* hfine = reinterpret_cast<uint32_t*>(smem + Ly.hfine);
  uint32_t* hf_own = hfine + kFuMaxCluster * 16;
  unsigned char* qt = smem + Ly.qt;
  double* s_q = reinterpret_cast<double*>(smem + Ly.sq);
  T* qraw = reinterpret_cast<T*>(smem + Ly.qraw);
  int* s_dom = reinterpret_cast<int*>(smem + Ly.dom);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Ly.bars);
  uint64_t* empty = full + kFuMaxStages;
  uint32_t* chist = reinterpret_cast<uint32_t*>(smem + Ly.chist);
  uint32_t* xch = reinterpret_cast<uint32_t*>(smem + Ly.xch);
  uint32_t* scan = reinterpret_cast<uint32_t*>(smem + Ly.scan);
  float* rml = reinterpret_cast<float*>(smem + Ly.rml);
  float* ro = reinterpret_cast<float*>(smem + Ly.ro);
  // after scoring, the ring holds the union of the boundary bin's tokens
  // (keys, then token indices, ucap each) and the radix scratch
  uint32_t* ukey_s = reinterpret_cast<uint32_t*>(ring);
  int32_t* uidx_s = reinterpret_cast<int32_t*>(ring + p.ucap * 4);
  uint32_t* rscr = reinterpret_cast<uint32_t*>(ring + p.ucap * 8);

  const int row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.group;
  const int bb = row / p.n_kv_heads, g = row % p.n_kv_heads;
  const int t0 = cr * p.n_loc;
  const int n = max(0, min(p.len - t0, p.n_loc));

  // ---------------------------------------------------------------- setup
  if (tid == 0) {
    for (int b = 0; b < p.n_stages; ++b) {
      mbar_init(&full[b], 1);
      mbar_init(&empty[b], kFuScoreWarps);
    }
    fence_mbar_init();
  }
  for (int i = tid; i < 4 * 256; i += kFuThreads) chist[i] = 0u;
  if (tid < 256) hloc[tid] = 0u;
  // the sketch rows do not change between decode steps except for appended
  // tokens: warm L2 with this CTA's range while the previous kernel in the
  // stream may still run (the reads proper wait for it), and let the next
  // kernel's CTAs start on free SMs to do the same
  if (!kFromScores && warp == kFuScoreWarps && lane == 0 && n > 0) {
    const char* src = reinterpret_cast<const char*>(p.sketch) + ((int64_t)row * p.max_len + t0) * S::ROWB;
    for (int t = 0; t < n; t += TPS) prefetch_l2(src + (int64_t)t * S::ROWB, (uint32_t)(min(TPS, n - t) * S::ROWB));
  }
  grid_dependents_launch();
  __syncthreads();
  cluster_arrive();  // every CTA of the cluster runs: waited for before the first remote access
  grid_dependency_wait();

  // ---------------------------------------------------------------- 1. score
  if constexpr (kFromScores) {
    {
      const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + ((int64_t)(bb * p.n_kv_heads + g) * G) * kD);
      for (int c = tid; c < G * kD / 8; c += kFuThreads) reinterpret_cast<uint4*>(qraw)[c] = __ldg(qsrc + c);
    }
    __syncthreads();
    query_terms(qraw, G, p.cosv, p.sinv, qt, tid, kFuThreads);
    // the row's scores of this CTA's range: keys and the top-8-bit histogram
    const float* src = p.scores + (int64_t)row * p.sld + t0;
    constexpr int U = 8;
    for (int i0 = tid; i0 < n; i0 += kFuThreads * U) {
      float f[U];
#pragma unroll
      for (int u = 0; u < U; ++u) f[u] = i0 + u * kFuThreads < n ? __ldcg(src + i0 + u * kFuThreads) : 0.0f;
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (i0 + u * kFuThreads < n) {
          const uint32_t key = score_key(f[u]);
          keys[i0 + u * kFuThreads] = key;
          atomicAdd(&hloc[key >> 24], 1u);
        }
    }
  } else if (warp == kFuScoreWarps) {
    // the stream starts before the query work of the other warps
    if (lane == 0 && n > 0) {
      const char* src = reinterpret_cast<const char*>(p.sketch) + ((int64_t)row * p.max_len + t0) * S::ROWB;
      int t = 0;
      for (int j = 0; t < n; ++j) {
        const int b = j % p.n_stages;
        if (j >= p.n_stages && !mbar_wait(&empty[b], (uint32_t)(((j / p.n_stages) - 1) & 1))) break;
        const int m = min(TPS, n - t);
        mbar_arrive_expect_tx(&full[b], (uint32_t)(m * S::ROWB));
        bulk_g2s(ring + b * kStage, src + (int64_t)t * S::ROWB, (uint32_t)(m * S::ROWB), &full[b]);
        t += m;
      }
    }
    __syncwarp();
  } else {
    {
      const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + ((int64_t)(bb * p.n_kv_heads + g) * G) * kD);
      for (int c = tid; c < G * kD / 8; c += kFuScoreWarps * 32) reinterpret_cast<uint4*>(qraw)[c] = __ldg(qsrc + c);
      if (tid < p.n_dom) s_dom[tid] = __ldg(p.dom_idx + g * p.n_dom + tid);
    }
    named_barrier_sync(1, kFuScoreWarps * 32);
    query_coefs<T>(qraw, s_dom, G, p.n_dom, p.stride, p.cosv, p.sinv, tid, s_q);
    query_terms(qraw, G, p.cosv, p.sinv, qt, tid, kFuScoreWarps * 32);
    named_barrier_sync(1, kFuScoreWarps * 32);
    double qr[S::EPL];
    load_coefs<T, LPT>(qr, s_q, lane);
    for (int j = 0, done = 0; done < n; ++j) {
      const int b = j % p.n_stages;
      if (!mbar_wait(&full[b], (uint32_t)((j / p.n_stages) & 1))) break;  // status already recorded
      const int m = min(TPS, n - done);
      uint32_t* kd = keys + done;
      score_block<T, LPT, kFuScoreWarps>(ring + b * kStage, m, qr, warp, lane, [&](int t, bool writer, float sc) {
        if (writer) {
          const uint32_t key = score_key(sc);
          kd[t] = key;
          atomicAdd(&hloc[key >> 24], 1u);
        }
      });
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[b]);
      done += m;
    }
  }
  __syncthreads();  // keys and histogram complete, ring free

  // ---------------------------------------------------------------- 2. select
  cluster_wait();
  for (int i = tid; i < C * 256; i += kFuThreads) cluster.map_shared_rank(hall, i >> 8)[cr * 256 + (i & 255)] = hloc[i & 255];
  cluster_arrive();  // histograms delivered; this CTA's ring is free for the union
  cluster_wait();
  // the row's histogram (one bin per thread), then the boundary bin B by one warp
  if (tid < 256) {
    uint32_t t = 0u;
    for (int r = 0; r < C; ++r) t += hall[r * 256 + tid];
    hloc[tid] = t;
  }
  if (tid < 16) hf_own[tid] = 0u;
  __syncthreads();
  if (warp == 0) {
    const uint2 b = warp_bin256(hloc, p.n_keep, lane);
    if (lane == 0) {
      scan[61] = b.x;
      scan[62] = b.y;
    }
  }
  __syncthreads();
  const uint32_t bin8 = scan[61], above8 = scan[62];
  // second level: the 16 sub-bins (key bits 20..23) of bin B, counted here
  // and written into every CTA
  for (int i = tid; i < n; i += kFuThreads) {
    const uint32_t x = keys[i];
    if ((x >> 24) == bin8) atomicAdd(&hf_own[(x >> 20) & 15u], 1u);
  }
  __syncthreads();
  if (tid < C * 16) cluster.map_shared_rank(hfine, tid >> 4)[cr * 16 + (tid & 15)] = hf_own[tid & 15];
  cluster_arrive();
  cluster_wait();
  // one warp: the 12-bit bin b12 holding the k_eff-th key, the count above
  // it, every rank's count inside it and their offsets in the union
  uint32_t* uoff = hloc;  // [16] (the row histogram is no longer needed)
  if (warp == 0) {
    uint32_t cf = 0u;  // lane l < 16: sub-bin 15 - l of the row
    if (lane < 16)
      for (int r = 0; r < C; ++r) cf += hfine[r * 16 + (15 - lane)];
    uint32_t incl = cf;
#pragma unroll
    for (int o2 = 1; o2 < 32; o2 <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o2);
      if (lane >= o2) incl += v;
    }
    const uint32_t excl = incl - cf;
    const unsigned hit = __ballot_sync(0xFFFFFFFFu, lane < 16 && above8 + excl < (uint32_t)p.n_keep &&
                                                        (uint32_t)p.n_keep <= above8 + incl);
    const int fl = hit ? __ffs(hit) - 1 : 0;
    const uint32_t f12 = 15u - (uint32_t)fl;
    const uint32_t ab = above8 + __shfl_sync(0xFFFFFFFFu, excl, fl);
    const uint32_t nr = lane < C ? hfine[lane * 16 + f12] : 0u;
    uint32_t inr = nr;
#pragma unroll
    for (int o2 = 1; o2 < 32; o2 <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, inr, o2);
      if (lane >= o2) inr += v;
    }
    if (lane < C) uoff[lane] = inr - nr;
    if (lane == 31) {
      scan[56] = (bin8 << 4) | f12;
      scan[57] = ab;
      scan[58] = inr;
    }
  }
  __syncthreads();
  const uint32_t b12 = scan[56], above12 = scan[57], n_b = scan[58];
  const int krem12 = p.n_keep - (int)above12;  // keys of bin b12 still to take (>= 1)
  const uint32_t off = uoff[cr];               // this CTA's offset in the union
  const bool exact = n_b <= (uint32_t)p.ucap;  // the same in every CTA
  auto in_bin = [keys, b12](int i) { return (keys[i] >> 20) == b12; };
  if (exact) {
    // this CTA's tokens of b12, compacted locally (in the radix scratch,
    // unused until the union is complete), then copied into every CTA with
    // consecutive threads on consecutive entries
    const uint2 cp = fu_count(n, scan, in_bin);
    const int mine = (int)min(cp.y, n_b - off);  // they agree unless a timeout was recorded
    uint32_t* lk = rscr;
    int32_t* li = reinterpret_cast<int32_t*>(rscr + kFuRadixBytes / 8);
    if (mine <= kFuRadixBytes / 8) {
      fu_visit(n, cp.x, in_bin, [&](int pos, int i) {
        if (pos < mine) {
          lk[pos] = keys[i];
          li[pos] = t0 + i;
        }
      });
      __syncthreads();
      for (int e = tid; e < C * mine; e += kFuThreads) {
        const int r = e / mine, j = e - r * mine;
        cluster.map_shared_rank(ukey_s, r)[off + j] = lk[j];
        cluster.map_shared_rank(uidx_s, r)[off + j] = li[j];
      }
    } else {
      fu_visit(n, cp.x, in_bin, [&](int pos, int i) {
        if (pos >= mine) return;
#pragma unroll 1
        for (int r = 0; r < C; ++r) {
          cluster.map_shared_rank(ukey_s, r)[off + pos] = keys[i];
          cluster.map_shared_rank(uidx_s, r)[off + pos] = t0 + i;
        }
      });
    }
  }
  cluster_arrive();
  cluster_wait();

  uint32_t thr = 0u, thr2 = 0u;
  if (exact) {
    // the exact krem8-th key of the union, and its ties (lower index first)
    const int n_u = (int)n_b;
    int quota;
    select_low20(ukey_s, n_u, krem12, b12 << 20, rscr, scan, thr, quota);
    uint32_t neq = 0u;
    for (int base = warp * 32; base < n_u; base += kFuThreads)
      neq += __popc(__ballot_sync(0xFFFFFFFFu, base + lane < n_u && ukey_s[base + lane] == thr));
    if (lane == 0) scan[warp] = neq;
    __syncthreads();
    uint32_t eq_total = 0u;
#pragma unroll
    for (int w = 0; w < kFuWarps; ++w) eq_total += scan[w];
    __syncthreads();
    const bool all_ties = (int)eq_total <= quota;
    if (!all_ties) {
      auto tie_key = [ukey_s, uidx_s, thr](int i) { return ukey_s[i] == thr ? ~(uint32_t)uidx_s[i] : 0u; };
      int q2;
      ballot_radix_fn<false>(tie_key, n_u, quota, 0u, 0, 32, rscr, nullptr, cluster, thr2, q2);
    }
    int w0, w1;
    fu_words(n, w0, w1);
    for (int w = w0; w < w1; ++w) {
      const int i = w * 32 + lane;
      const bool v = i < n;
      const uint32_t x = v ? keys[i] : 0u;
      const bool keep = v && (x > thr || (x == thr && (all_ties || ~(uint32_t)(t0 + i) >= thr2)));
      const unsigned kb = __ballot_sync(0xFFFFFFFFu, keep);
      if (lane == 0) bm[w] = kb;
    }
  } else {
    // exact distributed radix select over the keys of bin b12; the CTAs' tie
    // counts are exchanged once and CTA r keeps what the lower ranks left
    int krem;
    ballot_radix_fn<true>([keys](int i) { return keys[i]; }, n, krem12, b12 << 20, 12, 32, rscr, chist, cluster, thr,
                          krem);
    const uint2 eq = fu_count(n, scan, [keys, thr](int i) { return keys[i] == thr; });
    if (tid < C) cluster.map_shared_rank(xch, tid)[kXTies * kFuMaxCluster + cr] = eq.y;
    cluster_arrive();
    cluster_wait();
    uint32_t before = 0u;
    for (int r = 0; r < cr; ++r) before += xch[kXTies * kFuMaxCluster + r];
    const int take = max(0, min((int)eq.y, krem - (int)before));
    // ties kept: the first `take` in index order
    const unsigned lt = (1u << lane) - 1u;
    int w0, w1;
    fu_words(n, w0, w1);
    uint32_t er = eq.x;
    for (int w = w0; w < w1; ++w) {
      const int i = w * 32 + lane;
      const bool v = i < n;
      const uint32_t x = v ? keys[i] : 0u;
      const unsigned gt = __ballot_sync(0xFFFFFFFFu, v && x > thr);
      const unsigned eqm = __ballot_sync(0xFFFFFFFFu, v && x == thr);
      const bool take_eq = ((eqm >> lane) & 1u) && (int)(er + __popc(eqm & lt)) < take;
      const unsigned te = __ballot_sync(0xFFFFFFFFu, take_eq);
      if (lane == 0) bm[w] = gt | te;
      er += __popc(eqm);
    }
  }
  __syncthreads();
  // kept list (local indices, ascending); keys are no longer read
  auto is_kept = [bm](int i) { return ((bm[i >> 5] >> (i & 31)) & 1u) != 0u; };
  const uint2 kpos = fu_count(n, scan, is_kept);
  fu_visit(n, kpos.x, is_kept, [&](int pos, int i) { kept[pos] = i; });
  const int n_kept = (int)kpos.y;
  if (tid < C) cluster.map_shared_rank(xch, tid)[kXKept * kFuMaxCluster + cr] = (uint32_t)n_kept;
  __syncthreads();

  // ---------------------------------------------------------------- 3. attend
  float o[16][4];
#pragma unroll
  for (int nn = 0; nn < 16; ++nn)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[nn][e] = 0.0f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;  // heads lane/4 and lane/4 + 8
  const int nch = (n_kept + kAttChunk - 1) / kAttChunk;
  {
    const T* kb = p.k + ((int64_t)row * p.max_len + t0) * kD;
    const T* vb = p.v + ((int64_t)row * p.max_len + t0) * kD;
    unsigned char* buf = ring + warp * kAttStageBytes;
    for (int ci = warp; ci < nch; ci += kFuWarps) {
      const int j0 = ci * kAttChunk;
#pragma unroll
      for (int r = 0; r < kAttChunk; ++r) {  // 16 rows x (16 K + 16 V) 16-byte parts, one part per lane
        const int jj = j0 + r;
        const int t = jj < n_kept ? kept[jj] : 0;  // masked below
        const T* src = (lane < 16 ? kb : vb) + (int64_t)t * kD + (lane % 16) * 8;
        cp_async16(buf + (lane < 16 ? 0 : kAttHalf) + r * 256 + (((lane % 16) ^ (r & 7)) * 16), src);
      }
      cp_async_commit();
      cp_async_wait<0>();
      __syncwarp();
      const unsigned char* Ks = buf;
      const unsigned char* Vs = buf + kAttHalf;
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};  // rows 0-7, 8-15 of the chunk
      const int arow = (lane % 8) + ((lane / 8) % 2) * 8;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t b[4];
        ldsm_x4(b, Ks + ((lane / 16) * 8 + lane % 8) * 256 + (((ks * 2 + (lane / 8) % 2) ^ (lane % 8)) * 16));
        const int aoff = arow * 256 + (((ks * 2 + lane / 16) ^ (arow & 7)) * 16);
#pragma unroll
        for (int term = 0; term < 3; ++term) {  // low, middle, high bf16 term of Q
          uint32_t a[4];
          ldsm_x4(a, qt + term * 4096 + aoff);
          mma_16816(s0, a, b[0], b[1]);
          mma_16816(s1, a, b[2], b[3]);
        }
      }
      const int c0 = (lane % 4) * 2;
      if (j0 + c0 >= n_kept) s0[0] = s0[2] = -INFINITY;
      if (j0 + c0 + 1 >= n_kept) s0[1] = s0[3] = -INFINITY;
      if (j0 + 8 + c0 >= n_kept) s1[0] = s1[2] = -INFINITY;
      if (j0 + 8 + c0 + 1 >= n_kept) s1[1] = s1[3] = -INFINITY;
      float mx0 = fmaxf(fmaxf(s0[0], s0[1]), fmaxf(s1[0], s1[1]));
      float mx1 = fmaxf(fmaxf(s0[2], s0[3]), fmaxf(s1[2], s1[3]));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, 2));
      const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
      const float sc0 = (m0 == -INFINITY) ? 0.0f : exp2f(m0 - n0);
      const float sc1 = (m1 == -INFINITY) ? 0.0f : exp2f(m1 - n1);
      float pr[8];
      pr[0] = s0[0] == -INFINITY ? 0.f : exp2f(s0[0] - n0);
      pr[1] = s0[1] == -INFINITY ? 0.f : exp2f(s0[1] - n0);
      pr[2] = s0[2] == -INFINITY ? 0.f : exp2f(s0[2] - n1);
      pr[3] = s0[3] == -INFINITY ? 0.f : exp2f(s0[3] - n1);
      pr[4] = s1[0] == -INFINITY ? 0.f : exp2f(s1[0] - n0);
      pr[5] = s1[1] == -INFINITY ? 0.f : exp2f(s1[1] - n0);
      pr[6] = s1[2] == -INFINITY ? 0.f : exp2f(s1[2] - n1);
      pr[7] = s1[3] == -INFINITY ? 0.f : exp2f(s1[3] - n1);
      l0 = l0 * sc0 + (pr[0] + pr[1] + pr[4] + pr[5]);
      l1 = l1 * sc1 + (pr[2] + pr[3] + pr[6] + pr[7]);
      m0 = n0;
      m1 = n1;
#pragma unroll
      for (int nn = 0; nn < 16; ++nn) {
        o[nn][0] *= sc0;
        o[nn][1] *= sc0;
        o[nn][2] *= sc1;
        o[nn][3] *= sc1;
      }
      uint32_t ph[4], pl[4];
      split_pack(pr[0], pr[1], ph[0], pl[0]);
      split_pack(pr[2], pr[3], ph[1], pl[1]);
      split_pack(pr[4], pr[5], ph[2], pl[2]);
      split_pack(pr[6], pr[7], ph[3], pl[3]);
#pragma unroll
      for (int nn = 0; nn < 16; nn += 2) {
        uint32_t b[4];
        ldsm_x4_t(b, Vs + (((lane / 8) % 2) * 8 + lane % 8) * 256 + (((nn + lane / 16) ^ (lane % 8)) * 16));
        mma_16816(o[nn], ph, b[0], b[1]);
        mma_16816(o[nn], pl, b[0], b[1]);
        mma_16816(o[nn + 1], ph, b[2], b[3]);
        mma_16816(o[nn + 1], pl, b[2], b[3]);
      }
      __syncwarp();  // the buffer is refilled by the warp's next chunk
    }
  }

  // warps merged pairwise: warps [h, 2h) hand their fragments to warps [0, h);
  // rounds whose upper warps attended nothing are skipped (nch is uniform)
  float* slots = reinterpret_cast<float*>(ring);
#pragma unroll 1
  for (int half = kFuWarps / 2; half >= 1; half >>= 1) {
    if (nch <= half) continue;
    __syncthreads();
    if (warp >= half && warp < 2 * half) {
      float* sl = slots + (warp - half) * kFuSlot;
#pragma unroll
      for (int nn = 0; nn < 16; ++nn)
#pragma unroll
        for (int e = 0; e < 4; ++e) sl[(nn * 4 + e) * 32 + lane] = o[nn][e];
      sl[64 * 32 + lane] = m0;
      sl[65 * 32 + lane] = m1;
      sl[66 * 32 + lane] = l0;
      sl[67 * 32 + lane] = l1;
    }
    __syncthreads();
    if (warp < half) {
      const float* sl = slots + warp * kFuSlot;
      const float pm0 = sl[64 * 32 + lane], pm1 = sl[65 * 32 + lane];
      const float n0 = fmaxf(m0, pm0), n1 = fmaxf(m1, pm1);
      const float a0 = (m0 == -INFINITY) ? 0.0f : exp2f(m0 - n0), a1 = (m1 == -INFINITY) ? 0.0f : exp2f(m1 - n1);
      const float b0 = (pm0 == -INFINITY) ? 0.0f : exp2f(pm0 - n0), b1 = (pm1 == -INFINITY) ? 0.0f : exp2f(pm1 - n1);
#pragma unroll
      for (int nn = 0; nn < 16; ++nn) {
        o[nn][0] = o[nn][0] * a0 + sl[(nn * 4 + 0) * 32 + lane] * b0;
        o[nn][1] = o[nn][1] * a0 + sl[(nn * 4 + 1) * 32 + lane] * b0;
        o[nn][2] = o[nn][2] * a1 + sl[(nn * 4 + 2) * 32 + lane] * b1;
        o[nn][3] = o[nn][3] * a1 + sl[(nn * 4 + 3) * 32 + lane] * b1;
      }
      l0 = l0 * a0 + sl[66 * 32 + lane] * b0;
      l1 = l1 * a1 + sl[67 * 32 + lane] * b1;
      m0 = n0;
      m1 = n1;
    }
  }
  // the CTA's partial (m[16], l[16], o[16][kFuPStride]) in local memory, then
  // every thread forwards part of it: (m, l) to every CTA, o[h][d] to the CTA
  // that owns output element h*128 + d
  float* P = reinterpret_cast<float*>(ring + kFuPartOff);
  if (warp == 0) {
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 1);
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 2);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 1);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 2);
    if (lane % 4 == 0) {
      P[lane / 4] = m0;
      P[lane / 4 + 8] = m1;
      P[16 + lane / 4] = l0;
      P[16 + lane / 4 + 8] = l1;
    }
#pragma unroll
    for (int nn = 0; nn < 16; ++nn) {
      const int d = nn * 8 + (lane % 4) * 2;
      P[32 + (lane / 4) * kFuPStride + d] = o[nn][0];
      P[32 + (lane / 4) * kFuPStride + d + 1] = o[nn][1];
      P[32 + (lane / 4 + 8) * kFuPStride + d] = o[nn][2];
      P[32 + (lane / 4 + 8) * kFuPStride + d + 1] = o[nn][3];
    }
  }
  __syncthreads();
  const int total_el = G * kD;
  const int share = (total_el + C - 1) / C;
  for (int i = tid; i < C * 32; i += kFuThreads) cluster.map_shared_rank(rml, i / 32)[cr * 32 + i % 32] = P[i % 32];
  for (int e = tid; e < total_el; e += kFuThreads) {
    const int own = e / share;
    cluster.map_shared_rank(ro, own)[cr * share + (e - own * share)] = P[32 + (e / kD) * kFuPStride + e % kD];
  }
  cluster_arrive();  // every partial and kept count has arrived
  cluster_wait();
  // no CTA may leave while distributed shared memory operations aimed at it
  // could still be outstanding: a last barrier, its arrival here and its
  // wait at the end, so its latency overlaps the merge
  cluster_arrive();

  // this CTA's outputs [cr*share, (cr+1)*share), from local memory only
  float* wgt = reinterpret_cast<float*>(ring + kFuPartOff + (32 + 16 * kFuPStride) * 4);  // [C][16]
  float* den = wgt + kFuMaxCluster * 16;                                                  // [16]
  if (tid < 16) {
    float M = -INFINITY;
    for (int r = 0; r < C; ++r) M = fmaxf(M, rml[r * 32 + tid]);
    float dsum = 0.0f;
    for (int r = 0; r < C; ++r) {
      const float mr = rml[r * 32 + tid];
      const float w = (mr == -INFINITY || M == -INFINITY) ? 0.0f : exp2f(mr - M);
      wgt[r * 16 + tid] = w;
      dsum += w * rml[r * 32 + 16 + tid];
    }
    den[tid] = dsum;
  }
  __syncthreads();
  const int e0 = cr * share, e1 = min(total_el, e0 + share);
  T* outp = p.out + ((int64_t)row * G) * kD;
  for (int e = e0 + tid; e < e1; e += kFuThreads) {
    const int h = e / kD;
    float num = 0.0f;
    for (int r = 0; r < C; ++r) num += wgt[r * 16 + h] * ro[r * share + (e - e0)];
    const float dn = den[h];
    outp[e] = __float2bfloat16_rn(dn > 0.0f ? num / dn : 0.0f);
  }
  if (p.idx_out != nullptr) {
    uint32_t before = 0u;
    for (int r = 0; r < cr; ++r) before += xch[kXKept * kFuMaxCluster + r];
    int32_t* io = p.idx_out + (int64_t)row * p.n_keep;
    for (int i = tid; i < n_kept; i += kFuThreads) {
      if (before + (uint32_t)i < (uint32_t)p.n_keep)
        io[before + i] = t0 + kept[i];
      else
        flag_status(FASA_ERR_BAD_INDEX);
    }
  }
  cluster_wait();
}

}  // namespace fasa
