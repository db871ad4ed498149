// Critical-set selection and focused attention, one thread-block cluster per
// (sequence, KV head).
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2, FAC bullets): from the TIP scores pick the critical token set T_t, run
// full softmax attention over exactly those tokens, keep their original
// absolute positions (their keys were rotated at append time).
//
// Modes (one kernel template, chosen at launch):
//   kSelect     scores -> idx (fasa_select_topk)
//   kDecode     scores -> T_t -> attention -> out (second launch of fasa_decode)
//   kAttendIdx  given idx -> attention -> out (fasa_sparse_attend)
//   kDense      all rows -> attention -> out (fasa_dense_decode)
//
// Selection is exact: the k_eff largest order-preserving uint32 keys, ties to
// the lower token index. The C CTAs of a cluster each hold a contiguous chunk
// of the row's keys in shared memory.
//  1. Threshold guess: every CTA reads the same strided sample of the whole
//     row from L2 and takes a value t_lo at or below the sample's
//     j-th largest (j a few standard deviations above k_eff / stride), so
//     that about k_eff + margin keys are >= t_lo.
//  2. Every CTA counts its keys >= t_lo (warp ballots) and tells the others;
//     if the total is < k_eff or exceeds the candidate buffer, all CTAs take
//     the exact fallback (3 below on all keys).
//  3. Candidates (key, index) are written, in index order, into every CTA's
//     shared memory; each CTA finds the exact k_eff-th key and the number of
//     ties to keep with a radix select whose digit histograms are counted by
//     warp ballots (no atomics), and extracts its own slice of the kept list.
// Attention: each CTA gathers its slice's K and V rows with 16-byte cp.async
// (double-buffered), computes float32 logits with the query in registers and
// a butterfly transpose-reduce across the warp, keeps a base-2 online
// softmax, accumulates P.V per 4-dim quad, and the cluster merges its
// (m, l, o) partials over DSMEM. The dense mode streams contiguous rows with
// 1-D bulk copies (TMA engine, mbarrier completion, no multicast).
#pragma once

#include <cooperative_groups.h>

#include "fasa_device.cuh"

namespace fasa {
namespace cg = cooperative_groups;

constexpr int kSAThreads = 512;
constexpr int kSAWarps = kSAThreads / 32;
constexpr int kMaxCluster = 16;
constexpr int kMaxSamples = 2048;
constexpr int kStageBytes = 32768;  // K + V rows of one pipeline stage

enum SAMode { kSelect = 0, kDecode = 1, kAttendIdx = 2, kDense = 3 };

struct SAParams {
  const float* scores;       // [rows][len]
  const uint32_t* hist;      // [rows][4096] histogram of the top 12 key bits, or null
  int32_t* idx_out;          // [rows][n_keep] or null
  const int32_t* idx_in;     // [rows][n_keep] (kAttendIdx)
  const void* k;             // [rows][max_len][128]
  const void* v;
  const void* q;             // [B][Hq][128]
  void* out;                 // [B][Hq][128]
  int64_t max_len;
  int32_t len;
  int32_t n_keep;            // k_eff (select/decode) or n_idx (attend)
  int32_t chunk;             // keys (select) or rows (dense) per CTA
  int32_t slice;             // kept indices attended per CTA
  int32_t n_kv_heads;
  int32_t group;
  int32_t cap;               // candidate capacity per CTA
  int32_t sample_stride;     // s: every s-th score is sampled
  int32_t sample_rank;       // j: rank of the sample used as threshold
  int32_t n_stages;          // attention pipeline depth
  double cosv[kNFC];         // cos / sin of q_pos * theta_i (host, float64)
  double sinv[kNFC];
};

template <typename T> __host__ __device__ constexpr int stage_rows() {
  return kStageBytes / (2 * kD * (int)sizeof(T));
}

struct SALayout {
  int keys, stage, cand_key, cand_idx, samples, idx, rscr, chist, misc, qraw, qs, zs, acc, ml, mlall, red, bar, total;
};

__host__ __device__ inline int sa_align(int x, int a) { return (x + a - 1) / a * a; }

// Region A holds the keys and, after them, the candidate buffer during
// selection, and the attention stages afterwards.
__host__ __device__ inline SALayout sa_layout(int mode, int elem_bytes, int chunk, int slice, int cap, int maxg,
                                              int n_stages) {
  SALayout L;
  const int rb = kStageBytes / (2 * kD * elem_bytes);
  const bool sel = (mode == kSelect || mode == kDecode);
  const bool att = (mode != kSelect);
  const int keys_bytes = sel ? sa_align(chunk * 4, 128) : 0;
  const int cand_bytes = sel ? 2 * sa_align(cap * 4, 128) : 0;
  const int stage_bytes = att ? n_stages * kStageBytes : 0;
  int off = 0;
  L.keys = L.stage = 0;
  L.cand_key = keys_bytes;
  L.cand_idx = keys_bytes + cand_bytes / 2;
  off = sa_align(keys_bytes + cand_bytes > stage_bytes ? keys_bytes + cand_bytes : stage_bytes, 128);
  L.samples = off;
  off = sa_align(off + (sel ? kMaxSamples * 4 : 0), 128);
  L.idx = off;
  off = sa_align(off + ((mode == kDecode || mode == kAttendIdx) ? slice * 4 : 0), 128);
  L.rscr = off;
  off = sa_align(off + (sel ? (kSAWarps * 256 + 256 + 8) * 4 : 0), 128);
  L.chist = off;
  off = sa_align(off + (sel ? 4 * 256 * 4 : 0), 128);
  L.misc = off;
  off = sa_align(off + 128 * 4, 128);
  L.qraw = off;
  off = sa_align(off + (att ? maxg * kD * elem_bytes : 0), 128);
  L.qs = off;
  off = sa_align(off + (att ? maxg * kD * 4 : 0), 128);
  L.zs = off;
  off = sa_align(off + (att ? maxg * rb * 4 : 0), 128);
  L.acc = off;
  off = sa_align(off + (att ? maxg * kD * 4 : 0), 128);
  L.ml = off;
  off = sa_align(off + (att ? 4 * maxg * 4 : 0), 128);
  L.mlall = off;
  off = sa_align(off + (att ? kMaxCluster * 2 * maxg * 4 : 0), 128);
  L.red = off;
  off = sa_align(off + (att ? (maxg * kD + kMaxCluster) * 4 : 0), 128);
  L.bar = off;
  off = sa_align(off + 8 * 8, 128);
  L.total = off;
  return L;
}

// misc-area slots (uint32 words)
enum : int {
  kMiscWarpA = 0,     // [16] per-warp counts / exclusive offsets
  kMiscWarpB = 16,    // [16]
  kMiscCtaA = 32,     // [16] per-CTA counts, written by every CTA into every CTA
  kMiscCtaB = 48,     // [16]
  kMiscScan = 64,     // [16] scratch
  kMiscBcast = 80,    // [8]  broadcast values
};

// ----------------------------------------------------------- helpers

// Exclusive scan of the 16 per-warp values in misc[base..base+16) in place;
// returns the total. Call from one thread.
__device__ __forceinline__ uint32_t warp_offsets_serial(uint32_t* misc, int base) {
  uint32_t t = 0;
#pragma unroll
  for (int w = 0; w < kSAWarps; ++w) {
    const uint32_t a = misc[base + w];
    misc[base + w] = t;
    t += a;
  }
  return t;
}

// Exact radix select by 8-bit digits, most significant first, over
// keys[0..n) in shared memory. Digit histograms are counted with warp
// ballots, no atomics: one ballot per digit bit, and lane L counts bins
// 8L..8L+7 by intersecting the ballots. After `passes` passes (4 = exact),
// returns the prefix of the k-th largest key and how many keys equal to that
// prefix must still be taken (ties to the lower position). With kCluster the
// per-pass histograms are summed over the cluster in the leader's shared
// memory.
template <bool kCluster, typename KeyAt>
__device__ void ballot_radix_fn(KeyAt key_at, int n, int k, uint32_t prefix, int known, int stop, uint32_t* rscr,
                                uint32_t* chist, cg::cluster_group& cluster, uint32_t& out_prefix, int& out_krem) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t* tot = rscr + kSAWarps * 256;
  uint32_t* bc = tot + 256;
  uint32_t pmask = known ? ~0u << (32 - known) : 0u;
  int krem = k;
  for (int pass = 0; known < stop; ++pass) {
    const int width = min(8, stop - known);
    const int shift = 32 - known - width;
    known += width;
    uint32_t cnt[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    for (int base = warp * 32; base < n; base += kSAThreads) {
      const int i = base + lane;
      bool act = false;
      uint32_t d = 0u;
      if (i < n) {
        const uint32_t x = key_at(i);
        act = (x & pmask) == prefix;
        d = (x >> shift) & ((1u << width) - 1u);
      }
      unsigned b[8];
      const unsigned a = __ballot_sync(0xFFFFFFFFu, act);
#pragma unroll
      for (int j = 0; j < 8; ++j) b[j] = __ballot_sync(0xFFFFFFFFu, act && ((d >> j) & 1u));
      unsigned m = a;
#pragma unroll
      for (int j = 0; j < 5; ++j) m &= ((lane >> j) & 1) ? b[3 + j] : ~b[3 + j];
      const unsigned n0 = ~b[0], n1 = ~b[1], n2 = ~b[2];
      cnt[0] += __popc(m & n0 & n1 & n2);
      cnt[1] += __popc(m & b[0] & n1 & n2);
      cnt[2] += __popc(m & n0 & b[1] & n2);
      cnt[3] += __popc(m & b[0] & b[1] & n2);
      cnt[4] += __popc(m & n0 & n1 & b[2]);
      cnt[5] += __popc(m & b[0] & n1 & b[2]);
      cnt[6] += __popc(m & n0 & b[1] & b[2]);
      cnt[7] += __popc(m & b[0] & b[1] & b[2]);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) rscr[warp * 256 + lane * 8 + u] = cnt[u];
    __syncthreads();
    if (tid < 256) {
      uint32_t sum = 0u;
#pragma unroll
      for (int w = 0; w < kSAWarps; ++w) sum += rscr[w * 256 + tid];
      if (kCluster) {
        if (sum) atomicAdd(cluster.map_shared_rank(chist + pass * 256, 0) + tid, sum);
      } else {
        tot[tid] = sum;
      }
    }
    if (kCluster) {
      cluster_arrive();
      cluster_wait();
      if (tid < 256) tot[tid] = cluster.map_shared_rank(chist + pass * 256, 0)[tid];
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t g[8], gs = 0u;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        g[u] = tot[lane * 8 + u];
        gs += g[u];
      }
      // inclusive sum over this lane and all higher lanes (higher bins)
      uint32_t incl = gs;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, incl, off);
        if (lane + off < 32) incl += v;
      }
      const uint32_t excl = incl - gs;
      if (excl < (uint32_t)krem && (uint32_t)krem <= incl) {
        uint32_t acc = excl;
#pragma unroll
        for (int u = 7; u >= 0; --u) {
          if (acc + g[u] >= (uint32_t)krem) {
            bc[0] = (uint32_t)(lane * 8 + u);
            bc[1] = acc;
            break;
          }
          acc += g[u];
        }
      }
    }
    __syncthreads();
    prefix |= bc[0] << shift;
    pmask |= ((1u << width) - 1u) << shift;
    krem -= (int)bc[1];
  }
  out_prefix = prefix;
  out_krem = krem;
}

// From a row's 4096-bin histogram of the top 12 key bits, the bin holding
// the k-th largest key and the number of keys in higher bins. Block-wide
// suffix scan: thread t owns bins 4095-8t .. 4088-8t.
// (hist_threshold_fn takes the bin loader; hist_threshold reads global memory.)
template <typename Ld>
__device__ __forceinline__ void hist_threshold_fn(Ld ld, int k, uint32_t* scan, uint32_t& bin, uint32_t& above) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t c[8], sum = 0u;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    c[u] = ld(4095 - (8 * tid + u));
    sum += c[u];
  }
  uint32_t incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) scan[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kSAWarps ? scan[lane] : 0u;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, w, off);
      if (lane >= off) w += v;
    }
    if (lane < kSAWarps) scan[16 + lane] = w;
  }
  __syncthreads();
  incl += warp > 0 ? scan[16 + warp - 1] : 0u;
  const uint32_t excl = incl - sum;
  if (excl < (uint32_t)k && (uint32_t)k <= incl) {
    uint32_t acc = excl;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (acc + c[u] >= (uint32_t)k) {
        scan[32] = 4095u - (uint32_t)(8 * tid + u);
        scan[33] = acc;
        break;
      }
      acc += c[u];
    }
  }
  __syncthreads();
  bin = scan[32];
  above = scan[33];
  __syncthreads();
}
__device__ __forceinline__ void hist_threshold(const uint32_t* h, int k, uint32_t* scan, uint32_t& bin,
                                               uint32_t& above) {
  hist_threshold_fn([h](int i) { return __ldcg(h + i); }, k, scan, bin, above);
}

template <bool kCluster>
__device__ __forceinline__ void ballot_radix(const uint32_t* keys, int n, int k, uint32_t prefix, int known, int stop,
                                             uint32_t* rscr, uint32_t* chist, cg::cluster_group& cluster,
                                             uint32_t& out_prefix, int& out_krem) {
  ballot_radix_fn<kCluster>([keys](int i) { return keys[i]; }, n, k, prefix, known, stop, rscr, chist, cluster,
                            out_prefix, out_krem);
}

// Unrolled coalesced load of n score keys (global float -> order-preserving key).
__device__ __forceinline__ void load_keys(uint32_t* dst, const float* src, int n) {
  constexpr int U = 8;
  for (int base = threadIdx.x; base < n; base += kSAThreads * U) {
    float f[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * kSAThreads;
      f[u] = i < n ? __ldcg(src + i) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * kSAThreads;
      if (i < n) dst[i] = score_key(f[u]);
    }
  }
}

template <typename T, int MODE, int MAXG>
__global__ void __launch_bounds__(kSAThreads, 1) select_attend_kernel(const SAParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  grid_dependency_wait();  // inputs of an earlier kernel in the stream are complete
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr bool kSel = (MODE == kSelect || MODE == kDecode);
  constexpr bool kAtt = (MODE != kSelect);
  constexpr int RB = stage_rows<T>();
  constexpr int ES = (int)sizeof(T);
  constexpr int NV = (MAXG == 8) ? 32 : 16;  // partial logits per lane in one step
  constexpr int RPW = NV / MAXG;              // rows per warp in one logit step
  constexpr bool kQReg = MAXG <= 8;           // query slice held in registers
  const unsigned lt = (1u << lane) - 1u;

  const SALayout L = sa_layout(MODE, ES, p.chunk, p.slice, p.cap, MAXG, p.n_stages);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + L.keys);
  unsigned char* stage = smem + L.stage;
  uint32_t* cand_key = reinterpret_cast<uint32_t*>(smem + L.cand_key);
  int32_t* cand_idx = reinterpret_cast<int32_t*>(smem + L.cand_idx);
  uint32_t* samples = reinterpret_cast<uint32_t*>(smem + L.samples);
  int32_t* idx_s = reinterpret_cast<int32_t*>(smem + L.idx);
  uint32_t* rscr = reinterpret_cast<uint32_t*>(smem + L.rscr);
  uint32_t* chist = reinterpret_cast<uint32_t*>(smem + L.chist);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L.misc);
  float* qs = reinterpret_cast<float*>(smem + L.qs);
  float* zs = reinterpret_cast<float*>(smem + L.zs);
  float* acc_s = reinterpret_cast<float*>(smem + L.acc);
  float* ml = reinterpret_cast<float*>(smem + L.ml);  // m[MAXG], l[MAXG], scale[MAXG], weight[MAXG]
  float* mlall = reinterpret_cast<float*>(smem + L.mlall);
  float* red = reinterpret_cast<float*>(smem + L.red);
  unsigned char* qraw = smem + L.qraw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar);

  const int G = p.group;

  // ------------------------------------------------------------ set-up
  if (kSel && rank == 0)
    for (int i = tid; i < 4 * 256; i += kSAThreads) chist[i] = 0u;
  if (tid < 128) misc[tid] = 0u;
  if (MODE == kDecode)  // slots the selection never fills stay masked
    for (int i = tid; i < p.slice; i += kSAThreads) idx_s[i] = -1;
  if (kAtt) {
    // prefetch the group's raw queries; rotated just before attention
    const unsigned char* qsrc = static_cast<const unsigned char*>(p.q) + ((int64_t)row * G) * kD * ES;
    for (int c = tid; c < G * kD * ES / 16; c += kSAThreads) cp_async16(qraw + c * 16, qsrc + c * 16);
    cp_async_commit();
    if (MODE == kDense && tid == 0) {
      for (int s = 0; s < p.n_stages; ++s) mbar_init(&bars[s], 1);
      fence_mbar_init();
    }
    for (int i = tid; i < MAXG * kD; i += kSAThreads) acc_s[i] = 0.0f;
    if (tid < MAXG) {
      ml[tid] = -INFINITY;
      ml[MAXG + tid] = 0.0f;
      ml[2 * MAXG + tid] = 0.0f;
      ml[3 * MAXG + tid] = 0.0f;
    }
  }
  __syncthreads();
  if (C > 1) cluster_arrive();  // "all CTAs started": waited for before the first DSMEM access
  bool start_waited = (C == 1);

  int n_mine = 0;      // rows this CTA attends over
  int row_start = 0;   // first slice position (kept lists) or first row (dense)

  // ------------------------------------------------------------ select
  if constexpr (kSel) {
    const int start = rank * p.chunk;
    const int n_loc = max(0, min(p.chunk, p.len - start));
    const float* srow = p.scores + (int64_t)row * p.len;
    load_keys(keys, srow + start, n_loc);
    // 1. threshold t_lo <= the k_eff-th key. With the score kernel's key
    //    histogram it is the lower edge of the bin holding that key (exact:
    //    the leader then only resolves the low 20 bits); otherwise the top 16
    //    bits of the j-th largest of a strided sample of the row.
    uint32_t t_lo = 0u, lead_prefix = 0u;
    int lead_known = 0, lead_k = p.n_keep;
    if (p.hist != nullptr) {
      __syncthreads();
      uint32_t bin, above;
      hist_threshold(p.hist + (int64_t)row * 4096, p.n_keep, misc + kMiscScan, bin, above);
      t_lo = bin << 20;
      lead_prefix = t_lo;
      lead_known = 12;
      lead_k = p.n_keep - (int)above;
    } else {
      const int s_str = p.sample_stride;
      const int m = (p.len + s_str - 1) / s_str;
      const bool use_samples = p.sample_rank < m;
      if (use_samples)
        for (int i = tid; i < m; i += kSAThreads) samples[i] = score_key(__ldcg(srow + (int64_t)i * s_str));
      __syncthreads();
      if (use_samples) {
        uint32_t pre;
        int kr;
        ballot_radix<false>(samples, m, p.sample_rank, 0u, 0, 16, rscr, chist, cluster, pre, kr);
        t_lo = pre;
      }
    }
    __syncthreads();

    // 2. count local keys >= t_lo by warp segments (index order)
    const int seg = ((n_loc + kSAWarps * 32 - 1) / (kSAWarps * 32)) * 32;
    const int ws = min(n_loc, warp * seg), we = min(n_loc, ws + seg);
    uint32_t cnt = 0u;
    for (int base = ws; base < we; base += 32) {
      const int i = base + lane;
      cnt += __popc(__ballot_sync(0xFFFFFFFFu, i < we && keys[i] >= t_lo));
    }
    if (lane == 0) misc[kMiscWarpA + warp] = cnt;
    __syncthreads();
    if (tid == 0) misc[kMiscBcast] = warp_offsets_serial(misc, kMiscWarpA);
    __syncthreads();
    if (!start_waited) {
      cluster_wait();
      start_waited = true;
    }
    if (tid < C) cluster.map_shared_rank(misc, tid)[kMiscCtaA + rank] = misc[kMiscBcast];
    if (C > 1) {
      cluster_arrive();
      cluster_wait();
    } else {
      __syncthreads();
    }
    uint32_t total = 0u, before = 0u;
    for (int r = 0; r < C; ++r) {
      const uint32_t c = misc[kMiscCtaA + r];
      total += c;
      if (r < rank) before += c;
    }
    const bool fast = total >= (uint32_t)p.n_keep && total <= (uint32_t)p.cap;  // same in every CTA

    uint32_t thr = 0u;
    int quota = 0;
    if (fast) {
      // 3. candidates, in index order, into the leader
      uint32_t* lkey = cluster.map_shared_rank(cand_key, 0);
      int32_t* lidx = cluster.map_shared_rank(cand_idx, 0);
      uint32_t pos = before + misc[kMiscWarpA + warp];
      for (int base = ws; base < we; base += 32) {
        const int i = base + lane;
        const bool sel = i < we && keys[i] >= t_lo;
        const unsigned b = __ballot_sync(0xFFFFFFFFu, sel);
        if (sel) {
          const uint32_t at = pos + __popc(b & lt);
          lkey[at] = keys[i];
          lidx[at] = start + i;
        }
        pos += __popc(b);
      }
      if (C > 1) {
        cluster_arrive();
        cluster_wait();
      } else {
        __syncthreads();
      }
      if (rank == 0) {
        // exact k_eff-th key among the candidates; the kept list is the
        // candidates above it and the first `quota` equal to it
        ballot_radix<false>(cand_key, (int)total, lead_k, lead_prefix, lead_known, 32, rscr, chist, cluster, thr,
                            quota);
        const int n = (int)total;
        const int cseg = ((n + kSAWarps * 32 - 1) / (kSAWarps * 32)) * 32;
        const int cs = min(n, warp * cseg), ce = min(n, cs + cseg);
        uint32_t cg_ = 0u, ce_ = 0u;
        for (int base = cs; base < ce; base += 32) {
          const int i = base + lane;
          const bool v = i < ce;
          const uint32_t x = v ? cand_key[i] : 0u;
          cg_ += __popc(__ballot_sync(0xFFFFFFFFu, v && x > thr));
          ce_ += __popc(__ballot_sync(0xFFFFFFFFu, v && x == thr));
        }
        if (lane == 0) {
          misc[kMiscWarpA + warp] = cg_;
          misc[kMiscWarpB + warp] = ce_;
        }
        __syncthreads();
        if (tid == 0) {
          warp_offsets_serial(misc, kMiscWarpA);
          warp_offsets_serial(misc, kMiscWarpB);
        }
        __syncthreads();
        int gr = (int)misc[kMiscWarpA + warp], er = (int)misc[kMiscWarpB + warp];
        for (int base = cs; base < ce; base += 32) {
          const int i = base + lane;
          const bool v = i < ce;
          const uint32_t x = v ? cand_key[i] : 0u;
          const bool is_gt = v && x > thr, is_eq = v && x == thr;
          const unsigned bg = __ballot_sync(0xFFFFFFFFu, is_gt);
          const unsigned be = __ballot_sync(0xFFFFFFFFu, is_eq);
          const int my_gr = gr + __popc(bg & lt), my_er = er + __popc(be & lt);
          const int at = my_gr + min(my_er, quota);
          if ((is_gt || (is_eq && my_er < quota)) && at < p.n_keep) {
            const int token = cand_idx[i];
            const int owner = at / p.slice;
            if (MODE == kDecode) cluster.map_shared_rank(idx_s, owner)[at - owner * p.slice] = token;
            if (p.idx_out) p.idx_out[(int64_t)row * p.n_keep + at] = token;
          }
          gr += __popc(bg);
          er += __popc(be);
        }
      }
      if (C > 1) {
        cluster_arrive();
        cluster_wait();
      } else {
        __syncthreads();
      }
    } else {
      // exact fallback over all keys, histograms summed across the cluster
      ballot_radix<true>(keys, n_loc, p.n_keep, 0u, 0, 32, rscr, chist, cluster, thr, quota);
      uint32_t cgt = 0u, ceq = 0u;
      for (int base = ws; base < we; base += 32) {
        const int i = base + lane;
        const bool v = i < we;
        const uint32_t x = v ? keys[i] : 0u;
        cgt += __popc(__ballot_sync(0xFFFFFFFFu, v && x > thr));
        ceq += __popc(__ballot_sync(0xFFFFFFFFu, v && x == thr));
      }
      if (lane == 0) {
        misc[kMiscWarpA + warp] = cgt;
        misc[kMiscWarpB + warp] = ceq;
      }
      __syncthreads();
      if (tid == 0) {
        misc[kMiscBcast + 1] = warp_offsets_serial(misc, kMiscWarpA);
        misc[kMiscBcast + 2] = warp_offsets_serial(misc, kMiscWarpB);
      }
      __syncthreads();
      if (tid < C) {
        uint32_t* dst = cluster.map_shared_rank(misc, tid);
        dst[kMiscCtaA + rank] = misc[kMiscBcast + 1];
        dst[kMiscCtaB + rank] = misc[kMiscBcast + 2];
      }
      if (C > 1) {
        cluster_arrive();
        cluster_wait();
      } else {
        __syncthreads();
      }
      uint32_t gb = 0u, eb = 0u;
      for (int r = 0; r < rank; ++r) {
        gb += misc[kMiscCtaA + r];
        eb += misc[kMiscCtaB + r];
      }
      int gr = (int)(gb + misc[kMiscWarpA + warp]);
      int er = (int)(eb + misc[kMiscWarpB + warp]);
      for (int base = ws; base < we; base += 32) {
        const int i = base + lane;
        const bool v = i < we;
        const uint32_t x = v ? keys[i] : 0u;
        const bool is_gt = v && x > thr, is_eq = v && x == thr;
        const unsigned bg = __ballot_sync(0xFFFFFFFFu, is_gt);
        const unsigned be = __ballot_sync(0xFFFFFFFFu, is_eq);
        const int my_gr = gr + __popc(bg & lt), my_er = er + __popc(be & lt);
        const int at = my_gr + min(my_er, quota);
        if (is_gt || (is_eq && my_er < quota)) {
          if (at < p.n_keep) {
            const int owner = at / p.slice;
            if (MODE == kDecode) cluster.map_shared_rank(idx_s, owner)[at - owner * p.slice] = start + i;
            if (p.idx_out) p.idx_out[(int64_t)row * p.n_keep + at] = start + i;
          } else {
            flag_status(FASA_ERR_BAD_INDEX);
          }
        }
        gr += __popc(bg);
        er += __popc(be);
      }
      if (C > 1) {
        cluster_arrive();
        cluster_wait();
      } else {
        __syncthreads();
      }
    }
    if (MODE == kDecode) {
      row_start = rank * p.slice;
      n_mine = max(0, min(p.slice, p.n_keep - row_start));
    }
  }

  if constexpr (!kAtt) {
    // no DSMEM access follows the last cluster barrier
    if (!start_waited) cluster_wait();
    return;
  } else {
    if (MODE == kAttendIdx) {
      row_start = rank * p.slice;
      n_mine = max(0, min(p.slice, p.n_keep - row_start));
      const int32_t* src = p.idx_in + (int64_t)row * p.n_keep + row_start;
      for (int j = tid; j < n_mine; j += kSAThreads) {
        int t = src[j];
        if (t < 0 || t >= p.len) {
          flag_status(FASA_ERR_BAD_INDEX);
          t = -1;
        }
        idx_s[j] = t;
      }
    } else if (MODE == kDense) {
      row_start = rank * p.chunk;
      n_mine = max(0, min(p.chunk, p.len - row_start));
    }
    __syncthreads();

    // rotated, pre-scaled queries: q'_h * log2(e) / sqrt(128), float32
    cp_async_wait<0>();
    __syncthreads();
    {
      const T* qh = reinterpret_cast<const T*>(qraw);
      const double qscale = 1.4426950408889634 / 11.313708498984761;  // log2(e) / sqrt(128)
      for (int e = tid; e < MAXG * kD; e += kSAThreads) {
        const int h = e / kD, d = e % kD, i = d & (kNFC - 1);
        float val = 0.0f;
        if (h < G) {
          const double x = to_float(qh[h * kD + i]);
          const double y = to_float(qh[h * kD + i + kNFC]);
          const double c = p.cosv[i], s = p.sinv[i];
          const double r = (d < kNFC) ? (x * c - y * s) : (y * c + x * s);
          val = (float)(r * qscale);
        }
        qs[e] = val;
      }
    }
    __syncthreads();

    const T* kbase = static_cast<const T*>(p.k) + (int64_t)row * p.max_len * kD;
    const T* vbase = static_cast<const T*>(p.v) + (int64_t)row * p.max_len * kD;
    const int nbatch = (n_mine + RB - 1) / RB;
    const int NST = p.n_stages;
    constexpr int CPR = kD * ES / 16;  // 16-byte chunks per row

    // load batch bi into stage bi % NST (gather: cp.async; dense: bulk copies)
    auto issue = [&](int bi) {
      if (bi < nbatch) {
        const int s = bi % NST;
        const int j0 = bi * RB;
        const int nr = min(RB, n_mine - j0);
        unsigned char* ks = stage + (size_t)s * kStageBytes;
        unsigned char* vs = ks + RB * kD * ES;
        if (MODE == kDense) {
          if (tid == 0) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&bars[s], (uint32_t)(nr * 2 * kD * ES));
            bulk_g2s(ks, kbase + (int64_t)(row_start + j0) * kD, (uint32_t)(nr * kD * ES), &bars[s]);
            bulk_g2s(vs, vbase + (int64_t)(row_start + j0) * kD, (uint32_t)(nr * kD * ES), &bars[s]);
          }
        } else {
          const int tot = nr * CPR;
          for (int c = tid; c < 2 * tot; c += kSAThreads) {
            const int which = c >= tot;
            const int rem = c - which * tot;
            const int r = rem / CPR, part = rem % CPR;
            int t = idx_s[j0 + r];
            if (t < 0 || t >= p.len) t = 0;  // masked below
            const T* src = (which ? vbase : kbase) + (int64_t)t * kD;
            cp_async16((which ? vs : ks) + r * kD * ES + part * 16,
                       reinterpret_cast<const unsigned char*>(src) + part * 16);
          }
        }
      }
      if (MODE != kDense) cp_async_commit();
    };

    // per-lane query slice: dims 4*lane .. 4*lane+3 of every head
    float qreg[kQReg ? MAXG : 1][4];
    if (kQReg) {
#pragma unroll
      for (int h = 0; h < (kQReg ? MAXG : 1); ++h) {
        const float4 qq = *reinterpret_cast<const float4*>(qs + h * kD + 4 * lane);
        qreg[h][0] = qq.x;
        qreg[h][1] = qq.y;
        qreg[h][2] = qq.z;
        qreg[h][3] = qq.w;
      }
    }

    float acc[MAXG][4];
#pragma unroll
    for (int h = 0; h < MAXG; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[h][e] = 0.0f;

    for (int s = 0; s < NST; ++s) issue(s);

    for (int bi = 0; bi < nbatch; ++bi) {
      const int s = bi % NST;
      const int j0 = bi * RB;
      const int nr = min(RB, n_mine - j0);
      const unsigned char* ks = stage + (size_t)s * kStageBytes;
      const unsigned char* vs = ks + RB * kD * ES;
      if (MODE == kDense) {
        mbar_wait(&bars[s], (uint32_t)((bi / NST) & 1));
      } else {
        if (NST == 2) cp_async_wait<1>();
        else if (NST == 3) cp_async_wait<2>();
        else cp_async_wait<3>();
        __syncthreads();
      }

      // logits: RPW rows per warp; lane owns 4 dims; butterfly reduce
      for (int rg = warp; rg * RPW < RB; rg += kSAWarps) {
        float v[NV];
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
          const int rr = rg * RPW + r;
          float kf[4];
          if (ES == 2) {
            const uint2 u = *reinterpret_cast<const uint2*>(ks + (rr * kD + 4 * lane) * ES);
            kf[0] = __uint_as_float(u.x << 16);
            kf[1] = __uint_as_float(u.x & 0xFFFF0000u);
            kf[2] = __uint_as_float(u.y << 16);
            kf[3] = __uint_as_float(u.y & 0xFFFF0000u);
          } else {
            const float4 u = *reinterpret_cast<const float4*>(ks + (rr * kD + 4 * lane) * ES);
            kf[0] = u.x;
            kf[1] = u.y;
            kf[2] = u.z;
            kf[3] = u.w;
          }
#pragma unroll
          for (int h = 0; h < MAXG; ++h) {
            float q0, q1, q2, q3;
            if (kQReg) {
              q0 = qreg[kQReg ? h : 0][0];
              q1 = qreg[kQReg ? h : 0][1];
              q2 = qreg[kQReg ? h : 0][2];
              q3 = qreg[kQReg ? h : 0][3];
            } else {
              const float4 qq = *reinterpret_cast<const float4*>(qs + h * kD + 4 * lane);
              q0 = qq.x;
              q1 = qq.y;
              q2 = qq.z;
              q3 = qq.w;
            }
            float a = q0 * kf[0];
            a = fmaf(q1, kf[1], a);
            a = fmaf(q2, kf[2], a);
            v[h * RPW + r] = fmaf(q3, kf[3], a);
          }
        }
        // butterfly transpose-reduce: after it, lane l holds the full sum of
        // item l mod NV (with NV = 16 the lane-bit-4 pairs are summed first)
        if (NV == 16) {
#pragma unroll
          for (int j = 0; j < NV; ++j) v[j] += __shfl_xor_sync(0xFFFFFFFFu, v[j], 16);
        }
#pragma unroll
        for (int w = NV / 2; w >= 1; w >>= 1) {
          const bool upper = (lane & w) != 0;
#pragma unroll
          for (int j = 0; j < w; ++j) {
            const float send = upper ? v[j] : v[j + w];
            const float keep = upper ? v[j + w] : v[j];
            v[j] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, w);
          }
        }
        const int item = lane & (NV - 1);
        const int h = item / RPW, rr = rg * RPW + item % RPW;
        if (lane < NV && h < G) {
          bool valid = rr < nr;
          if (MODE != kDense && valid) {
            const int t = idx_s[j0 + rr];
            valid = t >= 0 && t < p.len;
            if (MODE == kDecode && !valid) flag_status(FASA_ERR_BAD_INDEX);
          }
          zs[h * RB + rr] = valid ? v[0] : -INFINITY;
        }
      }
      __syncthreads();
      // online softmax: one warp per query head
      if (warp < G) {
        const int h = warp;
        float mx = -INFINITY;
        for (int r = lane; r < RB; r += 32) mx = fmaxf(mx, zs[h * RB + r]);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
        const float m_old = ml[h];
        const float m_new = fmaxf(m_old, mx);
        const float sc = (m_old == -INFINITY) ? 0.0f : exp2f(m_old - m_new);
        float sum = 0.0f;
        for (int r = lane; r < RB; r += 32) {
          const float z = zs[h * RB + r];
          const float pz = (z == -INFINITY) ? 0.0f : exp2f(z - m_new);
          zs[h * RB + r] = pz;
          sum += pz;
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
        if (lane == 0) {
          ml[h] = m_new;
          ml[MAXG + h] = ml[MAXG + h] * sc + sum;
          ml[2 * MAXG + h] = sc;
        }
      }
      __syncthreads();
      // P.V: thread = (quad of dims = lane, row group = warp)
#pragma unroll
      for (int h = 0; h < MAXG; ++h) {
        if (h < G) {
          const float sc = ml[2 * MAXG + h];
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[h][e] *= sc;
        }
      }
      for (int r = warp; r < nr; r += kSAWarps) {
        float vf[4];
        if (ES == 2) {
          const uint2 u = *reinterpret_cast<const uint2*>(vs + (r * kD + lane * 4) * ES);
          vf[0] = __uint_as_float(u.x << 16);
          vf[1] = __uint_as_float(u.x & 0xFFFF0000u);
          vf[2] = __uint_as_float(u.y << 16);
          vf[3] = __uint_as_float(u.y & 0xFFFF0000u);
        } else {
          const float4 u = *reinterpret_cast<const float4*>(vs + (r * kD + lane * 4) * ES);
          vf[0] = u.x;
          vf[1] = u.y;
          vf[2] = u.z;
          vf[3] = u.w;
        }
#pragma unroll
        for (int h = 0; h < MAXG; ++h) {
          if (h < G) {
            const float pz = zs[h * RB + r];
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[h][e] = fmaf(pz, vf[e], acc[h][e]);
          }
        }
      }
      __syncthreads();  // stage s and zs fully consumed
      issue(bi + NST);
    }
    if (MODE != kDense) cp_async_wait<0>();

    // reduce the 16 row groups: per-warp partials through shared memory (the
    // stage area is free now), heads in chunks that fit
    float* part = reinterpret_cast<float*>(stage);
    const int hc = min(MAXG, (NST * kStageBytes) / (kSAWarps * kD * 4));
    __syncthreads();
    for (int h0 = 0; h0 < G; h0 += hc) {
#pragma unroll
      for (int h = 0; h < MAXG; ++h)
        if (h >= h0 && h < h0 + hc && h < G)
#pragma unroll
          for (int e = 0; e < 4; ++e) part[((h - h0) * kSAWarps + warp) * kD + lane * 4 + e] = acc[h][e];
      __syncthreads();
      for (int e = tid; e < hc * kD; e += kSAThreads) {
        const int hh = e / kD, d = e % kD;
        if (h0 + hh < G) {
          float s = 0.0f;
#pragma unroll
          for (int w = 0; w < kSAWarps; ++w) s += part[(hh * kSAWarps + w) * kD + d];
          acc_s[(h0 + hh) * kD + d] = s;
        }
      }
      __syncthreads();
    }

    T* out = static_cast<T*>(p.out) + ((int64_t)row * G) * kD;
    if (C == 1) {
      for (int e = tid; e < G * kD; e += kSAThreads) {
        const float l = ml[MAXG + e / kD];
        store_f(out + e, l > 0.0f ? acc_s[e] / l : 0.0f);
      }
      return;
    }
    if (!start_waited) {
      cluster_wait();
      start_waited = true;
    }
    // merge: (m, l) of every CTA to every CTA ...
    if (tid < C * G) {
      const int r = tid / G, h = tid % G;
      float* dst = cluster.map_shared_rank(mlall, r);
      dst[(rank * MAXG + h) * 2] = ml[h];
      dst[(rank * MAXG + h) * 2 + 1] = ml[MAXG + h];
    }
    cluster_arrive();
    cluster_wait();
    // ... then each CTA adds its rescaled o into the owner of each output
    if (tid < G) {
      float M = -INFINITY;
      for (int r = 0; r < C; ++r) M = fmaxf(M, mlall[(r * MAXG + tid) * 2]);
      float lsum = 0.0f;
      if (M != -INFINITY)
        for (int r = 0; r < C; ++r) {
          const float mr = mlall[(r * MAXG + tid) * 2];
          if (mr != -INFINITY) lsum += exp2f(mr - M) * mlall[(r * MAXG + tid) * 2 + 1];
        }
      ml[3 * MAXG + tid] = (ml[tid] == -INFINITY || M == -INFINITY) ? 0.0f : exp2f(ml[tid] - M);
      ml[2 * MAXG + tid] = lsum;
    }
    __syncthreads();
    // each source CTA has its own slot in the owner, summed in rank order
    // below, so the result does not depend on arrival order
    const int per_owner = (G * kD + C - 1) / C;
    for (int e = tid; e < G * kD; e += kSAThreads) {
      const int owner = e / per_owner;
      cluster.map_shared_rank(red, owner)[rank * per_owner + (e - owner * per_owner)] =
          ml[3 * MAXG + e / kD] * acc_s[e];
    }
    cluster_arrive();
    cluster_wait();
    const int e0 = rank * per_owner, e1 = min(G * kD, e0 + per_owner);
    for (int e = e0 + tid; e < e1; e += kSAThreads) {
      float s = 0.0f;
      for (int r = 0; r < C; ++r) s += red[r * per_owner + (e - e0)];
      const float l = ml[2 * MAXG + e / kD];
      store_f(out + e, l > 0.0f ? s / l : 0.0f);
    }
    // no DSMEM access follows the last cluster barrier
  }
}

}  // namespace fasa
