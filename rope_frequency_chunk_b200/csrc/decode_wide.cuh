// Fused decode for bf16 caches: each (batch, KV head) row is spread over
// n_split independent CTAs, so a layer fills the GPU whatever its row count.
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2): TIP scores from the dominant FCs only ("online prediction", a proxy at
// no significant compute cost), the critical set T_t = the k highest-scoring
// tokens (ties to the lower index, k_eff = min(k, L)), then full softmax
// attention of every query head of the group over exactly those rows at
// their original positions (FAC).
//
// Grid n_split x rows, 512 threads, no clusters. CTA s of a row owns the
// tokens [s*n_loc, (s+1)*n_loc). Every CTA:
//  1. prefetches its sketch range into L2 (a hint, issued before the wait on
//     the preceding grid, so a layer's stream overlaps the previous layer's
//     tail), waits, then forms the float32 TIP coefficients of its group
//     (tip.cuh);
//  2. streams its sketch rows straight into registers with 16-byte loads
//     (one token per lane, 2 or 4 lanes for wide rows), scores them in
//     float32 and keeps each score's order-preserving key in shared memory,
//     with a 4096-bin histogram of the top 12 key bits;
//  3. finds the bin b_loc holding its own k_eff-th key and publishes every
//     token in bins >= b_loc as a (key, token) pair: a token of the row's top
//     k_eff is in its CTA's top k_eff, so the published union holds the row's
//     whole critical set, and every token of the row in a bin at or above the
//     row's boundary bin (which is >= every b_loc);
//  4. takes a ticket on the row's semaphore word; the last CTA of the row to
//     arrive (no CTA ever waits on another) resolves the row:
//      - a histogram of the union gives the boundary bin B and the count
//        above it (exact: the union holds every token of bins >= B);
//      - tokens above B are kept; among the tokens of B the need largest keys
//        are kept, ties to the lower token index (rank counting for a few,
//        else an exact radix select);
//      - a bitmap of the kept tokens emits them in ascending order;
//      - with `direct` (k_eff <= 512, G <= 8) the same CTA attends them on
//        CUDA cores (attend_cc.cuh: each warp a contiguous part of the kept
//        list, then the warps merged); otherwise it writes the kept list for
//        attend_cc_kernel, launched next.
//
// Semaphore: sem[row] counts the row's CTAs that have published. It must be
// zero when a call starts; the last CTA of the row writes it back to zero,
// so a workspace zeroed once stays valid. A ticket beyond its range (a
// workspace that was not zero) is flagged FASA_ERR_WORKSPACE; region counts
// are clamped to the region size, so nothing is read out of bounds.
#pragma once

#include "attend_cc.cuh"
#include "select_attend.cuh"
#include "tip.cuh"

namespace fasa {

constexpr int kWdThreads = kSAThreads;  // 512 (the histogram and radix helpers' block size)
constexpr int kWdWarps = kWdThreads / 32;
constexpr int kWdMaxLoc = 16384;        // tokens per CTA (their keys live in shared memory)
constexpr int kWdTieCap = 2048;         // boundary-bin entries held in shared memory
constexpr int kWdRankMax = 128;         // entries of the finest bin resolved by rank counting
constexpr int kWdUnionUnroll = 8;       // union entries in flight per thread
constexpr int kWdMaxDirect = 16 * kWdWarps;  // kept rows the resolving CTA attends itself (16 per warp)
// radix scratch: the sub-bin histogram and entries, then ballot_radix_fn's
constexpr int kWdRadixWords = 256 + 2 * 128 + kSAWarps * 256 + 264;
constexpr int kWdMisc = 128;            // words of scan and flag scratch

struct WideParams {
  const __nv_bfloat16* sketch;  // [rows][max_len][stride]
  const __nv_bfloat16* k;       // [rows][max_len][128], rotated
  const __nv_bfloat16* v;
  const __nv_bfloat16* q;       // [B][Hq][128], pre-RoPE
  const int32_t* dom_idx;       // [Hkv][n_dom]
  __nv_bfloat16* out;           // [B][Hq][128]
  int32_t* idx_out;             // [rows][n_keep] kept tokens, ascending, or null
  int32_t* idx_ws;              // [rows][n_keep] for the attention launch, or null (direct)
  uint2* cand;                  // [rows][n_split][n_loc + 1] regions: (count, b_loc), then (key, token) pairs
  uint32_t* keys;               // [rows][len] every token's score key
  unsigned long long* sem;      // [rows], zero between calls
  int64_t max_len;
  int32_t len;
  int32_t stride;
  int32_t n_kv_heads;
  int32_t group;
  int32_t n_dom;
  int32_t n_keep;   // k_eff, 1 .. len
  int32_t n_pub;    // each CTA publishes its n_pub best tokens (with the rest of their bin), <= n_keep
  int32_t n_loc;    // tokens per CTA, <= kWdMaxLoc
  int32_t n_split;  // CTAs per row
  int32_t ucache;   // entries of each CTA's region the resolving CTA stages in shared memory (P, a power of two)
  int32_t ushift;   // log2(P)
  int32_t direct;   // 1: the resolving CTA attends (n_keep <= kWdMaxDirect, G <= 8)
  // per-sequence lengths and per-head budgets (fasa_decode_varlen), or null:
  // len and n_keep for every row; len and n_keep are then upper bounds and
  // the row strides of keys and the kept lists
  const int32_t* seq_len;  // [B]
  const int32_t* budget;   // [Hkv]
  int32_t* row_keep;       // [rows] each row's k_eff, for the attention launch (varlen), or null
  int32_t q_prerot;        // varlen: 1 if the queries are already rotated
  PageMap pm;              // paged pools (pm.table set), else [rows][max_len] planes
  // multi-query decode: n_q query tokens per sequence, q [B][n_q][Hq][128],
  // token j at position q_pos0 + j (angles from theta_i in cosv), or 1
  int32_t n_q;
  int32_t q_pos0;
  double cosv[kNFC];       // cos / sin of the query angle (uniform length), or
  double sinv[kNFC];       // theta_i in cosv (varlen: the angle is seq_len[b] * theta_i)
};

// The row's length and k_eff: uniform, or from the device arrays (clamped
// into range, a value outside flagged).
__device__ __forceinline__ int2 wd_row_shape(const WideParams& p, int row) {
  int L = p.len, k = p.n_keep;
  if (p.seq_len) {
    const int b = row / p.n_kv_heads, g = row % p.n_kv_heads;
    L = __ldg(p.seq_len + b);
    if (L < 1 || L > p.len) {
      if (threadIdx.x == 0) flag_status(FASA_ERR_BAD_INDEX);
      L = min(max(L, 1), p.len);
    }
    if (p.budget) {
      k = __ldg(p.budget + g);
      if (k < 1 || k > p.n_keep) {
        if (threadIdx.x == 0) flag_status(FASA_ERR_BAD_INDEX);
        k = min(max(k, 1), p.n_keep);
      }
    }
  }
  return make_int2(L, min(k, L));
}

__host__ __device__ constexpr int wd_al(int x, int a) { return (x + a - 1) / a * a; }

// Shared-memory layout. r1 is reused: the CTA's keys (steps 1-3); then, in
// the resolving CTA, the bitmap, boundary-bin entries, radix scratch and the
// staged union ([n_split][P] entries); then the attention's logits, warp
// sums and V rows.
struct WdLayout {
  int hist, misc, coef, qraw, dom, cs, qs, pgs, cnt, kept, r1, bitmap, ties, rscr, ucache, zs, ring, total;
};
__host__ __device__ inline WdLayout wd_layout(int n_loc, int len, int n_keep, int direct, int group, int n_split,
                                              int P, int paged, int n_q) {
  WdLayout L;
  const int MG = group <= 4 ? 4 : 8;
  int o = 0;
  L.hist = o;
  o += 4096 * 4;
  L.misc = o;
  o += kWdMisc * 4;
  L.coef = o;
  o += kD * 4;
  L.qraw = o;
  o += (n_q * group > FASA_MAX_GROUP ? n_q * group : FASA_MAX_GROUP) * kD * 2;
  L.dom = o;
  o += kNFC * 4;
  L.cs = o;  // cos, sin of each query token's angle (float64)
  o += 2 * kNFC * 8 * n_q;
  L.qs = o;  // attention queries [MG][128] f32
  o += direct ? MG * kD * 4 : 0;
  L.pgs = o;  // paged: the CTA's pages (block size >= 16)
  o += paged ? wd_al((n_loc / 16 + 2) * 4, 16) : 0;
  L.cnt = o;  // region counts, their prefix sums, the regions' b_loc
  o += wd_al((3 * n_split + 2) * 4, 16);
  L.kept = o;
  o += wd_al(direct ? n_keep * 4 : 0, 128);
  L.r1 = o;
  const int a = n_loc * 4;
  L.bitmap = o;
  int b = wd_al((len + 31) / 32 * 4, 16);
  L.ties = o + b;
  b += kWdTieCap * 8;
  L.rscr = o + b;
  b += wd_al(kWdRadixWords * 4, 16);
  L.ucache = o + b;
  b += n_split * P * 8;
  // the attention (cc_block_attend): logits [256][MG] f32, warp sums
  // [16][MG][128] f32, head sums [MG] (64 B), V rows [256][128] bf16
  L.zs = o;
  int c = 0;
  if (direct) {
    c = kWdMaxDirect * MG * 4;
    L.ring = o + c;
    c += kWdWarps * MG * kD * 4 + 64 + kWdMaxDirect * kD * 2;
  } else {
    L.ring = o;
  }
  L.total = o + (a > b ? (a > c ? a : c) : (b > c ? b : c));
  return L;
}

// Exclusive scan of one value per thread over the 512 threads; returns the
// thread's offset and, in *total, the sum. scr: 17 words. Ends synchronized.
__device__ __forceinline__ uint32_t wd_block_scan(uint32_t v, uint32_t* scr, uint32_t* total) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t x = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += x;
  }
  if (lane == 31) scr[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kWdWarps ? scr[lane] : 0u;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t x = __shfl_up_sync(0xFFFFFFFFu, w, off);
      if (lane >= off) w += x;
    }
    if (lane < kWdWarps) scr[lane] = w;  // inclusive warp sums
  }
  __syncthreads();
  const uint32_t before = warp > 0 ? scr[warp - 1] : 0u;
  *total = scr[kWdWarps - 1];
  __syncthreads();
  return before + incl - v;
}

__device__ __forceinline__ void wd_keep(uint32_t* bm, uint32_t t, int len) {
  if (t < (uint32_t)len) atomicOr(bm + (t >> 5), 1u << (t & 31));
}

// Exact choice of the `need` largest keys among the entries whose top
// `known` key bits equal those of `prefix` (ties to the lower token index), by
// two radix selects: the need-th key K, then, if only some of the keys equal
// to K fit, the lowest token indices among them. entry_at(i) gives entry i
// of n (any entries; only the prefix's take part). rscr: kSAWarps * 256 +
// 258 words.
template <typename At>
__device__ void wd_resolve_radix(At entry_at, int n, int need, uint32_t prefix, int known, uint32_t* rscr,
                                 uint32_t* misc, uint32_t* bm, int len) {
  cg::cluster_group cl = cg::this_cluster();
  const int tid = threadIdx.x;
  uint32_t K = 0;
  int krem = 0;
  ballot_radix_fn<false>([&](int i) { return entry_at(i).x; }, n, need, prefix, known, 32, rscr, nullptr, cl, K,
                         krem);
  // keys above K with the prefix are kept; count the keys equal to K
  const uint32_t pmask = ~0u << (32 - known);
  if (tid == 0) misc[0] = 0u;
  __syncthreads();
  for (int i = tid; i < n; i += kWdThreads) {
    const uint2 e = entry_at(i);
    if ((e.x & pmask) == prefix && e.x > K) wd_keep(bm, e.y, len);
    if (e.x == K) atomicAdd(misc, 1u);
  }
  __syncthreads();
  const int n_eq = (int)misc[0];
  __syncthreads();
  if (krem >= n_eq) {
    for (int i = tid; i < n; i += kWdThreads) {
      const uint2 e = entry_at(i);
      if (e.x == K) wd_keep(bm, e.y, len);
    }
    return;
  }
  // the krem lowest indices among the keys equal to K: select the largest ~t
  // (token indices are below 2^19, so ~t has its top 13 bits set)
  uint32_t T = 0;
  int trem = 0;
  ballot_radix_fn<false>([&](int i) {
    const uint2 e = entry_at(i);
    return e.x == K ? ~e.y : 0u;
  }, n, krem, 0xFFF80000u, 13, 32, rscr, nullptr, cl, T, trem);
  for (int i = tid; i < n; i += kWdThreads) {
    const uint2 e = entry_at(i);
    if (e.x == K && ~e.y >= T) wd_keep(bm, e.y, len);
  }
}

// One warp: in the 256-bin histogram h, the bin holding the k-th largest
// (k <= total) and the count in higher bins, written to out[0], out[1].
// Lane l owns bins 255 - 8l .. 248 - 8l.
__device__ __forceinline__ void wd_warp_bin256(const uint32_t* h, int k, uint32_t* out) {
  const int lane = threadIdx.x & 31;
  uint32_t c[8], sum = 0u;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    c[u] = h[255 - (8 * lane + u)];
    sum += c[u];
  }
  uint32_t incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t x = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += x;
  }
  const uint32_t excl = incl - sum;
  if (excl < (uint32_t)k && (uint32_t)k <= incl) {
    uint32_t acc = excl;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (acc + c[u] >= (uint32_t)k) {
        out[0] = 255u - (uint32_t)(8 * lane + u);
        out[1] = acc;
        break;
      }
      acc += c[u];
    }
  }
}

// Exact choice of the n_keep largest keys (ties to the lower token index)
// among n_src (key, token) entries, given their 4096-bin histogram of the
// top 12 key bits in hist: sets the kept tokens' bits in bm (zero before).
// for_src(fn) calls fn(entry) once per entry, spread over the CTA's threads;
// src_at(i) is entry i (for the rare radix path). *B_out: the boundary bin.
template <typename ForSrc, typename SrcAt>
__device__ void wd_select(ForSrc&& for_src, SrcAt&& src_at, int n_src, int n_keep, uint32_t* hist, uint32_t* misc,
                          uint32_t* bm, uint2* ties, uint32_t* rscr, int len, uint32_t* B_out) {
  const int tid = threadIdx.x, warp = tid >> 5;
  uint32_t B = 0u, above = 0u;
  if (n_keep > 0) hist_threshold_fn([&](int i) { return hist[i]; }, n_keep, misc, B, above);
  if (tid == 0) misc[100] = 0u;
  __syncthreads();
  for_src([&](const uint2& e) {
    const uint32_t b = e.x >> 20;
    if (b > B) {
      wd_keep(bm, e.y, len);
    } else if (b == B) {
      const uint32_t at = atomicAdd(misc + 100, 1u);
      if (at < (uint32_t)kWdTieCap) ties[at] = e;
    }
  });
  __syncthreads();
  const int n_b = (int)misc[100];
  const int need = n_keep - (int)above;
  __syncthreads();
  if (need > 0 && n_keep > 0) {
    if (n_b == need && n_b <= kWdTieCap) {
      for (int i = tid; i < n_b; i += kWdThreads) wd_keep(bm, ties[i].y, len);
    } else if (n_b <= kWdTieCap) {
      // next 8 key bits of the boundary bin's entries, then ranks (or a
      // radix select) among the entries of the boundary sub-bin
      uint32_t* h2 = rscr;             // 256 counts
      uint2* t2 = reinterpret_cast<uint2*>(rscr + 256);  // the sub-bin's entries
      for (int i = tid; i < 256; i += kWdThreads) h2[i] = 0u;
      if (tid == 0) misc[101] = 0u;
      __syncthreads();
      for (int i = tid; i < n_b; i += kWdThreads) atomicAdd(h2 + ((ties[i].x >> 12) & 255u), 1u);
      __syncthreads();
      if (warp == 0) wd_warp_bin256(h2, need, misc + 102);
      __syncthreads();
      const uint32_t B2 = misc[102];
      const int need2 = need - (int)misc[103];
      for (int i = tid; i < n_b; i += kWdThreads) {
        const uint2 e = ties[i];
        const uint32_t sb = (e.x >> 12) & 255u;
        if (sb > B2) {
          wd_keep(bm, e.y, len);
        } else if (sb == B2) {
          const uint32_t at = atomicAdd(misc + 101, 1u);
          if (at < (uint32_t)kWdRankMax) t2[at] = e;
        }
      }
      __syncthreads();
      const int n_b2 = (int)misc[101];
      __syncthreads();
      if (n_b2 == need2 && n_b2 <= kWdRankMax) {
        for (int i = tid; i < n_b2; i += kWdThreads) wd_keep(bm, t2[i].y, len);
      } else if (n_b2 <= kWdRankMax) {
        for (int i = tid; i < n_b2; i += kWdThreads) {
          const uint2 a = t2[i];
          int r = 0;
          for (int j = 0; j < n_b2; ++j) {
            const uint2 c = t2[j];
            r += (c.x > a.x) || (c.x == a.x && c.y < a.y);
          }
          if (r < need2) wd_keep(bm, a.y, len);
        }
      } else {
        // a crowded sub-bin (ties): exact radix select over the boundary
        // bin's entries, restricted to the sub-bin by its 20-bit prefix
        const uint32_t pre = (B << 20) | (B2 << 12);
        wd_resolve_radix([&](int i) { return ties[i]; }, n_b, need2, pre, 20, rscr + 256 + 2 * kWdRankMax, misc,
                         bm, len);
      }
    } else {
      wd_resolve_radix(src_at, n_src, need, B << 20, 12, rscr, misc, bm, len);
    }
  }
  __syncthreads();

  *B_out = B;
}

template <int LPT, int MG>
__global__ void __launch_bounds__(kWdThreads, 1) decode_wide_kernel(const WideParams p) {
  using S = TipShape<__nv_bfloat16, LPT>;
  constexpr int U = S::LPT2 == 1 ? 4 : 2;  // tokens in flight per lane
  extern __shared__ __align__(128) unsigned char smem[];
  const WdLayout Lo = wd_layout(p.n_loc, p.len, p.n_keep, p.direct, p.group, p.n_split, p.ucache, p.pm.table != nullptr,
                                p.n_q);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + Lo.hist);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lo.misc);
  float* coef = reinterpret_cast<float*>(smem + Lo.coef);
  __nv_bfloat16* qraw = reinterpret_cast<__nv_bfloat16*>(smem + Lo.qraw);
  int* s_dom = reinterpret_cast<int*>(smem + Lo.dom);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + Lo.r1);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, row = blockIdx.y;
  const int t_beg = split * p.n_loc;
  const int2 shp = wd_row_shape(p, row);
  const int Lr = shp.x, kr = shp.y;  // the row's length and k_eff
  // each CTA publishes its n_pub best (about twice its share of the kept set)
  const int n_pub = p.seq_len ? (p.n_split == 1 ? kr : min(kr, (2 * ((kr + p.n_split - 1) / p.n_split) + 63) / 32 * 32))
                              : p.n_pub;
  const int n_tok = max(0, min(Lr - t_beg, p.n_loc));
  const bool paged = p.pm.table != nullptr;
  const int bb = row / p.n_kv_heads, g = row % p.n_kv_heads;
  const char* src = reinterpret_cast<const char*>(p.sketch) + ((int64_t)row * p.max_len + t_beg) * S::ROWB;
  if (!paged) {  // L2 prefetch of this CTA's sketch range: a hint, safe before the wait
    const int64_t bytes = (int64_t)n_tok * S::ROWB;
    constexpr int kPf = 8192;
    for (int64_t o = (int64_t)tid * kPf; o < bytes; o += (int64_t)kWdThreads * kPf)
      prefetch_l2(src + o, (uint32_t)(bytes - o < kPf ? bytes - o : kPf));
  }
  double* cs_sm = reinterpret_cast<double*>(smem + Lo.cs);
  // the angle table from the parameters (no dependence on the previous
  // launch): read before the wait, so its constant-bank misses overlap it
  if (p.n_q == 1 && !p.seq_len) {
    if (tid < kNFC) cs_sm[tid] = p.cosv[tid];
    else if (tid < 2 * kNFC) cs_sm[tid] = p.sinv[tid - kNFC];
  }
  // the group's queries and dominant FCs to L2 (hints: the loads after the
  // wait still see what an earlier launch wrote)
  if (p.n_q == 1 && tid >= 2 * kNFC && tid < 2 * kNFC + p.group * 2)
    prefetch_line_l2(p.q + ((int64_t)(bb * p.n_kv_heads + g) * p.group) * kD + (tid - 2 * kNFC) * 64);
  if (tid == 2 * kNFC + 2 * FASA_MAX_GROUP) prefetch_line_l2(p.dom_idx + g * p.n_dom);
  grid_dependency_wait();
  grid_dependents_launch();
  // paged: the CTA's pages (read after the wait: an earlier launch may have
  // written the table), each prefetched to L2 whole
  int* s_pg = reinterpret_cast<int*>(smem + Lo.pgs);
  const int pg0 = paged ? t_beg >> p.pm.log2bs : 0;
  if (paged) {
    const int n_pg = n_tok > 0 ? ((t_beg + n_tok - 1) >> p.pm.log2bs) - pg0 + 1 : 0;
    for (int i = tid; i < n_pg; i += kWdThreads) {
      int pg = __ldg(p.pm.table + (int64_t)bb * p.pm.max_blocks + pg0 + i);
      if ((unsigned)pg >= (unsigned)p.pm.n_pages) {
        flag_status(FASA_ERR_BAD_INDEX);
        pg = -1;
      } else {
        prefetch_l2(reinterpret_cast<const char*>(p.sketch) +
                        ((int64_t)(pg * p.pm.n_kv_heads + g) << p.pm.log2bs) * S::ROWB,
                    (uint32_t)(S::ROWB << p.pm.log2bs));
      }
      s_pg[i] = pg;
    }
    __syncthreads();
  }
  // sketch row of the CTA's token t (< n_tok), or null for a page outside the pool
  auto sk_row = [&](int t) -> const char* {
    if (!paged) return src + (int64_t)t * S::ROWB;
    const int tt = t_beg + t, pg = s_pg[(tt >> p.pm.log2bs) - pg0];
    if (pg < 0) return nullptr;
    return reinterpret_cast<const char*>(p.sketch) +
           (int64_t)(((pg * p.pm.n_kv_heads + g) << p.pm.log2bs) | (tt & ((1 << p.pm.log2bs) - 1))) * S::ROWB;
  };

  // 1. the group's queries, dominant FCs and rotation table; the CTA's first
  // sketch rows are requested before the coefficients are formed, so the
  // query's round trip and the float64 work overlap the stream
  const int G = p.group;
  {
    if (p.n_q == 1) {  // one round trip: both loads in flight before either store
      const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + ((int64_t)(bb * p.n_kv_heads + g) * G) * kD);
      const uint4 qv = tid < G * kD / 8 ? __ldg(qsrc + tid) : make_uint4(0u, 0u, 0u, 0u);
      const int dv = tid < p.n_dom ? __ldg(p.dom_idx + g * p.n_dom + tid) : 0;
      if (tid < G * kD / 8) reinterpret_cast<uint4*>(qraw)[tid] = qv;
      if (tid < p.n_dom) s_dom[tid] = dv;
    } else {  // rows j * G + h: token j's group queries
      const int hq = p.n_kv_heads * G;
      for (int c = tid; c < p.n_q * G * kD / 8; c += kWdThreads) {
        const int r = c / (kD / 8), j = r / G, h = r % G;
        reinterpret_cast<uint4*>(qraw)[c] = __ldg(
            reinterpret_cast<const uint4*>(p.q + (((int64_t)bb * p.n_q + j) * hq + g * G + h) * kD) + c % (kD / 8));
      }
    }
    if (p.n_q > 1 && tid < p.n_dom) s_dom[tid] = __ldg(p.dom_idx + g * p.n_dom + tid);
    if (p.n_q > 1) {  // token j at position q_pos0 + j
      for (int e = tid; e < p.n_q * kNFC; e += kWdThreads) {
        const int j = e / kNFC, i = e % kNFC;
        double sn = 0.0, cn = 1.0;
        if (!p.q_prerot) sincos((double)(p.q_pos0 + j) * p.cosv[i], &sn, &cn);
        cs_sm[j * 2 * kNFC + i] = cn;
        cs_sm[j * 2 * kNFC + kNFC + i] = sn;
      }
    } else if (p.seq_len && tid < kNFC) {  // the query of sequence b sits at position Lr
      double sn = 0.0, cn = 1.0;
      if (!p.q_prerot) sincos((double)Lr * p.cosv[tid], &sn, &cn);
      cs_sm[tid] = cn;
      cs_sm[kNFC + tid] = sn;
    }
  }
  constexpr int kTokPass = kWdThreads / S::LPT2;
  const int my_tok = tid / S::LPT2;
  const int sub = tid % S::LPT2;  // the lane's chunk group; a token's lanes are adjacent
  uint4 v[U][S::CPL];
  auto load_rows = [&](int base) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = base + u * kTokPass + my_tok;
      const char* rp = t < n_tok ? sk_row(t) : nullptr;
#pragma unroll
      for (int c = 0; c < S::CPL; ++c)
        v[u][c] = rp ? __ldg(reinterpret_cast<const uint4*>(rp) + sub * S::CPL + c) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  load_rows(0);
  for (int i = tid; i < 4096; i += kWdThreads) hist[i] = 0u;
  __syncthreads();
  if (tid < p.stride)
    coef[tid] = tip_coef<__nv_bfloat16>(qraw, s_dom, G, p.n_dom, tid, cs_sm, cs_sm + kNFC, p.n_q, 2 * kNFC);
  // the attention queries, used by the row's resolving CTA
  if (p.direct) cc_queries(qraw, G, MG, cs_sm, cs_sm + kNFC, reinterpret_cast<float*>(smem + Lo.qs), tid, kWdThreads);
  __syncthreads();
  float cr[S::EPL];
#pragma unroll
  for (int e = 0; e < S::EPL; ++e) cr[e] = coef[sub * S::EPL + e];

  // 2. score the CTA's tokens straight from global memory
  for (int base = 0; base < n_tok; base += kTokPass * U) {  // block-uniform trip count
    if (base > 0) load_rows(base);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = base + u * kTokPass + my_tok;
      float part[S::CPL];
#pragma unroll
      for (int c = 0; c < S::CPL; ++c) part[c] = tip_chunk(v[u][c], cr + c * 8, __nv_bfloat16());
      const float sc = tip_lanes_sum<S::LPT2>(tip_lane_sum<S::CPL>(part));
      if (t < n_tok && sub == 0) {
        const uint32_t key = score_key(sc);
        keys[t] = key;
        atomicAdd(hist + (key >> 20), 1u);
      }
    }
  }
  __syncthreads();

  // 3. every key to the row's key array (for the exact fallback; written
  // first, so that the stores complete while the rest of this step runs);
  // the bin b_loc holding this CTA's n_pub-th key; publish the tokens at or
  // above it into the CTA's own region: [(count, b_loc)][(key, token) ...]
  {
    uint32_t* kdst = p.keys + (int64_t)row * p.len + t_beg;
    for (int i = tid; i < n_tok; i += kWdThreads) kdst[i] = keys[i];
  }
  uint32_t b_loc = 0u;
  if (n_tok > n_pub) {
    uint32_t above = 0u;
    hist_threshold_fn([&](int i) { return hist[i]; }, n_pub, misc, b_loc, above);
  }
  uint32_t wc = 0u;
  for (int i0 = warp * 32; i0 < n_tok; i0 += kWdThreads) {
    const int i = i0 + lane;
    wc += __popc(__ballot_sync(0xFFFFFFFFu, i < n_tok && (keys[i] >> 20) >= b_loc));
  }
  if (lane == 0) misc[64 + warp] = wc;
  __syncthreads();
  if (warp == 0) {  // exclusive offsets of the warps, and the total
    const uint32_t c = lane < kWdWarps ? misc[64 + lane] : 0u;
    uint32_t incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t x = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += x;
    }
    if (lane < kWdWarps) misc[64 + lane] = incl - c;
    if (lane == kWdWarps - 1) misc[96] = incl;
  }
  __syncthreads();
  const int64_t rstride = (int64_t)p.n_loc + 1;  // entries per region, with its header
  uint2* region = p.cand + ((int64_t)row * p.n_split + split) * rstride;
  {
    uint32_t pos = 1u + misc[64 + warp];
    for (int i0 = warp * 32; i0 < n_tok; i0 += kWdThreads) {
      const int i = i0 + lane;
      const uint32_t key = i < n_tok ? keys[i] : 0u;
      const bool q = i < n_tok && (key >> 20) >= b_loc;
      const unsigned m = __ballot_sync(0xFFFFFFFFu, q);
      if (q) region[pos + __popc(m & ((1u << lane) - 1u))] = make_uint2(key, (uint32_t)(t_beg + i));
      pos += __popc(m);
    }
    if (tid == 0) region[0] = make_uint2(misc[96], b_loc);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned long long old = atomicAdd(p.sem + row, 1ull);
    if (old >= (unsigned long long)p.n_split) flag_status(FASA_ERR_WORKSPACE);
    misc[98] = (old == (unsigned long long)p.n_split - 1) ? 1u : 0u;
  }
  __syncthreads();
  if (!misc[98]) return;

  // 4. the row's last CTA: exact selection over the published union. One
  // batched read brings every region's count and first P entries into
  // shared memory (entries beyond P, rare, are read from global memory).
  __threadfence();
  const int S_ = p.n_split, P = p.ucache;  // P: a power of two
  uint2* stage = reinterpret_cast<uint2*>(smem + Lo.ucache);  // [S][P]
  uint32_t* cnt = reinterpret_cast<uint32_t*>(smem + Lo.cnt);  // [S] counts, then [S + 1] prefix sums
  uint32_t* bm = reinterpret_cast<uint32_t*>(smem + Lo.bitmap);
  uint2* ties = reinterpret_cast<uint2*>(smem + Lo.ties);
  uint32_t* rscr = reinterpret_cast<uint32_t*>(smem + Lo.rscr);
  const int words = (Lr + 31) / 32;
  const uint2* rows0 = p.cand + (int64_t)row * p.n_split * rstride;
  if (tid == 0) p.sem[row] = 0ull;  // every CTA of the row has arrived: ready for the next call
  // the histogram and the bitmap are cleared while the union's loads are in flight
  for (int i = tid; i < 4096; i += kWdThreads) hist[i] = 0u;
  for (int i = tid; i < words; i += kWdThreads) bm[i] = 0u;
  if (tid == 0) misc[100] = 0u;
  {  // slots [0, S): the regions' counts; then entry j < P of region s at S + s*P + j
    const int nslots = S_ + (S_ << p.ushift);
    for (int base = 0; base < nslots; base += kWdThreads * kWdUnionUnroll) {
      uint2 e[kWdUnionUnroll];
#pragma unroll
      for (int u = 0; u < kWdUnionUnroll; ++u) {
        const int f = base + u * kWdThreads + tid;
        const int g = f - S_;
        const int64_t at = f < S_ ? (int64_t)f * rstride : (int64_t)(g >> p.ushift) * rstride + 1 + (g & (P - 1));
        e[u] = f < nslots ? __ldcg(rows0 + at) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kWdUnionUnroll; ++u) {
        const int f = base + u * kWdThreads + tid;
        if (f < S_) {
          cnt[f] = min(e[u].x, (uint32_t)p.n_loc);
          cnt[2 * S_ + 1 + f] = e[u].y;  // the region's b_loc
        }
        else if (f < nslots) stage[f - S_] = e[u];
      }
    }
  }
  __syncthreads();
  if (warp == 0) {  // prefix sums of the counts (S <= 32 per pass of the warp), the highest b_loc, overflow
    uint32_t run = 0u, bmx = 0u;
    bool ovf = false;
    for (int s0 = 0; s0 < S_; s0 += 32) {
      const uint32_t c = s0 + lane < S_ ? cnt[s0 + lane] : 0u;
      if (s0 + lane < S_) bmx = max(bmx, cnt[2 * S_ + 1 + s0 + lane]);
      ovf |= c > (uint32_t)P;
      uint32_t incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t x = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += x;
      }
      if (s0 + lane < S_) cnt[S_ + 1 + s0 + lane] = run + incl;
      run += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    bmx = __reduce_max_sync(0xFFFFFFFFu, bmx);
    ovf = __any_sync(0xFFFFFFFFu, ovf);
    if (lane == 0) {
      cnt[S_] = 0u;
      misc[110] = bmx;
      misc[111] = ovf ? 1u : 0u;
    }
  }
  __syncthreads();
  const uint32_t* pre = cnt + S_;  // pre[s] = entries of regions before s; pre[S] = all
  const uint32_t b_max = misc[110];  // the highest b_loc: a row boundary bin below it cannot be trusted
  const int nu = (int)min(pre[S_], (uint32_t)p.len);
  const bool overflow = misc[111] != 0u;
  // every union entry once: the staged ones, then (rare) the rest from global memory
  auto for_union = [&](auto&& fn) {
    for (int f = tid; f < (S_ << p.ushift); f += kWdThreads)
      if ((f & (P - 1)) < (int)cnt[f >> p.ushift]) fn(stage[f]);
    if (overflow)
      for (int sr = 0; sr < S_; ++sr)
        for (int j = P + tid; j < (int)cnt[sr]; j += kWdThreads) fn(__ldcg(rows0 + sr * rstride + 1 + j));
  };
  // entry i of the union in region order (binary search over the prefix sums)
  auto union_at = [&](int i) -> uint2 {
    int lo = 0, hi = S_;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if ((int)pre[mid] <= i) lo = mid; else hi = mid;
    }
    const int j = i - (int)pre[lo];
    return j < P ? stage[lo * P + j] : __ldcg(rows0 + lo * rstride + 1 + j);
  };
  for_union([&](const uint2& e) { atomicAdd(hist + (e.x >> 20), 1u); });
  __syncthreads();
  const int n_keep = min(kr, nu);
  uint32_t B = 0u;
  wd_select(for_union, union_at, nu, n_keep, hist, misc, bm, ties, rscr, Lr, &B);
  if (nu < kr || B < b_max) {
    // some CTA may hold unpublished tokens at or above the boundary: the exact
    // selection again, over every key of the row
    const uint32_t* krow = p.keys + (int64_t)row * p.len;
    auto for_keys = [&](auto&& fn) {
      for (int base = 0; base < Lr; base += kWdThreads * kWdUnionUnroll) {
        uint32_t kx[kWdUnionUnroll];
#pragma unroll
        for (int u = 0; u < kWdUnionUnroll; ++u) {
          const int i = base + u * kWdThreads + tid;
          kx[u] = i < Lr ? __ldcg(krow + i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < kWdUnionUnroll; ++u) {
          const int i = base + u * kWdThreads + tid;
          if (i < Lr) fn(make_uint2(kx[u], (uint32_t)i));
        }
      }
    };
    auto keys_at = [&](int i) -> uint2 { return make_uint2(__ldcg(krow + i), (uint32_t)i); };
    for (int i = tid; i < words; i += kWdThreads) bm[i] = 0u;
    for (int i = tid; i < 4096; i += kWdThreads) hist[i] = 0u;
    __syncthreads();
    for_keys([&](const uint2& e) { atomicAdd(hist + (e.x >> 20), 1u); });
    __syncthreads();
    wd_select(for_keys, keys_at, Lr, kr, hist, misc, bm, ties, rscr, Lr, &B);
  }

  // ascending emission from the bitmap
  int* kept = reinterpret_cast<int*>(smem + Lo.kept);
  const int wpt = (words + kWdThreads - 1) / kWdThreads;
  const int w0 = min(words, tid * wpt), w1 = min(words, w0 + wpt);
  uint32_t nbits = 0u;
  for (int w = w0; w < w1; ++w) nbits += __popc(bm[w]);
  uint32_t total = 0u;
  uint32_t pos = wd_block_scan(nbits, misc, &total);
  if (tid == 0 && total != (uint32_t)kr) flag_status(FASA_ERR_WORKSPACE);
  int32_t* io = p.idx_out ? p.idx_out + (int64_t)row * p.n_keep : nullptr;
  int32_t* iw = p.idx_ws ? p.idx_ws + (int64_t)row * p.n_keep : nullptr;
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = bm[w];
    while (bits) {
      const int t = w * 32 + __ffs(bits) - 1;
      bits &= bits - 1u;
      if (pos < (uint32_t)kr) {
        if (p.direct) kept[pos] = t;
        if (io) io[pos] = t;
        if (iw) iw[pos] = t;
      }
      ++pos;
    }
  }
  if (kr < p.n_keep)  // a shorter row: pad its kept lists
    for (int j = kr + tid; j < p.n_keep; j += kWdThreads) {
      if (io) io[j] = -1;
      if (iw) iw[j] = -1;
    }
  if (p.row_keep && tid == 0) p.row_keep[row] = kr;
  __syncthreads();
  const int n_att = min((int)total, kr);
  if (!p.direct) return;  // the split-K attention launch follows
  // the group's attention over the kept rows (at most 16 per warp)
  const float* qs = reinterpret_cast<const float*>(smem + Lo.qs);
  float* zs = reinterpret_cast<float*>(smem + Lo.zs);
  float* mo = reinterpret_cast<float*>(smem + Lo.ring);
  float* lsum = mo + kWdWarps * MG * kD;
  __nv_bfloat16* vst = reinterpret_cast<__nv_bfloat16*>(lsum + 16);
  const int64_t plane = paged ? 0 : (int64_t)row * p.max_len * kD;
  cc_block_attend<MG, kWdWarps>(p.k + plane, p.v + plane,
                                [&](int j) -> int { return paged ? paged_row(p.pm, bb, g, kept[j]) : kept[j]; },
                                n_att, G, qs, zs, mo, lsum, vst, p.out + (int64_t)row * G * kD);
}

}  // namespace fasa
