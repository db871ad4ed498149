// Critical-set selection for the fused decode, from the score kernel's
// per-row key histogram.
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2, FAC first bullet): T_t is the set of the k highest-scoring tokens
// (ties to the lower index; k_eff = min(k, L)). Two kernels:
//
//  filter   (grid: token tiles x rows) The bin b1 holding the k_eff-th key
//           (found once per row by the score kernel from the row's 4096-bin
//           histogram of the top 12 key bits) splits the row. Keys in
//           higher bins are certainly kept: each warp writes the bitmap word
//           of its 32 consecutive tokens (every word of [0, len) is written
//           exactly once, so the bitmap needs no clearing). Keys in bin b1
//           are gathered in shared memory and appended, (index, key) pairs,
//           to the row's candidate list with one global atomic per CTA (a
//           per-warp atomic on the row's counter serialises thousands of
//           warps on one cache line). Tile 0 of each row also prepares the
//           attention kernel's query terms, before waiting for the scores.
//  finalize (grid: rows) Exact k_eff-th key among the candidates (radix
//           select on the low 20 bits, digit histograms counted with warp
//           ballots); ties at it go to the lower token index. Their bits
//           are added to the bitmap, and the kept indices are emitted in
//           ascending order by a popcount scan of the bitmap. If the
//           candidate list overflowed, the row is resolved exactly from all
//           its scores instead (slow, rare).
#pragma once

#include "score.cuh"
#include "select_attend.cuh"

namespace fasa {

constexpr int kFilterThreads = kSAThreads;  // hist_threshold assumes 512 threads

constexpr int kFilterCands = 2048;  // candidates a CTA gathers in shared memory

struct FilterParams {
  const float* scores;      // [rows][ld], 16-byte aligned
  int64_t ld;               // row stride of scores, a multiple of 32
  const uint32_t* thr;      // [rows][2]: the bin of the k_eff-th key, the keys above it
  uint32_t* cand_cnt;       // [rows], zero before the launch
  int32_t* cand_idx;        // [rows][cap]
  uint32_t* cand_key;       // [rows][cap], the candidates' score keys
  uint32_t* bitmap;         // [rows][words]
  int32_t len;
  int32_t n_keep;           // k_eff
  int32_t cap;
  int32_t tile;             // tokens per CTA, a multiple of 128
  int32_t words;            // ceil(len / 32)
};

__global__ void __launch_bounds__(kFilterThreads, 4) filter_kernel(const FilterParams p) {
  __shared__ int32_t s_cidx[kFilterCands];
  __shared__ uint32_t s_ckey[kFilterCands];
  __shared__ uint32_t s_n, s_base;
  const int row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_n = 0u;
  grid_dependency_wait();
  const uint32_t bin = __ldcg(p.thr + 2 * row);
  __syncthreads();  // publishes s_n
  const int t0 = blockIdx.x * p.tile;
  const int t1 = min(p.len, t0 + p.tile);
  const float4* s4 = reinterpret_cast<const float4*>(p.scores + (int64_t)row * p.ld);
  uint32_t* bm = p.bitmap + (int64_t)row * p.words;
  int32_t* cidx = p.cand_idx + (int64_t)row * p.cap;
  // Lane l of a warp holds tokens base + 4l .. base + 4l + 3 of a 128-token
  // step, so lanes 8j .. 8j+7 hold the 32 tokens of bitmap word j of the
  // step (the row stride and the tile are multiples of 32 and 128, so every
  // float4 is aligned and inside the row's padded stride).
  constexpr int U = 2;  // 16-byte loads in flight per lane
  constexpr int kStep = 128, kPass = kFilterThreads / 32 * kStep;
  for (int base0 = t0 + warp * kStep; base0 < t1; base0 += kPass * U) {
    float4 f[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base0 + u * kPass + lane * 4;
      f[u] = i < t1 ? __ldcg(s4 + i / 4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int base = base0 + u * kPass;
      if (base >= t1) break;  // warp-uniform
      const int i = base + lane * 4;
      const float fv[4] = {f[u].x, f[u].y, f[u].z, f[u].w};
      uint32_t dn = 0u, cn = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool v = i + e < t1;
        const uint32_t b = score_key(fv[e]) >> 20;
        dn |= (uint32_t)(v && b > bin) << e;
        cn |= (uint32_t)(v && b == bin) << e;
      }
      uint32_t dw = dn << (4 * (lane & 7));
      dw |= __shfl_xor_sync(0xFFFFFFFFu, dw, 1);
      dw |= __shfl_xor_sync(0xFFFFFFFFu, dw, 2);
      dw |= __shfl_xor_sync(0xFFFFFFFFu, dw, 4);
      if ((lane & 7) == 0 && i < t1) bm[i >> 5] = dw;
      if (cn) {  // rare: this lane's threshold-bin tokens into the CTA's list
        uint32_t at = atomicAdd(&s_n, (uint32_t)__popc(cn));
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if ((cn >> e) & 1u) {
            if (at < (uint32_t)kFilterCands) {
              s_cidx[at] = i + e;
              s_ckey[at] = score_key(fv[e]);
            } else {  // this CTA's buffer is full (heavy ties): straight to the global list
              const uint32_t g = atomicAdd(p.cand_cnt + row, 1u);
              if (g < (uint32_t)p.cap) {
                cidx[g] = i + e;
                p.cand_key[(int64_t)row * p.cap + g] = score_key(fv[e]);
              }
            }
            ++at;
          }
      }
    }
  }
  __syncthreads();
  const uint32_t n = min(s_n, (uint32_t)kFilterCands);
  if (tid == 0) s_base = n ? atomicAdd(p.cand_cnt + row, n) : 0u;
  __syncthreads();
  uint32_t* ckey = p.cand_key + (int64_t)row * p.cap;
  for (uint32_t j = tid; j < n; j += kFilterThreads) {
    const uint32_t g = s_base + j;
    if (g < (uint32_t)p.cap) {
      cidx[g] = s_cidx[j];
      ckey[g] = s_ckey[j];
    }
  }
}

struct FinalParams {
  float* scores;            // [rows][ld]; the slow path turns a row into keys in place
  int64_t ld;
  const uint32_t* thr;      // [rows][2]
  uint32_t* cand_cnt;       // [rows]; finalize leaves it zero
  const int32_t* cand_idx;  // [rows][cap]
  const uint32_t* cand_key; // [rows][cap]
  const uint32_t* bitmap;   // [rows][words]
  int32_t* idx;             // [rows][n_keep]
  int32_t* idx_out;         // [rows][n_keep] or null
  int32_t len;
  int32_t n_keep;
  int32_t cap;              // candidate list capacity
  int32_t scap;             // candidates held in shared memory
  int32_t words;
};

__host__ __device__ inline int final_smem_bytes(int words, int scap) {
  return sa_align(words * 4, 128) + (kSAWarps * 256 + 264) * 4 + 64 * 4 + 2 * scap * 4;
}

__global__ void __launch_bounds__(kSAThreads, 1) finalize_kernel(const FinalParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  grid_dependency_wait();
  cg::cluster_group cluster = cg::this_cluster();  // a cluster of one; radix helpers take it
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  uint32_t* bm = reinterpret_cast<uint32_t*>(smem);
  uint32_t* rscr = reinterpret_cast<uint32_t*>(smem + sa_align(p.words * 4, 128));
  uint32_t* scan = rscr + kSAWarps * 256 + 264;
  uint32_t* ckey = scan + 64;                           // [scap]
  int32_t* cidx = reinterpret_cast<int32_t*>(ckey + p.scap);  // [scap]

  // the candidate count and, asynchronously, the filter's bitmap, while
  // the threshold bin is found again from the histogram
  const uint32_t n_c = __ldcg(p.cand_cnt + row);
  const uint32_t* gbm = p.bitmap + (int64_t)row * p.words;
  for (int w = tid; w < p.words; w += kSAThreads) cp_async4(bm + w, gbm + w);
  cp_async_commit();
  const bool fast = n_c <= (uint32_t)p.cap && n_c <= (uint32_t)p.scap;
  if (fast) {  // the (index, key) candidates, also in flight during the scan
    const int32_t* gi = p.cand_idx + (int64_t)row * p.cap;
    const uint32_t* gk = p.cand_key + (int64_t)row * p.cap;
    for (int j = tid; j < (int)n_c; j += kSAThreads) {
      cp_async4(cidx + j, gi + j);
      cp_async4(ckey + j, gk + j);
    }
  }
  cp_async_commit();
  const uint32_t bin = __ldcg(p.thr + 2 * row), above = __ldcg(p.thr + 2 * row + 1);
  const int krem = p.n_keep - (int)above;
  cp_async_wait<0>();
  __syncthreads();

  if (fast) {
    const int32_t* gc = cidx;
    auto key_of = [ckey](int j) { return ckey[j]; };
    __syncthreads();
    uint32_t thr;
    int quota;
    ballot_radix_fn<false>(key_of, (int)n_c, krem, bin << 20, 12, 32, rscr, nullptr, cluster, thr, quota);
    // how many candidates tie at thr: keep all of them, or the `quota` with
    // the lowest indices
    uint32_t neq = 0u;
    for (int base = warp * 32; base < (int)n_c; base += kSAThreads) {
      const int j = base + lane;
      neq += __popc(__ballot_sync(0xFFFFFFFFu, j < (int)n_c && key_of(j) == thr));
    }
    if (lane == 0) scan[warp] = neq;
    __syncthreads();
    uint32_t eq_total = 0u;
#pragma unroll
    for (int w = 0; w < kSAWarps; ++w) eq_total += scan[w];
    __syncthreads();
    uint32_t thr2 = 0u;
    if ((int)eq_total > quota) {
      // the tied candidates with the lowest indices: the largest ~index
      auto tie_key = [key_of, gc, thr](int j) { return key_of(j) == thr ? ~(uint32_t)gc[j] : 0u; };
      int q2;
      ballot_radix_fn<false>(tie_key, (int)n_c, quota, 0u, 0, 32, rscr, nullptr, cluster, thr2, q2);
    }
    for (int j = tid; j < (int)n_c; j += kSAThreads) {
      const uint32_t x = key_of(j);
      const int t = gc[j];
      const bool keep = x > thr || (x == thr && ((int)eq_total <= quota || ~(uint32_t)t >= thr2));
      if (keep) atomicOr(&bm[t >> 5], 1u << (t & 31));
    }
  } else {
    // slow exact path: this row's scores become keys in place, then a radix
    // select over all of them, then the bitmap from scratch in index order
    // (overwriting the copied filter bitmap)
    uint32_t* keys = reinterpret_cast<uint32_t*>(p.scores + (int64_t)row * p.ld);
    for (int i = tid; i < p.len; i += kSAThreads) keys[i] = score_key(__ldcg(p.scores + (int64_t)row * p.ld + i));
    __threadfence_block();
    __syncthreads();
    uint32_t thr;
    int quota;
    ballot_radix<false>(keys, p.len, p.n_keep, 0u, 0, 32, rscr, nullptr, cluster, thr, quota);
    // equal keys per warp range of words, in index order
    const int wseg = (p.words + kSAWarps - 1) / kSAWarps;
    const int w0 = min(p.words, warp * wseg), w1 = min(p.words, w0 + wseg);
    uint32_t neq = 0u;
    for (int w = w0; w < w1; ++w) {
      const int i = w * 32 + lane;
      neq += __popc(__ballot_sync(0xFFFFFFFFu, i < p.len && keys[i] == thr));
    }
    if (lane == 0) scan[warp] = neq;
    __syncthreads();
    uint32_t er = 0u;
    for (int w = 0; w < warp; ++w) er += scan[w];
    for (int w = w0; w < w1; ++w) {
      const int i = w * 32 + lane;
      const bool v = i < p.len;
      const uint32_t x = v ? keys[i] : 0u;
      const unsigned gt = __ballot_sync(0xFFFFFFFFu, v && x > thr);
      const unsigned eq = __ballot_sync(0xFFFFFFFFu, v && x == thr);
      const bool take_eq = ((eq >> lane) & 1u) && (int)(er + __popc(eq & lt)) < quota;
      const unsigned te = __ballot_sync(0xFFFFFFFFu, take_eq);
      if (lane == 0) bm[w] = gt | te;
      er += __popc(eq);
    }
  }
  __syncthreads();

  // emit the kept indices in ascending order: popcount scan of the bitmap
  const int per = (p.words + kSAThreads - 1) / kSAThreads;
  const int wb = min(p.words, tid * per), we_ = min(p.words, wb + per);
  uint32_t cnt = 0u;
  for (int w = wb; w < we_; ++w) cnt += __popc(bm[w]);
  uint32_t incl = cnt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) scan[warp] = incl;
  __syncthreads();
  uint32_t before = 0u;
  for (int w = 0; w < warp; ++w) before += scan[w];
  uint32_t pos = before + incl - cnt;
  int32_t* out = p.idx + (int64_t)row * p.n_keep;
  int32_t* out2 = p.idx_out ? p.idx_out + (int64_t)row * p.n_keep : nullptr;
  for (int w = wb; w < we_; ++w) {
    uint32_t m = bm[w];
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1;
      if (pos < (uint32_t)p.n_keep) {
        out[pos] = w * 32 + bit;
        if (out2) out2[pos] = w * 32 + bit;
      } else {
        flag_status(FASA_ERR_BAD_INDEX);
      }
      ++pos;
    }
  }
  if (tid == 0) p.cand_cnt[row] = 0u;  // the workspace is ready for the next call
}

}  // namespace fasa
