// Offline calibration of the dominant FCs.
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2, TIP first bullet): once, before decoding, each head's dominant FCs
// I_dom are the ones whose single-FC attention scores agree best with the
// full head's ("Contextual Agreement", CA) over a small calibration set. The
// pages give no formula for CA; the agreement measured here is that of the
// token sets each score selects at the decode budget K:
//   counts[g][i] = sum over sequences b and calibration queries w of
//                  |Top_K(P_i) ∩ Top_K(full)|,
// with P_i(t) = qs[i] k[t][i] + qs[i+64] k[t][i+64], qs the group's rotated
// queries added head by head, the full score the 64 shares added in FC
// order, every value rounded once to float32, and Top_K the decode's
// selection (ties to the lower index). I_dom = the n_dom largest counts,
// ties to the lower FC.
//
// Three steps, each a kernel:
//  calib_score_kernel   (grid: token tiles x rows) the 65 score planes of
//                       every calibration query, float64 with every product
//                       and sum rounded as written (no contraction), then
//                       float32; one token per thread, coalesced plane rows.
//  (select)             the decode library's exact top-K selection over
//                       every plane (select_attend_kernel, kSelect).
//  calib_overlap_kernel (grid: rows x queries) the full plane's selection
//                       as a bitmap in shared memory; one warp per FC counts
//                       its selection's members and adds to counts[g][i].
//  calib_rank_kernel    (grid: KV heads) ranks the 64 counts.
#pragma once

#include "fasa_device.cuh"

namespace fasa {

constexpr int kCalMaxWin = FASA_CAL_MAX_WIN;  // calibration queries per call
constexpr int kCalPlanes = kNFC + 1;          // 64 single-FC planes + the full head
constexpr int kCalThreads = 256;              // tokens per CTA of the score kernel

struct CalScoreParams {
  const void* k;        // [rows][max_len][128] dtype, rotated keys
  const void* q;        // [B][n_win][Hq][128] dtype, pre-RoPE
  float* planes;        // [rows][n_win][65][len]
  int64_t max_len;
  int32_t len;
  int32_t n_win;
  int32_t n_kv_heads;
  int32_t group;
  double cosv[kCalMaxWin][kNFC];  // cos / sin of (q_pos0 + w) * theta_i (host, float64)
  double sinv[kCalMaxWin][kNFC];
};

template <typename T>
__device__ __forceinline__ double cal_load(const T* p) {
  if constexpr (sizeof(T) == 2) {
    return (double)__bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
  } else {
    return (double)*reinterpret_cast<const float*>(p);
  }
}

template <typename T>
__global__ void __launch_bounds__(kCalThreads) calib_score_kernel(const CalScoreParams p) {
  __shared__ double qs[kCalMaxWin][kD];
  const int row = blockIdx.y;
  const int b = row / p.n_kv_heads, g = row % p.n_kv_heads;
  const int G = p.group, Hq = p.n_kv_heads * G;
  const int tid = threadIdx.x;
  // the group's rotated queries of every calibration query, added head by
  // head: x' = x cos - y sin (dim i < 64), y' = y cos + x sin (dim i + 64)
  for (int e = tid; e < p.n_win * kD; e += kCalThreads) {
    const int w = e / kD, d = e % kD, i = d & (kNFC - 1);
    const T* qw = static_cast<const T*>(p.q) + ((int64_t)(b * p.n_win + w) * Hq + (int64_t)g * G) * kD;
    const double c = p.cosv[w][i], s = p.sinv[w][i];
    double acc = 0.0;
    for (int h = 0; h < G; ++h) {
      const double x = cal_load(qw + h * kD + i), y = cal_load(qw + h * kD + i + kNFC);
      const double r = d < kNFC ? __dsub_rn(__dmul_rn(x, c), __dmul_rn(y, s))
                                : __dadd_rn(__dmul_rn(y, c), __dmul_rn(x, s));
      acc = h == 0 ? r : __dadd_rn(acc, r);
    }
    qs[w][d] = acc;
  }
  __syncthreads();
  const int t = blockIdx.x * kCalThreads + tid;
  if (t >= p.len) return;
  const T* kt = static_cast<const T*>(p.k) + ((int64_t)row * p.max_len + t) * kD;
  float* out = p.planes + (int64_t)row * p.n_win * kCalPlanes * p.len + t;
  double full[kCalMaxWin];
#pragma unroll 1
  for (int i = 0; i < kNFC; ++i) {
    const double x = cal_load(kt + i), y = cal_load(kt + i + kNFC);
#pragma unroll
    for (int w = 0; w < kCalMaxWin; ++w) {
      if (w < p.n_win) {
        const double share = __dadd_rn(__dmul_rn(qs[w][i], x), __dmul_rn(qs[w][i + kNFC], y));
        full[w] = i == 0 ? share : __dadd_rn(full[w], share);
        out[((int64_t)w * kCalPlanes + i) * p.len] = __double2float_rn(share);
      }
    }
  }
#pragma unroll
  for (int w = 0; w < kCalMaxWin; ++w)
    if (w < p.n_win) out[((int64_t)w * kCalPlanes + kNFC) * p.len] = __double2float_rn(full[w]);
}

// idx: [n_rows * n_win][65][keff] ascending selections; counts [n_kv][64]
// (cleared before the launch). Dynamic shared memory: ceil(len / 32) words.
__global__ void __launch_bounds__(kCalThreads) calib_overlap_kernel(const int32_t* idx, int32_t keff, int32_t len,
                                                                    int32_t n_kv_heads, int32_t n_win,
                                                                    uint32_t* counts) {
  extern __shared__ uint32_t cal_bm[];
  const int64_t rw = blockIdx.x;  // (row, calibration query)
  const int g = (int)((rw / n_win) % n_kv_heads);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int words = (len + 31) / 32;
  for (int w = tid; w < words; w += kCalThreads) cal_bm[w] = 0u;
  __syncthreads();
  const int32_t* full = idx + (rw * kCalPlanes + kNFC) * keff;
  for (int j = tid; j < keff; j += kCalThreads) {
    const int t = full[j];
    if (t >= 0 && t < len) {
      atomicOr(&cal_bm[t >> 5], 1u << (t & 31));
    } else {
      flag_status(FASA_ERR_BAD_INDEX);
    }
  }
  __syncthreads();
  for (int i = warp; i < kNFC; i += kCalThreads / 32) {
    const int32_t* sel = idx + (rw * kCalPlanes + i) * keff;
    uint32_t c = 0u;
    for (int j = lane; j < keff; j += 32) {
      const int t = sel[j];
      if (t >= 0 && t < len) c += (cal_bm[t >> 5] >> (t & 31)) & 1u;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
    if (lane == 0 && c) atomicAdd(counts + g * kNFC + i, c);
  }
}

// One CTA of 64 threads per KV head: FC i's rank among the counts
// (descending, ties to the lower FC); the first n_dom ranks go to dom_idx.
__global__ void __launch_bounds__(kNFC) calib_rank_kernel(const uint32_t* counts, int32_t n_dom, int32_t* dom_idx) {
  __shared__ uint32_t c[kNFC];
  const int g = blockIdx.x, i = threadIdx.x;
  c[i] = counts[g * kNFC + i];
  __syncthreads();
  int r = 0;
  for (int j = 0; j < kNFC; ++j) r += (c[j] > c[i] || (c[j] == c[i] && j < i)) ? 1 : 0;
  if (r < n_dom) dom_idx[g * n_dom + r] = i;
}

}  // namespace fasa
