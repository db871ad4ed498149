// TIP score kernel: token importance from the dominant frequency chunks only.
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2, TIP "online prediction"): each token's importance is the sum of the
// contributions of the pre-calibrated dominant FCs. An FC's contribution is
// its share of q'.k, q'[i]k[i] + q'[i+64]k[i+64]; the group's query heads are
// added. Because the score is linear in q', the G rotated queries are summed
// first (in float64) into one coefficient per sketch column, Q[c].
//
// Data path: the sketch holds 2*n_dom values per token, stride padded to a
// power-of-two number of 16-byte chunks. The grid is persistent (one CTA per
// SM) and splits the flattened (row, token) range evenly; a CTA takes its
// range row segment by row segment. Each warp streams its own 32-lane steps
// of consecutive tokens through a private ring of shared-memory slots with
// 16-byte cp.async copies (no block barrier inside a segment, many requests
// in flight per SM) and scores them, one token per lane (two or four lanes
// for rows wider than 32 elements).
//
// Arithmetic: float32, in the fixed order and with the error bound stated in
// tip.cuh (coefficients from a float64 rotation and group sum, rounded once).
#pragma once

#include "tip.cuh"

namespace fasa {

constexpr int kScoreWarps = 12;
constexpr int kScoreThreads = kScoreWarps * 32;
constexpr int kScoreWarpBytes = 12288;  // each warp's ring of copy slots

struct ScoreParams {
  const void* sketch;    // [rows][max_len][stride]
  const void* q;         // [B][Hq][128]
  const int32_t* dom_idx;
  float* scores;         // [rows][ld]
  int64_t ld;            // row stride of scores, >= len
  uint32_t* hist;        // [rows][4096] key-histogram counts (added to), or null
  // with hist: the row's last CTA (a ticket on row_done, zero between calls)
  // finds the bin of the row's n_keep-th largest key and the count above it
  // into thr[row] = (bin, above) and leaves the row's histogram zero
  uint32_t* row_done;    // [rows]
  uint32_t* thr;         // [rows][2]
  int32_t n_keep;
  int64_t max_len;
  int64_t total;         // rows * len
  int32_t len;
  int32_t stride;
  int32_t n_kv_heads;
  int32_t group;
  int32_t n_dom;
  double cosv[kNFC];   // cos / sin of q_pos * theta_i (host, float64)
  double sinv[kNFC];
};

constexpr int kHistBits = 12;                 // key bits of the per-row score histogram
constexpr int kHistBins = 1 << kHistBits;

// From a 4096-bin histogram of the top 12 key bits (ld(i) = bin i), the bin
// holding the k-th largest key (1 <= k <= total) and the number of keys in
// higher bins, for a block of NT threads: thread t owns bins 4095 - BPT*t ..
// down to 4096 - BPT*(t + 1), then a suffix scan over the threads. scan:
// 2 * (NT / 32) + 2 words.
template <int NT, typename Ld>
__device__ __forceinline__ void hist_bin_of_kth(Ld ld, int k, uint32_t* scan, uint32_t& bin, uint32_t& above) {
  constexpr int BPT = (kHistBins + NT - 1) / NT, NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t c[BPT], sum = 0u;
#pragma unroll
  for (int u = 0; u < BPT; ++u) {
    const int b = kHistBins - 1 - (BPT * tid + u);
    c[u] = b >= 0 ? ld(b) : 0u;
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
    uint32_t w = lane < NW ? scan[lane] : 0u;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, w, off);
      if (lane >= off) w += v;
    }
    if (lane < NW) scan[NW + lane] = w;
  }
  __syncthreads();
  incl += warp > 0 ? scan[NW + warp - 1] : 0u;
  const uint32_t excl = incl - sum;
  if (excl < (uint32_t)k && (uint32_t)k <= incl) {
    uint32_t acc = excl;
#pragma unroll
    for (int u = 0; u < BPT; ++u) {
      if (acc + c[u] >= (uint32_t)k) {
        scan[2 * NW] = (uint32_t)(kHistBins - 1 - (BPT * tid + u));
        scan[2 * NW + 1] = acc;
        break;
      }
      acc += c[u];
    }
  }
  __syncthreads();
  bin = scan[2 * NW];
  above = scan[2 * NW + 1];
  __syncthreads();
}

// Shape of the per-token work for sketch rows of LPT 16-byte chunks, with a
// chunk rotation per lane so that a quarter-warp's 16-byte shared-memory
// reads hit distinct banks (the lane's coefficients are rotated the same way).
template <typename T, int LPT>
struct ScoreShape : TipShape<T, LPT> {
  using B = TipShape<T, LPT>;
  static constexpr int TPW = 32 / B::LPT2;  // tokens per warp step
  __device__ static int rot(int lane) {
    return (B::LPT2 == 1) ? ((lane * B::CPL / 8) % B::CPL) : (B::LPT2 == 2 ? ((lane / 2) % B::CPL) : 0);
  }
};

// Sketch-column coefficients of one row (tip_coef): thread `tid` < stride
// writes column tid.
template <typename T>
__device__ __forceinline__ void query_coefs(const T* qraw, const int* dom, int group, int n_dom, int stride,
                                            const double* cosv, const double* sinv, int tid, float* s_q) {
  if (tid < stride) s_q[tid] = tip_coef<T>(qraw, dom, group, n_dom, tid, cosv, sinv);
}

// The lane's share of the coefficients, in its rotated chunk order.
template <typename T, int LPT>
__device__ __forceinline__ void load_coefs(float (&qr)[ScoreShape<T, LPT>::EPL], const float* s_q, int lane) {
  using S = ScoreShape<T, LPT>;
  const int sub = lane % S::LPT2, rot = S::rot(lane);
#pragma unroll
  for (int c = 0; c < S::CPL; ++c)
#pragma unroll
    for (int e = 0; e < S::EPC; ++e) qr[c * S::EPC + e] = s_q[(sub * S::CPL + (c + rot) % S::CPL) * S::EPC + e];
}

// Scores of the n tokens of one staged block of sketch rows, warps
// 0..NCW-1 in turn. sink(t, writer, score) is called by every lane of the
// warp (warp-uniform), writer set on the one lane that owns token t.
template <typename T, int LPT, int NCW, typename Sink>
__device__ __forceinline__ void score_block(const unsigned char* buf, int n, const float (&qr)[ScoreShape<T, LPT>::EPL],
                                            int warp, int lane, Sink&& sink) {
  using S = ScoreShape<T, LPT>;
  const int sub = lane % S::LPT2, rot = S::rot(lane);
  for (int gi = warp; gi * S::TPW < n; gi += NCW) {
    const int t = gi * S::TPW + lane / S::LPT2;
    const bool valid = t < n;
    uint4 v[S::CPL];
#pragma unroll
    for (int c = 0; c < S::CPL; ++c)
      v[c] = valid ? *reinterpret_cast<const uint4*>(buf + t * S::ROWB + (sub * S::CPL + (c + rot) % S::CPL) * 16)
                   : make_uint4(0, 0, 0, 0);
    // chunk partials in the lane's rotated order; the halving tree does not
    // depend on the rotation
    float part[S::CPL];
#pragma unroll
    for (int c = 0; c < S::CPL; ++c) part[c] = tip_chunk(v[c], qr + c * S::EPC, T());
    const float acc = tip_lanes_sum<S::LPT2>(tip_lane_sum<S::CPL>(part));
    sink(t, valid && sub == 0, acc);
  }
}

// Slots of a warp's ring: one warp step (32 lanes x their chunks) each.
template <typename T, int LPT>
struct ScoreRing {
  static constexpr int kSlot = 32 * ScoreShape<T, LPT>::CPL * 16;
  static constexpr int kRaw = kScoreWarpBytes / kSlot;
  static constexpr int kDepth = kRaw < 2 ? 2 : (kRaw > 16 ? 16 : kRaw);
  static_assert(kDepth * kSlot <= kScoreWarpBytes, "ring slots exceed the warp's ring");
};

__host__ __device__ constexpr int score_smem_bytes() { return kScoreWarps * kScoreWarpBytes + kHistBins * 4; }

template <typename T, int LPT, bool kHist>
__global__ void __launch_bounds__(kScoreThreads, 1) score_kernel(const ScoreParams p) {
  using S = ScoreShape<T, LPT>;
  using R = ScoreRing<T, LPT>;
  constexpr int D = R::kDepth;
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(smem + kScoreWarps * kScoreWarpBytes);
  __shared__ float s_q[kD];
  __shared__ __align__(16) T s_qraw[FASA_MAX_GROUP * kD];  // the group's raw queries
  __shared__ int s_dom[kNFC];
  __shared__ uint32_t s_scan[2 * kScoreWarps + 2];
  __shared__ uint32_t s_last;
  __shared__ double s_cs[2 * kNFC];  // cos, sin of the query angle
  // the angle table from the parameters (no dependence on the previous
  // launch): read before the wait, so its constant-bank misses overlap it
  if (threadIdx.x < kNFC) s_cs[threadIdx.x] = p.cosv[threadIdx.x];
  else if (threadIdx.x < 2 * kNFC) s_cs[threadIdx.x] = p.sinv[threadIdx.x - kNFC];
  grid_dependency_wait();
  grid_dependents_launch();  // the selection kernel may be scheduled now; it waits for our results

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned char* ring = smem + warp * kScoreWarpBytes;
  const int sub = lane % S::LPT2, tl = lane / S::LPT2;  // the lane's chunk group and token in a step
  const int64_t per = (p.total + gridDim.x - 1) / gridDim.x;
  const int64_t f_beg = min(p.total, (int64_t)blockIdx.x * per);
  const int64_t f_end = min(p.total, f_beg + per);
  if (kHist)
    for (int i = tid; i < kHistBins; i += kScoreThreads) s_hist[i] = 0u;

  // a segment: the CTA's tokens of one row. Its first D ring slots are
  // requested before the row's coefficients are formed (and, for every
  // segment after the first, before the previous row's histogram is
  // flushed), so the stream's first round trip overlaps that work.
  int row = 0, t0 = 0, n = 0, mine = 0;
  const char* src = nullptr;
  auto begin_seg = [&](int64_t seg) {
    row = (int)(seg / p.len);
    t0 = (int)(seg % p.len);
    n = (int)min((int64_t)(p.len - t0), f_end - seg);
    src = static_cast<const char*>(p.sketch) + ((int64_t)row * p.max_len + t0) * S::ROWB;
    const int nblk = (n + S::TPW - 1) / S::TPW;
    mine = nblk > warp ? (nblk - warp + kScoreWarps - 1) / kScoreWarps : 0;
  };
  // warp w takes the steps w, w + kScoreWarps, ... of TPW consecutive tokens
  auto issue = [&](int j) {
    if (j < mine) {
      const int tok = (j * kScoreWarps + warp) * S::TPW + tl;
      if (tok < n) {
        unsigned char* slot = ring + (j % D) * R::kSlot + tl * S::ROWB;
#pragma unroll
        for (int c = 0; c < S::CPL; ++c)
          cp_async16(slot + (sub * S::CPL + c) * 16, src + (int64_t)tok * S::ROWB + (sub * S::CPL + c) * 16);
      }
    }
    cp_async_commit();
  };
  if (f_beg < f_end) {
    begin_seg(f_beg);
#pragma unroll
    for (int j = 0; j < D; ++j) issue(j);
  }
  for (int64_t seg = f_beg; seg < f_end;) {
    // the row's query coefficients (float64), every thread taking part
    __syncthreads();
    {
      const int bb = row / p.n_kv_heads, g = row % p.n_kv_heads;
      const uint4* qsrc = reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) +
                                                         ((int64_t)(bb * p.n_kv_heads + g) * p.group) * kD);
      for (int c = tid; c < p.group * kD * (int)sizeof(T) / 16; c += kScoreThreads)
        reinterpret_cast<uint4*>(s_qraw)[c] = __ldg(qsrc + c);
      if (tid < p.n_dom) s_dom[tid] = __ldg(p.dom_idx + g * p.n_dom + tid);
    }
    __syncthreads();
    query_coefs<T>(s_qraw, s_dom, p.group, p.n_dom, p.stride, s_cs, s_cs + kNFC, tid, s_q);
    __syncthreads();
    float qr[S::EPL];
    load_coefs<T, LPT>(qr, s_q, lane);

    float* out = p.scores + (int64_t)row * p.ld + t0;
    for (int j = 0; j < mine; ++j) {
      cp_async_wait<D - 1>();
      __syncwarp();
      const int b0 = (j * kScoreWarps + warp) * S::TPW;
      score_block<T, LPT, 1>(ring + (j % D) * R::kSlot, min(S::TPW, n - b0), qr, 0, lane,
                             [&](int t, bool writer, float sc) {
                               if (writer) out[b0 + t] = sc;
                               if (kHist && writer) atomicAdd(&s_hist[score_key(sc) >> (32 - kHistBits)], 1u);
                             });
      __syncwarp();
      issue(j + D);
    }
    cp_async_wait<0>();
    __syncwarp();  // the warp's ring is consumed: the next segment may fill it
    const int cur_row = row, cur_n = n;
    const int64_t next = seg + n;
    if (next < f_end) {
      begin_seg(next);
#pragma unroll
      for (int j = 0; j < D; ++j) issue(j);
    }
    if (kHist) {
      __syncthreads();
      for (int i = tid; i < kHistBins; i += kScoreThreads) {
        const uint32_t v = s_hist[i];
        if (v) {
          atomicAdd(p.hist + (int64_t)cur_row * kHistBins + i, v);
          s_hist[i] = 0u;
        }
      }
      if (p.thr) {  // the row's last segment: its threshold bin, once per row
        __threadfence();
        __syncthreads();
        if (tid == 0) s_last = atomicAdd(p.row_done + cur_row, (uint32_t)cur_n) + (uint32_t)cur_n == (uint32_t)p.len;
        __syncthreads();
        if (s_last) {
          __threadfence();
          uint32_t* hr = p.hist + (int64_t)cur_row * kHistBins;
          uint32_t bin, above;
          hist_bin_of_kth<kScoreThreads>([hr](int i) { return __ldcg(hr + i); }, p.n_keep, s_scan, bin, above);
          if (tid == 0) {
            p.thr[2 * cur_row] = bin;
            p.thr[2 * cur_row + 1] = above;
            p.row_done[cur_row] = 0u;
          }
          for (int i = tid; i < kHistBins; i += kScoreThreads) hr[i] = 0u;  // ready for the next call
        }
      }
    }
    seg = next;
  }
}

}  // namespace fasa
