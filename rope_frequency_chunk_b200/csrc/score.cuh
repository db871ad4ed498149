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
// power-of-two number of 16-byte chunks. A token is read by LPT lanes, one
// 16-byte chunk each, so a warp's load covers 512 contiguous bytes. The grid
// is persistent and splits the flattened (row, token) range evenly.
//
// Arithmetic: float64. Each stored element e is widened exactly to the double
// e * 2^-896 by placing its sign, exponent and mantissa bits in the double's
// high word (bf16: 7 mantissa bits; f32: 23); the coefficients carry the
// compensating 2^896, so each product equals Q[c]*e rounded once. This avoids
// the float->double conversion unit in the hot loop. The sum is rounded to
// float32 once at the end.
#pragma once

#include "fasa_device.cuh"

namespace fasa {

constexpr int kScoreThreads = 256;
constexpr int kScoreUnroll = 4;

struct ScoreParams {
  const void* sketch;    // [rows][max_len][stride]
  const void* q;         // [B][Hq][128]
  const int32_t* dom_idx;
  float* scores;         // [rows][len]
  int64_t max_len;
  int64_t total;         // rows * len
  int32_t len;
  int32_t stride;
  int32_t n_kv_heads;
  int32_t group;
  int32_t n_dom;
  int32_t q_pos;
  double theta[kNFC];
};

// Widen the two bf16 halves of w to (value * 2^-896) doubles, exactly.
__device__ __forceinline__ void widen_scaled(uint32_t w, double& lo, double& hi, __nv_bfloat16) {
  const uint32_t lo_hi = ((w << 16) & 0x80000000u) | ((w << 13) & 0x0FFFE000u);
  const uint32_t hi_hi = (w & 0x80000000u) | ((w >> 3) & 0x0FFFE000u);
  lo = __hiloint2double((int)lo_hi, 0);
  hi = __hiloint2double((int)hi_hi, 0);
}
// Widen one float32 to (value * 2^-896) double, exactly.
__device__ __forceinline__ double widen_scaled_f32(uint32_t w) {
  const uint32_t h = (w & 0x80000000u) | ((w & 0x7FFFFFFFu) >> 3);
  return __hiloint2double((int)h, (int)(w << 29));
}

template <typename T>
__device__ __forceinline__ double chunk_dot(const uint4& u, const double (&qr)[Elem<T>::kPer16]);

template <>
__device__ __forceinline__ double chunk_dot<__nv_bfloat16>(const uint4& u, const double (&qr)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  double acc = 0.0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    double a, b;
    widen_scaled(w[i], a, b, __nv_bfloat16());
    acc = fma(a, qr[2 * i], acc);
    acc = fma(b, qr[2 * i + 1], acc);
  }
  return acc;
}
template <>
__device__ __forceinline__ double chunk_dot<float>(const uint4& u, const double (&qr)[4]) {
  double acc = 0.0;
  acc = fma(widen_scaled_f32(u.x), qr[0], acc);
  acc = fma(widen_scaled_f32(u.y), qr[1], acc);
  acc = fma(widen_scaled_f32(u.z), qr[2], acc);
  acc = fma(widen_scaled_f32(u.w), qr[3], acc);
  return acc;
}

template <typename T, int LPT>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(const ScoreParams p) {
  constexpr int EPC = Elem<T>::kPer16;
  constexpr int TPW = 32 / LPT;  // tokens per warp load
  constexpr int U = kScoreUnroll;
  __shared__ double s_q[kD];
  grid_dependency_wait();
  grid_dependents_launch();  // the selection kernel may be scheduled now; it waits for our results

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int nw = kScoreThreads / 32;
  const int sub = lane % LPT, tl = lane / LPT;
  const double two896 = __hiloint2double(0x77F00000, 0);  // 2^896: exponent field 1919

  const int64_t per = (p.total + gridDim.x - 1) / gridDim.x;
  int64_t f = (int64_t)blockIdx.x * per;
  const int64_t f_end = min(p.total, f + per);

  while (f < f_end) {
    const int row = (int)(f / p.len);
    const int t0 = (int)(f % p.len);
    const int t1 = (int)min((int64_t)p.len, (int64_t)t0 + (f_end - f));
    const int b = row / p.n_kv_heads, g = row % p.n_kv_heads;

    __syncthreads();  // previous segment done with s_q
    if (tid < p.stride) {
      double acc = 0.0;
      const int j = tid >> 1;
      if (j < p.n_dom) {
        const int i = p.dom_idx[g * p.n_dom + j];
        if (i >= 0 && i < kNFC) {
          double s, c;
          sincos((double)p.q_pos * p.theta[i], &s, &c);
          const T* qh = static_cast<const T*>(p.q) + ((int64_t)(b * p.n_kv_heads + g) * p.group) * kD;
          for (int h = 0; h < p.group; ++h) {
            const double x = to_float(qh[h * kD + i]);
            const double y = to_float(qh[h * kD + i + kNFC]);
            // rotated query, first (x) or second (y) dim of FC i
            acc += (tid & 1) ? __dadd_rn(__dmul_rn(y, c), __dmul_rn(x, s))
                             : __dsub_rn(__dmul_rn(x, c), __dmul_rn(y, s));
          }
        } else {
          flag_status(FASA_ERR_BAD_INDEX);
        }
      }
      s_q[tid] = acc * two896;
    }
    __syncthreads();
    double qr[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) qr[e] = s_q[sub * EPC + e];

    const char* base = static_cast<const char*>(p.sketch) +
                       ((int64_t)row * p.max_len) * p.stride * (int64_t)sizeof(T) + sub * 16;
    const int64_t row_bytes = (int64_t)p.stride * sizeof(T);
    float* out = p.scores + (int64_t)row * p.len;
    const int ngroups = (t1 - t0 + TPW - 1) / TPW;

    for (int gi = warp; gi < ngroups; gi += nw * U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tg = gi + u * nw;
        const int t = t0 + tg * TPW + tl;
        if (tg < ngroups && t < t1) v[u] = ld_stream16(base + (int64_t)t * row_bytes);
        else v[u] = make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tg = gi + u * nw;
        const int t = t0 + tg * TPW + tl;
        double acc = chunk_dot<T>(v[u], qr);
#pragma unroll
        for (int off = LPT / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
        if (sub == 0 && tg < ngroups && t < t1) out[t] = (float)acc;
      }
    }
    f += (t1 - t0);
  }
}

}  // namespace fasa
