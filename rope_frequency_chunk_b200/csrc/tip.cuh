// TIP score arithmetic, shared by every kernel that scores cached tokens.
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2, TIP "online prediction"): the importance of cached token t for KV head
// g is the sum, over the dominant FCs i of g, of each FC's share of the
// group's attention logits,
//   s_t = sum_{h in g} sum_{i in D_g} q'_h[i] k_t[i] + q'_h[i+64] k_t[i+64].
// The score is linear in q', so the group's rotated queries are added first,
// one coefficient per sketch column: column 2j (2j+1) of dominant FC
// i = D_g[j] carries c = sum_h q'_h[i] (sum_h q'_h[i+64]). The rotation and
// that sum are float64; c is rounded once to float32 (c^).
//
// Evaluation order, fixed so that every kernel gives bit-identical scores:
// a sketch row is cut into 16-byte chunks (8 bf16 or 4 f32 elements); a
// chunk's partial is a float32 chain in element order (a product, then one
// fma per element); a lane owning CPL consecutive chunks adds their partials
// as a halving tree (chunk j + CPL/2 onto chunk j, then j + CPL/4, ...), and
// the LPT2 lanes that share one token add their sums as an xor butterfly
// (offset LPT2/2 first). The halving tree is invariant under a cyclic
// rotation of the chunks (up to the order of the two operands of an add), so
// a kernel may visit a lane's chunks in rotated order.
//
// Error bound (u = 2^-24, n = elements per chunk + log2(chunks per row), the
// longest chain of roundings from one product to the score; the product of
// c^ and a stored element is exact inside the fma, and c^ = c (1 + d),
// |d| <= u):
//   |s^ - s| <= ((1 + u) gamma_n + u) * sum_j |c_j| |x_j|,
//   gamma_n = n u / (1 - n u).
// Rows have at most 16 bf16 chunks (n <= 8 + 4) or 32 f32 chunks
// (n <= 4 + 5), so |s^ - s| < 13.01 u sum_j |c_j| |x_j| for every shape.
#pragma once

#include "fasa_device.cuh"

namespace fasa {

// Chunks per row and lanes per token for rows of LPT 16-byte chunks of T.
template <typename T, int LPT>
struct TipShape {
  static constexpr int EPC = Elem<T>::kPer16;            // elements per chunk
  static constexpr int ROWE = LPT * EPC;                 // elements per row
  static constexpr int ROWB = LPT * 16;                  // bytes per row
  static constexpr int LPT2 = ROWE > 32 ? ROWE / 32 : 1;  // lanes per token
  static constexpr int EPL = ROWE / LPT2;                // elements per lane (<= 32)
  static constexpr int CPL = EPL / EPC;                  // chunks per lane
};

// Coefficient of sketch column col (float64 rotation and group sum, rounded
// once to float32). qraw holds the group's G pre-RoPE queries [G][128];
// cosv/sinv are cos and sin of q_pos * theta_i. Padding columns (col >=
// 2 n_dom) are zero. An FC index outside [0, 64) is flagged and gives zero.
// With n_tok query tokens per sequence (multi-query decode), qraw holds
// n_tok * G rows, token-major, and the rows of token j take the angle table
// at cosv + j * cs_stride (sinv likewise); the sum runs over every row in
// that order.
template <typename T>
__device__ __forceinline__ float tip_coef(const T* qraw, const int* dom, int group, int n_dom, int col,
                                          const double* cosv, const double* sinv, int n_tok = 1,
                                          int cs_stride = 0) {
  const int jj = col >> 1;
  if (jj >= n_dom) return 0.0f;
  const int i = dom[jj];
  if (i < 0 || i >= kNFC) {
    flag_status(FASA_ERR_BAD_INDEX);
    return 0.0f;
  }
  double acc = 0.0;
  for (int h = 0; h < group * n_tok; ++h) {
    const int j = h / group;
    const double c = cosv[j * cs_stride + i], s = sinv[j * cs_stride + i];
    const double x = to_float(qraw[h * kD + i]);
    const double y = to_float(qraw[h * kD + i + kNFC]);
    // rotated query, first (x') or second (y') dim of FC i
    acc = __dadd_rn(acc, (col & 1) ? __dadd_rn(__dmul_rn(y, c), __dmul_rn(x, s))
                                   : __dsub_rn(__dmul_rn(x, c), __dmul_rn(y, s)));
  }
  return __double2float_rn(acc);
}

// Partial of one 16-byte chunk: a float32 product-then-fma chain in element
// order over the chunk's elements, c[e] the matching coefficients.
__device__ __forceinline__ float tip_chunk(const uint4& u, const float* c, __nv_bfloat16) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  float acc = __fmul_rn(c[0], __uint_as_float(w[0] << 16));
  acc = __fmaf_rn(c[1], __uint_as_float(w[0] & 0xFFFF0000u), acc);
#pragma unroll
  for (int i = 1; i < 4; ++i) {
    acc = __fmaf_rn(c[2 * i], __uint_as_float(w[i] << 16), acc);
    acc = __fmaf_rn(c[2 * i + 1], __uint_as_float(w[i] & 0xFFFF0000u), acc);
  }
  return acc;
}
__device__ __forceinline__ float tip_chunk(const uint4& u, const float* c, float) {
  float acc = __fmul_rn(c[0], __uint_as_float(u.x));
  acc = __fmaf_rn(c[1], __uint_as_float(u.y), acc);
  acc = __fmaf_rn(c[2], __uint_as_float(u.z), acc);
  acc = __fmaf_rn(c[3], __uint_as_float(u.w), acc);
  return acc;
}

// Halving tree over a lane's chunk partials (p is overwritten).
template <int CPL>
__device__ __forceinline__ float tip_lane_sum(float (&p)[CPL]) {
#pragma unroll
  for (int r = CPL / 2; r >= 1; r /= 2)
#pragma unroll
    for (int j = 0; j < r; ++j) p[j] = __fadd_rn(p[j], p[j + r]);
  return p[0];
}

// Xor butterfly over the LPT2 lanes of one token (every lane of the warp
// must take part); each of them ends with the same value.
template <int LPT2>
__device__ __forceinline__ float tip_lanes_sum(float acc) {
#pragma unroll
  for (int off = LPT2 / 2; off >= 1; off /= 2) acc = __fadd_rn(acc, __shfl_xor_sync(0xFFFFFFFFu, acc, off));
  return acc;
}

}  // namespace fasa
