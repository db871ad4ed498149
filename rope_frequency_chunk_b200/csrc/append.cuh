// Append kernel: rotate new keys at their absolute positions, store K and V,
// and write the dominant-FC sketch rows.
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2 "A Descoberta": RoPE splits a head into 2-D frequency chunks, each with
// its own angular frequency; FAC bullet 3: tokens keep their original
// absolute positions). A key is rotated exactly once, here, at its slot's
// position, so a later gather of the row needs no re-rotation.
//
// Grid: x = blocks of kAppendTok tokens, y = groups of `heads_per_cta`
// consecutive (b, g) rows. cos/sin of a token block are computed once in
// float64 and reused across the CTA's heads (recomputed per sequence when
// every sequence appends at its own position). Slots are addressed through
// a PageMap, so the same kernel fills contiguous and paged caches.
#pragma once

#include "fasa_device.cuh"

namespace fasa {

constexpr int kAppendTok = 8;
constexpr int kAppendThreads = 256;

struct AppendParams {
  const void* k_new;     // [B*Hkv][n_new][128]
  const void* v_new;
  void* k;               // [B*Hkv][max_len][128]
  void* v;
  void* sketch;          // [B*Hkv][max_len][stride]
  const int32_t* dom_idx;  // [Hkv][n_dom]
  int64_t max_len;
  int32_t n_rows;        // B*Hkv
  int32_t n_kv_heads;
  int32_t n_new;
  int32_t pos0;
  int32_t n_dom;
  int32_t stride;
  int32_t heads_per_cta;
  const int32_t* pos0v;  // [B] each sequence's first new position, or null: pos0 for all
  PageMap pm;            // paged pools, or pm.table null: [B*Hkv][max_len] planes
  double theta[kNFC];    // base^(-2i/128), computed on the host in float64
};

template <typename T>
__global__ void __launch_bounds__(kAppendThreads) append_kernel(const AppendParams p) {
  __shared__ double s_cos[kAppendTok][kNFC];
  __shared__ double s_sin[kAppendTok][kNFC];
  __shared__ T s_row[kAppendTok][kD];
  __shared__ int s_dom[kNFC];
  __shared__ int64_t s_dst[kAppendTok];  // each token's row in the K / V / sketch planes, or -1

  const int tid = threadIdx.x;
  const int tok0 = blockIdx.x * kAppendTok;
  const int ntok = min(kAppendTok, p.n_new - tok0);
  const int row0 = blockIdx.y * p.heads_per_cta;
  const int row1 = min(p.n_rows, row0 + p.heads_per_cta);

  auto angles = [&](int pos) {
    for (int e = tid; e < ntok * kNFC; e += kAppendThreads) {
      const int t = e / kNFC, i = e % kNFC;
      const double ang = (double)(pos + tok0 + t) * p.theta[i];
      double s, c;
      sincos(ang, &s, &c);
      s_cos[t][i] = c;
      s_sin[t][i] = s;
    }
  };
  int cur = p.pos0;
  if (!p.pos0v) angles(cur);

  for (int row = row0; row < row1; ++row) {
    const int b = row / p.n_kv_heads, g = row % p.n_kv_heads;
    int pos = p.pos0;
    if (p.pos0v) {
      pos = __ldg(p.pos0v + b);
      if (pos < 0 || (int64_t)pos + p.n_new > p.max_len) {  // block-uniform: skip the row
        if (tid == 0 && blockIdx.x == 0) flag_status(FASA_ERR_BAD_INDEX);
        continue;
      }
      if (row == row0 || pos != cur) {
        __syncthreads();  // the previous row is done with the angles
        angles(pos);
        cur = pos;
      }
    }
    __syncthreads();  // s_cos ready; previous row done with s_row / s_dom / s_dst
    if (tid < ntok) {
      const int t = pos + tok0 + tid;
      s_dst[tid] = p.pm.table ? (int64_t)paged_row(p.pm, b, g, t) : (int64_t)row * p.max_len + t;
    }
    if (tid < p.n_dom) {
      int d = p.dom_idx[g * p.n_dom + tid];
      if (d < 0 || d >= kNFC) {
        flag_status(FASA_ERR_BAD_INDEX);
        d = -1;
      }
      s_dom[tid] = d;
    }
    const T* kin = static_cast<const T*>(p.k_new) + ((int64_t)row * p.n_new + tok0) * kD;
    const T* vin = static_cast<const T*>(p.v_new) + ((int64_t)row * p.n_new + tok0) * kD;
    T* kc = static_cast<T*>(p.k);
    T* vc = static_cast<T*>(p.v);
    T* sk = static_cast<T*>(p.sketch);
    __syncthreads();  // s_dst ready

    // RoPE of FC i: (x, y) -> (x cos - y sin, y cos + x sin), float64, no
    // contraction, one rounding to the cache dtype.
    for (int e = tid; e < ntok * kNFC; e += kAppendThreads) {
      const int t = e / kNFC, i = e % kNFC;
      const double x = to_float(kin[t * kD + i]);
      const double y = to_float(kin[t * kD + i + kNFC]);
      const double c = s_cos[t][i], s = s_sin[t][i];
      const double xr = __dsub_rn(__dmul_rn(x, c), __dmul_rn(y, s));
      const double yr = __dadd_rn(__dmul_rn(y, c), __dmul_rn(x, s));
      T xs, ys;
      round_store(&xs, xr);
      round_store(&ys, yr);
      const int64_t dst = s_dst[t];
      if (dst >= 0) {
        kc[dst * kD + i] = xs;
        kc[dst * kD + i + kNFC] = ys;
      }
      s_row[t][i] = xs;
      s_row[t][i + kNFC] = ys;
    }
    // values are stored as given (16-byte vectors)
    constexpr int kVecRow = kD * (int)sizeof(T) / 16;  // 16-byte vectors per row
    for (int e = tid; e < ntok * kVecRow; e += kAppendThreads) {
      const int64_t dst = s_dst[e / kVecRow];
      if (dst >= 0)
        reinterpret_cast<uint4*>(vc + dst * kD)[e % kVecRow] = reinterpret_cast<const uint4*>(vin)[e];
    }
    __syncthreads();
    // sketch row: dims (dom[j], dom[j]+64) at 2j, 2j+1, zero padding
    for (int e = tid; e < ntok * p.stride; e += kAppendThreads) {
      const int t = e / p.stride, c = e % p.stride, j = c >> 1;
      T val = T(0.0f);
      if (j < p.n_dom) {
        const int d = s_dom[j];
        if (d >= 0) val = s_row[t][d + (c & 1) * kNFC];
      }
      const int64_t dst = s_dst[t];
      if (dst >= 0) sk[dst * p.stride + c] = val;
    }
  }
}

}  // namespace fasa
