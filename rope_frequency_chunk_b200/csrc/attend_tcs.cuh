// Focused (and dense) attention for up to 16 query rows per KV head on the
// 5th-generation tensor cores, kept rows along the tensor-memory lanes.
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2, FAC): softmax attention of a group's query heads over the kept rows
// only, each at its original position; §4: the full-KV comparison is the
// same over every row. With G (or n_q * G) <= 16 query rows a tile of 128
// kept rows gives S^T = K Q^T (M = 128 kept rows, N = 16 query rows, K = 128
// dims) and O^T = V^T P^T (M = 128 dims, N = 16, K = 128 kept rows). The
// softmax is then per column of S^T: each thread holds one kept row's 16
// logits, and a column's maximum and sum are warp reductions plus a 4-warp
// combine. Every thread keeps its dim's 16 output values in registers. Per
// tile a thread issues about a hundred instructions; the gather of the K
// and V rows (16-byte cp.async into the swizzled layout) bounds the kernel,
// and two CTAs per SM overlap their chains.
//
// The rotated, scaled queries are split into three bf16 terms (hi + mid +
// lo) and the probabilities into two (hi + lo), one MMA per term: about 24
// and 16 significant bits, float32 accumulation. A kept row outside [0, len) is masked (its logit is
// -inf) and flagged; a multi-query row does not see kept slots after its
// own position. Splits of a row write (m, l, o) partials in the layout of
// the CUDA-core split-K kernel's; the row's last CTA merges them in order.
#pragma once

#include "attend_tc.cuh"

namespace fasa {

constexpr int kTsThreads = 128;
constexpr int kTsTile = 128;   // kept rows per tile
constexpr int kTsN = 16;       // query rows (N of both products)
constexpr int kTsMaxSplits = 256;
constexpr uint32_t kTsCols = 32;  // TMEM columns: S^T [0, 16), O^T tile [16, 32)
constexpr uint32_t kTsMasked = 0x7FFFFFFFu;

struct TsParams {
  const __nv_bfloat16* k;  // [rows][max_len][128], or paged pools
  const __nv_bfloat16* v;
  const int32_t* idx;      // [rows][n_keep] kept slots, or null: slots 0 .. n_keep-1
  const __nv_bfloat16* q;  // [B][n_q][Hq][128]
  __nv_bfloat16* out;      // [B][n_q][Hq][128]
  float* part;             // [rows][splits][kCcPartStride]
  uint32_t* counter;       // [rows], zero before the launch; left zero
  int64_t max_len;
  int32_t len;             // kept slots lie in [0, len) (upper bound with seq_len)
  int32_t n_keep;          // kept entries per row (upper bound and idx row stride with row_keep)
  int32_t slice;           // list positions per CTA, a multiple of kTsTile
  int32_t splits;
  int32_t group;
  int32_t n_q;
  int32_t n_kv_heads;
  int32_t q_pos0;          // token j at position q_pos0 + j (no mask when q_prerot)
  int32_t q_prerot;
  int32_t mask_after;      // 1: a row does not see kept slots after its position (multi-query)
  const int32_t* seq_len;  // [B] per-sequence lengths (the query at seq_len[b]), or null
  const int32_t* row_keep; // [rows] per-row kept counts, or null
  PageMap pm;
  double cosv[kNFC];       // cos / sin of the angle (one token, uniform length), or theta_i (varlen, n_q > 1)
  double sinv[kNFC];
};

__host__ __device__ constexpr int ts_smem_bytes(int n_q) {
  // Q hi / lo and P hi / lo tile pairs of 16 rows, K and V tiles, Q mid, kept slots,
  // column maxima / sums / weights, mbarrier and TMEM address, angle tables,
  // 1 KB to align the tiles
  return 5 * 2 * kTsN * 128 + 2 * 32768 + kTsTile * 4 + (2 * 4 * kTsN + 3 * kTsN) * 4 + 16 +
         n_q * 2 * kNFC * 8 + 1024;
}

__global__ void __launch_bounds__(kTsThreads, 2) attend_tcs_kernel(const TsParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, row = blockIdx.y;
  const int G = p.group, MQ = p.n_q * G;
  constexpr uint32_t kPair = 2u * kTsN * 128u;  // one 16-row tile pair (4 KB)
  unsigned char* qhi = smem;
  unsigned char* qmd = qhi + kPair;
  unsigned char* qlo = qmd + kPair;
  unsigned char* phi = qlo + kPair;
  unsigned char* plo = phi + kPair;
  unsigned char* ks = plo + kPair;  // 1024-aligned
  unsigned char* vs = ks + 32768;
  uint32_t* tok_s = reinterpret_cast<uint32_t*>(vs + 32768);
  float* red = reinterpret_cast<float*>(tok_s + kTsTile);  // [2][4 warps][16]: maxima, sums
  float* m_run = red + 2 * 4 * kTsN;                       // [16]
  float* l_run = m_run + kTsN;                             // [16]
  float* alpha = l_run + kTsN;                             // [16]
  uint64_t* bar = reinterpret_cast<uint64_t*>(alpha + kTsN);
  uint32_t* tbase_s = reinterpret_cast<uint32_t*>(bar + 1);
  double* cs = reinterpret_cast<double*>(tbase_s + 2);     // [n_q][cos 64 | sin 64]

  const int b = row / p.n_kv_heads, g = row % p.n_kv_heads;
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tc_alloc(tbase_s, kTsCols);
  // angle tables from the parameters, before the wait (they do not depend on
  // the earlier launch)
  const bool dev_angle = p.seq_len != nullptr || p.n_q > 1;  // cosv holds theta_i
  for (int e = tid; e < p.n_q * kNFC; e += kTsThreads) {
    const int j = e / kNFC, i = e % kNFC;
    cs[j * 2 * kNFC + i] = p.cosv[i];
    cs[j * 2 * kNFC + kNFC + i] = p.sinv[i];
  }
  if (tid < kTsN) {
    m_run[tid] = -INFINITY;
    l_run[tid] = 0.0f;
  }
  grid_dependency_wait();
  int len = p.len, n_keep = p.n_keep;
  int qpos = p.q_pos0;
  if (p.seq_len) {
    len = min(max(__ldg(p.seq_len + b), 1), p.len);  // range flagged by the selecting kernel
    qpos = len;
  }
  if (p.row_keep) n_keep = min(max(p.row_keep[row], 0), p.n_keep);
  __syncthreads();
  if (dev_angle) {  // token j at position qpos + j (or already rotated)
    for (int e = tid; e < p.n_q * kNFC; e += kTsThreads) {
      const int j = e / kNFC, i = e % kNFC;
      double sn = 0.0, cn = 1.0;
      if (!p.q_prerot) sincos((double)(qpos + j) * cs[j * 2 * kNFC + i], &sn, &cn);
      cs[j * 2 * kNFC + i] = cn;
      cs[j * 2 * kNFC + kNFC + i] = sn;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tbase_s;

  // the query rows n = j * G + h: staged raw in the P hi tiles, rotated
  // (float64), scaled by log2(e) / sqrt(128), split into bf16 hi + lo
  const int hq = p.n_kv_heads * G;
  {
    uint4* qst = reinterpret_cast<uint4*>(phi);  // [MQ][16] raw chunks (MQ * 256 <= 4 KB)
    for (int c = tid; c < MQ * 16; c += kTsThreads) {
      const int r = c >> 4, j = r / G, h = r % G;
      qst[c] = __ldg(reinterpret_cast<const uint4*>(p.q + (((int64_t)b * p.n_q + j) * hq + g * G + h) * kD) +
                     (c & 15));
    }
    __syncthreads();
    const __nv_bfloat16* qs = reinterpret_cast<const __nv_bfloat16*>(phi);
    const double qscale = 1.4426950408889634 / 11.313708498984761;
    for (int c = tid; c < MQ * 16; c += kTsThreads) {
      const int r = c >> 4, ch = c & 15;
      const double* cz = cs + (r / G) * 2 * kNFC;
      float x[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int d = ch * 8 + e, i = d & (kNFC - 1);
        const double a = __bfloat162float(qs[r * kD + i]), bb = __bfloat162float(qs[r * kD + i + kNFC]);
        const double rr = d < kNFC ? __dsub_rn(__dmul_rn(a, cz[i]), __dmul_rn(bb, cz[kNFC + i]))
                                   : __dadd_rn(__dmul_rn(bb, cz[i]), __dmul_rn(a, cz[kNFC + i]));
        x[e] = (float)(rr * qscale);
      }
      uint4 hi, md, lo;
      tc_split8x3(x, hi, md, lo);
      *reinterpret_cast<uint4*>(qhi + tc_sw(r, ch, kTsN)) = hi;
      *reinterpret_cast<uint4*>(qmd + tc_sw(r, ch, kTsN)) = md;
      *reinterpret_cast<uint4*>(qlo + tc_sw(r, ch, kTsN)) = lo;
    }
  }

  const int r_beg = split * p.slice, r_end = min(n_keep, r_beg + p.slice);
  const int32_t* idx = p.idx ? p.idx + (int64_t)row * p.n_keep : nullptr;
  const bool paged = p.pm.table != nullptr;
  const int64_t plane = paged ? 0 : (int64_t)row * p.max_len * kD;
  const __nv_bfloat16* kb = p.k + plane;
  const __nv_bfloat16* vb = p.v + plane;
  // the limit on a column's visible slots (the row's own position)
  auto col_lim = [&](int n) -> uint32_t {
    return (p.mask_after && !p.q_prerot) ? (uint32_t)min(qpos + n / G, (int)kTsMasked - 1) : kTsMasked - 1;
  };
  float o[kTsN];  // this thread's dim, every query row
#pragma unroll
  for (int n = 0; n < kTsN; ++n) o[n] = 0.0f;
  uint32_t phase = 0;
  bool failed = false;
  const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);

  for (int jb = r_beg; jb < r_end && !failed; jb += kTsTile) {
    {  // gather: thread = kept row (masked entries read row 0)
      const int j = jb + tid;
      int t = -1;
      if (j < r_end) {
        t = idx ? __ldg(idx + j) : j;
        if (t < 0 || t >= len) {
          flag_status(FASA_ERR_BAD_INDEX);
          t = -1;
        }
      }
      int prow = t;
      if (t >= 0 && paged) prow = paged_row(p.pm, b, g, t);
      tok_s[tid] = prow < 0 ? kTsMasked : (uint32_t)t;
      const uint4* kr = reinterpret_cast<const uint4*>(kb + (int64_t)(prow < 0 ? 0 : prow) * kD);
      const uint4* vr = reinterpret_cast<const uint4*>(vb + (int64_t)(prow < 0 ? 0 : prow) * kD);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        cp_async16(ks + tc_sw(tid, c, kTsTile), kr + c);
        cp_async16(vs + tc_sw(tid, c, kTsTile), vr + c);
      }
      cp_async_commit();
      cp_async_wait<0>();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // S^T = K (Q hi + Q mid + Q lo)^T: M 128 kept rows, N 16 query rows, K 128 dims
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int s8 = 0; s8 < 8; ++s8) {
        const uint32_t ko = (s8 >> 2) * kTsTile * 128 + (s8 & 3) * 32;
        const uint32_t qo = (s8 >> 2) * kTsN * 128 + (s8 & 3) * 32;
        const uint64_t ad = tc_desc(smem_u32(ks) + ko, 16, 1024);
        tc_mma(tbase, ad, tc_desc(smem_u32(qhi) + qo, 16, 1024), tc_idesc_n(kTsN, 0, 0), s8 > 0);
        tc_mma(tbase, ad, tc_desc(smem_u32(qmd) + qo, 16, 1024), tc_idesc_n(kTsN, 0, 0), 1);
        tc_mma(tbase, ad, tc_desc(smem_u32(qlo) + qo, 16, 1024), tc_idesc_n(kTsN, 0, 0), 1);
      }
      tc_commit(bar);
    }
    failed = __syncthreads_or(!mbar_wait(bar, phase));
    phase ^= 1u;
    if (failed) break;
    tc_fence_after();
    // column maxima of the tile (the thread's kept row, every query row)
    float s[kTsN];
    tc_ld16(tl, s);
    const uint32_t tok = tok_s[tid];
#pragma unroll
    for (int n = 0; n < kTsN; ++n) {
      if (n >= MQ || tok > col_lim(n)) s[n] = -INFINITY;
      float m = s[n];
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
      if (lane == n) red[warp * kTsN + n] = m;
    }
    __syncthreads();
    if (tid < kTsN) {
      const float mt = fmaxf(fmaxf(red[tid], red[kTsN + tid]), fmaxf(red[2 * kTsN + tid], red[3 * kTsN + tid]));
      const float mo = m_run[tid], mn = fmaxf(mo, mt);
      alpha[tid] = (mn == -INFINITY) ? 1.0f : exp2f(mo - mn);
      m_run[tid] = mn;
    }
    __syncthreads();
    // probabilities: P^T hi / lo, element (query row n, kept row tid); column sums
    {
      const int c = tid >> 3, e = tid & 7;
#pragma unroll
      for (int n = 0; n < kTsN; ++n) {
        const float mn = m_run[n];
        const float pz = (s[n] == -INFINITY || mn == -INFINITY) ? 0.0f : exp2f(s[n] - mn);
        const __nv_bfloat16 h = __float2bfloat16_rn(pz);
        const __nv_bfloat16 lo = __float2bfloat16_rn(pz - __bfloat162float(h));
        const uint32_t at = tc_sw(n, c, kTsN) + e * 2;
        *reinterpret_cast<__nv_bfloat16*>(phi + at) = h;
        *reinterpret_cast<__nv_bfloat16*>(plo + at) = lo;
        float sm = pz;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) sm += __shfl_xor_sync(0xFFFFFFFFu, sm, off);
        if (lane == n) red[4 * kTsN + warp * kTsN + n] = sm;
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid < kTsN) {
      const float* rs = red + 4 * kTsN;
      l_run[tid] = __fmaf_rn(l_run[tid], alpha[tid], (rs[tid] + rs[kTsN + tid]) + (rs[2 * kTsN + tid] + rs[3 * kTsN + tid]));
    }
    // O^T tile = V^T (P hi + P lo)^T: M 128 dims, N 16 query rows, K 128 kept rows
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int s8 = 0; s8 < 8; ++s8) {
        const uint64_t ad = tc_desc(smem_u32(vs) + s8 * 2048, kTsTile * 128, 1024);
        const uint32_t po = (s8 >> 2) * kTsN * 128 + (s8 & 3) * 32;
        tc_mma(tbase + kTsN, ad, tc_desc(smem_u32(phi) + po, 16, 1024), tc_idesc_n(kTsN, 1, 0), s8 > 0);
        tc_mma(tbase + kTsN, ad, tc_desc(smem_u32(plo) + po, 16, 1024), tc_idesc_n(kTsN, 1, 0), 1);
      }
      tc_commit(bar);
    }
    failed = __syncthreads_or(!mbar_wait(bar, phase));
    phase ^= 1u;
    if (failed) break;
    tc_fence_after();
    {
      float dv[kTsN];
      tc_ld16(tl + kTsN, dv);  // lane = this thread's dim
#pragma unroll
      for (int n = 0; n < kTsN; ++n) o[n] = __fmaf_rn(o[n], alpha[n], dv[n]);
    }
    tc_fence_before();
    __syncthreads();  // TMEM, the tiles and the column state are free for the next tile
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tc_dealloc(tbase, kTsCols);
  if (failed) return;

  // this split's partial (m, l, o), or the output when the row has one split
  const int d = tid;  // the thread's dim
  auto out_at = [&](int n) -> __nv_bfloat16* {
    return p.out + (((int64_t)b * p.n_q + n / G) * hq + g * G + n % G) * kD + d;
  };
  if (p.splits == 1) {
#pragma unroll
    for (int n = 0; n < kTsN; ++n)
      if (n < MQ) {
        const float l = l_run[n];
        *out_at(n) = __float2bfloat16_rn(l > 0.0f ? o[n] / l : 0.0f);
      }
    return;
  }
  float* pp = p.part + ((int64_t)row * p.splits + split) * kCcPartStride;
#pragma unroll
  for (int n = 0; n < kTsN; ++n)
    if (n < MQ) pp[32 + n * kD + d] = o[n];
  if (tid < MQ) {
    pp[tid] = m_run[tid];
    pp[16 + tid] = l_run[tid];
  }
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(p.counter + row, 1u) == (uint32_t)(p.splits - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // merge in split order: weights w[s][n] = 2^(m_s - M), denominators
  const float* rp = p.part + (int64_t)row * p.splits * kCcPartStride;
  float* w = reinterpret_cast<float*>(ks);  // [splits][16]
  float* den = w + p.splits * kTsN;         // [16]
  for (int it = tid; it < p.splits * MQ; it += kTsThreads) {
    const int sr = it / MQ, n = it % MQ;
    w[sr * kTsN + n] = __ldcg(rp + sr * kCcPartStride + n);
  }
  __syncthreads();
  if (tid < MQ) {
    float M = -INFINITY;
    for (int sr = 0; sr < p.splits; ++sr) M = fmaxf(M, w[sr * kTsN + tid]);
    float dn = 0.0f;
    for (int sr = 0; sr < p.splits; ++sr) {
      const float ms = w[sr * kTsN + tid];
      const float ws = (ms == -INFINITY || M == -INFINITY) ? 0.0f : exp2f(ms - M);
      w[sr * kTsN + tid] = ws;
      dn = __fmaf_rn(ws, __ldcg(rp + sr * kCcPartStride + 16 + tid), dn);
    }
    den[tid] = dn;
  }
  __syncthreads();
  float num[kTsN];
#pragma unroll
  for (int n = 0; n < kTsN; ++n) num[n] = 0.0f;
  for (int sr = 0; sr < p.splits; ++sr) {  // the thread's dim of every row, loads of one split in flight
    float v[kTsN];
#pragma unroll
    for (int n = 0; n < kTsN; ++n) v[n] = n < MQ ? __ldcg(rp + sr * kCcPartStride + 32 + n * kD + d) : 0.0f;
#pragma unroll
    for (int n = 0; n < kTsN; ++n) num[n] = __fmaf_rn(w[sr * kTsN + n], v[n], num[n]);
  }
#pragma unroll
  for (int n = 0; n < kTsN; ++n)
    if (n < MQ) *out_at(n) = __float2bfloat16_rn(den[n] > 0.0f ? num[n] / den[n] : 0.0f);
  if (tid == 0) p.counter[row] = 0u;
}

}  // namespace fasa
