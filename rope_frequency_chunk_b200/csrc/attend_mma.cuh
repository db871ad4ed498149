// Focused attention of the staged decode on tensor cores (bf16 caches).
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2, FAC bullets): full softmax attention of each query head over exactly
// the kept rows of its KV head, each row at its original position (keys were
// rotated at append).
//
// Layout of the work: grid = (splits, rows); a CTA takes a contiguous slice
// of the row's kept list and its 3 warps take 16-row chunks of it in turn
// (four CTAs per SM at G <= 8). Each warp gathers its chunks' K and V rows
// with 16-byte cp.async into its own 2-stage ring (no block barriers in the
// main loop; 16-byte chunks
// XOR-swizzled by row so ldmatrix reads are bank-conflict-free) and runs
// mma.sync.m16n8k16 (bf16 in, float32 accumulate):
//   S[16 x 16] = Q[16 x 128] K^T   (M = the group's query heads padded to 16,
//                                   N = 16 rows, K = head dim)
//   O[16 x 128] += P[16 x 16] V     (K = 16 rows, N = head dim)
// with an online base-2 softmax in registers (the 1/sqrt(128) and log2(e)
// scale folded into Q). Q is split into three bf16 terms (about 24 bits, as
// float32), prepared once per row by the filter kernel and read here with
// ldmatrix; each term accumulates in its own registers so the three MMA
// chains run side by side. P is split into two terms (P is in [0, 1] and only
// weights V); K and V are bf16 already and enter exactly. The warps of a CTA
// are merged as a tree through shared memory; the CTA writes its partial
// (m, l, o) to the workspace and the row's last CTA (atomic counter) merges
// the splits and writes the bf16 output.
#pragma once

#include "fasa_device.cuh"

namespace fasa {

constexpr int kAttWarps = 3;  // four CTAs (12 warps) per SM at G <= 8
constexpr int kAttThreads = kAttWarps * 32;
constexpr int kAttChunk = 16;                          // rows per warp step
constexpr int kAttStages = 2;                          // per-warp ring depth
constexpr int kAttHalf = kAttChunk * kD * 2;           // bytes of 16 bf16 rows (K or V)
constexpr int kAttStageBytes = 2 * kAttHalf;           // K + V
constexpr int kAttPartStride = 16 * kD + 32;           // floats: m[16], l[16], o[16][128]
constexpr int kQTermBytes = 3 * 16 * kD * 2;           // the three bf16 terms of 16 query rows
constexpr int kAttSlot = 68 * 32;                      // floats of one warp's (o, m, l) fragments

struct AttParams {
  const __nv_bfloat16* k;   // [rows][max_len][128]
  const __nv_bfloat16* v;
  const int32_t* idx;       // [rows][n_keep] kept rows; null: rows 0 .. n_keep-1
  const unsigned char* qterms;  // [rows][kQTermBytes] query terms (see query_terms), or null:
                                // each CTA forms its row's terms from q (query_terms_compact)
  const __nv_bfloat16* q;   // [B][Hq][128] pre-RoPE (with qterms null)
  int32_t n_kv_heads;       // (with qterms null)
  __nv_bfloat16* out;       // [B][Hq][128]
  float* part;              // [rows][splits][kAttPartStride]
  uint32_t* counter;        // [rows], zero before the launch; the last CTA resets it
  int64_t max_len;
  int32_t len;              // kept indices must lie in [0, len)
  int32_t n_keep;
  int32_t slice;            // rows per CTA, a multiple of kAttChunk
  int32_t splits;
  int32_t group;
  double cosv[kNFC];        // cos / sin of q_pos * theta_i (with qterms null)
  double sinv[kNFC];
};

// The ring, then the G query rows of each term (256 B each) and one zero row
// that stands in for the padding heads G..15.
__host__ __device__ constexpr int att_smem_bytes(int G) { return kAttWarps * kAttStages * kAttStageBytes + (3 * G + 1) * 256; }
static_assert(kAttSlot * 4 * (kAttWarps / 2) <= kAttWarps * kAttStages * kAttStageBytes, "merge slots exceed the ring");
// The last CTA of a row merges the splits in the ring's space: (m, l, weight)
// of 16 heads per split, then 16 denominators.
__host__ __device__ constexpr int att_merge_bytes(int splits) { return splits * 3 * 16 * 4 + 16 * 4; }
constexpr int kAttMaxSplits = (kAttWarps * kAttStages * kAttStageBytes - 16 * 4) / (3 * 16 * 4);
static_assert(att_merge_bytes(kAttMaxSplits) <= kAttWarps * kAttStages * kAttStageBytes, "split merge exceeds the ring");

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
// (x, y) -> bf16x2 with x in the low half (the lower k index), and the
// residuals (x - bf16(x), y - bf16(y)) likewise; returns the residuals too.
__device__ __forceinline__ float2 split_pack(float x, float y, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  const float2 hf = __bfloat1622float2(h);
  const float2 r = make_float2(x - hf.x, y - hf.y);
  const __nv_bfloat162 l = __floats2bfloat162_rn(r.x, r.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
  return r;
}

// Attention queries of the group: rotated, scaled by log2(e)/sqrt(128),
// rounded to float32, then split into three bf16 terms (low, middle, high)
// stored as rows of 256 B with 16-byte chunks XOR-swizzled by row for
// ldmatrix; heads >= G are zero. Threads tid < nthreads share the work.
__device__ __forceinline__ void query_terms(const __nv_bfloat16* qraw, int G, const double* cosv, const double* sinv,
                                            unsigned char* qt, int tid, int nthreads) {
  const double qscale = 1.4426950408889634 / 11.313708498984761;
  for (int e = tid; e < 16 * kD / 2; e += nthreads) {
    const int h = e / (kD / 2), d = 2 * (e % (kD / 2));
    float v2[2] = {0.0f, 0.0f};
    if (h < G) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int dd = d + u, i = dd & (kNFC - 1);
        const double x = __bfloat162float(qraw[h * kD + i]);
        const double y = __bfloat162float(qraw[h * kD + i + kNFC]);
        const double c = cosv[i], sn = sinv[i];
        v2[u] = (float)(((dd < kNFC) ? (x * c - y * sn) : (y * c + x * sn)) * qscale);
      }
    }
    uint32_t hi, mid, lo;
    const float2 r = split_pack(v2[0], v2[1], hi, mid);
    const float2 mf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&mid));
    const __nv_bfloat162 ll = __floats2bfloat162_rn(r.x - mf.x, r.y - mf.y);
    lo = *reinterpret_cast<const uint32_t*>(&ll);
    const int off = h * 256 + (((d / 8) ^ (h & 7)) * 16) + (d % 8) * 2;
    *reinterpret_cast<uint32_t*>(qt + 0 * 4096 + off) = lo;
    *reinterpret_cast<uint32_t*>(qt + 1 * 4096 + off) = mid;
    *reinterpret_cast<uint32_t*>(qt + 2 * 4096 + off) = hi;
  }
}

// The same terms in the compact layout chunk_logits reads: term t (low,
// middle, high) of head r at row t*G + r, then a zero row at 3G; the values
// are query_terms' bit for bit. qraw: the group's G pre-RoPE query rows.
__device__ __forceinline__ void query_terms_compact(const __nv_bfloat16* qraw, int G, const double* cosv,
                                                    const double* sinv, unsigned char* qt, int tid, int nthreads) {
  const double qscale = 1.4426950408889634 / 11.313708498984761;
  for (int e = tid; e < G * (kD / 2); e += nthreads) {
    const int h = e / (kD / 2), d = 2 * (e % (kD / 2));
    float v2[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int dd = d + u, i = dd & (kNFC - 1);
      const double x = __bfloat162float(qraw[h * kD + i]);
      const double y = __bfloat162float(qraw[h * kD + i + kNFC]);
      const double c = cosv[i], sn = sinv[i];
      v2[u] = (float)(((dd < kNFC) ? (x * c - y * sn) : (y * c + x * sn)) * qscale);
    }
    uint32_t hi, mid, lo;
    const float2 r = split_pack(v2[0], v2[1], hi, mid);
    const float2 mf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&mid));
    const __nv_bfloat162 ll = __floats2bfloat162_rn(r.x - mf.x, r.y - mf.y);
    lo = *reinterpret_cast<const uint32_t*>(&ll);
    const int off = (((d / 8) ^ (h & 7)) * 16) + (d % 8) * 2;
    *reinterpret_cast<uint32_t*>(qt + (0 * G + h) * 256 + off) = lo;
    *reinterpret_cast<uint32_t*>(qt + (1 * G + h) * 256 + off) = mid;
    *reinterpret_cast<uint32_t*>(qt + (2 * G + h) * 256 + off) = hi;
  }
  for (int c = tid; c < 16; c += nthreads) reinterpret_cast<uint4*>(qt + 3 * G * 256)[c] = make_uint4(0u, 0u, 0u, 0u);
}

// S = Q K^T for one 16-row chunk staged at Ks: s0 rows 0-7, s1 rows 8-15 of
// the chunk (fragment layout of m16n8k16), each Q term in its own chain.
// Query row r of term t is at qt + (t * G + r) * 256 for r < G, the zero
// row (qt + 3 * G * 256) otherwise.
__device__ __forceinline__ void chunk_logits(const unsigned char* qt, int G, const unsigned char* Ks, int lane,
                                             float (&s0)[4], float (&s1)[4]) {
  float a0[3][4], a1[3][4];
#pragma unroll
  for (int t = 0; t < 3; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) a0[t][e] = a1[t][e] = 0.0f;
  const int arow = (lane % 8) + ((lane / 8) % 2) * 8;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    uint32_t b[4];
    ldsm_x4(b, Ks + ((lane / 16) * 8 + lane % 8) * 256 + (((ks * 2 + (lane / 8) % 2) ^ (lane % 8)) * 16));
    const int aoff = (((ks * 2 + lane / 16) ^ (arow & 7)) * 16);
#pragma unroll
    for (int t = 0; t < 3; ++t) {  // low, middle, high bf16 term of Q
      uint32_t a[4];
      ldsm_x4(a, qt + (arow < G ? (t * G + arow) : 3 * G) * 256 + aoff);
      mma_16816(a0[t], a, b[0], b[1]);
      mma_16816(a1[t], a, b[2], b[3]);
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    s0[e] = (a0[0][e] + a0[1][e]) + a0[2][e];
    s1[e] = (a1[0][e] + a1[1][e]) + a1[2][e];
  }
}

__global__ void __launch_bounds__(kAttThreads) attend_mma_kernel(const AttParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  grid_dependency_wait();
  const int split = blockIdx.x, row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.group;
  unsigned char* qt = smem + kAttWarps * kAttStages * kAttStageBytes;
  if (p.qterms) {
    // the G real rows of each term (rows of the staged terms keep their
    // swizzle, which depends on the row index only), then a zero row
    const unsigned char* src = p.qterms + (int64_t)row * kQTermBytes;
    for (int c = tid; c < 3 * G * 16; c += kAttThreads) {
      const int t = c / (G * 16), r = (c / 16) % G, part = c % 16;
      cp_async16(qt + (t * G + r) * 256 + part * 16, src + t * 4096 + r * 256 + part * 16);
    }
    if (tid < 16) reinterpret_cast<uint4*>(qt + 3 * G * 256)[tid] = make_uint4(0u, 0u, 0u, 0u);
    cp_async_commit();
  } else {
    // the row's query terms from q, staged through the (not yet used) ring
    __nv_bfloat16* qraw = reinterpret_cast<__nv_bfloat16*>(smem);
    const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + (int64_t)row * G * kD);
    for (int c = tid; c < G * kD / 8; c += kAttThreads) reinterpret_cast<uint4*>(qraw)[c] = __ldg(qsrc + c);
    __syncthreads();
    query_terms_compact(qraw, G, p.cosv, p.sinv, qt, tid, kAttThreads);
    __syncthreads();
    cp_async_commit();  // an empty group: the pipeline below counts one group for the terms
  }

  const int r_beg = split * p.slice;
  const int r_end = min(p.n_keep, r_beg + p.slice);
  const int nchunks = max(0, (r_end - r_beg + kAttChunk - 1) / kAttChunk);
  const int mine = nchunks > warp ? (nchunks - warp + kAttWarps - 1) / kAttWarps : 0;
  unsigned char* ring = smem + warp * kAttStages * kAttStageBytes;
  const __nv_bfloat16* kb = p.k + (int64_t)row * p.max_len * kD;
  const __nv_bfloat16* vb = p.v + (int64_t)row * p.max_len * kD;
  const int32_t* idx = p.idx ? p.idx + (int64_t)row * p.n_keep : nullptr;

  // kept row of list position j (-1: past the end or an invalid index)
  auto row_of = [&](int j) -> int {
    if (j >= r_end) return -1;
    const int t = idx ? __ldg(idx + j) : j;
    return (t >= 0 && t < p.len) ? t : -1;
  };
  auto issue = [&](int ci) {
    if (ci < mine) {
      const int j0 = r_beg + (warp + ci * kAttWarps) * kAttChunk;
      unsigned char* st = ring + (ci % kAttStages) * kAttStageBytes;
      int tr = lane < kAttChunk ? row_of(j0 + lane) : 0;
      if (tr < 0) {
        if (lane < kAttChunk && j0 + lane < r_end) flag_status(FASA_ERR_BAD_INDEX);
        tr = 0;  // masked below
      }
#pragma unroll
      for (int r = 0; r < kAttChunk; ++r) {  // 16 rows x (16 K + 16 V) 16-byte parts, one part per lane
        const int t = __shfl_sync(0xFFFFFFFFu, tr, r);
        const __nv_bfloat16* src = (lane < 16 ? kb : vb) + (int64_t)t * kD + (lane % 16) * 8;
        // 16-byte chunk c of row r is stored at chunk c ^ (r & 7) (bank-conflict-free ldmatrix)
        cp_async16(st + (lane < 16 ? 0 : kAttHalf) + r * 256 + (((lane % 16) ^ (r & 7)) * 16), src);
      }
    }
    cp_async_commit();
  };

  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[n][e] = 0.0f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;  // heads lane/4 and lane/4 + 8

#pragma unroll
  for (int s = 0; s < kAttStages; ++s) issue(s);
  cp_async_wait<kAttStages>();  // the query terms (the oldest group)
  __syncthreads();
  for (int ci = 0; ci < mine; ++ci) {
    cp_async_wait<kAttStages - 1>();
    __syncwarp();
    const unsigned char* Ks = ring + (ci % kAttStages) * kAttStageBytes;
    const unsigned char* Vs = Ks + kAttHalf;
    float s0[4], s1[4];  // rows 0-7, 8-15 of the chunk
    chunk_logits(qt, G, Ks, lane, s0, s1);
    // mask the chunk's missing or invalid rows (columns of S)
    const int j0 = r_beg + (warp + ci * kAttWarps) * kAttChunk;
    const int c0 = (lane % 4) * 2;
    if (row_of(j0 + c0) < 0) s0[0] = s0[2] = -INFINITY;
    if (row_of(j0 + c0 + 1) < 0) s0[1] = s0[3] = -INFINITY;
    if (row_of(j0 + 8 + c0) < 0) s1[0] = s1[2] = -INFINITY;
    if (row_of(j0 + 8 + c0 + 1) < 0) s1[1] = s1[3] = -INFINITY;
    // online softmax over this chunk for heads lane/4 (x0) and lane/4 + 8 (x1)
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
    for (int n = 0; n < 16; ++n) {
      o[n][0] *= sc0;
      o[n][1] *= sc0;
      o[n][2] *= sc1;
      o[n][3] *= sc1;
    }
    // P as the A operand (heads x 16 rows), high and residual parts
    uint32_t ph[4], pl[4];
    split_pack(pr[0], pr[1], ph[0], pl[0]);
    split_pack(pr[2], pr[3], ph[1], pl[1]);
    split_pack(pr[4], pr[5], ph[2], pl[2]);
    split_pack(pr[6], pr[7], ph[3], pl[3]);
#pragma unroll
    for (int n = 0; n < 16; n += 2) {
      uint32_t b[4];
      ldsm_x4_t(b, Vs + (((lane / 8) % 2) * 8 + lane % 8) * 256 + (((n + lane / 16) ^ (lane % 8)) * 16));
      mma_16816(o[n], ph, b[0], b[1]);
      mma_16816(o[n], pl, b[0], b[1]);
      mma_16816(o[n + 1], ph, b[2], b[3]);
      mma_16816(o[n + 1], pl, b[2], b[3]);
    }
    __syncwarp();
    issue(ci + kAttStages);
  }
  cp_async_wait<0>();

  // warps merged as a tree through shared memory (the rings are free now):
  // of the cnt warps still holding a partial, warps [h, cnt) hand their
  // fragments to warps [0, cnt - h), h = ceil(cnt / 2); lane-major slots
  float* slots = reinterpret_cast<float*>(smem);
#pragma unroll 1
  for (int cnt = kAttWarps; cnt > 1;) {
    const int h = (cnt + 1) / 2;
    __syncthreads();
    if (warp >= h && warp < cnt) {
      float* sl = slots + (warp - h) * kAttSlot;
#pragma unroll
      for (int n = 0; n < 16; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) sl[(n * 4 + e) * 32 + lane] = o[n][e];
      sl[64 * 32 + lane] = m0;
      sl[65 * 32 + lane] = m1;
      sl[66 * 32 + lane] = l0;
      sl[67 * 32 + lane] = l1;
    }
    __syncthreads();
    if (warp < cnt - h) {
      const float* sl = slots + warp * kAttSlot;
      const float pm0 = sl[64 * 32 + lane], pm1 = sl[65 * 32 + lane];
      const float n0 = fmaxf(m0, pm0), n1 = fmaxf(m1, pm1);
      const float a0 = (m0 == -INFINITY) ? 0.0f : exp2f(m0 - n0), a1 = (m1 == -INFINITY) ? 0.0f : exp2f(m1 - n1);
      const float b0 = (pm0 == -INFINITY) ? 0.0f : exp2f(pm0 - n0), b1 = (pm1 == -INFINITY) ? 0.0f : exp2f(pm1 - n1);
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        o[n][0] = o[n][0] * a0 + sl[(n * 4 + 0) * 32 + lane] * b0;
        o[n][1] = o[n][1] * a0 + sl[(n * 4 + 1) * 32 + lane] * b0;
        o[n][2] = o[n][2] * a1 + sl[(n * 4 + 2) * 32 + lane] * b1;
        o[n][3] = o[n][3] * a1 + sl[(n * 4 + 3) * 32 + lane] * b1;
      }
      l0 = l0 * a0 + sl[66 * 32 + lane] * b0;
      l1 = l1 * a1 + sl[67 * 32 + lane] * b1;
      m0 = n0;
      m1 = n1;
    }
    cnt = h;
  }
  // warp 0: the CTA's partial (m, l, o) to the workspace
  float* pp = p.part + ((int64_t)row * p.splits + split) * kAttPartStride;
  if (warp == 0) {
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 1);
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 2);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 1);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 2);
    if (lane % 4 == 0) {
      pp[lane / 4] = m0;
      pp[lane / 4 + 8] = m1;
      pp[16 + lane / 4] = l0;
      pp[16 + lane / 4 + 8] = l1;
    }
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      const int d = n * 8 + (lane % 4) * 2;
      *reinterpret_cast<float2*>(pp + 32 + (lane / 4) * kD + d) = make_float2(o[n][0], o[n][1]);
      *reinterpret_cast<float2*>(pp + 32 + (lane / 4 + 8) * kD + d) = make_float2(o[n][2], o[n][3]);
    }
  }
  // the row's last CTA merges all splits
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(p.counter + row, 1u) == (uint32_t)(p.splits - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // merge: first every split's (m, l) into shared memory, then per head the
  // split weights and the denominator, then each output with all split loads
  // independent of one another
  const float* rp = p.part + (int64_t)row * p.splits * kAttPartStride;
  __nv_bfloat16* out = p.out + ((int64_t)row * G) * kD;
  float* sm_m = reinterpret_cast<float*>(smem);            // [splits][16]
  float* sm_l = sm_m + p.splits * 16;                     // [splits][16]
  float* sm_w = sm_l + p.splits * 16;                     // [splits][16] weights
  float* sm_den = sm_w + p.splits * 16;                   // [16]
  for (int i = tid; i < p.splits * 16; i += kAttThreads) {
    sm_m[i] = __ldcg(rp + (i / 16) * kAttPartStride + i % 16);
    sm_l[i] = __ldcg(rp + (i / 16) * kAttPartStride + 16 + i % 16);
  }
  __syncthreads();
  if (tid < 16) {
    float M = -INFINITY;
    for (int s = 0; s < p.splits; ++s) M = fmaxf(M, sm_m[s * 16 + tid]);
    float den = 0.0f;
    for (int s = 0; s < p.splits; ++s) {
      const float ms = sm_m[s * 16 + tid];
      const float w = (ms == -INFINITY || M == -INFINITY) ? 0.0f : exp2f(ms - M);
      sm_w[s * 16 + tid] = w;
      den += w * sm_l[s * 16 + tid];
    }
    sm_den[tid] = den;
  }
  __syncthreads();
  for (int e = tid; e < G * kD; e += kAttThreads) {
    const int h = e / kD;
    float num = 0.0f;
    int s = 0;
    for (; s + 4 <= p.splits; s += 4) {
      const float v0 = __ldcg(rp + (s + 0) * kAttPartStride + 32 + e);
      const float v1 = __ldcg(rp + (s + 1) * kAttPartStride + 32 + e);
      const float v2 = __ldcg(rp + (s + 2) * kAttPartStride + 32 + e);
      const float v3 = __ldcg(rp + (s + 3) * kAttPartStride + 32 + e);
      num += sm_w[(s + 0) * 16 + h] * v0 + sm_w[(s + 1) * 16 + h] * v1 + sm_w[(s + 2) * 16 + h] * v2 +
             sm_w[(s + 3) * 16 + h] * v3;
    }
    for (; s < p.splits; ++s) num += sm_w[s * 16 + h] * __ldcg(rp + s * kAttPartStride + 32 + e);
    const float den = sm_den[h];
    out[e] = __float2bfloat16_rn(den > 0.0f ? num / den : 0.0f);
  }
  if (tid == 0) p.counter[row] = 0u;
}

}  // namespace fasa
