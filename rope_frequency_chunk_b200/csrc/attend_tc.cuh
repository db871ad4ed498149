// Multi-query focused attention on the 5th-generation tensor cores.
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2, FAC): attention runs over the critical set only. With n_q query tokens
// per sequence (speculative drafts or batched rows) the n_q * G query rows of
// a KV head share one kept list, so Q K^T and P V over a tile of kept rows
// are dense products of (query rows) x 128 x (tile rows): tensor-core work.
//
// Design (one CTA of 4 warps per slice of a row's kept list; no clusters):
//  - the 128 TMEM lanes are query rows (M = 128; rows past n_q * G are never
//    read), a tile is 128 kept rows (the N of S = Q K^T and the K of O = P V);
//  - K and V rows are gathered with 16-byte cp.async into shared memory in
//    the 128-byte-swizzled layout the tensor core reads (K-major for K, the
//    same bytes read MN-major for V);
//  - the scaled rotated queries are split into three bf16 terms (hi + mid +
//    lo) and the probabilities into two (hi + lo), one MMA per term, so the
//    logits keep about 24 significant bits of the queries and O about 16 of
//    the probabilities (bf16 alone keeps 8);
//  - one thread issues tcgen05.mma; completion is signalled by
//    tcgen05.commit on an mbarrier (bounded wait); each query row's thread
//    reads its S row from TMEM (tcgen05.ld), runs the online softmax in base 2
//    and keeps its O row in registers;
//  - splits of a row write (m, l, o) partials; the row's last CTA (atomic
//    ticket, no waiting) merges them in a fixed order.
#pragma once

#include "fasa_device.cuh"

namespace fasa {

constexpr int kTcThreads = 128;   // warp w reads TMEM lanes 32w .. 32w + 31
constexpr int kTcTile = 128;      // kept rows per tile
constexpr int kTcMaxRows = 64;    // query rows per KV head (n_q * G)
constexpr int kTcMaxTok = 16;     // query tokens per sequence
constexpr int kTcPartStride = kTcMaxRows * kD + 2 * kTcMaxRows;  // m[64], l[64], o[64][128]
constexpr int kTcMaxSplits = 64;
constexpr uint32_t kTcCols = 256;  // TMEM columns: S [0, 128), the tile's P V [128, 256)

struct TcParams {
  const __nv_bfloat16* k;  // [rows][max_len][128]
  const __nv_bfloat16* v;
  const int32_t* idx;      // [rows][n_keep], ascending kept slots
  const __nv_bfloat16* q;  // [B][n_q][Hq][128] pre-RoPE (or rotated)
  __nv_bfloat16* out;      // [B][n_q][Hq][128]
  float* part;             // [rows][splits][kTcPartStride]
  uint32_t* counter;       // [rows], zero before the launch; left zero
  int64_t max_len;
  int32_t len;             // kept slots lie in [0, len)
  int32_t n_keep;
  int32_t slice;           // list positions per CTA, a multiple of kTcTile
  int32_t splits;
  int32_t group;
  int32_t n_q;
  int32_t n_kv_heads;
  int32_t q_pos0;          // token j at position q_pos0 + j
  int32_t q_prerot;        // 1: queries already rotated, no position mask
  double theta[kNFC];
};

// Shared memory: five K-major tile pairs of RQ rows (Q hi, Q mid, Q lo, P hi, P lo),
// the K and V tiles (128 rows each), kept slots, mbarrier, TMEM address, the
// tokens' rotation tables; plus 1 KB to align the tiles to 1024 bytes.
__host__ __device__ constexpr int tc_rows_pad(int mq) { return (mq + 7) / 8 * 8; }
__host__ __device__ constexpr int tc_smem_bytes(int mq, int n_q) {
  return 5 * 2 * tc_rows_pad(mq) * 128 + 2 * 32768 + kTcTile * 4 + 16 + n_q * 2 * kNFC * 8 + 1024;
}

// Byte offset of 16-byte chunk c (0 .. 15) of row r in a tile pair of R rows
// stored for the 128-byte swizzle: dims 0-63 then 64-127, 8-row atoms of
// 1024 bytes, chunk index xor (row mod 8).
__device__ __forceinline__ uint32_t tc_sw(int r, int c, int R) {
  return (uint32_t)((c >> 3) * R * 128 + (r >> 3) * 1024 + (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Shared-memory matrix descriptor (tcgen05): start, leading and stride byte
// offsets, descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: bf16 A and B, f32 accumulator,
// M = 128, N = 128, A K-major, B K-major (b_mn 0) or MN-major (1).
__host__ __device__ constexpr uint32_t tc_idesc(uint32_t b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
}
__device__ __forceinline__ void tc_alloc(uint32_t* dst, uint32_t ncols) {  // one warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t ncols) {  // one warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// 32 consecutive TMEM columns of the warp's 32 lanes (one per thread).
__device__ __forceinline__ void tc_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t tc_pack(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// hi + mid + lo split of 8 floats into three 16-byte bf16 chunks (each
// difference is exact in float32): about 24 significant bits.
__device__ __forceinline__ void tc_split8x3(const float* x, uint4& hi, uint4& mid, uint4& lo) {
  float r[8], t[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    r[i] = x[i] - __bfloat162float(__float2bfloat16_rn(x[i]));
    t[i] = r[i] - __bfloat162float(__float2bfloat16_rn(r[i]));
  }
  hi = make_uint4(tc_pack(x[0], x[1]), tc_pack(x[2], x[3]), tc_pack(x[4], x[5]), tc_pack(x[6], x[7]));
  mid = make_uint4(tc_pack(r[0], r[1]), tc_pack(r[2], r[3]), tc_pack(r[4], r[5]), tc_pack(r[6], r[7]));
  lo = make_uint4(tc_pack(t[0], t[1]), tc_pack(t[2], t[3]), tc_pack(t[4], t[5]), tc_pack(t[6], t[7]));
}

// hi + lo split of 8 floats into two 16-byte bf16 chunks.
__device__ __forceinline__ void tc_split8(const float* x, uint4& hi, uint4& lo) {
  float r[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) r[i] = x[i] - __bfloat162float(__float2bfloat16_rn(x[i]));
  hi = make_uint4(tc_pack(x[0], x[1]), tc_pack(x[2], x[3]), tc_pack(x[4], x[5]), tc_pack(x[6], x[7]));
  lo = make_uint4(tc_pack(r[0], r[1]), tc_pack(r[2], r[3]), tc_pack(r[4], r[5]), tc_pack(r[6], r[7]));
}

__global__ void __launch_bounds__(kTcThreads, 1) attend_tc_kernel(const TcParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int split = blockIdx.x, row = blockIdx.y;
  const int G = p.group, MQ = p.n_q * G, RQ = tc_rows_pad(MQ);
  const uint32_t pair = 2u * RQ * 128u;  // bytes of one Q / P tile pair
  // the Q and P tile pairs come first: an MMA reads all 128 rows of a pair
  // (rows past RQ only feed accumulator rows that are never read), so each
  // pair's reads stay inside the allocation, within the K and V tiles
  unsigned char* qhi = smem;
  unsigned char* qmd = qhi + pair;
  unsigned char* qlo = qmd + pair;
  unsigned char* phi = qlo + pair;
  unsigned char* plo = phi + pair;
  unsigned char* ks = plo + pair;  // K tile pair, 128 rows (1024-aligned: pair is a multiple of 1024)
  unsigned char* vs = ks + 32768;
  int* tok_s = reinterpret_cast<int*>(vs + 32768);
  uint64_t* bar = reinterpret_cast<uint64_t*>(tok_s + kTcTile);
  uint32_t* tbase_s = reinterpret_cast<uint32_t*>(bar + 1);
  double* cs = reinterpret_cast<double*>(tbase_s + 2);  // [n_q][cos 64 | sin 64]

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tc_alloc(tbase_s, kTcCols);
  for (int e = tid; e < p.n_q * kNFC; e += kTcThreads) {
    const int j = e / kNFC, i = e % kNFC;
    double sn = 0.0, cn = 1.0;
    if (!p.q_prerot) sincos((double)(p.q_pos0 + j) * p.theta[i], &sn, &cn);
    cs[j * 2 * kNFC + i] = cn;
    cs[j * 2 * kNFC + kNFC + i] = sn;
  }
  grid_dependency_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tbase_s;

  const int b = row / p.n_kv_heads, g = row % p.n_kv_heads;
  const int hq = p.n_kv_heads * G;
  // the query rows: row r = token j, head h of the group; staged raw in the
  // P hi tiles (free until the first softmax), then rotated (float64),
  // scaled by log2(e) / sqrt(128) and split into bf16 hi + lo, 8 dims per
  // thread and step
  {
    uint4* qst = reinterpret_cast<uint4*>(phi);  // [MQ][16] raw chunks
    for (int c = tid; c < MQ * 16; c += kTcThreads) {
      const int r = c >> 4, j = r / G, h = r % G;
      qst[c] = __ldg(reinterpret_cast<const uint4*>(p.q + (((int64_t)b * p.n_q + j) * hq + g * G + h) * kD) +
                     (c & 15));
    }
    __syncthreads();
    const __nv_bfloat16* qs = reinterpret_cast<const __nv_bfloat16*>(phi);
    const double qscale = 1.4426950408889634 / 11.313708498984761;
    for (int c = tid; c < MQ * 16; c += kTcThreads) {
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
      *reinterpret_cast<uint4*>(qhi + tc_sw(r, ch, RQ)) = hi;
      *reinterpret_cast<uint4*>(qmd + tc_sw(r, ch, RQ)) = md;
      *reinterpret_cast<uint4*>(qlo + tc_sw(r, ch, RQ)) = lo;
    }
  }

  const int r_beg = split * p.slice, r_end = min(p.n_keep, r_beg + p.slice);
  const int32_t* idx = p.idx + (int64_t)row * p.n_keep;
  const __nv_bfloat16* kb = p.k + (int64_t)row * p.max_len * kD;
  const __nv_bfloat16* vb = p.v + (int64_t)row * p.max_len * kD;
  const bool soft = warp * 32 < MQ;  // warps holding query rows (whole warps: tcgen05.ld is warp-wide)
  const int jq = tid / G;
  // visible columns: kept slot <= lim (masked entries hold kTcMasked)
  constexpr int kTcMasked = 0x7FFFFFFF;
  const int lim = p.q_prerot ? kTcMasked - 1 : min(p.q_pos0 + jq, kTcMasked - 1);
  const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
  float m_run = -INFINITY, l_run = 0.0f;
  float o[kD];
#pragma unroll
  for (int d = 0; d < kD; ++d) o[d] = 0.0f;
  uint32_t phase = 0;
  bool failed = false;

  for (int jb = r_beg; jb < r_end && !failed; jb += kTcTile) {
    {  // gather the tile's K and V rows (masked entries read row 0)
      const int j = jb + tid;
      int t = -1;
      if (j < r_end) {
        t = __ldg(idx + j);
        if (t < 0 || t >= p.len) {
          flag_status(FASA_ERR_BAD_INDEX);
          t = -1;
        }
      }
      tok_s[tid] = t < 0 ? kTcMasked : t;
      const uint4* kr = reinterpret_cast<const uint4*>(kb + (int64_t)(t < 0 ? 0 : t) * kD);
      const uint4* vr = reinterpret_cast<const uint4*>(vb + (int64_t)(t < 0 ? 0 : t) * kD);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        cp_async16(ks + tc_sw(tid, c, kTcTile), kr + c);
        cp_async16(vs + tc_sw(tid, c, kTcTile), vr + c);
      }
      cp_async_commit();
      cp_async_wait<0>();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // S = (Q hi + Q mid + Q lo) K^T
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int s8 = 0; s8 < 8; ++s8) {
        const uint32_t qo = (s8 >> 2) * RQ * 128 + (s8 & 3) * 32;
        const uint64_t bd = tc_desc(smem_u32(ks) + (s8 >> 2) * kTcTile * 128 + (s8 & 3) * 32, 16, 1024);
        tc_mma(tbase, tc_desc(smem_u32(qhi) + qo, 16, 1024), bd, tc_idesc(0), s8 > 0);
        tc_mma(tbase, tc_desc(smem_u32(qmd) + qo, 16, 1024), bd, tc_idesc(0), 1);
        tc_mma(tbase, tc_desc(smem_u32(qlo) + qo, 16, 1024), bd, tc_idesc(0), 1);
      }
      tc_commit(bar);
    }
    failed = __syncthreads_or(!mbar_wait(bar, phase));
    phase ^= 1u;
    if (failed) break;
    tc_fence_after();
    // online softmax of the row's 128 logits; P hi / lo to shared memory
    float alpha = 1.0f;
    if (soft) {
      float cmax = -INFINITY;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float s[32];
        tc_ld32(tl + ch * 32, s);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (tok_s[ch * 32 + i] <= lim) cmax = fmaxf(cmax, s[i]);
        }
      }
      const float m_new = fmaxf(m_run, cmax);
      alpha = (m_new == -INFINITY) ? 1.0f : exp2f(m_run - m_new);
      float lsum = 0.0f;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float s[32];
        tc_ld32(tl + ch * 32, s);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = (tok_s[ch * 32 + i] <= lim && m_new != -INFINITY) ? exp2f(s[i] - m_new) : 0.0f;
          lsum += s[i];
        }
        if (tid < MQ) {
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            uint4 hi, lo;
            tc_split8(s + q8 * 8, hi, lo);
            *reinterpret_cast<uint4*>(phi + tc_sw(tid, ch * 4 + q8, RQ)) = hi;
            *reinterpret_cast<uint4*>(plo + tc_sw(tid, ch * 4 + q8, RQ)) = lo;
          }
        }
      }
      l_run = l_run * alpha + lsum;
      m_run = m_new;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // the tile's O = (P hi + P lo) V
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int s8 = 0; s8 < 8; ++s8) {
        const uint32_t po = (s8 >> 2) * RQ * 128 + (s8 & 3) * 32;
        const uint64_t bd = tc_desc(smem_u32(vs) + s8 * 2048, kTcTile * 128, 1024);
        tc_mma(tbase + 128, tc_desc(smem_u32(phi) + po, 16, 1024), bd, tc_idesc(1), s8 > 0);
        tc_mma(tbase + 128, tc_desc(smem_u32(plo) + po, 16, 1024), bd, tc_idesc(1), 1);
      }
      tc_commit(bar);
    }
    failed = __syncthreads_or(!mbar_wait(bar, phase));
    phase ^= 1u;
    if (failed) break;
    tc_fence_after();
    if (soft) {
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float dv[32];
        tc_ld32(tl + 128 + ch * 32, dv);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[ch * 32 + i] = __fmaf_rn(o[ch * 32 + i], alpha, dv[i]);
      }
    }
    tc_fence_before();
    __syncthreads();  // TMEM columns and the tiles are free for the next tile
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tc_dealloc(tbase, kTcCols);
  if (failed) return;

  // this split's partial, or the output when the row has one split
  const int hrow = g * G;  // first query head of the group
  auto out_at = [&](int r, int d) -> __nv_bfloat16* {
    return p.out + (((int64_t)b * p.n_q + r / G) * hq + hrow + r % G) * kD + d;
  };
  if (p.splits == 1) {
    if (tid < MQ) {
      const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
#pragma unroll
      for (int d = 0; d < kD; d += 2)
        *reinterpret_cast<__nv_bfloat162*>(out_at(tid, d)) = __floats2bfloat162_rn(o[d] * inv, o[d + 1] * inv);
    }
    return;
  }
  float* pp = p.part + ((int64_t)row * p.splits + split) * kTcPartStride;
  if (tid < MQ) {
    pp[tid] = m_run;
    pp[kTcMaxRows + tid] = l_run;
    float4* po = reinterpret_cast<float4*>(pp + 2 * kTcMaxRows + tid * kD);
#pragma unroll
    for (int d = 0; d < kD; d += 4) po[d / 4] = make_float4(o[d], o[d + 1], o[d + 2], o[d + 3]);
  }
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(p.counter + row, 1u) == (uint32_t)(p.splits - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // merge in split order: weights w[s][r] = 2^(m_s - M), denominators; then
  // each thread sums its float4 groups of o over the splits (the loads of one
  // split are independent of each other, so they overlap)
  const float* rp = p.part + (int64_t)row * p.splits * kTcPartStride;
  float* w = reinterpret_cast<float*>(ks);  // [splits][64]
  float* den = w + p.splits * kTcMaxRows;   // [64]
  if (tid < MQ) {
    float M = -INFINITY;
#pragma unroll 8
    for (int s = 0; s < p.splits; ++s) M = fmaxf(M, __ldcg(rp + s * kTcPartStride + tid));
    float dn = 0.0f;
#pragma unroll 8
    for (int s = 0; s < p.splits; ++s) {
      const float ms = __ldcg(rp + s * kTcPartStride + tid);
      const float ws = (ms == -INFINITY || M == -INFINITY) ? 0.0f : exp2f(ms - M);
      w[s * kTcMaxRows + tid] = ws;
      dn += ws * __ldcg(rp + s * kTcPartStride + kTcMaxRows + tid);
    }
    den[tid] = dn;
  }
  __syncthreads();
  constexpr int kGroups = kTcMaxRows * kD / 4 / kTcThreads;  // float4 groups per thread at most
  const int n4 = MQ * kD / 4;
  float4 acc[kGroups];
#pragma unroll
  for (int i = 0; i < kGroups; ++i) acc[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (int s = 0; s < p.splits; ++s) {
    const float4* src = reinterpret_cast<const float4*>(rp + s * kTcPartStride + 2 * kTcMaxRows);
#pragma unroll
    for (int i = 0; i < kGroups; ++i) {
      const int f = tid + i * kTcThreads;
      if (f < n4) {
        const float4 v = __ldcg(src + f);
        const float ws = w[s * kTcMaxRows + f / (kD / 4)];
        acc[i].x = __fmaf_rn(ws, v.x, acc[i].x);
        acc[i].y = __fmaf_rn(ws, v.y, acc[i].y);
        acc[i].z = __fmaf_rn(ws, v.z, acc[i].z);
        acc[i].w = __fmaf_rn(ws, v.w, acc[i].w);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kGroups; ++i) {
    const int f = tid + i * kTcThreads;
    if (f < n4) {
      const int r = f / (kD / 4), d = (f % (kD / 4)) * 4;
      const float inv = den[r] > 0.0f ? 1.0f / den[r] : 0.0f;
      __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(out_at(r, d));
      o2[0] = __floats2bfloat162_rn(acc[i].x * inv, acc[i].y * inv);
      o2[1] = __floats2bfloat162_rn(acc[i].z * inv, acc[i].w * inv);
    }
  }
  if (tid == 0) p.counter[row] = 0u;
}

}  // namespace fasa
