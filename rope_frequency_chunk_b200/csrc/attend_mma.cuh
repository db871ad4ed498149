// Focused attention of the fused decode on tensor cores (bf16 caches).
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2, FAC bullets): full softmax attention of each query head over exactly
// the kept rows of its KV head, each row at its original position (keys were
// rotated at append).
//
// Layout of the work: grid = (splits, rows); a CTA takes a contiguous slice
// of the row's kept list and its 4 warps take 16-row chunks of it in turn.
// Each warp gathers its chunks' K and V rows with 16-byte cp.async into its
// own 3-stage ring (no block barriers in the main loop; 16-byte chunks
// XOR-swizzled by row so ldmatrix reads are bank-conflict-free) and runs
// mma.sync.m16n8k16 (bf16 in, float32 accumulate):
//   S[16 x 16] = Q[16 x 128] K^T   (M = the group's query heads padded to 16,
//                                   N = 16 rows, K = head dim)
//   O[16 x 128] += P[16 x 16] V     (K = 16 rows, N = head dim)
// with an online base-2 softmax in registers (the 1/sqrt(128) and log2(e)
// scale folded into Q). Q is split into three bf16 terms (about 24 bits, as
// float32) and P into two (P is in [0, 1] and only weights V); K and V are
// bf16 already and enter exactly. The warps
// of a CTA are merged in shared memory; the CTA writes its partial
// (m, l, o) to the workspace and the row's last CTA (atomic counter) merges
// the splits and writes the bf16 output.
#pragma once

#include "fasa_device.cuh"

namespace fasa {

constexpr int kAttWarps = 4;
constexpr int kAttThreads = kAttWarps * 32;
constexpr int kAttChunk = 16;                          // rows per warp step
constexpr int kAttStages = 3;                          // per-warp ring depth
constexpr int kAttHalf = kAttChunk * kD * 2;           // bytes of 16 bf16 rows (K or V)
constexpr int kAttStageBytes = 2 * kAttHalf;           // K + V
constexpr int kAttPartStride = 16 * kD + 32;           // floats: m[16], l[16], o[16][128]

struct AttParams {
  const __nv_bfloat16* k;   // [rows][max_len][128]
  const __nv_bfloat16* v;
  const int32_t* idx;       // [rows][n_keep] kept rows; null: rows 0 .. n_keep-1
  const __nv_bfloat16* q;   // [B][Hq][128], pre-RoPE
  __nv_bfloat16* out;       // [B][Hq][128]
  float* part;              // [rows][splits][kAttPartStride]
  uint32_t* counter;        // [rows], zero before the launch; the last CTA resets it
  int64_t max_len;
  int32_t len;              // kept indices must lie in [0, len)
  int32_t n_keep;
  int32_t slice;            // rows per CTA, a multiple of kAttChunk
  int32_t splits;
  int32_t group;
  double cosv[kNFC];        // cos / sin of q_pos * theta_i (host, float64)
  double sinv[kNFC];
};

__host__ __device__ constexpr int att_smem_bytes() { return kAttWarps * kAttStages * kAttStageBytes + 16 * kD * 4; }

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

__global__ void __launch_bounds__(kAttThreads) attend_mma_kernel(const AttParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  grid_dependency_wait();
  const int split = blockIdx.x, row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.group;
  float* qs = reinterpret_cast<float*>(smem + kAttWarps * kAttStages * kAttStageBytes);  // [16][128]

  // rotated, pre-scaled queries: q'_h * log2(e) / sqrt(128); rows >= G are
  // zero. The raw rows are first brought into shared memory in one go.
  {
    __nv_bfloat16* qraw = reinterpret_cast<__nv_bfloat16*>(smem);  // ring area, free until the gathers
    const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + ((int64_t)row * G) * kD);
    for (int c = tid; c < G * kD / 8; c += kAttThreads) reinterpret_cast<uint4*>(qraw)[c] = __ldg(qsrc + c);
    __syncthreads();
    const double qscale = 1.4426950408889634 / 11.313708498984761;
    for (int e = tid; e < 16 * kD; e += kAttThreads) {
      const int h = e / kD, d = e % kD, i = d & (kNFC - 1);
      float val = 0.0f;
      if (h < G) {
        const double x = __bfloat162float(qraw[h * kD + i]);
        const double y = __bfloat162float(qraw[h * kD + i + kNFC]);
        const double c = p.cosv[i], s = p.sinv[i];
        val = (float)(((d < kNFC) ? (x * c - y * s) : (y * c + x * s)) * qscale);
      }
      qs[e] = val;
    }
  }
  __syncthreads();
  // A fragments of Q for the 8 k-steps as three bf16 terms (about 24 bits,
  // so large logits keep float32 accuracy)
  uint32_t ah[8][4], am[8][4], al[8][4];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = lane / 4 + (j & 1) * 8;
      const int c = ks * 16 + (lane % 4) * 2 + (j >> 1) * 8;
      const float2 res = split_pack(qs[r * kD + c], qs[r * kD + c + 1], ah[ks][j], am[ks][j]);
      const __nv_bfloat162 mm = *reinterpret_cast<const __nv_bfloat162*>(&am[ks][j]);
      const float2 mf = __bfloat1622float2(mm);
      const __nv_bfloat162 ll = __floats2bfloat162_rn(res.x - mf.x, res.y - mf.y);
      al[ks][j] = *reinterpret_cast<const uint32_t*>(&ll);
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
#pragma unroll
      for (int x = lane; x < kAttChunk * 32; x += 32) {  // 16 rows x (16 K + 16 V) 16-byte parts
        const int r = x / 32, part = x % 32;
        int t = row_of(j0 + r);
        if (t < 0) t = 0;  // masked below
        const __nv_bfloat16* src = (part < 16 ? kb : vb) + (int64_t)t * kD + (part % 16) * 8;
        // 16-byte chunk c of row r is stored at chunk c ^ (r & 7) (bank-conflict-free ldmatrix)
        cp_async16(st + (part < 16 ? 0 : kAttHalf) + r * 256 + (((part % 16) ^ (r & 7)) * 16), src);
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
  for (int ci = 0; ci < mine; ++ci) {
    cp_async_wait<kAttStages - 1>();
    __syncwarp();
    const unsigned char* Ks = ring + (ci % kAttStages) * kAttStageBytes;
    const unsigned char* Vs = Ks + kAttHalf;
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};  // rows 0-7, 8-15 of the chunk
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t b[4];
      ldsm_x4(b, Ks + ((lane / 16) * 8 + lane % 8) * 256 + (((ks * 2 + (lane / 8) % 2) ^ (lane % 8)) * 16));
      mma_16816(s0, al[ks], b[0], b[1]);
      mma_16816(s0, am[ks], b[0], b[1]);
      mma_16816(s0, ah[ks], b[0], b[1]);
      mma_16816(s1, al[ks], b[2], b[3]);
      mma_16816(s1, am[ks], b[2], b[3]);
      mma_16816(s1, ah[ks], b[2], b[3]);
    }
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
  l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 1);
  l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 2);
  l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 1);
  l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 2);

  // merge the CTA's warps through shared memory (the rings are free now)
  __syncthreads();
  float* wm = reinterpret_cast<float*>(smem);   // [warp][16] running max
  float* wl = wm + kAttWarps * 16;              // [warp][16] sums
  float* wo = wl + kAttWarps * 16;              // [warp][16][128]
  if (lane % 4 == 0) {
    wm[warp * 16 + lane / 4] = m0;
    wm[warp * 16 + lane / 4 + 8] = m1;
    wl[warp * 16 + lane / 4] = l0;
    wl[warp * 16 + lane / 4 + 8] = l1;
  }
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    const int d = n * 8 + (lane % 4) * 2;
    wo[(warp * 16 + lane / 4) * kD + d] = o[n][0];
    wo[(warp * 16 + lane / 4) * kD + d + 1] = o[n][1];
    wo[(warp * 16 + lane / 4 + 8) * kD + d] = o[n][2];
    wo[(warp * 16 + lane / 4 + 8) * kD + d + 1] = o[n][3];
  }
  __syncthreads();
  float* pp = p.part + ((int64_t)row * p.splits + split) * kAttPartStride;
  for (int e = tid; e < 16 * kD; e += kAttThreads) {
    const int h = e / kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttWarps; ++w) M = fmaxf(M, wm[w * 16 + h]);
    float acc = 0.0f;
    if (M != -INFINITY)
#pragma unroll
      for (int w = 0; w < kAttWarps; ++w) {
        const float mw = wm[w * 16 + h];
        if (mw != -INFINITY) acc += exp2f(mw - M) * wo[(w * 16 + h) * kD + e % kD];
      }
    pp[32 + e] = acc;
    if (e % kD == 0) {
      float L = 0.0f;
      if (M != -INFINITY)
#pragma unroll
        for (int w = 0; w < kAttWarps; ++w) {
          const float mw = wm[w * 16 + h];
          if (mw != -INFINITY) L += exp2f(mw - M) * wl[w * 16 + h];
        }
      pp[h] = M;
      pp[16 + h] = L;
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
