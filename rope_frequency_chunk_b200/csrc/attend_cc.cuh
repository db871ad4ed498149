// Focused attention on CUDA cores (bf16 caches): flash decode in float32.
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2, FAC bullets): full softmax attention of each query head of a KV-head
// group over exactly the kept rows, each row at its original position (keys
// were rotated at append time). The dense comparison decode is the same
// attention over every row ([tech §4] "Resultados Experimentais", FKV).
//
// Decode attention has G (<= 16) query rows per KV head, so QK^T and PV are
// matrix-vector products at about G flops per byte: the path is bound by
// HBM, and float32 fma on CUDA cores keeps up with it at these group sizes.
//
// Warp step: 8 rows. Lane l owns head dims 4l .. 4l+3: it loads those 8
// bytes of each K and V row, forms the partial dot products of its 4 dims
// with every head's query (an fma chain), and a reduce-scatter butterfly
// over the 32 lanes (5 rounds of shuffles, each halving the values a lane
// holds) leaves lane l with the full logit of (row l/4, head 4g + l%4) for
// head group g. Each lane takes the rows and heads in an order permuted by
// its own lane bits, so every round keeps the lower half of the registers
// and sends the upper half (no selects). Online softmax in
// base 2 (the 1/sqrt(128) and log2(e) scale is folded into the queries):
// per-head chunk maxima and sums by shuffles among the lanes of one head,
// running (m, l) in the warp's shared-memory scratch, probabilities
// broadcast through it; o[h][4l..4l+3] += p * v in registers.
//
// Error: a logit is a float32 sum of 128 products (query rounded once from
// float64; keys exact) along a 4-fma chain and a 5-level tree, so its error
// is below 10 * 2^-24 * sum_d |q_d k_d|; probabilities and the output
// accumulate in float32.
#pragma once

#include "fasa_device.cuh"

namespace fasa {

constexpr int kCcStep = 8;  // rows per warp step

// Per-warp shared-memory scratch (floats): p[8][MG], then running max, sum
// and the last rescale factor per head.
__host__ __device__ constexpr int cc_warp_scratch(int MG) { return (kCcStep + 3) * MG; }

// Attention queries of one KV-head group, [MG][128] floats: query h rotated
// at the query position and scaled by log2(e)/sqrt(128), in float64, rounded
// to float32; rows h >= G are zero. qraw: the group's G pre-RoPE rows.
template <typename T>
__device__ __forceinline__ void cc_queries(const T* qraw, int G, int MG, const double* cosv, const double* sinv,
                                           float* qs, int tid, int nthreads) {
  const double qscale = 1.4426950408889634 / 11.313708498984761;
  for (int e = tid; e < MG * kD; e += nthreads) {
    const int h = e / kD, dd = e % kD, i = dd & (kNFC - 1);
    float v = 0.0f;
    if (h < G) {
      const double x = to_float(qraw[h * kD + i]);
      const double y = to_float(qraw[h * kD + i + kNFC]);
      const double c = cosv[i], s = sinv[i];
      const double r = (dd < kNFC) ? __dsub_rn(__dmul_rn(x, c), __dmul_rn(y, s))
                                   : __dadd_rn(__dmul_rn(y, c), __dmul_rn(x, s));
      v = (float)(r * qscale);
    }
    qs[e] = v;
  }
}

// A warp's running attention state: o for the lane's 4 dims of every head
// (the running max and sum live in the warp's scratch).
template <int MG>
struct CcAcc {
  float o[MG][4];
};

template <int MG>
__device__ __forceinline__ void cc_init(CcAcc<MG>& a, float* ws, int lane) {
#pragma unroll
  for (int h = 0; h < MG; ++h)
#pragma unroll
    for (int d = 0; d < 4; ++d) a.o[h][d] = 0.0f;
  float* wm = ws + kCcStep * MG;
  for (int h = lane; h < MG; h += 32) {
    wm[h] = -INFINITY;
    wm[MG + h] = 0.0f;
  }
  __syncwarp();
}

__device__ __forceinline__ void cc_bf16x4(const uint2& u, float (&f)[4]) {
  f[0] = __uint_as_float(u.x << 16);
  f[1] = __uint_as_float(u.x & 0xFFFF0000u);
  f[2] = __uint_as_float(u.y << 16);
  f[3] = __uint_as_float(u.y & 0xFFFF0000u);
}

// One step of 8 rows: kk[r] is the lane's 8 bytes of K row r, and vs the
// 8 V rows in shared memory ([8][128] bf16, the lane reads its own 8 bytes
// of each); bit r of `valid` says whether row r takes part. qs: [MG][128]
// queries; ws: the warp's scratch (cc_warp_scratch floats).
template <int MG>
__device__ __forceinline__ void cc_step8(CcAcc<MG>& a, const uint2 (&kk)[kCcStep], const __nv_bfloat16* vs,
                                         unsigned valid, const float* qs, float* ws, int lane) {
  constexpr int NG = MG / 4;
  float* wp = ws;                    // p[8][MG]
  float* wm = ws + kCcStep * MG;     // running max [MG]
  float* wl = wm + MG;               // running sum [MG]
  float* wsc = wl + MG;              // rescale of this step [MG]
  // kk[r'] holds row r' ^ (lane >> 2) (cc_warp_rows loads the rows in that
  // lane-permuted order), and register r'*4 + h' takes head h' ^ (lane & 3):
  // register p then holds the partial of logical (row, head) index p ^ lane,
  // so each butterfly round keeps the lower half of the registers and sends
  // the upper half, with no selects
  float kf[kCcStep][4];
#pragma unroll
  for (int r = 0; r < kCcStep; ++r) cc_bf16x4(kk[r], kf[r]);
  const int r_me = lane >> 2;           // the row and head (within a group) whose logit this lane ends with
  const bool row_ok = (valid >> r_me) & 1u;
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    float v[32];  // register p: logical index (p ^ lane) = row * 4 + head
#pragma unroll
    for (int hh = 0; hh < 4; ++hh) {
      const float4 q4 = *reinterpret_cast<const float4*>(qs + (g * 4 + (hh ^ (lane & 3))) * kD + 4 * lane);
#pragma unroll
      for (int r = 0; r < kCcStep; ++r)
        v[r * 4 + hh] = __fmaf_rn(q4.w, kf[r][3], __fmaf_rn(q4.z, kf[r][2], __fmaf_rn(q4.y, kf[r][1],
                                                                                    __fmul_rn(q4.x, kf[r][0]))));
    }
    // reduce-scatter: the round with offset o adds the partner's upper half
    // onto the lower half (the partner's registers i + o hold the logical
    // indices this lane keeps at registers i)
#pragma unroll
    for (int s = 0; s < 5; ++s) {
      const int off = 16 >> s;
#pragma unroll
      for (int i = 0; i < off; ++i) v[i] = __fadd_rn(v[i], __shfl_xor_sync(0xFFFFFFFFu, v[i + off], off));
    }
    const int h = g * 4 + (lane & 3);
    const float z = row_ok ? v[0] : -INFINITY;
    float cm = z;
    cm = fmaxf(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, 4));
    cm = fmaxf(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, 8));
    cm = fmaxf(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, 16));
    const float mold = wm[h];
    const float mnew = fmaxf(mold, cm);
    const float p = (z == -INFINITY) ? 0.0f : exp2f(z - mnew);
    float cs = p;
    cs += __shfl_xor_sync(0xFFFFFFFFu, cs, 4);
    cs += __shfl_xor_sync(0xFFFFFFFFu, cs, 8);
    cs += __shfl_xor_sync(0xFFFFFFFFu, cs, 16);
    const float sc = (mold == -INFINITY) ? 0.0f : exp2f(mold - mnew);
    wp[r_me * MG + h] = p;
    __syncwarp();
    if (lane < 4) {
      wm[h] = mnew;
      wl[h] = wl[h] * sc + cs;
      wsc[h] = sc;
    }
  }
  __syncwarp();
  // rescale, then o += p v
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const float4 s4 = *reinterpret_cast<const float4*>(wsc + g * 4);
    const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
    for (int hh = 0; hh < 4; ++hh)
#pragma unroll
      for (int d = 0; d < 4; ++d) a.o[g * 4 + hh][d] *= sv[hh];
  }
#pragma unroll
  for (int r = 0; r < kCcStep; ++r) {
    float vf[4];
    cc_bf16x4(*reinterpret_cast<const uint2*>(vs + r * kD + 4 * lane), vf);
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const float4 p4 = *reinterpret_cast<const float4*>(wp + r * MG + g * 4);
      const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
      for (int hh = 0; hh < 4; ++hh)
#pragma unroll
        for (int d = 0; d < 4; ++d) a.o[g * 4 + hh][d] = __fmaf_rn(pv[hh], vf[d], a.o[g * 4 + hh][d]);
    }
  }
  __syncwarp();
}

// A warp attends rows j0 .. j1-1 of a list: token(j) gives the cache slot
// of list position j, or -1 for a position to skip. kb, vb: the row's K and
// V planes [max_len][128]. K rows go to registers, V rows to the warp's
// shared-memory buffer vbuf ([2][8][128] bf16) with 8-byte cp.async; the
// next step's rows are loaded before the current step is computed.
template <int MG, typename Tok>
__device__ __forceinline__ void cc_warp_rows(CcAcc<MG>& a, const __nv_bfloat16* kb, const __nv_bfloat16* vb,
                                             Tok token, int j0, int j1, const float* qs, float* ws,
                                             __nv_bfloat16* vbuf, int lane) {
  auto load = [&](uint2 (&kk)[kCcStep], __nv_bfloat16* vs, unsigned& valid, int jb) {
    const int mine = (lane < kCcStep && jb + lane < j1) ? token(jb + lane) : -1;
    valid = __ballot_sync(0xFFFFFFFFu, mine >= 0) & 0xFFu;
#pragma unroll
    for (int r = 0; r < kCcStep; ++r) {
      int t = __shfl_sync(0xFFFFFFFFu, mine, r);
      int tk = __shfl_sync(0xFFFFFFFFu, mine, r ^ (lane >> 2));  // K rows in the lane-permuted order
      if (t < 0) t = 0;  // masked out; row 0 is a valid address
      if (tk < 0) tk = 0;
      kk[r] = __ldcg(reinterpret_cast<const uint2*>(kb + (int64_t)tk * kD) + lane);
      asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(vs + r * kD + 4 * lane)),
                   "l"(vb + (int64_t)t * kD + 4 * lane)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  if (j0 >= j1) return;
  uint2 k0[kCcStep], k1[kCcStep];
  unsigned m0, m1;
  __nv_bfloat16* vs0 = vbuf;
  __nv_bfloat16* vs1 = vbuf + kCcStep * kD;
  load(k0, vs0, m0, j0);
  for (int jb = j0; jb < j1; jb += 2 * kCcStep) {
    const bool more = jb + kCcStep < j1;
    if (more) {
      load(k1, vs1, m1, jb + kCcStep);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    cc_step8<MG>(a, k0, vs0, m0, qs, ws, lane);
    if (!more) break;
    const bool more2 = jb + 2 * kCcStep < j1;
    if (more2) {
      load(k0, vs0, m0, jb + 2 * kCcStep);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    cc_step8<MG>(a, k1, vs1, m1, qs, ws, lane);
  }
}

// Merges the nw warps' states of a CTA in shared memory. Warp w writes its
// o to mo[w][MG][128] and its (m, l) are in its scratch ws0 + w * stride;
// afterwards thread tid < MG*128 ... handles output element e = tid (and
// e + nthreads ...): returns nothing, calls emit(h, d, m, l, o) once per
// element (head h, dim d) with the merged state. Must be called by every
// thread of the CTA.
template <int MG, typename Emit>
__device__ __forceinline__ void cc_block_merge(const CcAcc<MG>& a, float* mo, const float* ws0, int ws_stride, int nw,
                                               Emit emit) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthreads = nw * 32;
#pragma unroll
  for (int h = 0; h < MG; ++h)
    *reinterpret_cast<float4*>(mo + (warp * MG + h) * kD + 4 * lane) =
        make_float4(a.o[h][0], a.o[h][1], a.o[h][2], a.o[h][3]);
  __syncthreads();
  for (int e = tid; e < MG * kD; e += nthreads) {
    const int h = e / kD, d = e % kD;
    float M = -INFINITY;
    for (int w = 0; w < nw; ++w) M = fmaxf(M, ws0[w * ws_stride + kCcStep * MG + h]);
    float L = 0.0f, O = 0.0f;
    for (int w = 0; w < nw; ++w) {
      const float mw = ws0[w * ws_stride + kCcStep * MG + h];
      const float f = (mw == -INFINITY) ? 0.0f : exp2f(mw - M);
      L += f * ws0[w * ws_stride + kCcStep * MG + MG + h];
      O += f * mo[(w * MG + h) * kD + d];
    }
    emit(h, d, M, L, O);
  }
}

}  // namespace fasa

namespace fasa {

constexpr int kCcWarps = 8;
constexpr int kCcThreads = kCcWarps * 32;
constexpr int kCcPartStride = 16 * kD + 32;  // floats per split partial: m[16], l[16], o[16][128]

struct CcParams {
  const __nv_bfloat16* k;   // [rows][max_len][128]
  const __nv_bfloat16* v;
  const int32_t* idx;       // [rows][n_keep] kept rows, or null: rows 0 .. n_keep-1 (dense)
  const __nv_bfloat16* q;   // [B][Hq][128], pre-RoPE
  __nv_bfloat16* out;       // [B][Hq][128]
  float* part;              // [rows][splits][kCcPartStride] split partials (attend_merge_kernel merges them)
  int64_t max_len;
  int32_t len;              // kept indices must lie in [0, len)
  int32_t n_keep;
  int32_t slice;            // list positions per CTA, a multiple of 8 * kCcWarps
  int32_t splits;
  int32_t group;
  // per-sequence lengths (fasa_decode_varlen), or null: len and n_keep for
  // every row (then the upper bounds, n_keep the kept lists' row stride)
  const int32_t* seq_len;   // [B]
  const int32_t* row_keep;  // [rows] each row's kept count
  int32_t n_kv_heads;
  int32_t q_prerot;         // varlen: 1 if the queries are already rotated
  PageMap pm;               // paged pools (pm.table set), else [rows][max_len] planes
  double cosv[kNFC];        // cos / sin of q_pos * theta_i; varlen: theta_i in cosv
  double sinv[kNFC];
};

// Shared memory of attend_cc_kernel: group queries (raw), queries (scaled
// float32), warp scratch, warp partials.
__host__ __device__ constexpr int cc_smem_bytes(int MG) {
  return FASA_MAX_GROUP * kD * 2 + MG * kD * 4 + kCcWarps * cc_warp_scratch(MG) * 4 + kCcWarps * MG * kD * 4 +
         kCcWarps * 2 * kCcStep * kD * 2 + 2 * kNFC * 8;
}
constexpr int kCcMaxSplits = 85;  // splits per row at most (the merge kernel holds a quarter of them in registers)

// Prologue of the split-K attention kernels, in two parts called by all NT
// threads. cc_row_begin: the angle tables to cs (before the launch-
// dependency wait, so their constant-bank misses overlap it), then the
// row's length and kept count. cc_row_queries: the group's G pre-RoPE
// queries to qraw and the rotated, scaled queries qs [MG][128]
// (cc_queries; rows h >= G zero); varlen rows rotate at their own length
// with theta_i from the table, unless the queries come rotated. A kernel may
// start its first row loads between the two.
template <int NT>
__device__ __forceinline__ void cc_row_begin(const CcParams& p, int row, double* cs, int& len, int& n_keep) {
  const int tid = threadIdx.x;
  if (tid < kNFC) {
    cs[tid] = p.cosv[tid];
    cs[kNFC + tid] = p.sinv[tid];
  } else if (tid < kNFC + 2 * p.group) {  // the group's queries to L2 (a hint)
    prefetch_line_l2(p.q + (int64_t)row * p.group * kD + (tid - kNFC) * 64);
  }
  grid_dependency_wait();
  len = p.len;
  n_keep = p.n_keep;
  if (p.seq_len) {
    len = min(max(__ldg(p.seq_len + row / p.n_kv_heads), 1), p.len);  // range flagged by the fused kernel
    n_keep = min(max(p.row_keep[row], 0), p.n_keep);
  }
}

// kStaged: the caller has copied the queries to qraw (cc_stage_queries) and
// waited for that copy; otherwise they are loaded here.
template <int MG, int NT, bool kStaged = false>
__device__ __forceinline__ void cc_row_queries(const CcParams& p, int row, int len, __nv_bfloat16* qraw, double* cs,
                                               float* qs) {
  const int tid = threadIdx.x;
  const int G = p.group;
  if (!kStaged) {
    const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + (int64_t)row * G * kD);
    for (int c = tid; c < G * kD / 8; c += NT) reinterpret_cast<uint4*>(qraw)[c] = __ldg(qsrc + c);
  }
  if (p.seq_len && tid < kNFC) {  // the query of sequence b sits at position len
    double sn = 0.0, cn = 1.0;
    if (!p.q_prerot) sincos((double)len * cs[tid], &sn, &cn);
    cs[tid] = cn;
    cs[kNFC + tid] = sn;
  }
  __syncthreads();
  cc_queries(qraw, G, MG, cs, cs + kNFC, qs, tid, NT);
  __syncthreads();
}

// The group's G query rows to qraw with 16-byte cp.async, committed as one
// group (so that they can be issued ahead of the row loads and waited for
// on their own).
template <int NT>
__device__ __forceinline__ void cc_stage_queries(const CcParams& p, int row, __nv_bfloat16* qraw) {
  const int G = p.group;
  const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + (int64_t)row * G * kD);
  for (int c = threadIdx.x; c < G * kD / 8; c += NT) cp_async16(reinterpret_cast<uint4*>(qraw) + c, qsrc + c);
  cp_async_commit();
}

// Split merge of the split-K attention: a kernel of its own, launched after
// the attention (its grid's completion orders the partials before the
// reads, so there is no ticket or fence). Grid (G, rows), kMgThreads
// threads: CTA (h, row) merges head h of the row. Warp w takes a contiguous
// quarter of the splits; lane l owns dims 4l .. 4l+3. Every warp forms the
// head's maximum M over all splits, the weights w_s = 2^(m_s - M) and the
// denominator sum_s w_s l_s by one fixed shuffle tree (so all warps agree
// bit for bit); the warps' weighted sums of o, each in split order, are
// added in warp order and divided by the denominator.
constexpr int kMgThreads = 128;
constexpr int kMgWarps = kMgThreads / 32;
constexpr int kMgMaxPer = (kCcMaxSplits + kMgWarps - 1) / kMgWarps;  // splits per warp, at most

struct MergeParams {
  const float* part;   // [rows][splits][kCcPartStride]: m[16], l[16], o[16][128]
  __nv_bfloat16* out;  // [rows][G][128]
  int32_t splits;      // 2 .. kCcMaxSplits
  int32_t group;
};

__global__ void __launch_bounds__(kMgThreads) attend_merge_kernel(const MergeParams p) {
  __shared__ float ws[kMgWarps][kCcMaxSplits];
  __shared__ float4 acc[kMgWarps][32];
  const int h = blockIdx.x, row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = p.splits;
  const float* rp = p.part + (int64_t)row * S * kCcPartStride;
  grid_dependency_wait();
  const int per = (S + kMgWarps - 1) / kMgWarps;
  const int s0 = min(S, warp * per), n = min(S, s0 + per) - s0;
  // the warp's splits' o for the lane's 4 dims, all loads in flight
  float4 v[kMgMaxPer];
#pragma unroll
  for (int i = 0; i < kMgMaxPer; ++i)
    if (i < n) v[i] = __ldcg(reinterpret_cast<const float4*>(rp + (int64_t)(s0 + i) * kCcPartStride + 32 + h * kD) + lane);
  // m and l of every split, lanes over the splits
  constexpr int kLanesPer = (kCcMaxSplits + 31) / 32;
  float m[kLanesPer], l[kLanesPer];
#pragma unroll
  for (int i = 0; i < kLanesPer; ++i) {
    const int sp = lane + 32 * i;
    m[i] = sp < S ? __ldcg(rp + (int64_t)sp * kCcPartStride + h) : -INFINITY;
    l[i] = sp < S ? __ldcg(rp + (int64_t)sp * kCcPartStride + 16 + h) : 0.0f;
  }
  float M = m[0];
#pragma unroll
  for (int i = 1; i < kLanesPer; ++i) M = fmaxf(M, m[i]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, off));
  float den = 0.0f;
#pragma unroll
  for (int i = 0; i < kLanesPer; ++i) {
    const int sp = lane + 32 * i;
    const float w = (m[i] == -INFINITY || M == -INFINITY) ? 0.0f : exp2f(m[i] - M);
    if (sp < S) ws[warp][sp] = w;
    den += w * l[i];
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) den += __shfl_xor_sync(0xFFFFFFFFu, den, off);
  __syncwarp();
  float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
  for (int i = 0; i < kMgMaxPer; ++i)
    if (i < n) {
      const float w = ws[warp][s0 + i];
      a.x = __fmaf_rn(w, v[i].x, a.x);
      a.y = __fmaf_rn(w, v[i].y, a.y);
      a.z = __fmaf_rn(w, v[i].z, a.z);
      a.w = __fmaf_rn(w, v[i].w, a.w);
    }
  acc[warp][lane] = a;
  __syncthreads();
  if (warp == 0) {
    float4 t = acc[0][lane];
#pragma unroll
    for (int w = 1; w < kMgWarps; ++w) {
      const float4 b = acc[w][lane];
      t.x += b.x;
      t.y += b.y;
      t.z += b.z;
      t.w += b.w;
    }
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(p.out + ((int64_t)row * p.group + h) * kD + 4 * lane);
    o2[0] = __floats2bfloat162_rn(den > 0.0f ? t.x / den : 0.0f, den > 0.0f ? t.y / den : 0.0f);
    o2[1] = __floats2bfloat162_rn(den > 0.0f ? t.z / den : 0.0f, den > 0.0f ? t.w / den : 0.0f);
  }
}

// Split-K attention over a row's kept list (or all its rows): grid
// (splits, rows); CTA `split` takes list positions [split*slice, ...), its
// 8 warps contiguous eighths of them; the warps merge in shared memory and
// the CTA writes its partial (m, l, o), or with one split the output
// (attend_merge_kernel merges the partials).
template <int MG>
__global__ void __launch_bounds__(kCcThreads, MG <= 8 ? 2 : 1) attend_cc_kernel(const CcParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16* qraw = reinterpret_cast<__nv_bfloat16*>(smem);
  float* qs = reinterpret_cast<float*>(smem + FASA_MAX_GROUP * kD * 2);
  float* wsall = qs + MG * kD;
  float* mo = wsall + kCcWarps * cc_warp_scratch(MG);
  __nv_bfloat16* vball = reinterpret_cast<__nv_bfloat16*>(mo + kCcWarps * MG * kD);
  double* cs = reinterpret_cast<double*>(vball + kCcWarps * 2 * kCcStep * kD);
  const int split = blockIdx.x, row = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = p.group;
  int len, n_keep;  // the row's length and kept count
  cc_row_begin<kCcThreads>(p, row, cs, len, n_keep);
  cc_row_queries<MG, kCcThreads>(p, row, len, qraw, cs, qs);
  float* ws = wsall + warp * cc_warp_scratch(MG);
  CcAcc<MG> acc;
  cc_init<MG>(acc, ws, lane);
  const int r_beg = split * p.slice, r_end = min(n_keep, r_beg + p.slice);
  const int per_warp = ((max(0, r_end - r_beg) + kCcWarps * kCcStep - 1) / (kCcWarps * kCcStep)) * kCcStep;
  const int j0 = min(r_end, r_beg + warp * per_warp), j1 = min(r_end, j0 + per_warp);
  const bool paged = p.pm.table != nullptr;
  const int64_t plane = paged ? 0 : (int64_t)row * p.max_len * kD;
  const __nv_bfloat16* kb = p.k + plane;
  const __nv_bfloat16* vb = p.v + plane;
  const int32_t* idx = p.idx ? p.idx + (int64_t)row * p.n_keep : nullptr;
  cc_warp_rows<MG>(acc, kb, vb, [&](int j) -> int {
    const int t = idx ? __ldg(idx + j) : j;
    if (t < 0 || t >= len) {
      flag_status(FASA_ERR_BAD_INDEX);
      return -1;
    }
    return paged ? paged_row(p.pm, row / p.n_kv_heads, row % p.n_kv_heads, t) : t;
  }, j0, j1, qs, ws, vball + warp * 2 * kCcStep * kD, lane);
  grid_dependents_launch();  // the merge (or the next kernel) may start its prologue on SMs this grid frees
  __nv_bfloat16* out = p.out + (int64_t)row * G * kD;
  float* pp = p.part + ((int64_t)row * p.splits + split) * kCcPartStride;
  const bool single = p.splits == 1;
  cc_block_merge<MG>(acc, mo, wsall, cc_warp_scratch(MG), kCcWarps, [&](int h, int d, float M, float L, float O) {
    if (single) {
      if (h < G) out[h * kD + d] = __float2bfloat16_rn(L > 0.0f ? O / L : 0.0f);
    } else {
      pp[32 + h * kD + d] = O;
      if (d == 0) {
        pp[h] = M;
        pp[16 + h] = L;
      }
    }
  });
}

}  // namespace fasa

namespace fasa {

// One CTA of NW warps attends a short kept list (n <= 16 * NW rows) in
// phases, with every load in flight at once: (1) warp w loads the K and V
// rows of its list positions [16w, 16w + 16) into registers (the lane's 8
// bytes of each) and forms their logits (cc_step8's dot products and
// reduce-scatter), stored to zs[j][h]; (2) warp h < G takes the softmax of
// head h over all n logits (max, exp2, sum; zs becomes the probabilities);
// (3) each warp adds p * v over its rows for the lane's 4 dims; (4) the warp
// sums are added in a fixed order and divided by the head's sum.
// Shared memory: zs [16 * NW][MG] floats, mo [NW][MG][128] floats, lsum [16]
// floats, vst [16 * NW][128] bf16 (the V rows, staged with cp.async).
template <int MG, int NW, typename Tok>
__device__ __forceinline__ void cc_block_attend(const __nv_bfloat16* kb, const __nv_bfloat16* vb, Tok token, int n,
                                                int G, const float* qs, float* zs, float* mo, float* lsum,
                                                __nv_bfloat16* vst, __nv_bfloat16* out) {
  constexpr int NG = MG / 4;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int jb = warp * 16;
  uint2 kk[2][kCcStep];
  const int mine = (lane < 16 && jb + lane < n) ? token(jb + lane) : -1;
  const unsigned valid = __ballot_sync(0xFFFFFFFFu, mine >= 0) & 0xFFFFu;
#pragma unroll
  for (int s = 0; s < 2; ++s)
#pragma unroll
    for (int r = 0; r < kCcStep; ++r) {
      int t = __shfl_sync(0xFFFFFFFFu, mine, s * kCcStep + r);
      int tk = __shfl_sync(0xFFFFFFFFu, mine, s * kCcStep + (r ^ (lane >> 2)));  // lane-permuted K rows
      if (t < 0) t = 0;  // masked out; row 0 is a valid address
      if (tk < 0) tk = 0;
      kk[s][r] = __ldcg(reinterpret_cast<const uint2*>(kb + (int64_t)tk * kD) + lane);
      asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(vst + (jb + s * kCcStep + r) * kD + 4 * lane)),
                   "l"(vb + (int64_t)t * kD + 4 * lane)
                   : "memory");
    }
  asm volatile("cp.async.commit_group;" ::: "memory");
  // (1) logits
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    float kf[kCcStep][4];
#pragma unroll
    for (int r = 0; r < kCcStep; ++r) cc_bf16x4(kk[s][r], kf[r]);
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      float v[32];
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        const float4 q4 = *reinterpret_cast<const float4*>(qs + (g * 4 + (hh ^ (lane & 3))) * kD + 4 * lane);
#pragma unroll
        for (int r = 0; r < kCcStep; ++r)
          v[r * 4 + hh] = __fmaf_rn(q4.w, kf[r][3], __fmaf_rn(q4.z, kf[r][2], __fmaf_rn(q4.y, kf[r][1],
                                                                                      __fmul_rn(q4.x, kf[r][0]))));
      }
#pragma unroll
      for (int st = 0; st < 5; ++st) {
        const int off = 16 >> st;
#pragma unroll
        for (int i = 0; i < off; ++i) v[i] = __fadd_rn(v[i], __shfl_xor_sync(0xFFFFFFFFu, v[i + off], off));
      }
      const int r = s * kCcStep + (lane >> 2);
      zs[(jb + r) * MG + g * 4 + (lane & 3)] = ((valid >> r) & 1u) ? v[0] : -INFINITY;
    }
  }
  __syncthreads();
  // (2) softmax of head `warp` over the n rows
  const int nr = 16 * NW;  // every row written in (1); padding rows are -inf and become 0
  if (warp < G) {
    float m = -INFINITY;
    for (int j = lane; j < nr; j += 32) m = fmaxf(m, zs[j * MG + warp]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
    float l = 0.0f;
    for (int j = lane; j < nr; j += 32) {
      const float z = zs[j * MG + warp];
      const float pz = (z == -INFINITY) ? 0.0f : exp2f(z - m);
      zs[j * MG + warp] = pz;
      l += pz;
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, off);
    if (lane == 0) lsum[warp] = l;
  }
  __syncthreads();
  // (3) p * v over the warp's rows
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncwarp();
  float o[MG][4];
#pragma unroll
  for (int h = 0; h < MG; ++h)
#pragma unroll
    for (int d = 0; d < 4; ++d) o[h][d] = 0.0f;
#pragma unroll
  for (int s = 0; s < 2; ++s)
#pragma unroll
    for (int r = 0; r < kCcStep; ++r) {
      const int j = jb + s * kCcStep + r;
      float vf[4];
      cc_bf16x4(*reinterpret_cast<const uint2*>(vst + j * kD + 4 * lane), vf);
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const float4 p4 = *reinterpret_cast<const float4*>(zs + j * MG + g * 4);
        const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
        for (int hh = 0; hh < 4; ++hh)
#pragma unroll
          for (int d = 0; d < 4; ++d) o[g * 4 + hh][d] = __fmaf_rn(pv[hh], vf[d], o[g * 4 + hh][d]);
      }
    }
#pragma unroll
  for (int h = 0; h < MG; ++h)
    *reinterpret_cast<float4*>(mo + (warp * MG + h) * kD + 4 * lane) = make_float4(o[h][0], o[h][1], o[h][2], o[h][3]);
  __syncthreads();
  // (4) warp sums in warp order, divided by the head's sum
  for (int e = tid; e < G * kD; e += NW * 32) {
    const int h = e / kD, d = e % kD;
    float acc = 0.0f;
    for (int w = 0; w < NW; ++w) acc += mo[(w * MG + h) * kD + d];
    const float l = lsum[h];
    out[e] = __float2bfloat16_rn(l > 0.0f ? acc / l : 0.0f);
  }
}

}  // namespace fasa
