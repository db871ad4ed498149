// Focused attention with warp-level tensor-core products (bf16 caches,
// G <= 8 query heads per KV head): split-K flash decode.
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2, FAC bullets): softmax attention of each query head of a KV-head group
// over exactly the kept rows (keys rotated at append time); the dense
// comparison decode is the same attention over every row ([tech §4]
// "Resultados Experimentais", FKV).
//
// Decode attention is bound by HBM: a kept row is 512 bytes of K and V for
// G * 128 * 4 flops. What limits a CUDA-core version is instruction issue
// (the dot products, a reduce-scatter of the logits and the p * v fmas: some
// 50 to 170 warp instructions per row). Here one warp takes 16 rows per
// step with mma.sync.m16n8k16 (bf16 in, float32 accumulate), and the M = 16
// rows of each A operand hold two terms of the same 8 heads, so every
// product the decode needs costs 3 MMAs per row and never leaves the
// registers of the thread that owns its head:
//
//   logits  S = Q K^T: A1 = [Q_hi; Q_mid] (rows 0-7 / 8-15 the G heads'
//           high and middle bf16 terms), A2 = [Q_lo; 0], B = K^T from the
//           staged K rows (ldmatrix); head h's logit of key n is
//           (S1[h][n] + S1[8+h][n]) + S2[h][n]. Q_hi + Q_mid + Q_lo is the
//           float32 query exactly, the bf16 x bf16 products are exact, so a
//           logit carries only the float32 accumulation error of three
//           128-term sums (below 3 * 2^-23 * sum_d |q_d k_d|).
//   softmax online in base 2 (the 1/sqrt(128) and log2(e) scale is in the
//           queries), per head: the four lanes of a quad hold one head.
//   output  O = P V: A = [P_hi; P_lo] (p split into two bf16 terms, relative
//           error 2^-17), B = V from the staged V rows (ldmatrix.trans);
//           rows 0-7 and 8-15 of the accumulator are added at the end.
//
// The accumulator fragment of S (row h / 8+h, keys 2q, 2q+1) is exactly the
// A fragment P needs for the 16 keys of the step, so the probabilities go
// from the logits to the second product in registers.
//
// Rows are staged per warp with 16-byte cp.async into a ring of kAmStages
// steps (K and V, 8 KB a step), each row's 16 chunks stored XOR-swizzled by
// the row index so that ldmatrix reads are free of bank conflicts; masked
// rows (past the list, or a bad index) are zero-filled and get p = 0.
#pragma once

#include "attend_cc.cuh"

namespace fasa {

constexpr int kAmStages = 3;                    // steps in flight per warp
constexpr int kAmRows = 16;                     // rows per warp step
constexpr int kAmTile = kAmRows * kD * 2;       // bytes of one K (or V) step
// A CTA has 4 warps, two CTAs per SM; with many rows and one split each, 2
// warps, four CTAs per SM (one wave of rows, twice the steps per warp).
static_assert(4 * kAmRows == kCcWarps * kCcStep, "the attention launchers share one list unit");

// Shared memory: raw queries [8][128] bf16, scaled queries [8][128] f32, angle tables,
// then the per-warp rings (K step, V step per stage); the warps' states
// reuse the rings after the last step.
__host__ __device__ constexpr int am_smem_bytes(int NW) {
  return 8 * kD * 2 + 8 * kD * 4 + 2 * kNFC * 8 + NW * kAmStages * 2 * kAmTile;
}

__device__ __forceinline__ uint32_t am_pack(float lo_elem, float hi_elem) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo_elem, hi_elem);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void am_mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void am_ldsm4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void am_ldsm4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// 16-byte copy, zero-filled when src_bytes is 0 (nothing is read then).
__device__ __forceinline__ void am_cp16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// Byte offset of 16-byte chunk c of row r in a staged step.
__device__ __forceinline__ uint32_t am_swz(int r, int c) { return (uint32_t)(r * (kD * 2) + ((c ^ (r & 7)) << 4)); }

// The A fragments of the queries: thread (g = lane/4, q = lane%4) holds head
// g's terms at dims 16s + 2q + {0, 1, 8, 9} of every k-step s.
struct AmQuery {
  uint32_t a1[8][4];  // [Q_hi; Q_mid]
  uint32_t a2[8][2];  // [Q_lo; 0] (the zero half is not stored)
};

__device__ __forceinline__ void am_split3(float x, float& hi, float& mid, float& lo) {
  hi = __bfloat162float(__float2bfloat16_rn(x));
  const float r1 = x - hi;  // exact
  mid = __bfloat162float(__float2bfloat16_rn(r1));
  lo = r1 - mid;            // exact, and exactly a bf16
}

__device__ __forceinline__ void am_query_frags(AmQuery& Q, const float* qs, int lane) {
  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const float2 x = *reinterpret_cast<const float2*>(qs + g * kD + 16 * s + 8 * half + 2 * q);
      float h0, m0, l0, h1, m1, l1;
      am_split3(x.x, h0, m0, l0);
      am_split3(x.y, h1, m1, l1);
      Q.a1[s][2 * half] = am_pack(h0, h1);
      Q.a1[s][2 * half + 1] = am_pack(m0, m1);
      Q.a2[s][half] = am_pack(l0, l1);
    }
  }
}

// A warp's running state for head g = lane/4: o[t] holds dims 8t + 2q,
// 8t + 2q + 1 of the P_hi (o[t][0..1]) and P_lo (o[t][2..3]) products; m is
// the running maximum (shared by the quad), l the lane's part of the sum.
struct AmState {
  float o[16][4];
  float m, l;
};

// One step of 16 staged rows (ks, vs: shared addresses of the K and V
// steps); bit r of `valid` says whether row r takes part.
__device__ __forceinline__ void am_step(AmState& st, const AmQuery& Q, uint32_t ks, uint32_t vs, unsigned valid,
                                        int lane) {
  const int q = lane & 3;
  const int mi = lane >> 3, r8 = lane & 7;
  float s1[2][4], s2[2][4];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) s1[j][e] = s2[j][e] = 0.0f;
  // S = Q K^T: ldmatrix x4 of key rows 8j .. 8j+7 gives k-steps 2u, 2u+1
#pragma unroll
  for (int u = 0; u < 4; ++u) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint32_t b[4];
      am_ldsm4(b, ks + am_swz(8 * j + r8, 4 * u + mi));
      const int s0 = 2 * u, s1i = 2 * u + 1;
      am_mma(s1[j], Q.a1[s0][0], Q.a1[s0][1], Q.a1[s0][2], Q.a1[s0][3], b[0], b[1]);
      am_mma(s2[j], Q.a2[s0][0], 0u, Q.a2[s0][1], 0u, b[0], b[1]);
      am_mma(s1[j], Q.a1[s1i][0], Q.a1[s1i][1], Q.a1[s1i][2], Q.a1[s1i][3], b[2], b[3]);
      am_mma(s2[j], Q.a2[s1i][0], 0u, Q.a2[s1i][1], 0u, b[2], b[3]);
    }
  }
  // logits of head g for keys 8j + 2q + e
  float z[2][2];
  float mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int key = 8 * j + 2 * q + e;
      const float v = __fadd_rn(__fadd_rn(s1[j][e], s1[j][e + 2]), s2[j][e]);
      z[j][e] = ((valid >> key) & 1u) ? v : -INFINITY;
      mx = fmaxf(mx, z[j][e]);
    }
  mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
  if (mx > st.m) {  // the quad's maximum rises: rescale (st.m = -inf: the state is empty)
    const float sc = (st.m == -INFINITY) ? 0.0f : exp2f(st.m - mx);
    st.m = mx;
    st.l *= sc;
#pragma unroll
    for (int t = 0; t < 16; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) st.o[t][e] *= sc;
  }
  uint32_t pa[4];  // [P_hi; P_lo] for keys 2q, 2q+1 (j = 0) and 8 + 2q, 9 + 2q (j = 1)
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float ph[2], pl[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float pz = (z[j][e] == -INFINITY) ? 0.0f : exp2f(z[j][e] - st.m);
      st.l += pz;
      ph[e] = __bfloat162float(__float2bfloat16_rn(pz));
      pl[e] = pz - ph[e];
    }
    pa[2 * j] = am_pack(ph[0], ph[1]);
    pa[2 * j + 1] = am_pack(pl[0], pl[1]);
  }
  // O += P V: ldmatrix x4.trans gives the B fragments of dim tiles 2v, 2v+1
  const int vr = ((mi & 1) << 3) + r8;
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    uint32_t b[4];
    am_ldsm4_t(b, vs + am_swz(vr, 2 * v + (mi >> 1)));
    am_mma(st.o[2 * v], pa[0], pa[1], pa[2], pa[3], b[0], b[1]);
    am_mma(st.o[2 * v + 1], pa[0], pa[1], pa[2], pa[3], b[2], b[3]);
  }
}

// Merge of NW warps' states in shared memory: wm, wl [NW][8] the maxima and
// sums, wo(w) warp w's o [8][128]. Threads tid < NW * 8 form the weight of
// (warp w, head h) = 2^(m_wh - M_h) into wf [NW][8]; after a barrier every
// output element e = h * 128 + d of the G heads (e = tid, tid + NT, ...)
// sums its warps' weighted o and l in warp order and calls emit(e, O, L).
// Called by all NT threads after a barrier that follows the state writes.
template <int NW, int NT, typename WoAt, typename Emit>
__device__ __forceinline__ void am_merge_warps(const float* wm, const float* wl, float* wf, WoAt wo, int G, Emit emit) {
  const int tid = threadIdx.x;
  if (tid < NW * 8) {
    const int h = tid & 7;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, wm[w * 8 + h]);
    wf[tid] = (wm[tid] == -INFINITY) ? 0.0f : exp2f(wm[tid] - M);
  }
  __syncthreads();
  for (int e = tid; e < G * kD; e += NT) {
    const int h = e / kD;
    float L = 0.0f, O = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float f = wf[w * 8 + h];
      L += f * wl[w * 8 + h];
      O += f * wo(w)[e];
    }
    emit(e, O, L);
  }
}

// Split-K attention over a row's kept list (or all its rows) for G <= 8:
// grid (splits, rows); CTA `split` takes list positions [split*slice, ...),
// its NW warps (4, or 2 for many rows of one split each) contiguous parts of
// them in steps of 16 rows; the warps merge in shared memory and the CTA
// writes its partial (m, l, o), or with one split the output
// (attend_merge_kernel merges the partials).
template <int NW>
__global__ void __launch_bounds__(NW * 32, 8 / NW) attend_mma_kernel(const CcParams p) {
  constexpr int kAmWarps = NW, kAmThreads = NW * 32;
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16* qraw = reinterpret_cast<__nv_bfloat16*>(smem);
  float* qs = reinterpret_cast<float*>(smem + 8 * kD * 2);  // after the raw queries (G <= 8 rows)
  double* cs = reinterpret_cast<double*>(qs + 8 * kD);
  unsigned char* ring = reinterpret_cast<unsigned char*>(cs + 2 * kNFC);
  const int split = blockIdx.x, row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.group;
  int len, n_keep;
  cc_row_begin<kAmThreads>(p, row, cs, len, n_keep);

  const int r_beg = split * p.slice, r_end = min(n_keep, r_beg + p.slice);
  const int per_warp = ((max(0, r_end - r_beg) + kAmWarps * kAmRows - 1) / (kAmWarps * kAmRows)) * kAmRows;
  const int j0 = min(r_end, r_beg + warp * per_warp), j1 = min(r_end, j0 + per_warp);
  const int n_steps = (j1 - j0 + kAmRows - 1) / kAmRows;
  const bool paged = p.pm.table != nullptr;
  const int64_t plane = paged ? 0 : (int64_t)row * p.max_len * kD;
  const __nv_bfloat16* kb = p.k + plane;
  const __nv_bfloat16* vb = p.v + plane;
  const int32_t* idx = p.idx ? p.idx + (int64_t)row * p.n_keep : nullptr;
  const uint32_t ring_w = smem_u32(ring) + (uint32_t)(warp * kAmStages * 2 * kAmTile);

  // lanes 0..15 hold the list entry of row `lane` of a step: raw() reads it
  // (no wait), resolve() checks it and maps it to its cache row (-1: masked)
  auto raw = [&](int step) -> int {
    const int j = j0 + step * kAmRows + lane;
    if (lane >= kAmRows || step >= n_steps || j >= j1) return -1;
    return idx ? __ldg(idx + j) : j;
  };
  auto resolve = [&](int t, int step) -> int {
    const int j = j0 + step * kAmRows + lane;
    if (lane >= kAmRows || step >= n_steps || j >= j1) return -1;
    if (t < 0 || t >= len) {
      flag_status(FASA_ERR_BAD_INDEX);
      return -1;
    }
    return paged ? paged_row(p.pm, row / p.n_kv_heads, row % p.n_kv_heads, t) : t;
  };
  // issue step `step` into its stage: lane l copies chunk l%16 of rows
  // 2i + l/16, K then V; returns the step's valid mask
  auto issue = [&](int tok, int step) -> unsigned {
    const unsigned valid = __ballot_sync(0xFFFFFFFFu, tok >= 0) & 0xFFFFu;
    const uint32_t kst = ring_w + (uint32_t)((step % kAmStages) * 2 * kAmTile);
    const uint32_t vst = kst + kAmTile;
    const int c = lane & 15;
#pragma unroll
    for (int i = 0; i < kAmRows / 2; ++i) {
      const int r = 2 * i + (lane >> 4);
      const int t = __shfl_sync(0xFFFFFFFFu, tok, r);
      const int64_t off = (int64_t)(t < 0 ? 0 : t) * kD + c * 8;
      const uint32_t nb = t < 0 ? 0u : 16u;
      am_cp16(kst + am_swz(r, c), kb + off, nb);
      am_cp16(vst + am_swz(r, c), vb + off, nb);
    }
    return valid;
  };

  // the queries first, then the first steps' rows: the rows are in flight
  // while the queries are formed
  cc_stage_queries<kAmThreads>(p, row, qraw);
  unsigned valid[kAmStages];
#pragma unroll
  for (int s = 0; s < kAmStages; ++s) {
    valid[s] = (s < n_steps) ? issue(resolve(raw(s), s), s) : 0u;
    cp_async_commit();
  }
  int nxt = raw(kAmStages);
  cp_async_wait<kAmStages>();  // the queries' group
  cc_row_queries<8, kAmThreads, true>(p, row, len, qraw, cs, qs);
  AmQuery Q;
  am_query_frags(Q, qs, lane);
  AmState st;
#pragma unroll
  for (int t = 0; t < 16; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) st.o[t][e] = 0.0f;
  st.m = -INFINITY;
  st.l = 0.0f;
  for (int step = 0; step < n_steps; ++step) {
    cp_async_wait<kAmStages - 1>();
    __syncwarp();
    const int stage = step % kAmStages;
    const uint32_t kst = ring_w + (uint32_t)(stage * 2 * kAmTile);
    unsigned vm = valid[0];
#pragma unroll
    for (int s = 1; s < kAmStages; ++s)
      if (stage == s) vm = valid[s];
    am_step(st, Q, kst, kst + kAmTile, vm, lane);
    __syncwarp();  // every lane is done with the stage before it is refilled
    const int ns = step + kAmStages;
    if (ns < n_steps) {
      const unsigned v = issue(resolve(nxt, ns), ns);
#pragma unroll
      for (int s = 0; s < kAmStages; ++s)
        if (stage == s) valid[s] = v;
    }
    cp_async_commit();
    nxt = raw(ns + 1);
  }
  cp_async_wait<0>();
  grid_dependents_launch();  // the merge (or the next kernel) may start its prologue on SMs this grid frees
  st.l += __shfl_xor_sync(0xFFFFFFFFu, st.l, 1);
  st.l += __shfl_xor_sync(0xFFFFFFFFu, st.l, 2);
  __syncthreads();  // every warp is past its ring: the states reuse it

  // warp states: m, l [kAmWarps][8], merge weights [kAmWarps][8], o [kAmWarps][8][128]
  float* wm = reinterpret_cast<float*>(ring);
  float* wl = wm + kAmWarps * 8;
  float* wf = wl + kAmWarps * 8;
  float* wo = wf + kAmWarps * 8;
  const int g = lane >> 2, q = lane & 3;
  if (q == 0) {
    wm[warp * 8 + g] = st.m;
    wl[warp * 8 + g] = st.l;
  }
#pragma unroll
  for (int t = 0; t < 16; ++t)
    *reinterpret_cast<float2*>(wo + (warp * 8 + g) * kD + 8 * t + 2 * q) =
        make_float2(__fadd_rn(st.o[t][0], st.o[t][2]), __fadd_rn(st.o[t][1], st.o[t][3]));
  __syncthreads();
  __nv_bfloat16* out = p.out + (int64_t)row * G * kD;
  float* pp = p.part + ((int64_t)row * p.splits + split) * kCcPartStride;
  const bool single = p.splits == 1;
  am_merge_warps<kAmWarps, kAmThreads>(wm, wl, wf, [&](int w) { return wo + w * 8 * kD; }, G,
                                       [&](int e, float O, float L) {
    if (single) {
      out[e] = __float2bfloat16_rn(L > 0.0f ? O / L : 0.0f);
    } else {
      pp[32 + e] = O;
      if (e % kD == 0) {  // the head's maximum and sum
        const int h = e / kD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kAmWarps; ++w) M = fmaxf(M, wm[w * 8 + h]);
        pp[h] = M;
        pp[16 + h] = L;
      }
    }
  });
}

}  // namespace fasa
