// Critical-set selection and focused attention, one thread-block cluster per
// (sequence, KV head).
//
// "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
// §2, FAC bullets): from the TIP scores pick the critical token set T_t, run
// full softmax attention over exactly those tokens, keep their original
// absolute positions (their keys were rotated at append time).
//
// Modes (one kernel template, chosen at launch):
//   kSelect     scores -> idx (fasa_select_topk)
//   kDecode     scores -> T_t -> attention -> out (second launch of fasa_decode)
//   kAttendIdx  given idx -> attention -> out (fasa_sparse_attend)
//   kDense      all rows -> attention -> out (fasa_dense_decode)
//
// Select: exact top-k by a 3-pass radix select (11, 11, 10 bits) on
// order-preserving uint32 keys. The C CTAs of a cluster each hold a contiguous
// chunk of the row's keys in shared memory; per-pass histograms are summed
// into the leader CTA's shared memory over DSMEM and every CTA reads the
// total back, so no pass touches global memory. Ties at the threshold key go
// to the lower token index; the kept indices are emitted in ascending order
// straight into the shared memory of the CTA that will attend over them.
//
// Attention: each CTA takes an equal slice of the kept indices, gathers their
// K and V rows with 1-D bulk copies (TMA engine, mbarrier completion,
// double-buffered, no multicast), computes float32 logits for the G query
// heads with 8 lanes per row, keeps a float32 online softmax (base-2, scale
// folded into q), and accumulates P.V per 4-dim quad. Partials (m, l, o) are
// merged across the cluster over DSMEM.
#pragma once

#include <cooperative_groups.h>

#include "fasa_device.cuh"

namespace fasa {
namespace cg = cooperative_groups;

constexpr int kSAThreads = 512;
constexpr int kSAWarps = kSAThreads / 32;
constexpr int kBins = 2048;
constexpr int kMaxCluster = 16;

enum SAMode { kSelect = 0, kDecode = 1, kAttendIdx = 2, kDense = 3 };

struct SAParams {
  const float* scores;       // [rows][len]
  int32_t* idx_out;          // [rows][n_keep] or null
  const int32_t* idx_in;     // [rows][n_keep] (kAttendIdx)
  const void* k;             // [rows][max_len][128]
  const void* v;
  const void* q;             // [B][Hq][128]
  void* out;                 // [B][Hq][128]
  int64_t max_len;
  int32_t len;
  int32_t n_keep;            // k_eff (select/decode) or n_idx (attend)
  int32_t chunk;             // keys (select) or rows (dense) per CTA
  int32_t slice;             // kept indices attended per CTA
  int32_t n_kv_heads;
  int32_t group;
  int32_t q_pos;
  double theta[kNFC];
};

// Rows per pipeline stage: 32 KB of K+V per stage.
template <typename T> __host__ __device__ constexpr int stage_rows() { return 32768 / (2 * kD * (int)sizeof(T)); }

// Shared-memory layout, identical on host and device.
struct SALayout {
  int off_keys, off_stage, off_idx, off_hist, off_ghist, off_q, off_z, off_o, off_ml, off_cs, off_misc, off_bar, total;
};

__host__ __device__ inline int sa_align(int x, int a) { return (x + a - 1) / a * a; }

__host__ __device__ inline SALayout sa_layout(int mode, int elem_bytes, int chunk, int slice, int maxg) {
  SALayout L;
  const int rb = 32768 / (2 * kD * elem_bytes);
  const bool sel = (mode == kSelect || mode == kDecode);
  const bool att = (mode != kSelect);
  const int keys_bytes = sel ? chunk * 4 : 0;
  const int stage_bytes = att ? 2 * 32768 : 0;
  const int a_bytes = keys_bytes > stage_bytes ? keys_bytes : stage_bytes;
  int off = 0;
  L.off_keys = off;
  L.off_stage = off;  // stages reuse the key region after selection
  off = sa_align(off + a_bytes, 128);
  L.off_idx = off;
  off = sa_align(off + ((mode == kDecode || mode == kAttendIdx) ? slice * 4 : 0), 128);
  L.off_hist = off;
  off = sa_align(off + (sel ? kBins * 4 : 0), 128);
  L.off_ghist = off;
  off = sa_align(off + (sel ? 3 * kBins * 4 : 0), 128);
  L.off_q = off;
  off = sa_align(off + (att ? maxg * kD * 4 : 0), 128);
  L.off_z = off;
  off = sa_align(off + (att ? maxg * rb * 4 : 0), 128);
  L.off_o = off;
  off = sa_align(off + (att ? maxg * kD * 4 : 0), 128);
  L.off_ml = off;
  off = sa_align(off + (att ? 3 * maxg * 4 : 0), 128);
  L.off_cs = off;
  off = sa_align(off + (att ? 2 * kNFC * 8 : 0), 128);
  L.off_misc = off;
  off = sa_align(off + 256 * 4, 128);
  L.off_bar = off;
  off = sa_align(off + 2 * 8, 128);
  L.total = off;
  return L;
}

// misc-area slots (uint32 words)
enum : int {
  kMiscWarpGt = 0,     // [16]
  kMiscWarpEq = 16,    // [16]
  kMiscCtaGt = 32,     // [16]  written remotely into the leader
  kMiscCtaEq = 48,     // [16]
  kMiscScan = 64,      // [16]  block-scan scratch
  kMiscBin = 80,       // broadcast: selected bin
  kMiscAbove = 81,     // broadcast: count above it
  kMiscGtBefore = 82,
  kMiscEqBefore = 83,
};

// Inclusive scan of one value per thread (thread order), block-wide.
__device__ __forceinline__ uint32_t block_incl_scan(uint32_t v, uint32_t* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t n = __shfl_up_sync(0xFFFFFFFFu, v, off);
    if (lane >= off) v += n;
  }
  if (lane == 31) scratch[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kSAWarps ? scratch[lane] : 0u;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t n = __shfl_up_sync(0xFFFFFFFFu, w, off);
      if (lane >= off) w += n;
    }
    if (lane < kSAWarps) scratch[lane] = w;
  }
  __syncthreads();
  const uint32_t before = warp > 0 ? scratch[warp - 1] : 0u;
  __syncthreads();
  return v + before;
}

template <typename T, int MODE, int MAXG>
__global__ void __launch_bounds__(kSAThreads, (MAXG <= 4 ? 2 : 1)) select_attend_kernel(const SAParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  grid_dependency_wait();  // inputs of an earlier kernel in the stream are complete
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr bool kSel = (MODE == kSelect || MODE == kDecode);
  constexpr bool kAtt = (MODE != kSelect);
  constexpr int RB = stage_rows<T>();
  constexpr int ES = (int)sizeof(T);

  const SALayout L = sa_layout(MODE, ES, p.chunk, p.slice, MAXG);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + L.off_keys);
  T* stage = reinterpret_cast<T*>(smem + L.off_stage);
  int32_t* idx_s = reinterpret_cast<int32_t*>(smem + L.off_idx);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + L.off_hist);
  uint32_t* ghist = reinterpret_cast<uint32_t*>(smem + L.off_ghist);
  float* qs = reinterpret_cast<float*>(smem + L.off_q);
  float* zs = reinterpret_cast<float*>(smem + L.off_z);
  float* os = reinterpret_cast<float*>(smem + L.off_o);
  float* ml = reinterpret_cast<float*>(smem + L.off_ml);  // m[MAXG], l[MAXG], scale[MAXG]
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L.off_misc);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.off_bar);

  const int G = p.group;

  // ------------------------------------------------------------ set-up
  if (kSel && rank == 0)
    for (int i = tid; i < 3 * kBins; i += kSAThreads) ghist[i] = 0u;
  if (MODE == kDecode)  // slots the selection never fills stay masked
    for (int i = tid; i < p.slice; i += kSAThreads) idx_s[i] = -1;
  if (kAtt) {
    if (tid == 0) {
      mbar_init(&bars[0], 1);
      mbar_init(&bars[1], 1);
      fence_mbar_init();
    }
    for (int i = tid; i < MAXG * kD; i += kSAThreads) os[i] = 0.0f;
    if (tid < MAXG) {
      ml[tid] = -INFINITY;
      ml[MAXG + tid] = 0.0f;
      ml[2 * MAXG + tid] = 0.0f;
    }
    // rotated, pre-scaled queries: q'_h * log2(e) / sqrt(128), float32
    double* cs = reinterpret_cast<double*>(smem + L.off_cs);  // 64 x (cos, sin)
    if (tid < kNFC) {
      double s, c;
      sincos((double)p.q_pos * p.theta[tid], &s, &c);
      cs[2 * tid] = c;
      cs[2 * tid + 1] = s;
    }
    __syncthreads();
    const T* qh = static_cast<const T*>(p.q) + ((int64_t)row * G) * kD;
    const double qscale = 1.4426950408889634 / 11.313708498984761;  // log2(e) / sqrt(128)
    for (int e = tid; e < G * kD; e += kSAThreads) {
      const int h = e / kD, d = e % kD, i = d & (kNFC - 1);
      const double x = to_float(qh[h * kD + i]);
      const double y = to_float(qh[h * kD + i + kNFC]);
      const double c = cs[2 * i], s = cs[2 * i + 1];
      const double r = (d < kNFC) ? (x * c - y * s) : (y * c + x * s);
      qs[h * kD + d] = (float)(r * qscale);
    }
    for (int e = G * kD + tid; e < MAXG * kD; e += kSAThreads) qs[e] = 0.0f;
  }
  __syncthreads();
  if (C > 1) cluster.sync();  // all CTAs started; leader histograms zeroed

  int n_mine = 0;      // rows this CTA attends over
  int row_start = 0;   // first row (dense) / first slice position (kept lists)

  // ------------------------------------------------------------ select
  if constexpr (kSel) {
    const int start = rank * p.chunk;
    const int n_loc = max(0, min(p.chunk, p.len - start));
    const float* srow = p.scores + (int64_t)row * p.len + start;
    for (int i = tid; i < n_loc; i += kSAThreads) keys[i] = score_key(srow[i]);
    __syncthreads();

    uint32_t prefix = 0u, pmask = 0u;
    int krem = p.n_keep;
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const int nb = pass == 2 ? 1024 : 2048;
      for (int i = tid; i < kBins; i += kSAThreads) hist[i] = 0u;
      __syncthreads();
      for (int base = warp * 32; base < n_loc; base += kSAThreads) {
        const int i = base + lane;
        bool ok = false;
        uint32_t bin = 0u;
        if (i < n_loc) {
          const uint32_t x = keys[i];
          ok = (x & pmask) == prefix;
          bin = (x >> shift) & (uint32_t)(nb - 1);
        }
        const unsigned act = __ballot_sync(0xFFFFFFFFu, ok);
        if (ok) {
          const unsigned peers = __match_any_sync(act, bin);
          if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
        }
      }
      __syncthreads();
      uint32_t* gh = cluster.map_shared_rank(ghist + pass * kBins, 0);
      for (int i = tid; i < nb; i += kSAThreads) {
        const uint32_t h = hist[i];
        if (h) atomicAdd(gh + i, h);
      }
      if (C > 1) cluster.sync(); else __syncthreads();
      // find the bin holding the krem-th largest key, scanning from the top
      const int per = nb / kSAThreads;  // 4 or 2 bins per thread
      uint32_t c[4] = {0u, 0u, 0u, 0u};
      uint32_t sum = 0u;
      for (int j = 0; j < per; ++j) {
        c[j] = gh[nb - 1 - (tid * per + j)];
        sum += c[j];
      }
      const uint32_t incl = block_incl_scan(sum, misc + kMiscScan);
      const uint32_t excl = incl - sum;
      if (excl < (uint32_t)krem && (uint32_t)krem <= incl) {
        uint32_t acc = excl;
        for (int j = 0; j < per; ++j) {
          if (acc + c[j] >= (uint32_t)krem) {
            misc[kMiscBin] = (uint32_t)(nb - 1 - (tid * per + j));
            misc[kMiscAbove] = acc;
            break;
          }
          acc += c[j];
        }
      }
      __syncthreads();
      const uint32_t bin = misc[kMiscBin];
      krem -= (int)misc[kMiscAbove];
      prefix |= bin << shift;
      pmask |= (uint32_t)(nb - 1) << shift;
      __syncthreads();
    }
    const uint32_t thr = prefix;  // the k_eff-th largest key; take krem of the keys equal to it

    // count keys above / at the threshold per warp (warp segments in index order)
    const int seg = ((n_loc + kSAWarps * 32 - 1) / (kSAWarps * 32)) * 32;
    const int ws = min(n_loc, warp * seg), we = min(n_loc, ws + seg);
    uint32_t cgt = 0u, ceq = 0u;
    for (int base = ws; base < we; base += 32) {
      const int i = base + lane;
      const bool valid = i < we;
      const uint32_t x = valid ? keys[i] : 0u;
      cgt += __popc(__ballot_sync(0xFFFFFFFFu, valid && x > thr));
      ceq += __popc(__ballot_sync(0xFFFFFFFFu, valid && x == thr));
    }
    if (lane == 0) {
      misc[kMiscWarpGt + warp] = cgt;
      misc[kMiscWarpEq + warp] = ceq;
    }
    __syncthreads();
    if (tid == 0) {
      uint32_t tg = 0u, te = 0u;
      for (int w = 0; w < kSAWarps; ++w) {
        const uint32_t a = misc[kMiscWarpGt + w], e = misc[kMiscWarpEq + w];
        misc[kMiscWarpGt + w] = tg;  // exclusive offsets
        misc[kMiscWarpEq + w] = te;
        tg += a;
        te += e;
      }
      uint32_t* lead = cluster.map_shared_rank(misc, 0);
      lead[kMiscCtaGt + rank] = tg;
      lead[kMiscCtaEq + rank] = te;
    }
    if (C > 1) cluster.sync(); else __syncthreads();
    if (tid == 0) {
      const uint32_t* lead = cluster.map_shared_rank(misc, 0);
      uint32_t gb = 0u, eb = 0u;
      for (int r = 0; r < rank; ++r) {
        gb += lead[kMiscCtaGt + r];
        eb += lead[kMiscCtaEq + r];
      }
      misc[kMiscGtBefore] = gb;
      misc[kMiscEqBefore] = eb;
    }
    __syncthreads();

    // emit the kept indices in ascending order
    int gr = (int)(misc[kMiscGtBefore] + misc[kMiscWarpGt + warp]);
    int er = (int)(misc[kMiscEqBefore] + misc[kMiscWarpEq + warp]);
    const unsigned lt = (1u << lane) - 1u;
    for (int base = ws; base < we; base += 32) {
      const int i = base + lane;
      const bool valid = i < we;
      const uint32_t x = valid ? keys[i] : 0u;
      const bool is_gt = valid && x > thr, is_eq = valid && x == thr;
      const unsigned bg = __ballot_sync(0xFFFFFFFFu, is_gt);
      const unsigned be = __ballot_sync(0xFFFFFFFFu, is_eq);
      const int my_gr = gr + __popc(bg & lt), my_er = er + __popc(be & lt);
      const int pos = my_gr + min(my_er, krem);
      if ((is_gt || (is_eq && my_er < krem)) && pos >= p.n_keep) flag_status(FASA_ERR_BAD_INDEX);
      if ((is_gt || (is_eq && my_er < krem)) && pos < p.n_keep) {
        const int token = start + i;
        if (MODE == kDecode) {
          const int owner = pos / p.slice;
          int32_t* dst = cluster.map_shared_rank(idx_s, owner);
          dst[pos - owner * p.slice] = token;
        }
        if (p.idx_out) p.idx_out[(int64_t)row * p.n_keep + pos] = token;
      }
      gr += __popc(bg);
      er += __popc(be);
    }
    fence_proxy_async_smem();  // key region is reused by bulk copies below
    if (C > 1) cluster.sync(); else __syncthreads();
    if (MODE == kDecode) {
      row_start = rank * p.slice;
      n_mine = max(0, min(p.slice, p.n_keep - row_start));
    }
  }

  if constexpr (!kAtt) {
    return;  // the last cluster barrier above keeps the leader alive while read
  } else {
    if (MODE == kAttendIdx) {
      row_start = rank * p.slice;
      n_mine = max(0, min(p.slice, p.n_keep - row_start));
      const int32_t* src = p.idx_in + (int64_t)row * p.n_keep + row_start;
      for (int j = tid; j < n_mine; j += kSAThreads) {
        int t = src[j];
        if (t < 0 || t >= p.len) {
          flag_status(FASA_ERR_BAD_INDEX);
          t = -1;
        }
        idx_s[j] = t;
      }
      __syncthreads();
    } else if (MODE == kDense) {
      row_start = rank * p.chunk;
      n_mine = max(0, min(p.chunk, p.len - row_start));
    }

    const T* kbase = static_cast<const T*>(p.k) + (int64_t)row * p.max_len * kD;
    const T* vbase = static_cast<const T*>(p.v) + (int64_t)row * p.max_len * kD;
    const int nbatch = (n_mine + RB - 1) / RB;

    auto issue = [&](int bi) {
      const int s = bi & 1;
      const int j0 = bi * RB;
      const int nr = min(RB, n_mine - j0);
      T* ks = stage + (size_t)s * 2 * RB * kD;
      T* vs = ks + RB * kD;
      if (lane == 0) mbar_arrive_expect_tx(&bars[s], (uint32_t)(nr * 2 * kD * ES));
      __syncwarp();
      if (MODE == kDense) {
        if (lane == 0) {
          bulk_g2s(ks, kbase + (int64_t)(row_start + j0) * kD, (uint32_t)(nr * kD * ES), &bars[s]);
          bulk_g2s(vs, vbase + (int64_t)(row_start + j0) * kD, (uint32_t)(nr * kD * ES), &bars[s]);
        }
      } else {
        for (int r = lane; r < nr; r += 32) {
          int t = idx_s[j0 + r];  // this CTA's slice of the kept list
          if (t < 0 || t >= p.len) t = 0;  // skipped index: copy a valid row, masked below
          bulk_g2s(ks + r * kD, kbase + (int64_t)t * kD, kD * ES, &bars[s]);
          bulk_g2s(vs + r * kD, vbase + (int64_t)t * kD, kD * ES, &bars[s]);
        }
      }
    };

    if (warp == 0) {
      if (nbatch > 0) issue(0);
      if (nbatch > 1) issue(1);
    }

    // per-thread P.V accumulators: quad of dims 4*lq .. 4*lq+3, row group warp
    float acc[MAXG][4];
#pragma unroll
    for (int h = 0; h < MAXG; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[h][e] = 0.0f;

    for (int bi = 0; bi < nbatch; ++bi) {
      const int s = bi & 1;
      const int j0 = bi * RB;
      const int nr = min(RB, n_mine - j0);
      const T* ks = stage + (size_t)s * 2 * RB * kD;
      const T* vs = ks + RB * kD;
      mbar_wait(&bars[s], (uint32_t)((bi >> 1) & 1));

      // logits: 8 lanes per row, 16 dims per lane
      for (int r = warp * 4 + (lane >> 3); r < RB; r += kSAWarps * 4) {
        const int sub = lane & 7;
        float kf[16];
        const uint4* src = reinterpret_cast<const uint4*>(ks + r * kD + sub * 16);
        if (ES == 2) {
          float f8[8];
          unpack16(src[0], f8, T());
#pragma unroll
          for (int e = 0; e < 8; ++e) kf[e] = f8[e];
          unpack16(src[1], f8, T());
#pragma unroll
          for (int e = 0; e < 8; ++e) kf[8 + e] = f8[e];
        } else {
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const uint4 u = src[c4];
            kf[4 * c4 + 0] = __uint_as_float(u.x);
            kf[4 * c4 + 1] = __uint_as_float(u.y);
            kf[4 * c4 + 2] = __uint_as_float(u.z);
            kf[4 * c4 + 3] = __uint_as_float(u.w);
          }
        }
        bool valid = r < nr;
        if (MODE != kDense && valid) {
          const int t = idx_s[j0 + r];
          valid = t >= 0 && t < p.len;
          if (MODE == kDecode && !valid) flag_status(FASA_ERR_BAD_INDEX);
        }
#pragma unroll
        for (int h = 0; h < MAXG; ++h) {
          if (h < G) {
            const float4* qv = reinterpret_cast<const float4*>(qs + h * kD + sub * 16);
            float a = 0.0f;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
              const float4 qq = qv[c4];
              a = fmaf(qq.x, kf[4 * c4 + 0], a);
              a = fmaf(qq.y, kf[4 * c4 + 1], a);
              a = fmaf(qq.z, kf[4 * c4 + 2], a);
              a = fmaf(qq.w, kf[4 * c4 + 3], a);
            }
            a += __shfl_xor_sync(0xFFFFFFFFu, a, 1);
            a += __shfl_xor_sync(0xFFFFFFFFu, a, 2);
            a += __shfl_xor_sync(0xFFFFFFFFu, a, 4);
            if (sub == 0) zs[h * RB + r] = valid ? a : -INFINITY;
          }
        }
      }
      __syncthreads();
      // online softmax: one warp per query head
      if (warp < G) {
        const int h = warp;
        float mx = -INFINITY;
        for (int r = lane; r < RB; r += 32) mx = fmaxf(mx, zs[h * RB + r]);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
        const float m_old = ml[h];
        const float m_new = fmaxf(m_old, mx);
        const float sc = (m_old == -INFINITY) ? 0.0f : exp2f(m_old - m_new);
        float sum = 0.0f;
        for (int r = lane; r < RB; r += 32) {
          const float z = zs[h * RB + r];
          const float pz = (z == -INFINITY) ? 0.0f : exp2f(z - m_new);
          zs[h * RB + r] = pz;
          sum += pz;
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
        if (lane == 0) {
          ml[h] = m_new;
          ml[MAXG + h] = ml[MAXG + h] * sc + sum;
          ml[2 * MAXG + h] = sc;
        }
      }
      __syncthreads();
      // P.V: thread = (quad lane, row group warp)
#pragma unroll
      for (int h = 0; h < MAXG; ++h) {
        if (h < G) {
          const float sc = ml[2 * MAXG + h];
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[h][e] *= sc;
        }
      }
      for (int r = warp; r < nr; r += kSAWarps) {
        float vf[4];
        if (ES == 2) {
          const uint2 u = *reinterpret_cast<const uint2*>(vs + r * kD + lane * 4);
          vf[0] = __uint_as_float(u.x << 16);
          vf[1] = __uint_as_float(u.x & 0xFFFF0000u);
          vf[2] = __uint_as_float(u.y << 16);
          vf[3] = __uint_as_float(u.y & 0xFFFF0000u);
        } else {
          const uint4 u = *reinterpret_cast<const uint4*>(vs + r * kD + lane * 4);
          vf[0] = __uint_as_float(u.x);
          vf[1] = __uint_as_float(u.y);
          vf[2] = __uint_as_float(u.z);
          vf[3] = __uint_as_float(u.w);
        }
#pragma unroll
        for (int h = 0; h < MAXG; ++h) {
          if (h < G) {
            const float pz = zs[h * RB + r];
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[h][e] = fmaf(pz, vf[e], acc[h][e]);
          }
        }
      }
      fence_proxy_async_smem();
      __syncthreads();  // stage s fully consumed
      if (warp == 0 && bi + 2 < nbatch) issue(bi + 2);
    }

    // reduce the 16 row groups into this CTA's partial o
#pragma unroll
    for (int h = 0; h < MAXG; ++h) {
      if (h < G) {
#pragma unroll
        for (int e = 0; e < 4; ++e) atomicAdd(&os[h * kD + lane * 4 + e], acc[h][e]);
      }
    }
    __syncthreads();
    if (C > 1) cluster.sync();

    // merge the cluster's partials; each CTA finishes a share of the outputs
    T* out = static_cast<T*>(p.out) + ((int64_t)row * G) * kD;
    for (int e = rank * kSAThreads + tid; e < G * kD; e += C * kSAThreads) {
      const int h = e / kD, d = e % kD;
      float M = -INFINITY;
      for (int r = 0; r < C; ++r) M = fmaxf(M, cluster.map_shared_rank(ml, r)[h]);
      float num = 0.0f, den = 0.0f;
      if (M != -INFINITY) {
        for (int r = 0; r < C; ++r) {
          const float* mlr = cluster.map_shared_rank(ml, r);
          const float mr = mlr[h];
          const float w = (mr == -INFINITY) ? 0.0f : exp2f(mr - M);
          den = fmaf(w, mlr[MAXG + h], den);
          num = fmaf(w, cluster.map_shared_rank(os, r)[h * kD + d], num);
        }
      }
      store_f(out + h * kD + d, den > 0.0f ? num / den : 0.0f);
    }
    if (C > 1) cluster.sync();  // partials stay readable until everyone is done
  }
}

}  // namespace fasa
