// C ABI of the FASA decode hot path (declared in include/fasa.h).
//
// Host side only: argument validation (before any launch), launch-shape
// choice, and dispatch to the kernels in append.cuh, score.cuh and
// select_attend.cuh. Nothing here allocates device memory.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <unordered_map>

#include "append.cuh"
#include "fasa_device.cuh"
#include "score.cuh"
#include "select_attend.cuh"
#include "select_hist.cuh"
#include "attend_cc.cuh"
#include "attend_mma.cuh"
#include "attend_tc.cuh"
#include "decode_wide.cuh"
#include "calibrate.cuh"

using namespace fasa;

// Fixed scratch of fasa_decode_static_scratch: one copy per device, living as
// long as the library is loaded. Host code must not use its address directly
// (the host-side symbol is only a stand-in); the device address comes from
// cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_static_scratch[FASA_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxChunkKeys = 32768;  // keys per CTA held in shared memory
constexpr int kMaxSlice = 8192;       // kept indices per CTA
constexpr int kMaxDevices = 64;

struct DevInfo {
  bool ready = false;
  int sms = 0;
  int smem_optin = 0;
};
DevInfo g_dev[kMaxDevices];
std::mutex g_mu;
std::unordered_map<uint64_t, int> g_cache;  // (device, kernel, key) -> value

fasa_status device_info(DevInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FASA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return FASA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return FASA_ERR_CUDA;
    d.ready = true;
  }
  *out = d;
  return FASA_OK;
}

// A query position: >= 0, or FASA_Q_PREROTATED.
inline bool bad_qpos(int32_t q_pos) { return q_pos < 0 && q_pos != FASA_Q_PREROTATED; }
inline bool aligned(const void* p, uintptr_t a) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int pow2ceil(int64_t x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}
inline int elem_bytes(int dtype) { return dtype == FASA_F32 ? 4 : 2; }

void fill_theta(double* th, double base) {
  for (int i = 0; i < kNFC; ++i) th[i] = std::pow(base, -2.0 * (double)i / (double)kD);
}

// cos / sin of the query's rotation angle pos * theta_i, float64 on the host.
void fill_query_angle(double* cosv, double* sinv, double base, int32_t pos) {
  if (pos == FASA_Q_PREROTATED) {  // q is already rotated: the identity
    for (int i = 0; i < kNFC; ++i) {
      cosv[i] = 1.0;
      sinv[i] = 0.0;
    }
    return;
  }
  double th[kNFC];
  fill_theta(th, base);
  for (int i = 0; i < kNFC; ++i) {
    const double a = (double)pos * th[i];
    cosv[i] = std::cos(a);
    sinv[i] = std::sin(a);
  }
}

fasa_status check_cache(const fasa_cache* c) {
  if (c == nullptr) return FASA_ERR_INVALID_ARG;
  if (c->head_dim != kD) return FASA_ERR_UNSUPPORTED;
  if (c->dtype != FASA_F32 && c->dtype != FASA_BF16) return FASA_ERR_UNSUPPORTED;
  if (c->batch < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1 || c->n_q_heads % c->n_kv_heads != 0)
    return FASA_ERR_INVALID_ARG;
  if (c->n_q_heads / c->n_kv_heads > FASA_MAX_GROUP) return FASA_ERR_UNSUPPORTED;
  if ((int64_t)c->batch * c->n_kv_heads > 65535) return FASA_ERR_UNSUPPORTED;
  if (c->n_dom < 1 || c->n_dom > kNFC) return FASA_ERR_INVALID_ARG;
  if (c->sketch_stride != fasa_sketch_stride(c->n_dom, c->dtype)) return FASA_ERR_INVALID_ARG;
  if (c->max_len < 1 || c->max_len > (1 << 30)) return FASA_ERR_INVALID_ARG;
  if (!(c->rope_base > 1.0) || !std::isfinite(c->rope_base)) return FASA_ERR_INVALID_ARG;
  if (!aligned(c->k, 16) || !aligned(c->v, 16) || !aligned(c->sketch, 16) || !aligned(c->dom_idx, 4))
    return FASA_ERR_INVALID_ARG;
  return FASA_OK;
}

// True when p lies in host memory (a FASA-M cache's K or V).
bool host_resident(const void* p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

thread_local const char* t_last_cuda_error = "no error";

fasa_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return FASA_OK;
  t_last_cuda_error = cudaGetErrorString(e);
  (void)cudaGetLastError();  // clear a non-sticky launch error
  return FASA_ERR_CUDA;
}

// Cached per (device, kernel, key) integer, computed once by `fn`.
template <typename F>
fasa_status cached_int(const void* kernel, uint64_t key, int* out, F fn) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FASA_ERR_CUDA;
  const uint64_t h = (reinterpret_cast<uint64_t>(kernel) * 1000003ull) ^ (key * 131ull) ^ (uint64_t)dev;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_cache.find(h);
    if (it != g_cache.end()) {
      *out = it->second;
      return FASA_OK;
    }
  }
  int v = 0;
  const fasa_status st = fn(&v);
  if (st != FASA_OK) return st;
  std::lock_guard<std::mutex> lk(g_mu);
  g_cache[h] = v;
  *out = v;
  return FASA_OK;
}

// True when a cache's K or V lies in host memory (FASA-M), cached per
// pointer (a reused address of the other kind would only change the plan's
// speed, not its result).
bool kv_on_host(const fasa_cache* c) {
  int h = 0;
  if (cached_int(c->k, 11, &h, [&](int* v) {
        *v = host_resident(c->k) || host_resident(c->v) ? 1 : 0;
        return FASA_OK;
      }) != FASA_OK)
    return false;
  return h != 0;
}

// Plain launch with programmatic stream serialization (the kernel waits
// for its predecessor with griddepcontrol.wait).
template <typename K, typename P>
fasa_status launch_pdl(K kern, dim3 grid, int threads, size_t smem, cudaStream_t st, const P& p) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, p));
}

// ------------------------------------------------------------ score

template <typename T, int LPT, bool kHist>
fasa_status launch_score_t(const ScoreParams& p, const DevInfo& d, cudaStream_t st) {
  auto kern = score_kernel<T, LPT, kHist>;
  const int smem = score_smem_bytes();
  int set = 0;
  fasa_status s = cached_int((const void*)kern, 0, &set, [&](int* v) {
    *v = 1;
    return cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  });
  if (s != FASA_OK) return s;
  const int64_t cap = ceil_div(p.total, 256);  // at least 256 tokens per CTA
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(d.sms, cap));
  return launch_pdl(kern, dim3((unsigned)grid, 1, 1), kScoreThreads, (size_t)smem, st, p);
}

template <typename T, bool kHist>
fasa_status launch_score_lpt(const ScoreParams& p, const DevInfo& d, cudaStream_t st) {
  const int lpt = p.stride * (int)sizeof(T) / 16;
  switch (lpt) {
    case 1: return launch_score_t<T, 1, kHist>(p, d, st);
    case 2: return launch_score_t<T, 2, kHist>(p, d, st);
    case 4: return launch_score_t<T, 4, kHist>(p, d, st);
    case 8: return launch_score_t<T, 8, kHist>(p, d, st);
    case 16: return launch_score_t<T, 16, kHist>(p, d, st);
    case 32: return launch_score_t<T, 32, kHist>(p, d, st);
    default: return FASA_ERR_UNSUPPORTED;
  }
}

// TIP scores for every (b, g, t < len); with `hist` also the per-row
// histogram of the top 12 bits of each score's order-preserving key (added
// into `hist`, which must be zero).
fasa_status launch_score(const fasa_cache* c, int32_t len, const void* q, int32_t q_pos, float* scores,
                         int64_t ld, uint32_t* hist, cudaStream_t st, uint32_t* row_done = nullptr,
                         uint32_t* thr = nullptr, int32_t n_keep = 0) {
  DevInfo d;
  fasa_status s = device_info(&d);
  if (s != FASA_OK) return s;
  ScoreParams p{};
  p.sketch = c->sketch;
  p.q = q;
  p.dom_idx = c->dom_idx;
  p.scores = scores;
  p.ld = ld;
  p.hist = hist;
  p.row_done = row_done;
  p.thr = thr;
  p.n_keep = n_keep;
  p.max_len = c->max_len;
  p.total = (int64_t)c->batch * c->n_kv_heads * len;
  p.len = len;
  p.stride = c->sketch_stride;
  p.n_kv_heads = c->n_kv_heads;
  p.group = c->n_q_heads / c->n_kv_heads;
  p.n_dom = c->n_dom;
  fill_query_angle(p.cosv, p.sinv, c->rope_base, q_pos);
  if (c->dtype == FASA_F32)
    return hist ? launch_score_lpt<float, true>(p, d, st) : launch_score_lpt<float, false>(p, d, st);
  return hist ? launch_score_lpt<__nv_bfloat16, true>(p, d, st) : launch_score_lpt<__nv_bfloat16, false>(p, d, st);
}

// ---------------------------------------------------- select / attend

constexpr int kMaxCap = 16384;  // candidate keys per CTA in the sampled selection

inline int maxg_for(int g) { return g <= 4 ? 4 : (g <= 8 ? 8 : 16); }

template <typename T, int MODE, int MAXG>
fasa_status launch_sa_t(SAParams p, int rows, int C, bool pdl, cudaStream_t st, const DevInfo& d) {
  auto kern = select_attend_kernel<T, MODE, MAXG>;
  SALayout L = sa_layout(MODE, (int)sizeof(T), p.chunk, p.slice, p.cap, MAXG, p.n_stages);
  // a smaller candidate buffer only sends more rows to the exact fallback
  while (L.total > d.smem_optin && p.cap > 1024) {
    p.cap /= 2;
    L = sa_layout(MODE, (int)sizeof(T), p.chunk, p.slice, p.cap, MAXG, p.n_stages);
  }
  if (L.total > d.smem_optin) return FASA_ERR_UNSUPPORTED;
  int set = 0;
  fasa_status s = cached_int((const void*)kern, 1, &set, [&](int* v) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, d.smem_optin);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    *v = 1;
    return cuda_status(e);
  });
  if (s != FASA_OK) return s;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attrs[2];
  cfg.gridDim = dim3((unsigned)C, (unsigned)rows, 1);
  cfg.blockDim = dim3(kSAThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)L.total;
  cfg.stream = st;
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = (unsigned)C;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  int na = 1;
  if (pdl) {
    attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[1].val.programmaticStreamSerializationAllowed = 1;
    na = 2;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = na;

  if (C > 8) {  // non-portable cluster size: make sure it can be co-scheduled
    int nclus = 0;
    s = cached_int((const void*)kern, 1000ull + (uint64_t)C * 1000003ull + (uint64_t)L.total, &nclus, [&](int* v) {
      return cuda_status(cudaOccupancyMaxActiveClusters(v, kern, &cfg));
    });
    if (s != FASA_OK) return s;
    if (nclus < 1) return FASA_ERR_UNSUPPORTED;
  }
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, p));
}

template <typename T, int MODE>
fasa_status launch_sa_g(const SAParams& p, int rows, int C, bool pdl, cudaStream_t st, const DevInfo& d) {
  switch (maxg_for(p.group)) {
    case 4: return launch_sa_t<T, MODE, 4>(p, rows, C, pdl, st, d);
    case 8: return launch_sa_t<T, MODE, 8>(p, rows, C, pdl, st, d);
    default: return launch_sa_t<T, MODE, 16>(p, rows, C, pdl, st, d);
  }
}

// Cluster size: enough CTAs to cover the GPU, within the shared-memory
// limits on keys and kept indices per CTA.
int choose_cluster(int mode, int rows, int64_t len, int64_t keep, int sms) {
  int cmin = 1;
  if (mode == kSelect || mode == kDecode) cmin = std::max(cmin, pow2ceil(ceil_div(len, kMaxChunkKeys)));
  if (mode == kDecode || mode == kAttendIdx) cmin = std::max(cmin, pow2ceil(ceil_div(keep, kMaxSlice)));
  const int64_t target = (mode == kDense ? 1 : 2) * (int64_t)sms;
  const int cfill = pow2ceil(ceil_div(target, rows));
  return std::max(cmin, std::min(cfill, kMaxCluster));
}

// Sampling parameters of the selection: stride s (at most kMaxSamples samples
// per row), rank j of the sample used as threshold (k_eff / s plus four
// standard deviations and a constant), candidate capacity.
void choose_sampling(SAParams& p) {
  const int64_t len = p.len, k = p.n_keep;
  int s = 8;
  while (ceil_div(len, s) > kMaxSamples) s <<= 1;
  const int64_t m = ceil_div(len, s);
  const int64_t mu = ceil_div(k, s);
  const int64_t j = mu + (int64_t)std::ceil(4.0 * std::sqrt((double)mu)) + 4;
  p.sample_stride = s;
  if (j >= m) {
    p.sample_rank = (int)m;  // no sampling: every key is a candidate
    p.cap = (int)std::min<int64_t>(kMaxCap, std::max<int64_t>(1024, pow2ceil(len)));
  } else {
    p.sample_rank = (int)j;
    const int64_t expect = (j + (int64_t)std::ceil(3.0 * std::sqrt((double)j)) + 2) * s;
    p.cap = (int)std::min<int64_t>(kMaxCap, std::max<int64_t>(1024, pow2ceil(expect)));
  }
}

template <int MODE>
fasa_status launch_sa(const fasa_cache* c, SAParams p, int rows, bool pdl, cudaStream_t st, int dtype,
                      int32_t q_pos) {
  DevInfo d;
  fasa_status s = device_info(&d);
  if (s != FASA_OK) return s;
  int C = choose_cluster(MODE, rows, p.len, p.n_keep, d.sms);
  if (C > kMaxCluster) return FASA_ERR_UNSUPPORTED;
  if (c) fill_query_angle(p.cosv, p.sinv, c->rope_base, q_pos);
  if (MODE == kSelect || MODE == kDecode) choose_sampling(p);
  p.n_stages = (MODE == kDense) ? 4 : 2;
  for (;;) {
    p.chunk = (int)ceil_div(p.len, C);
    p.slice = (int)ceil_div(p.n_keep, C);
    if constexpr (MODE == kSelect) {
      s = launch_sa_t<float, MODE, 4>(p, rows, C, pdl, st, d);
    } else {
      if (dtype == FASA_F32)
        s = launch_sa_g<float, MODE>(p, rows, C, pdl, st, d);
      else
        s = launch_sa_g<__nv_bfloat16, MODE>(p, rows, C, pdl, st, d);
    }
    // a 16-CTA cluster that cannot be co-scheduled: retry with 8 when allowed
    if (s == FASA_ERR_UNSUPPORTED && C == 16) {
      const int cmin = choose_cluster(MODE, 1 << 30, p.len, p.n_keep, d.sms);
      if (cmin <= 8) {
        C = 8;
        continue;
      }
    }
    return s;
  }
}

// Device address of this device's g_static_scratch, looked up once per
// device with that device current.
void* g_static_scratch_addr[kMaxDevices] = {nullptr};

fasa_status static_scratch_addr(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FASA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_static_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || p == nullptr) return cuda_status(e == cudaSuccess ? cudaErrorInvalidSymbol : e);
    g_static_scratch_addr[dev] = p;
  }
  *out = g_static_scratch_addr[dev];
  return FASA_OK;
}

// ------------------------------------------------- wide fused decode

std::atomic<int> g_decode_path{FASA_DECODE_AUTO};

// Launch plan of the wide fused decode (decode_wide.cuh).
struct WidePlan {
  int n_split = 0, n_loc = 0, n_pub = 0, direct = 0, ucache = 0, ushift = 0, smem = 0;
};

template <int LPT, int MG>
fasa_status wide_attrs(const DevInfo& d) {
  auto kern = decode_wide_kernel<LPT, MG>;
  int set = 0;
  return cached_int((const void*)kern, 0, &set, [&](int* v) {
    *v = 1;
    return cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, d.smem_optin));
  });
}

// Published-candidate slots per row in the decode workspace: the CTAs'
// regions (n_split * (n_loc + 1) entries) stay within len + len/64 + 64.
inline int64_t wide_region_slots(int64_t len) { return len + len / 64 + 64; }

// Device view of a paged cache's block table (table null: contiguous).
PageMap page_map(const fasa_cache* c, const fasa_paged* pg) {
  PageMap m{};
  m.n_kv_heads = c->n_kv_heads;
  if (pg == nullptr) return m;
  m.table = pg->block_table;
  m.max_blocks = pg->max_blocks;
  m.n_pages = pg->n_pages;
  int l = 0;
  while ((1 << l) < pg->block_size) ++l;
  m.log2bs = l;
  return m;
}

// Host checks of a paged description against the cache.
fasa_status check_paged(const fasa_cache* c, const fasa_paged* pg) {
  if (pg == nullptr || !aligned(pg->block_table, 4)) return FASA_ERR_INVALID_ARG;
  const int32_t bs = pg->block_size;
  if (bs < 16 || bs > (1 << 16) || (bs & (bs - 1)) != 0) return FASA_ERR_INVALID_ARG;
  if (pg->max_blocks < 1 || pg->n_pages < 1) return FASA_ERR_INVALID_ARG;
  if ((int64_t)pg->max_blocks * bs != c->max_len) return FASA_ERR_INVALID_ARG;
  // pool rows are addressed with 32-bit indices
  if ((int64_t)pg->n_pages * c->n_kv_heads * bs > INT32_MAX) return FASA_ERR_UNSUPPORTED;
  return FASA_OK;
}

// CTAs per row: about one per SM over all rows (never fewer than the
// shared-memory limit on keys per CTA allows); tokens per CTA. The
// resolving CTA attends itself for budgets up to kWdMaxDirect when its ring
// fits, and caches as much of the published union as shared memory allows.
bool wide_plan(const fasa_cache* c, int32_t len, int32_t keff, const DevInfo& d, WidePlan* pl, int paged = 0,
               int n_q = 0) {
  if (c->dtype != FASA_BF16) return false;
  const int64_t rows = (int64_t)c->batch * c->n_kv_heads;
  // about one CTA per SM, leaving one SM per row free: the rows' resolving
  // CTAs then never hold back a CTA of the next launch
  int64_t S = std::max<int64_t>(1, (d.sms - std::min<int64_t>(rows, d.sms / 2)) / rows);
  S = std::max<int64_t>(S, ceil_div(len, kWdMaxLoc));
  S = std::min<int64_t>(S, std::max<int64_t>(1, ceil_div(len, 256)));
  pl->n_split = (int)S;
  pl->n_loc = (int)ceil_div(len, S);
  if (pl->n_loc > kWdMaxLoc || S > 65535) return false;
  if ((int64_t)pl->n_split * (pl->n_loc + 1) > wide_region_slots(len)) return false;
  // each CTA publishes about twice its expected share of the kept set (and
  // the rest of its boundary bin); the resolving CTA falls back to every key
  // of the row when a CTA turns out to hold more of the kept set than that
  pl->n_pub = pl->n_split == 1 ? keff
                                : (int)std::min<int64_t>(keff, (2 * ceil_div(keff, pl->n_split) + 32 + 31) / 32 * 32);
  const int G = c->n_q_heads / c->n_kv_heads;
  // n_q > 0: the multi-query decode (n_q tokens, the attention in its own launch)
  const int nq = n_q > 0 ? n_q : 1;
  // K and V in host memory (FASA-M): the kept rows cross the host link
  // faster from the split-K attention's many CTAs than through the one
  // resolving CTA (measured at c2: 51.5 us against 62.1 us per layer)
  const bool in_cta = keff <= kWdMaxDirect && G <= 8 && n_q == 0 && !kv_on_host(c);
  for (int direct = in_cta ? 1 : 0; direct >= 0; --direct) {
    const WdLayout base = wd_layout(pl->n_loc, len, keff, direct, G, pl->n_split, 0, paged, nq);
    if (base.total > d.smem_optin) continue;
    // entries of each CTA's region the resolving CTA stages in shared memory:
    // a power of two covering what a CTA usually publishes (its k_eff best
    // and the rest of their bin), as far as shared memory allows
    const int64_t room = std::max<int64_t>(1, (int64_t)(d.smem_optin - base.ucache) / (8 * pl->n_split));
    const int64_t want = std::min<int64_t>(pl->n_loc, (int64_t)pl->n_pub + pl->n_pub / 4 + 32);
    int64_t P = 1;
    while (P < want && 2 * P <= room) P *= 2;
    pl->direct = direct;
    pl->ucache = (int)P;
    pl->ushift = 0;
    while ((1 << pl->ushift) < P) ++pl->ushift;
    pl->smem = wd_layout(pl->n_loc, len, keff, direct, G, pl->n_split, pl->ucache, paged, nq).total;
    if (pl->smem > d.smem_optin) continue;
    return true;
  }
  return false;
}

// The plan fasa_decode picks by itself: the fused plan while each row can
// have about eight or more SMs and its budget stays small enough for the
// one resolving CTA of a row to select it quickly (measured on B200: c2, 8
// rows, 21.3 us fused against 35 us staged at k 256, 27.9 against 30.7 at
// k 1024; 64 and 512 rows 20% faster staged, where the fused plan's
// per-row resolving CTAs no longer pay; 16 rows at k 6193 58.7 us fused
// against 52.2 staged).
constexpr int kFusedMaxKeep = 1024;
inline bool fused_preferred(const fasa_cache* c, int keff, const DevInfo& d) {
  return (int64_t)c->batch * c->n_kv_heads * 8 <= d.sms && keff <= kFusedMaxKeep;
}

template <int LPT, int MG>
fasa_status launch_wide_t(const WideParams& p, int rows, const WidePlan& pl, cudaStream_t st, const DevInfo& d) {
  auto kern = decode_wide_kernel<LPT, MG>;
  fasa_status s = wide_attrs<LPT, MG>(d);
  if (s != FASA_OK) return s;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attrs[1];
  cfg.gridDim = dim3((unsigned)pl.n_split, (unsigned)rows, 1);
  cfg.blockDim = dim3(kWdThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)pl.smem;
  cfg.stream = st;
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, p));
}

// Decode workspace, each part 256-byte aligned:
//   zero between calls (every call leaves them zero), at offsets fixed by
//   the row count: sem [rows] u64 | att_cnt [rows] u32 |
//     hist [rows][4096] u32, cnt [rows], thr [rows][2], rdone [rows] (staged plan) |
//   scores [rows][ld] f32 (ld = len rounded up to 32), or, in the fused plan,
//     the CTAs' published candidates [rows][len + len/64 + 64] u32x2 |
//   keys [rows][len] u32 (fused plan: every token's score key) | rowk [rows] i32 (varlen: each row's k_eff) |
//   bitmap [rows][ceil(len/32)] u32 | cand_idx [rows][cap] i32 | cand_key [rows][cap] u32 |
//   idx [rows][k_eff] i32 | part [rows][splits_max][kCcPartStride] f32
constexpr int kAssumedMaxSms = 256;  // sizes the split-K partials for any GPU
constexpr int kAttMaxPerSm = 4;      // attention CTAs resident per SM, an upper bound
constexpr int kAttUnit = kCcWarps * kCcStep;  // kept rows per CTA step of the attention
struct DecodeWs {
  size_t sem, att_cnt, scores, keys, rowk, hist, cnt, thr, rdone, bitmap, cand, ckey, idx, part, total;
  int64_t ld;
  int cap, words, splits_max;
};
inline size_t al256(size_t x) { return (x + 255) / 256 * 256; }
inline int att_chunks(int keff) { return (keff + kAttUnit - 1) / kAttUnit; }
// Splits per row so that the attention grid fills, without exceeding, one
// wave of resident CTAs; at most kCcMaxSplits, whose merge state fits in
// the kernel's shared memory.
inline int att_splits(int rows, int keff, int sms, int per_sm) {
  const int64_t s = std::min<int64_t>(att_chunks(keff), (int64_t)per_sm * sms / rows);
  return (int)std::max<int64_t>(1, std::min<int64_t>(s, kCcMaxSplits));
}
DecodeWs decode_layout(const fasa_cache* c, int32_t len, int32_t k) {
  DecodeWs w;
  const size_t rows = (size_t)c->batch * c->n_kv_heads;
  const size_t L = (size_t)std::max(len, 0);
  const int keff = std::max(0, std::min(k, len));
  w.words = (int)((L + 31) / 32);
  w.cap = (int)std::min<size_t>(std::max<size_t>(L, 1), 8192);
  w.splits_max = att_splits((int)rows, std::max(keff, 1), kAssumedMaxSms, kAttMaxPerSm);
  w.ld = (int64_t)((L + 31) / 32 * 32);
  // the parts that must be zero between calls first, at offsets that depend
  // on the row count only: a workspace sized for the largest len and k
  // serves calls at any smaller len and k
  w.sem = 0;
  w.att_cnt = rows * 8;
  w.hist = al256(w.att_cnt + rows * 4);
  w.cnt = w.hist + rows * kHistBins * 4;
  w.thr = w.cnt + rows * 4;
  w.rdone = w.thr + rows * 8;
  w.scores = al256(w.rdone + rows * 4);
  w.keys = al256(w.scores + rows * std::max<size_t>((size_t)w.ld * 4, (size_t)wide_region_slots((int64_t)L) * 8));
  w.rowk = al256(w.keys + rows * L * 4);
  w.bitmap = al256(w.rowk + rows * 4);
  w.cand = al256(w.bitmap + rows * (size_t)w.words * 4);
  w.ckey = al256(w.cand + rows * (size_t)w.cap * 4);
  w.idx = al256(w.ckey + rows * (size_t)w.cap * 4);
  w.part = al256(w.idx + rows * (size_t)keff * 4);
  w.total = al256(w.part + rows * (size_t)w.splits_max * kCcPartStride * 4) + 256;
  return w;
}
size_t decode_ws(const fasa_cache* c, int32_t len, int32_t k) { return decode_layout(c, len, k).total; }


// Calibration workspace: score planes [rows][n_win][65][len] f32, then the
// selections [rows][n_win][65][k_eff] i32.
struct CalWs {
  size_t planes, idx, total;
};
CalWs cal_layout(int64_t rows, int32_t len, int32_t n_win, int32_t budget) {
  CalWs w;
  const int64_t keff = std::min<int64_t>(budget, len);
  w.planes = 0;
  w.idx = al256((size_t)rows * n_win * kCalPlanes * (size_t)len * 4);
  w.total = al256(w.idx + (size_t)rows * n_win * kCalPlanes * (size_t)keff * 4);
  return w;
}

template <typename T>
fasa_status launch_cal_scores(const fasa_cache* c, int32_t len, const void* q_win, int32_t q_pos0, int32_t n_win,
                              float* planes, cudaStream_t st) {
  CalScoreParams p{};
  p.k = c->k;
  p.q = q_win;
  p.planes = planes;
  p.max_len = c->max_len;
  p.len = len;
  p.n_win = n_win;
  p.n_kv_heads = c->n_kv_heads;
  p.group = c->n_q_heads / c->n_kv_heads;
  for (int w = 0; w < n_win; ++w) fill_query_angle(p.cosv[w], p.sinv[w], c->rope_base, q_pos0 + w);
  const dim3 grid((unsigned)ceil_div(len, kCalThreads), (unsigned)(c->batch * c->n_kv_heads), 1);
  calib_score_kernel<T><<<grid, kCalThreads, 0, st>>>(p);
  return cuda_status(cudaGetLastError());
}

// Split-K attention of every row over its kept list idx [rows][n_keep], or
// over rows 0 .. n_keep-1 when idx is null (the dense decode): the
// tensor-core kernel (attend_mma_kernel) for groups of up to 8 query heads,
// the CUDA-core one (attend_cc_kernel) for larger groups. Every CTA forms its
// group's queries from q. A row whose list is split over several CTAs leaves
// partials in part [rows][splits_max][kCcPartStride], and a second launch
// (attend_merge_kernel) merges them.
struct AttendKernel {
  const void* fn;
  int threads, smem;
};
AttendKernel attend_kernel(int group, int nw) {
  if (group > 8) return {(const void*)attend_cc_kernel<16>, kCcThreads, cc_smem_bytes(16)};
  if (nw == 2) return {(const void*)attend_mma_kernel<2>, 64, am_smem_bytes(2)};
  return {(const void*)attend_mma_kernel<4>, 128, am_smem_bytes(4)};
}

fasa_status attend_per_sm(const AttendKernel& k, int* per_sm) {
  fasa_status s = cached_int(k.fn, 7, per_sm, [&](int* v) {
    cudaError_t e = cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, k.smem);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(v, k.fn, k.threads, (size_t)k.smem);
    return cuda_status(e);
  });
  *per_sm = std::max(1, *per_sm);
  return s;
}

// Splits per row of the attention over n_keep list positions: one wave of
// resident CTAs at most, each with at least one step per warp; sets the
// slice (list positions per CTA) too. *nw: warps per CTA of the tensor-core
// kernel, 2 when the rows alone (one split each) would overfill a wave of
// 4-warp CTAs but fill one of 2-warp CTAs, for short lists (at most
// kAm2MaxKeep positions: c5's kept lists; the dense decode's 16K-row lists
// stream faster from 4-warp CTAs, 596 against 658 us).
constexpr int kAm2MaxKeep = 2048;
fasa_status attend_split(int group, int rows, int n_keep, int splits_max, const DevInfo& d, int* splits, int* slice,
                         int* nw) {
  int per_sm = 0;
  fasa_status s = attend_per_sm(attend_kernel(group, 4), &per_sm);
  if (s != FASA_OK) return s;
  constexpr int kUnit = kCcWarps * kCcStep;
  const int64_t units = std::max<int64_t>(1, ceil_div(n_keep, kUnit));
  int64_t sp = std::min<int64_t>(units, std::max<int64_t>(1, (int64_t)per_sm * d.sms / rows));
  sp = std::min<int64_t>(sp, std::min<int64_t>(splits_max, kCcMaxSplits));
  sp = std::max<int64_t>(sp, 1);
  *slice = (int)(ceil_div(units, sp) * kUnit);
  *splits = (int)ceil_div(std::max(n_keep, 1), *slice);
  *nw = 4;
  if (group <= 8 && *splits == 1 && n_keep <= kAm2MaxKeep && (int64_t)rows > (int64_t)per_sm * d.sms) {
    int per_sm2 = 0;
    if ((s = attend_per_sm(attend_kernel(group, 2), &per_sm2)) != FASA_OK) return s;
    if ((int64_t)rows <= (int64_t)per_sm2 * d.sms) *nw = 2;
  }
  return FASA_OK;
}

fasa_status launch_attend_k(CcParams& ap, int rows, int splits_max, const DevInfo& d, cudaStream_t st) {
  int nw = 4;
  fasa_status s = attend_split(ap.group, rows, ap.n_keep, splits_max, d, &ap.splits, &ap.slice, &nw);
  if (s != FASA_OK) return s;
  const dim3 grid((unsigned)ap.splits, (unsigned)rows, 1);
  if (ap.group > 8)
    s = launch_pdl(attend_cc_kernel<16>, grid, kCcThreads, (size_t)cc_smem_bytes(16), st, ap);
  else if (nw == 2)
    s = launch_pdl(attend_mma_kernel<2>, grid, 64, (size_t)am_smem_bytes(2), st, ap);
  else
    s = launch_pdl(attend_mma_kernel<4>, grid, 128, (size_t)am_smem_bytes(4), st, ap);
  if (s != FASA_OK || ap.splits == 1) return s;
  MergeParams mp{ap.part, ap.out, ap.splits, ap.group};
  return launch_pdl(attend_merge_kernel, dim3((unsigned)ap.group, (unsigned)rows, 1), kMgThreads, 0, st, mp);
}

fasa_status launch_attend(const fasa_cache* c, int32_t len, int n_keep, void* out, const int32_t* idx,
                          const void* q, int32_t q_pos, float* part, int splits_max,
                          const DevInfo& d, cudaStream_t st, const fasa_varlen* vl = nullptr,
                          const int32_t* row_keep = nullptr, const fasa_paged* pg = nullptr) {
  const int rows = c->batch * c->n_kv_heads;
  CcParams ap{};
  ap.k = static_cast<const __nv_bfloat16*>(c->k);
  ap.v = static_cast<const __nv_bfloat16*>(c->v);
  ap.idx = idx;
  ap.q = static_cast<const __nv_bfloat16*>(q);
  ap.out = static_cast<__nv_bfloat16*>(out);
  ap.part = part;
  ap.max_len = c->max_len;
  ap.len = len;
  ap.n_keep = n_keep;
  ap.group = c->n_q_heads / c->n_kv_heads;
  ap.n_kv_heads = c->n_kv_heads;
  ap.pm = page_map(c, pg);
  if (vl) {  // per-row lengths and kept counts; the angles from the lengths on the device
    ap.seq_len = vl->seq_len;
    ap.row_keep = row_keep;
    ap.q_prerot = vl->q_prerotated;
    fill_theta(ap.cosv, c->rope_base);
  } else {
    fill_query_angle(ap.cosv, ap.sinv, c->rope_base, q_pos);
  }
  return launch_attend_k(ap, rows, splits_max, d, st);
}

// The decode's attention over the kept lists in the workspace.
fasa_status launch_attend_ws(const fasa_cache* c, int32_t len, int keff, const void* q, int32_t q_pos, void* out,
                             const DecodeWs& w, char* base, const DevInfo& d, cudaStream_t st,
                             const fasa_varlen* vl = nullptr, const fasa_paged* pg = nullptr) {
  return launch_attend(c, len, keff, out, reinterpret_cast<const int32_t*>(base + w.idx), q, q_pos,
                       reinterpret_cast<float*>(base + w.part), w.splits_max, d, st, vl,
                       reinterpret_cast<const int32_t*>(base + w.rowk), pg);
}

// Dense decode workspace: att_cnt [rows] u32 (zero between calls) | part
// [rows][splits_max][kCcPartStride] f32.
struct DenseWs {
  size_t att_cnt, part, total;
  int splits_max;
};
DenseWs dense_layout(const fasa_cache* c, int32_t len) {
  DenseWs w;
  const size_t rows = (size_t)c->batch * c->n_kv_heads;
  w.splits_max = att_splits((int)rows, std::max(len, 1), kAssumedMaxSms, kAttMaxPerSm);
  w.att_cnt = 0;
  w.part = al256(rows * 4);
  w.total = al256(w.part + rows * (size_t)w.splits_max * kCcPartStride * 4) + 256;
  return w;
}

// The append kernel's launch: every sequence at pos0, or at pos0v[b].
fasa_status launch_append(const fasa_cache* c, const void* k_new, const void* v_new, int32_t n_new, int32_t pos0,
                          const int32_t* pos0v, const fasa_paged* pg, const DevInfo& d, cudaStream_t stream) {
  AppendParams p{};
  p.k_new = k_new;
  p.v_new = v_new;
  p.k = c->k;
  p.v = c->v;
  p.sketch = c->sketch;
  p.dom_idx = c->dom_idx;
  p.max_len = c->max_len;
  p.n_rows = c->batch * c->n_kv_heads;
  p.n_kv_heads = c->n_kv_heads;
  p.n_new = n_new;
  p.pos0 = pos0;
  p.pos0v = pos0v;
  p.pm = page_map(c, pg);
  p.n_dom = c->n_dom;
  p.stride = c->sketch_stride;
  fill_theta(p.theta, c->rope_base);
  const int64_t tok_blocks = ceil_div(n_new, kAppendTok);
  const int64_t groups = std::max<int64_t>(1, std::min<int64_t>(p.n_rows, ceil_div(4LL * d.sms, tok_blocks)));
  p.heads_per_cta = (int)ceil_div(p.n_rows, groups);
  const dim3 grid((unsigned)tok_blocks, (unsigned)ceil_div(p.n_rows, p.heads_per_cta), 1);
  if (c->dtype == FASA_F32)
    append_kernel<float><<<grid, kAppendThreads, 0, stream>>>(p);
  else
    append_kernel<__nv_bfloat16><<<grid, kAppendThreads, 0, stream>>>(p);
  return cuda_status(cudaGetLastError());
}

// Multi-query decode workspace: the decode workspace, then the tensor-core
// attention's split partials [rows][splits][kTcPartStride] f32.
struct MultiWs {
  DecodeWs w;
  size_t tpart, total;
  int splits_max;
};
inline int tc_splits(int rows, int keff, int sms) {
  const int64_t tiles = ceil_div(std::max(keff, 1), kTcTile);
  const int64_t s = std::min<int64_t>(tiles, std::max<int64_t>(1, (int64_t)sms / rows));
  return (int)std::max<int64_t>(1, std::min<int64_t>(s, kTcMaxSplits));
}
MultiWs multi_layout(const fasa_cache* c, int32_t len, int32_t k) {
  MultiWs m;
  m.w = decode_layout(c, len, k);
  const size_t rows = (size_t)c->batch * c->n_kv_heads;
  m.splits_max = tc_splits((int)rows, std::max(0, std::min(k, len)), kAssumedMaxSms);
  m.tpart = al256(m.w.total);
  m.total = al256(m.tpart + rows * (size_t)m.splits_max * kTcPartStride * 4) + 256;
  return m;
}

fasa_status launch_tc(const fasa_cache* c, int32_t len, int keff, const void* q, int32_t q_pos0, int32_t n_q,
                      void* out, const MultiWs& m, char* base, const DevInfo& d, cudaStream_t st) {
  const int rows = c->batch * c->n_kv_heads;
  TcParams tp{};
  tp.k = static_cast<const __nv_bfloat16*>(c->k);
  tp.v = static_cast<const __nv_bfloat16*>(c->v);
  tp.idx = reinterpret_cast<const int32_t*>(base + m.w.idx);
  tp.q = static_cast<const __nv_bfloat16*>(q);
  tp.out = static_cast<__nv_bfloat16*>(out);
  tp.part = reinterpret_cast<float*>(base + m.tpart);
  tp.counter = reinterpret_cast<uint32_t*>(base + m.w.att_cnt);
  tp.max_len = c->max_len;
  tp.len = len;
  tp.n_keep = keff;
  tp.group = c->n_q_heads / c->n_kv_heads;
  tp.n_q = n_q;
  tp.n_kv_heads = c->n_kv_heads;
  tp.q_prerot = q_pos0 == FASA_Q_PREROTATED ? 1 : 0;
  tp.q_pos0 = tp.q_prerot ? 0 : q_pos0;
  fill_theta(tp.theta, c->rope_base);
  const int splits = std::min(m.splits_max, tc_splits(rows, keff, d.sms));
  const int64_t tiles = ceil_div(keff, kTcTile);
  tp.slice = (int)(ceil_div(tiles, splits) * kTcTile);
  tp.splits = (int)ceil_div(keff, tp.slice);
  const int smem = tc_smem_bytes(n_q * tp.group, n_q);
  int ok = 0;
  fasa_status s = cached_int(reinterpret_cast<const void*>(attend_tc_kernel), 0, &ok, [&](int* r) {
    *r = 1;
    return cuda_status(cudaFuncSetAttribute(attend_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            tc_smem_bytes(kTcMaxRows, kTcMaxTok)));
  });
  if (s != FASA_OK) return s;
  return launch_pdl(attend_tc_kernel, dim3((unsigned)tp.splits, (unsigned)rows, 1), kTcThreads, (size_t)smem, st,
                    tp);
}

// The fused kernel's instance for the sketch row length (16-byte chunks) and
// the padded head count of its in-CTA attention.
fasa_status launch_wide_sel(const WideParams& p, int rows, const WidePlan& pl, const DevInfo& d, cudaStream_t st) {
  const bool g4 = p.group <= 4;  // padded heads of the in-CTA attention: 4 or 8
  switch (p.stride / 8) {
    case 1: return g4 ? launch_wide_t<1, 4>(p, rows, pl, st, d) : launch_wide_t<1, 8>(p, rows, pl, st, d);
    case 2: return g4 ? launch_wide_t<2, 4>(p, rows, pl, st, d) : launch_wide_t<2, 8>(p, rows, pl, st, d);
    case 4: return g4 ? launch_wide_t<4, 4>(p, rows, pl, st, d) : launch_wide_t<4, 8>(p, rows, pl, st, d);
    case 8: return g4 ? launch_wide_t<8, 4>(p, rows, pl, st, d) : launch_wide_t<8, 8>(p, rows, pl, st, d);
    case 16: return g4 ? launch_wide_t<16, 4>(p, rows, pl, st, d) : launch_wide_t<16, 8>(p, rows, pl, st, d);
    default: return FASA_ERR_UNSUPPORTED;
  }
}

// The wide fused decode: one launch, plus the split-K attention when the
// budget is beyond what the resolving CTA attends itself.
fasa_status launch_wide(const fasa_cache* c, int32_t len, const void* q, int32_t q_pos, int keff, void* out,
                        int32_t* idx_out, const DecodeWs& w, char* base, const WidePlan& pl, const DevInfo& d,
                        cudaStream_t st, const fasa_varlen* vl = nullptr, const fasa_paged* pg = nullptr) {
  WideParams p{};
  p.pm = page_map(c, pg);
  p.n_q = 1;
  p.sketch = static_cast<const __nv_bfloat16*>(c->sketch);
  p.k = static_cast<const __nv_bfloat16*>(c->k);
  p.v = static_cast<const __nv_bfloat16*>(c->v);
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.dom_idx = c->dom_idx;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.idx_out = idx_out;
  p.idx_ws = pl.direct ? nullptr : reinterpret_cast<int32_t*>(base + w.idx);
  p.cand = reinterpret_cast<uint2*>(base + w.scores);
  p.sem = reinterpret_cast<unsigned long long*>(base + w.sem);
  p.max_len = c->max_len;
  p.len = len;
  p.stride = c->sketch_stride;
  p.n_kv_heads = c->n_kv_heads;
  p.group = c->n_q_heads / c->n_kv_heads;
  p.n_dom = c->n_dom;
  p.n_keep = keff;
  p.n_pub = pl.n_pub;
  p.keys = reinterpret_cast<uint32_t*>(base + w.keys);
  p.n_loc = pl.n_loc;
  p.n_split = pl.n_split;
  p.ucache = pl.ucache;
  p.ushift = pl.ushift;
  p.direct = pl.direct;
  if (vl) {  // per-sequence lengths and per-head budgets; len and keff are their bounds
    p.seq_len = vl->seq_len;
    p.budget = vl->budget;
    p.row_keep = pl.direct ? nullptr : reinterpret_cast<int32_t*>(base + w.rowk);
    p.q_prerot = vl->q_prerotated;
    fill_theta(p.cosv, c->rope_base);
  } else {
    fill_query_angle(p.cosv, p.sinv, c->rope_base, q_pos);
  }
  const fasa_status s = launch_wide_sel(p, c->batch * c->n_kv_heads, pl, d, st);
  if (s != FASA_OK || pl.direct) return s;
  return launch_attend_ws(c, len, keff, q, q_pos, out, w, base, d, st, vl, pg);
}

}  // namespace

// =================================================================== ABI

extern "C" {

int32_t fasa_abi_version(void) { return FASA_ABI_VERSION; }

const char* fasa_last_cuda_error(void) { return t_last_cuda_error; }

const char* fasa_status_string(int32_t s) {
  switch (s) {
    case FASA_OK: return "FASA_OK";
    case FASA_ERR_INVALID_ARG: return "FASA_ERR_INVALID_ARG";
    case FASA_ERR_UNSUPPORTED: return "FASA_ERR_UNSUPPORTED";
    case FASA_ERR_CAPACITY: return "FASA_ERR_CAPACITY";
    case FASA_ERR_WORKSPACE: return "FASA_ERR_WORKSPACE";
    case FASA_ERR_CUDA: return "FASA_ERR_CUDA";
    case FASA_ERR_TIMEOUT: return "FASA_ERR_TIMEOUT";
    case FASA_ERR_BAD_INDEX: return "FASA_ERR_BAD_INDEX";
    default: return "FASA_ERR_UNKNOWN";
  }
}

int32_t fasa_sketch_stride(int32_t n_dom, int32_t dtype) {
  if (n_dom < 1 || n_dom > kNFC) return -1;
  if (dtype != FASA_F32 && dtype != FASA_BF16) return -1;
  const int per16 = 16 / elem_bytes(dtype);
  const int chunks = pow2ceil(ceil_div(2 * n_dom, per16));
  return chunks * per16;
}

fasa_status fasa_check_dom_idx(const int32_t* dom, int32_t n_kv_heads, int32_t n_dom) {
  if (dom == nullptr || n_kv_heads < 1 || n_dom < 1 || n_dom > kNFC) return FASA_ERR_INVALID_ARG;
  for (int g = 0; g < n_kv_heads; ++g) {
    bool seen[kNFC] = {false};
    for (int j = 0; j < n_dom; ++j) {
      const int v = dom[g * n_dom + j];
      if (v < 0 || v >= kNFC || seen[v]) return FASA_ERR_INVALID_ARG;
      seen[v] = true;
    }
  }
  return FASA_OK;
}

fasa_status fasa_host_kv_pointer(void* host, void** dev) {
  if (host == nullptr || dev == nullptr) return FASA_ERR_INVALID_ARG;
  void* d = nullptr;
  const cudaError_t e = cudaHostGetDevicePointer(&d, host, 0);
  if (e != cudaSuccess || d == nullptr) {
    (void)cudaGetLastError();
    return FASA_ERR_INVALID_ARG;
  }
  *dev = d;
  return FASA_OK;
}

fasa_status fasa_append_kv(const fasa_cache* c, const void* k_new, const void* v_new, int32_t n_new,
                           int32_t pos0, cudaStream_t stream) {
  fasa_status s = check_cache(c);
  if (s != FASA_OK) return s;
  if (n_new < 0 || pos0 < 0) return FASA_ERR_INVALID_ARG;
  if ((int64_t)pos0 + n_new > c->max_len) return FASA_ERR_CAPACITY;
  if (n_new == 0) return FASA_OK;
  if (!aligned(k_new, 16) || !aligned(v_new, 16)) return FASA_ERR_INVALID_ARG;
  DevInfo d;
  if ((s = device_info(&d)) != FASA_OK) return s;
  return launch_append(c, k_new, v_new, n_new, pos0, nullptr, nullptr, d, stream);
}

fasa_status fasa_score(const fasa_cache* c, int32_t len, const void* q, int32_t q_pos, float* scores,
                       cudaStream_t stream) {
  fasa_status s = check_cache(c);
  if (s != FASA_OK) return s;
  if (len < 0 || bad_qpos(q_pos)) return FASA_ERR_INVALID_ARG;
  if (len > c->max_len) return FASA_ERR_CAPACITY;
  if (len == 0) return FASA_OK;
  if (!aligned(q, 16) || !aligned(scores, 4)) return FASA_ERR_INVALID_ARG;
  return launch_score(c, len, q, q_pos, scores, len, nullptr, stream);
}

fasa_status fasa_select_topk(const float* scores, int32_t n_rows, int32_t len, int32_t k, int32_t* idx,
                             cudaStream_t stream) {
  if (!aligned(scores, 4) || !aligned(idx, 4)) return FASA_ERR_INVALID_ARG;
  if (n_rows < 1 || len < 1 || k < 1) return FASA_ERR_INVALID_ARG;
  if (len > FASA_MAX_LEN || k > FASA_MAX_K || n_rows > 65535) return FASA_ERR_UNSUPPORTED;
  SAParams p{};
  p.scores = scores;
  p.idx_out = idx;
  p.len = len;
  p.n_keep = std::min(k, len);
  p.group = 1;
  return launch_sa<kSelect>(nullptr, p, n_rows, false, stream, FASA_F32, 0);
}

fasa_status fasa_sparse_attend(const fasa_cache* c, int32_t len, const void* q, int32_t q_pos,
                               const int32_t* idx, int32_t n_idx, void* out, cudaStream_t stream) {
  fasa_status s = check_cache(c);
  if (s != FASA_OK) return s;
  if (len < 1 || bad_qpos(q_pos) || n_idx < 1) return FASA_ERR_INVALID_ARG;
  if (len > c->max_len) return FASA_ERR_CAPACITY;
  if (n_idx > FASA_MAX_K) return FASA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(idx, 4)) return FASA_ERR_INVALID_ARG;
  SAParams p{};
  p.idx_in = idx;
  p.k = c->k;
  p.v = c->v;
  p.q = q;
  p.out = out;
  p.max_len = c->max_len;
  p.len = len;
  p.n_keep = n_idx;
  p.n_kv_heads = c->n_kv_heads;
  p.group = c->n_q_heads / c->n_kv_heads;
  return launch_sa<kAttendIdx>(c, p, c->batch * c->n_kv_heads, false, stream, c->dtype, q_pos);
}

size_t fasa_decode_workspace_bytes(const fasa_cache* c, int32_t len, int32_t k) {
  if (check_cache(c) != FASA_OK || len < 0 || k < 0) return 0;
  return decode_ws(c, len, k);
}

fasa_status fasa_decode(const fasa_cache* c, int32_t len, const void* q, int32_t q_pos, int32_t k, void* out,
                        int32_t* idx_out, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  fasa_status s = check_cache(c);
  if (s != FASA_OK) return s;
  if (len < 1 || bad_qpos(q_pos) || k < 1) return FASA_ERR_INVALID_ARG;
  if (len > c->max_len) return FASA_ERR_CAPACITY;
  if (len > FASA_MAX_LEN || k > FASA_MAX_K) return FASA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(out, 16)) return FASA_ERR_INVALID_ARG;
  if (idx_out != nullptr && !aligned(idx_out, 4)) return FASA_ERR_INVALID_ARG;
  const DecodeWs w = decode_layout(c, len, k);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < w.total) return FASA_ERR_WORKSPACE;
  DevInfo d;
  if ((s = device_info(&d)) != FASA_OK) return s;
  const int rows = c->batch * c->n_kv_heads;
  const int keff = std::min(k, len);
  const int path = g_decode_path.load();
  char* base = static_cast<char*>(workspace);
  if ((path == FASA_DECODE_AUTO && fused_preferred(c, keff, d)) || path == FASA_DECODE_FUSED) {
    WidePlan pl;
    if (wide_plan(c, len, keff, d, &pl)) return launch_wide(c, len, q, q_pos, keff, out, idx_out, w, base, pl, d, stream);
    if (path == FASA_DECODE_FUSED) return FASA_ERR_UNSUPPORTED;
  }
  float* scores = reinterpret_cast<float*>(base + w.scores);
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + w.hist);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(base + w.cnt);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(base + w.bitmap);
  int32_t* cand = reinterpret_cast<int32_t*>(base + w.cand);
  uint32_t* ckey = reinterpret_cast<uint32_t*>(base + w.ckey);
  int32_t* idx = reinterpret_cast<int32_t*>(base + w.idx);

  // 1. TIP scores, the per-row key histogram and its threshold bin (the
  // histograms, candidate counters and row tickets are zero between calls:
  // the score kernel and finalize leave them so)
  uint32_t* thr = reinterpret_cast<uint32_t*>(base + w.thr);
  if ((s = launch_score(c, len, q, q_pos, scores, w.ld, hist, stream, reinterpret_cast<uint32_t*>(base + w.rdone),
                        thr, keff)) != FASA_OK)
    return s;

  // 2. filter: certain tokens into the bitmap, threshold-bin tokens into the candidate list
  FilterParams fp{};
  fp.scores = scores;
  fp.ld = w.ld;
  fp.thr = thr;
  fp.cand_cnt = cnt;
  fp.cand_idx = cand;
  fp.cand_key = ckey;
  fp.bitmap = bitmap;
  fp.len = len;
  fp.n_keep = keff;
  fp.cap = w.cap;
  // one wave of four resident filter CTAs per SM
  const int64_t tiles_per_row = std::max<int64_t>(1, 4LL * d.sms / rows);
  fp.tile = (int)std::max<int64_t>(2048, ceil_div(ceil_div(len, tiles_per_row), 128) * 128);
  fp.words = w.words;
  if ((s = launch_pdl(filter_kernel, dim3((unsigned)ceil_div(len, fp.tile), (unsigned)rows, 1), kFilterThreads, 0,
                      stream, fp)) != FASA_OK)
    return s;

  // 3. finalize: exact threshold among the candidates, kept indices in ascending order
  FinalParams np{};
  np.scores = scores;
  np.ld = w.ld;
  np.thr = thr;
  np.cand_cnt = cnt;
  np.cand_idx = cand;
  np.cand_key = ckey;
  np.bitmap = bitmap;
  np.idx = idx;
  np.idx_out = idx_out;
  np.len = len;
  np.n_keep = keff;
  np.cap = w.cap;
  np.words = w.words;
  np.scap = w.cap;
  while (np.scap > 256 && final_smem_bytes(np.words, np.scap) > d.smem_optin) np.scap /= 2;
  const int fsmem = final_smem_bytes(np.words, np.scap);
  if (fsmem > d.smem_optin) return FASA_ERR_UNSUPPORTED;
  int set = 0;
  if ((s = cached_int((const void*)finalize_kernel, 0, &set, [&](int* v) {
         *v = 1;
         return cuda_status(
             cudaFuncSetAttribute(finalize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, d.smem_optin));
       })) != FASA_OK)
    return s;
  if ((s = launch_pdl(finalize_kernel, dim3((unsigned)rows, 1, 1), kSAThreads, (size_t)fsmem, stream, np)) !=
      FASA_OK)
    return s;

  // 4. focused attention over the kept rows
  if (c->dtype == FASA_BF16) return launch_attend_ws(c, len, keff, q, q_pos, out, w, base, d, stream);
  SAParams p{};
  p.idx_in = idx;
  p.k = c->k;
  p.v = c->v;
  p.q = q;
  p.out = out;
  p.max_len = c->max_len;
  p.len = len;
  p.n_keep = keff;
  p.n_kv_heads = c->n_kv_heads;
  p.group = c->n_q_heads / c->n_kv_heads;
  return launch_sa<kAttendIdx>(c, p, rows, true, stream, c->dtype, q_pos);
}

fasa_status fasa_set_decode_path(int32_t path) {
  if (path != FASA_DECODE_AUTO && path != FASA_DECODE_FUSED && path != FASA_DECODE_STAGED)
    return FASA_ERR_INVALID_ARG;
  g_decode_path.store(path);
  return FASA_OK;
}

int32_t fasa_decode_path(const fasa_cache* c, int32_t len, int32_t k) {
  fasa_status s = check_cache(c);
  if (s != FASA_OK) return -s;
  if (len < 1 || k < 1 || len > c->max_len) return -FASA_ERR_INVALID_ARG;
  DevInfo d;
  if ((s = device_info(&d)) != FASA_OK) return -s;
  const int path = g_decode_path.load();
  if (path != FASA_DECODE_AUTO) return path;
  WidePlan pl;
  const int keff = std::min(k, len);
  return fused_preferred(c, keff, d) && wide_plan(c, len, keff, d, &pl) ? FASA_DECODE_FUSED : FASA_DECODE_STAGED;
}

int32_t fasa_decode_launches(const fasa_cache* c, int32_t len, int32_t k) {
  const int32_t path = fasa_decode_path(c, len, k);
  if (path < 0) return path;
  DevInfo d;
  if (device_info(&d) != FASA_OK) return -FASA_ERR_CUDA;
  // the split-K attention of bf16 caches adds the split merge when a row's
  // kept list spans several CTAs
  auto merge = [&]() -> int32_t {
    if (c->dtype != FASA_BF16) return 0;
    int splits = 1, slice = 0, nw = 4;
    const DecodeWs w = decode_layout(c, len, k);
    if (attend_split(c->n_q_heads / c->n_kv_heads, c->batch * c->n_kv_heads, std::min(k, len), w.splits_max, d,
                     &splits, &slice, &nw) != FASA_OK)
      return -1;
    return splits > 1 ? 1 : 0;
  };
  if (path == FASA_DECODE_STAGED) {
    const int32_t m = merge();
    return m < 0 ? -FASA_ERR_CUDA : 4 + m;
  }
  WidePlan pl;
  if (!wide_plan(c, len, std::min(k, len), d, &pl)) return -FASA_ERR_UNSUPPORTED;
  if (pl.direct) return 1;
  const int32_t m = merge();
  return m < 0 ? -FASA_ERR_CUDA : 2 + m;
}

}  // extern "C"

namespace {
// Host checks of a varlen description against the cache.
fasa_status check_varlen(const fasa_cache* c, const fasa_varlen* vl) {
  if (vl == nullptr || !aligned(vl->seq_len, 4)) return FASA_ERR_INVALID_ARG;
  if (vl->budget != nullptr && !aligned(vl->budget, 4)) return FASA_ERR_INVALID_ARG;
  if (vl->max_seq_len < 1 || vl->max_budget < 1 || (vl->q_prerotated != 0 && vl->q_prerotated != 1))
    return FASA_ERR_INVALID_ARG;
  if (vl->max_seq_len > c->max_len) return FASA_ERR_CAPACITY;
  if (vl->max_seq_len > FASA_MAX_LEN || vl->max_budget > FASA_MAX_K) return FASA_ERR_UNSUPPORTED;
  return FASA_OK;
}

// fasa_decode_varlen / fasa_decode_paged after the cache checks.
fasa_status decode_varlen(const fasa_cache* c, const fasa_varlen* vl, const void* q, void* out, int32_t* idx_out,
                          void* workspace, size_t workspace_bytes, cudaStream_t stream, const fasa_paged* pg) {
  fasa_status s;
  if ((s = check_varlen(c, vl)) != FASA_OK) return s;
  if (c->dtype != FASA_BF16) return FASA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(out, 16)) return FASA_ERR_INVALID_ARG;
  if (idx_out != nullptr && !aligned(idx_out, 4)) return FASA_ERR_INVALID_ARG;
  const int32_t len = vl->max_seq_len, keff = std::min(vl->max_budget, vl->max_seq_len);
  const DecodeWs w = decode_layout(c, len, vl->max_budget);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < w.total) return FASA_ERR_WORKSPACE;
  DevInfo d;
  if ((s = device_info(&d)) != FASA_OK) return s;
  WidePlan pl;
  if (!wide_plan(c, len, keff, d, &pl, pg != nullptr)) return FASA_ERR_UNSUPPORTED;
  return launch_wide(c, len, q, 0, keff, out, idx_out, w, static_cast<char*>(workspace), pl, d, stream, vl, pg);
}
}  // namespace

extern "C" {

size_t fasa_decode_varlen_workspace_bytes(const fasa_cache* c, const fasa_varlen* vl) {
  if (check_cache(c) != FASA_OK || check_varlen(c, vl) != FASA_OK) return 0;
  return decode_ws(c, vl->max_seq_len, vl->max_budget);
}

fasa_status fasa_decode_varlen(const fasa_cache* c, const fasa_varlen* vl, const void* q, void* out,
                               int32_t* idx_out, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  fasa_status s = check_cache(c);
  if (s != FASA_OK) return s;
  return decode_varlen(c, vl, q, out, idx_out, workspace, workspace_bytes, stream, nullptr);
}


fasa_status fasa_append_kv_paged(const fasa_cache* c, const fasa_paged* pg, const void* k_new, const void* v_new,
                                 int32_t n_new, const int32_t* pos0, cudaStream_t stream) {
  fasa_status s = check_cache(c);
  if (s != FASA_OK) return s;
  if (pg != nullptr && (s = check_paged(c, pg)) != FASA_OK) return s;
  if (n_new < 0 || !aligned(pos0, 4)) return FASA_ERR_INVALID_ARG;
  if (n_new > c->max_len) return FASA_ERR_CAPACITY;
  if (n_new == 0) return FASA_OK;
  if (!aligned(k_new, 16) || !aligned(v_new, 16)) return FASA_ERR_INVALID_ARG;
  DevInfo d;
  if ((s = device_info(&d)) != FASA_OK) return s;
  return launch_append(c, k_new, v_new, n_new, 0, pos0, pg, d, stream);
}

size_t fasa_decode_paged_workspace_bytes(const fasa_cache* c, const fasa_paged* pg, const fasa_varlen* vl) {
  if (check_cache(c) != FASA_OK || check_paged(c, pg) != FASA_OK || check_varlen(c, vl) != FASA_OK) return 0;
  return decode_ws(c, vl->max_seq_len, vl->max_budget);
}

fasa_status fasa_decode_paged(const fasa_cache* c, const fasa_paged* pg, const fasa_varlen* vl, const void* q,
                              void* out, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
  fasa_status s = check_cache(c);
  if (s != FASA_OK) return s;
  if ((s = check_paged(c, pg)) != FASA_OK) return s;
  return decode_varlen(c, vl, q, out, idx_out, workspace, workspace_bytes, stream, pg);
}

size_t fasa_decode_multi_workspace_bytes(const fasa_cache* c, int32_t len, int32_t n_q, int32_t k) {
  if (check_cache(c) != FASA_OK || len < 1 || k < 1 || n_q < 1) return 0;
  return multi_layout(c, len, k).total;
}

fasa_status fasa_decode_multi(const fasa_cache* c, int32_t len, const void* q, int32_t q_pos0, int32_t n_q,
                              int32_t k, void* out, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
  fasa_status s = check_cache(c);
  if (s != FASA_OK) return s;
  if (len < 1 || k < 1 || n_q < 1 || bad_qpos(q_pos0)) return FASA_ERR_INVALID_ARG;
  if (q_pos0 != FASA_Q_PREROTATED && (int64_t)q_pos0 + n_q - 1 > INT32_MAX) return FASA_ERR_INVALID_ARG;
  if (len > c->max_len) return FASA_ERR_CAPACITY;
  if (len > FASA_MAX_LEN || k > FASA_MAX_K || c->dtype != FASA_BF16) return FASA_ERR_UNSUPPORTED;
  if (n_q > kTcMaxTok || n_q * (c->n_q_heads / c->n_kv_heads) > kTcMaxRows) return FASA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(out, 16)) return FASA_ERR_INVALID_ARG;
  if (idx_out != nullptr && !aligned(idx_out, 4)) return FASA_ERR_INVALID_ARG;
  const int keff = std::min(k, len);
  const MultiWs m = multi_layout(c, len, k);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < m.total) return FASA_ERR_WORKSPACE;
  DevInfo d;
  if ((s = device_info(&d)) != FASA_OK) return s;
  WidePlan pl;
  if (!wide_plan(c, len, keff, d, &pl, 0, n_q)) return FASA_ERR_UNSUPPORTED;
  char* base = static_cast<char*>(workspace);
  // scoring and selection: the fused kernel with the n_q tokens' coefficients
  WideParams p{};
  p.sketch = static_cast<const __nv_bfloat16*>(c->sketch);
  p.k = static_cast<const __nv_bfloat16*>(c->k);
  p.v = static_cast<const __nv_bfloat16*>(c->v);
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.dom_idx = c->dom_idx;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.idx_out = idx_out;
  p.idx_ws = reinterpret_cast<int32_t*>(base + m.w.idx);
  p.cand = reinterpret_cast<uint2*>(base + m.w.scores);
  p.sem = reinterpret_cast<unsigned long long*>(base + m.w.sem);
  p.keys = reinterpret_cast<uint32_t*>(base + m.w.keys);
  p.max_len = c->max_len;
  p.len = len;
  p.stride = c->sketch_stride;
  p.n_kv_heads = c->n_kv_heads;
  p.group = c->n_q_heads / c->n_kv_heads;
  p.n_dom = c->n_dom;
  p.n_keep = keff;
  p.n_pub = pl.n_pub;
  p.n_loc = pl.n_loc;
  p.n_split = pl.n_split;
  p.ucache = pl.ucache;
  p.ushift = pl.ushift;
  p.direct = 0;
  p.pm = page_map(c, nullptr);
  p.n_q = n_q;
  p.q_prerot = q_pos0 == FASA_Q_PREROTATED ? 1 : 0;
  p.q_pos0 = p.q_prerot ? 0 : q_pos0;
  if (n_q == 1)  // the single-token path takes the angle's cos / sin
    fill_query_angle(p.cosv, p.sinv, c->rope_base, q_pos0);
  else
    fill_theta(p.cosv, c->rope_base);
  if ((s = launch_wide_sel(p, c->batch * c->n_kv_heads, pl, d, stream)) != FASA_OK) return s;
  return launch_tc(c, len, keff, q, q_pos0, n_q, out, m, base, d, stream);
}

fasa_status fasa_decode_static_scratch(const fasa_cache* c, int32_t len, const void* q, int32_t q_pos, int32_t k,
                                       void* out, int32_t* idx_out, cudaStream_t stream) {
  // fasa_decode's own checks first, so a call both unsupported and too large
  // gets the same status as from fasa_decode; then the scratch limit
  fasa_status s = check_cache(c);
  if (s != FASA_OK) return s;
  if (len < 1 || bad_qpos(q_pos) || k < 1) return FASA_ERR_INVALID_ARG;
  if (len > c->max_len) return FASA_ERR_CAPACITY;
  if (len > FASA_MAX_LEN || k > FASA_MAX_K) return FASA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(out, 16)) return FASA_ERR_INVALID_ARG;
  if (idx_out != nullptr && !aligned(idx_out, 4)) return FASA_ERR_INVALID_ARG;
  const DecodeWs w = decode_layout(c, len, k);
  if (w.total > FASA_STATIC_SCRATCH_BYTES) return FASA_ERR_WORKSPACE;
  void* ws = nullptr;
  if ((s = static_scratch_addr(&ws)) != FASA_OK) return s;
  // the semaphores, histograms and counters start zero at load and every
  // call leaves them zero; clear them anyway, so that a call that ended in an
  // error cannot poison the next
  if ((s = cuda_status(cudaMemsetAsync(ws, 0, w.scores, stream))) != FASA_OK) return s;
  return fasa_decode(c, len, q, q_pos, k, out, idx_out, ws, FASA_STATIC_SCRATCH_BYTES, stream);
}

size_t fasa_dense_workspace_bytes(const fasa_cache* c, int32_t len) {
  if (check_cache(c) != FASA_OK || len < 0) return 0;
  return dense_layout(c, len).total;
}

fasa_status fasa_dense_decode(const fasa_cache* c, int32_t len, const void* q, int32_t q_pos, void* out,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  fasa_status s = check_cache(c);
  if (s != FASA_OK) return s;
  if (len < 1 || bad_qpos(q_pos)) return FASA_ERR_INVALID_ARG;
  if (len > c->max_len) return FASA_ERR_CAPACITY;
  if (!aligned(q, 16) || !aligned(out, 16)) return FASA_ERR_INVALID_ARG;
  const DenseWs w = dense_layout(c, len);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < w.total) return FASA_ERR_WORKSPACE;
  if (c->dtype == FASA_BF16) {
    DevInfo d;
    if ((s = device_info(&d)) != FASA_OK) return s;
    char* base = static_cast<char*>(workspace);
    return launch_attend(c, len, len, out, nullptr, q, q_pos, reinterpret_cast<float*>(base + w.part), w.splits_max,
                         d, stream);
  }
  // the f32 dense kernel stages K and V with bulk copies, which are kept to
  // device memory: a FASA-M cache (host-resident K/V) is refused here
  if (host_resident(c->k) || host_resident(c->v)) return FASA_ERR_UNSUPPORTED;
  SAParams p{};
  p.k = c->k;
  p.v = c->v;
  p.q = q;
  p.out = out;
  p.max_len = c->max_len;
  p.len = len;
  p.n_keep = len;
  p.n_kv_heads = c->n_kv_heads;
  p.group = c->n_q_heads / c->n_kv_heads;
  return launch_sa<kDense>(c, p, c->batch * c->n_kv_heads, false, stream, c->dtype, q_pos);
}

size_t fasa_calibrate_workspace_bytes(const fasa_cache* c, int32_t len, int32_t n_win, int32_t budget) {
  if (check_cache(c) != FASA_OK || len < 1 || len > c->max_len || n_win < 1 || n_win > kCalMaxWin || budget < 1)
    return 0;
  return cal_layout((int64_t)c->batch * c->n_kv_heads, len, n_win, budget).total;
}

fasa_status fasa_calibrate_scores(const fasa_cache* c, int32_t len, const void* q_win, int32_t q_pos0,
                                  int32_t n_win, float* planes, cudaStream_t stream) {
  fasa_status s = check_cache(c);
  if (s != FASA_OK) return s;
  if (len < 1 || n_win < 1 || n_win > kCalMaxWin || q_pos0 < 0 || (int64_t)q_pos0 + n_win > INT32_MAX)
    return FASA_ERR_INVALID_ARG;
  if (len > c->max_len) return FASA_ERR_CAPACITY;
  if (!aligned(q_win, 16) || !aligned(planes, 4)) return FASA_ERR_INVALID_ARG;
  return c->dtype == FASA_F32 ? launch_cal_scores<float>(c, len, q_win, q_pos0, n_win, planes, stream)
                              : launch_cal_scores<__nv_bfloat16>(c, len, q_win, q_pos0, n_win, planes, stream);
}

fasa_status fasa_calibrate_counts(const float* planes, int32_t n_rows, int32_t n_kv_heads, int32_t n_win,
                                  int32_t len, int32_t budget, uint32_t* counts, void* workspace,
                                  size_t workspace_bytes, cudaStream_t stream) {
  if (!aligned(planes, 4) || !aligned(counts, 4)) return FASA_ERR_INVALID_ARG;
  if (n_kv_heads < 1 || n_rows < 1 || n_rows % n_kv_heads != 0 || n_win < 1 || n_win > kCalMaxWin || len < 1 ||
      budget < 1)
    return FASA_ERR_INVALID_ARG;
  if (len > FASA_MAX_LEN || budget > FASA_MAX_K) return FASA_ERR_UNSUPPORTED;
  const int64_t keff = std::min<int64_t>(budget, len);
  const int64_t sel_rows = (int64_t)n_rows * n_win * kCalPlanes;
  if (sel_rows > INT32_MAX) return FASA_ERR_UNSUPPORTED;
  if (workspace == nullptr || !aligned(workspace, 4) || workspace_bytes < (size_t)(sel_rows * keff * 4))
    return FASA_ERR_WORKSPACE;
  DevInfo d;
  fasa_status s = device_info(&d);
  if (s != FASA_OK) return s;
  int32_t* idx = static_cast<int32_t*>(workspace);
  if ((s = cuda_status(cudaMemsetAsync(counts, 0, (size_t)n_kv_heads * kNFC * 4, stream))) != FASA_OK) return s;
  // every plane's selection, in launches of at most 65535 rows
  for (int64_t r0 = 0; r0 < sel_rows; r0 += 65535) {
    SAParams p{};
    p.scores = planes + r0 * len;
    p.idx_out = idx + r0 * keff;
    p.len = len;
    p.n_keep = (int32_t)keff;
    p.group = 1;
    if ((s = launch_sa<kSelect>(nullptr, p, (int)std::min<int64_t>(65535, sel_rows - r0), false, stream, FASA_F32,
                                0)) != FASA_OK)
      return s;
  }
  const size_t bm_bytes = (size_t)(len + 31) / 32 * 4;
  if (bm_bytes > (size_t)d.smem_optin) return FASA_ERR_UNSUPPORTED;
  int set = 0;
  if ((s = cached_int((const void*)calib_overlap_kernel, 0, &set, [&](int* v) {
         *v = 1;
         return cuda_status(
             cudaFuncSetAttribute(calib_overlap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, d.smem_optin));
       })) != FASA_OK)
    return s;
  calib_overlap_kernel<<<(unsigned)((int64_t)n_rows * n_win), kCalThreads, bm_bytes, stream>>>(
      idx, (int32_t)keff, len, n_kv_heads, n_win, counts);
  return cuda_status(cudaGetLastError());
}

fasa_status fasa_calibrate_dominant(const uint32_t* counts, int32_t n_kv_heads, int32_t n_dom, int32_t* dom_idx,
                                    cudaStream_t stream) {
  if (!aligned(counts, 4) || !aligned(dom_idx, 4) || n_kv_heads < 1 || n_dom < 1 || n_dom > kNFC)
    return FASA_ERR_INVALID_ARG;
  calib_rank_kernel<<<(unsigned)n_kv_heads, kNFC, 0, stream>>>(counts, n_dom, dom_idx);
  return cuda_status(cudaGetLastError());
}

fasa_status fasa_calibrate(const fasa_cache* c, int32_t len, const void* q_win, int32_t q_pos0, int32_t n_win,
                           int32_t budget, int32_t n_dom, uint32_t* counts, int32_t* dom_idx, void* workspace,
                           size_t workspace_bytes, cudaStream_t stream) {
  fasa_status s = check_cache(c);
  if (s != FASA_OK) return s;
  if (budget < 1 || n_dom < 1 || n_dom > kNFC || n_win < 1 || n_win > kCalMaxWin || len < 1)
    return FASA_ERR_INVALID_ARG;
  if (len > c->max_len) return FASA_ERR_CAPACITY;
  const int64_t rows = (int64_t)c->batch * c->n_kv_heads;
  const CalWs w = cal_layout(rows, len, n_win, budget);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < w.total) return FASA_ERR_WORKSPACE;
  unsigned char* base = static_cast<unsigned char*>(workspace);
  float* planes = reinterpret_cast<float*>(base + w.planes);
  if ((s = fasa_calibrate_scores(c, len, q_win, q_pos0, n_win, planes, stream)) != FASA_OK) return s;
  if ((s = fasa_calibrate_counts(planes, (int32_t)rows, c->n_kv_heads, n_win, len, budget, counts, base + w.idx,
                                 w.total - w.idx, stream)) != FASA_OK)
    return s;
  return fasa_calibrate_dominant(counts, c->n_kv_heads, n_dom, dom_idx, stream);
}

fasa_status fasa_device_status(int32_t clear) {
  if (cudaDeviceSynchronize() != cudaSuccess) return FASA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return FASA_ERR_CUDA;
  if (clear && v != 0) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(g_status, &z, sizeof(z)) != cudaSuccess) return FASA_ERR_CUDA;
  }
  return v == 0 ? FASA_OK : (fasa_status)v;
}

}  // extern "C"
