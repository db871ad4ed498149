// Device helpers shared by the FASA kernels: element types, exact rounding,
// order-preserving score keys, the sticky status word, and thin inline-PTX
// wrappers for mbarriers and 1-D bulk (TMA) copies on sm_100a.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/fasa.h"

namespace fasa {

constexpr int kD = 128;        // head dim
constexpr int kNFC = 64;       // frequency chunks per head
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // bounded waits give up after ~1 s

// Sticky per-device status: the first device-side problem wins.
__device__ unsigned int g_status;

__device__ __forceinline__ void flag_status(unsigned int code) { atomicCAS(&g_status, 0u, code); }

// Where slot t of row (b, g) lives. Contiguous caches: row t of the (b, g)
// plane [max_len][W]. Paged caches: the pools are [n_pages][Hkv][bs][W]
// and logical block t / bs of sequence b is page table[b][t / bs]; the row
// index below counts W-element rows from the pool's start.
struct PageMap {
  const int32_t* table;  // [B][max_blocks], or null for a contiguous cache
  int32_t max_blocks;
  int32_t n_pages;
  int32_t log2bs;        // log2 of the block size
  int32_t n_kv_heads;
};

// Pool row of slot t of (b, g) given the page, or -1 for a page outside the
// pool (flagged FASA_ERR_BAD_INDEX).
__device__ __forceinline__ int page_row(const PageMap& m, int pg, int g, int t) {
  if ((unsigned)pg >= (unsigned)m.n_pages) {
    flag_status(FASA_ERR_BAD_INDEX);
    return -1;
  }
  return ((pg * m.n_kv_heads + g) << m.log2bs) | (t & ((1 << m.log2bs) - 1));
}
// The same, looking the page up in the table.
__device__ __forceinline__ int paged_row(const PageMap& m, int b, int g, int t) {
  return page_row(m, __ldg(m.table + (int64_t)b * m.max_blocks + (t >> m.log2bs)), g, t);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------ element types

template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int kBytes = 4;
  static constexpr int kPer16 = 4;   // elements per 16-byte chunk
};
template <> struct Elem<__nv_bfloat16> {
  static constexpr int kBytes = 2;
  static constexpr int kPer16 = 8;
};

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }

// Unpack a 16-byte chunk into floats (exact for both element types).
__device__ __forceinline__ void unpack16(const uint4& u, float (&f)[4], float) {
  f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ void unpack16(const uint4& u, float (&f)[8], __nv_bfloat16) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Round a float64 to bfloat16, nearest-even, in effect one rounding step.
// Going through float32 first can only go wrong when the float32 result lands
// exactly on a bfloat16 tie while the float64 value was off it; that case is
// resolved from the float64 value directly.
__device__ __forceinline__ __nv_bfloat16 round_bf16(double x) {
  const float f = __double2float_rn(x);
  const uint32_t u = __float_as_uint(f);
  uint32_t r;
  if ((u & 0xFFFFu) == 0x8000u && (double)f != x) {
    r = (u >> 16) + (fabs(x) > fabs((double)f) ? 1u : 0u);
  } else {
    r = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
  }
  return __ushort_as_bfloat16((unsigned short)r);
}
__device__ __forceinline__ void round_store(float* p, double x) { *p = __double2float_rn(x); }
__device__ __forceinline__ void round_store(__nv_bfloat16* p, double x) { *p = round_bf16(x); }
__device__ __forceinline__ void store_f(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_f(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// ---------------------------------------------------------- score keys

// Order-preserving map float32 -> uint32 (larger score, larger key); -0.0 is
// folded onto +0.0 so that equal scores compare equal.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ------------------------------------------------------------ PTX: smem

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------- PTX: mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}
// Bounded wait for the phase with the given parity to complete. Gives up after
// ~1 s, records FASA_ERR_TIMEOUT and returns false; never spins forever.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      flag_status(FASA_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) writes to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16. No multicast.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Hint: bring [src, src + bytes) into L2 (16-byte aligned, multiple of 16).
// Safe before griddepcontrol.wait: later loads still see the latest data.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// Hint: bring the line holding p into L2 (any address).
__device__ __forceinline__ void prefetch_line_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p) : "memory");
}
// Programmatic dependent launch: wait until the preceding kernel in the
// stream has completed and its memory is visible (no-op without PDL); let
// the next kernel in the stream be scheduled.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace fasa

namespace fasa {

// ------------------------------------------------------- PTX: cluster

// Split cluster barrier: arrive (release) now, wait (acquire) later, so the
// barrier's latency overlaps local work.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ------------------------------------------------------- PTX: cp.async

// 16-byte global -> shared copy through L2 only (no L1 allocation).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// 4-byte global -> shared copy (through L1).
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace fasa
