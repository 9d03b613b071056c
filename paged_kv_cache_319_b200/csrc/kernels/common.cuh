// Device helpers for the sm_100a kernels of libkvp: device error word,
// mbarriers with bounded waits, TMA (cp.async.bulk.tensor, no multicast),
// tcgen05 (TMEM allocation, MMA, commit, loads).
//
// Every wait on an mbarrier is bounded by a wall-clock limit read from
// %globaltimer; a wait that runs out records KVP_DEVERR_TIMEOUT in the device
// error word and returns false so the kernel can drain and exit.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

namespace kvp {
namespace dev {

// ---- device error word ---------------------------------------------------
// bits 56..63: kind, bits 0..55: payload (the offending index). First error wins.
enum DevErr : uint32_t {
  KVP_DEVERR_SLOT = 1,      // reshape_and_cache: slot >= num_blocks * block_size
  KVP_DEVERR_BLOCK_ID = 2,  // decode: block table entry outside [0, num_blocks)
  KVP_DEVERR_CTX = 3,       // decode: context length outside [0, max_context_len]
  KVP_DEVERR_PAIR = 4,      // copy_blocks: src or dst outside [0, num_blocks)
  KVP_DEVERR_TIMEOUT = 5,   // a bounded wait ran out
};

// Defined here: all device code is compiled as one translation unit.
__device__ unsigned long long g_error_word = 0ull;

__device__ __forceinline__ void record_error(uint32_t kind, uint64_t payload) {
  const unsigned long long v =
      (static_cast<unsigned long long>(kind) << 56) | (payload & ((1ull << 56) - 1));
  atomicCAS(&g_error_word, 0ull, v);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// One second: every wait in these kernels normally completes in microseconds.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// ---- mbarrier ---------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return done != 0;
}

// Waits for the phase with the given parity to complete; false on timeout
// (recorded with `where` as payload).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t where,
                                          uint64_t limit_ns = kWaitLimitNs) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(a, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) {
      record_error(KVP_DEVERR_TIMEOUT, where);
      return false;
    }
  }
}

// ---- programmatic dependent launch ---------------------------------------------
// A kernel launched with programmatic stream serialisation may start while the
// previous kernel of the stream still runs; pdl_wait() blocks until that kernel
// has completed and its writes are visible. pdl_trigger() lets the dependent
// kernel launch once every CTA of this grid has triggered or exited.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Coherent load of a word that an earlier kernel of the stream wrote while
// this one may already have been running (programmatic dependent launch):
// issued after pdl_wait(), never through the read-only (.nc) path, whose loads
// the compiler may treat as invariant and move above the wait.
__device__ __forceinline__ int32_t ld_relaxed_gpu(const int32_t* p) {
  int32_t v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// ---- proxies, named barriers -----------------------------------------------
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---- TMA ----------------------------------------------------------------------
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// L2 policy of the K/V tile loads (0: evict first, 1: normal, 2: evict last).
#ifndef KVP_KV_L2_POLICY
#define KVP_KV_L2_POLICY 0
#endif
__device__ __forceinline__ uint64_t l2_policy_evict_last();
__device__ __forceinline__ uint64_t l2_policy_kv() {
  if constexpr (KVP_KV_L2_POLICY == 1) return l2_policy_evict_normal();
  if constexpr (KVP_KV_L2_POLICY == 2) return l2_policy_evict_last();
  return l2_policy_evict_first();
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled load of box {x-extent, y-extent} at element coordinates (x, y)
// into shared memory; completes `bar`'s transaction count. x * element size
// must be a multiple of 16 bytes (callers pass x in {0, 64} for 2-byte data).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// 3-D tiled load at element coordinates (x, y, z); x as for tma_load_2d.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y, int32_t z, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)),
      "l"(policy)
      : "memory");
}

// 3-D tiled store of a shared-memory box to global memory at element
// coordinates (x, y, z), tracked by the issuing thread's bulk async-group; x
// times the element size is a multiple of 16 bytes and no coordinate is
// negative. The box must not be written again before bulk_wait_read().
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int32_t x,
                                             int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// The issuing thread's committed bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// The issuing thread's committed bulk stores have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 4-D tiled load at element coordinates (x, y, z, w); x as for tma_load_2d.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y, int32_t z, int32_t w,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar)),
      "l"(policy)
      : "memory");
}

// ---- tcgen05 -------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (fp16 or bf16 in, fp32 out).
__device__ __forceinline__ void umma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on `bar` when every tcgen05.mma issued so far by this thread completes.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Each thread of the warp reads 4 consecutive 32-bit columns of its TMEM lane.
__device__ __forceinline__ void tmem_ld_x4(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr)
               : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- 16-bit element helpers -------------------------------------------------------
template <typename T>
struct Elem;

template <>
struct Elem<__half> {
  static __device__ __forceinline__ float2 to_float2(uint32_t packed) {
    return __half22float2(*reinterpret_cast<const __half2*>(&packed));
  }
  static __device__ __forceinline__ uint16_t from_float(float x) {
    return __half_as_ushort(__float2half_rn(x));
  }
  static __device__ __forceinline__ uint32_t pack2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

template <>
struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float2 to_float2(uint32_t packed) {
    // bf16 is the upper half of an fp32: widen by shifting into place.
    return make_float2(__uint_as_float(packed << 16), __uint_as_float(packed & 0xffff0000u));
  }
  static __device__ __forceinline__ uint16_t from_float(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
  }
  static __device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

// E4M3 (8-bit float: 1 sign, 4 exponent, 3 mantissa bits, bias 7, largest
// finite 448) by the PTX conversions of sm_89 and later. Two codes per 16 bits,
// the lower byte first.
// Two codes -> their exact values (every E4M3 value is an fp16 value).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two_codes) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(two_codes)));
  return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}
// Two E4M3 codes (lower byte first) -> two values of T packed in 32 bits,
// exactly: fp16 by one cvt; bf16 through fp32 (every E4M3 value is a bf16).
template <typename T>
__device__ __forceinline__ uint32_t e4m3x2_to_x2(uint32_t two_codes) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(two_codes)));
  if constexpr (std::is_same<T, __half>::value) {
    return h2;
  } else {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<const uint32_t*>(&b);
  }
}
// Two fp32 values -> their codes: round to nearest even, saturated to +-448
// (infinities too), NaN to NaN; lo goes to the lower byte.
__device__ __forceinline__ uint32_t float2_to_e4m3x2(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

// Order-preserving map of fp32 to int32 (for integer max reductions).
__device__ __forceinline__ int32_t float_to_ordered(float f) {
  const int32_t i = __float_as_int(f);
  return i >= 0 ? i : (i ^ 0x7fffffff);
}
__device__ __forceinline__ float ordered_to_float(int32_t i) {
  return __int_as_float(i >= 0 ? i : (i ^ 0x7fffffff));
}

__device__ __forceinline__ float warp_max(float v) {
  return ordered_to_float(__reduce_max_sync(0xffffffffu, float_to_ordered(v)));
}

}  // namespace dev
}  // namespace kvp
