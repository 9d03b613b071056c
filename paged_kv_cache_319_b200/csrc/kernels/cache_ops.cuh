// reshape_and_cache and copy_blocks: the two writes into the paged KV pool.
//
// Both are pure data movement, bound by HBM bandwidth. Every thread moves
// 16-byte vectors; a warp covers contiguous 512-byte spans, so loads and
// stores are fully coalesced. Out-of-range indices are skipped and recorded.
#pragma once

#include "common.cuh"

namespace kvp {
namespace dev {

// New tokens' K and V rows go to their slots: decode appends new cache state
// ["PagedAttention: KV cache memory management", section "A request
// lifecycle: allocation, growth, sharing and release"].
// k_new/v_new: [T][Hkv][D]; cache: [NB][Hkv][bs][D]. Thread-iteration c moves
// the 16-byte chunk j = c % cpr of row (t, h) = c / cpr, where cpr = D / 8
// chunks per row; cpr and block_size are powers of two (shifts), and the
// host guarantees T * Hkv * cpr < 2^31.
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, const int64_t* __restrict__ slot_mapping, uint32_t num_chunks,
    uint32_t num_kv_heads, uint32_t log2_cpr, uint32_t log2_bs, int64_t num_slots) {
  const uint32_t stride = gridDim.x * blockDim.x;
  const uint32_t cpr_mask = (1u << log2_cpr) - 1u;
  for (uint32_t c = blockIdx.x * blockDim.x + threadIdx.x; c < num_chunks; c += stride) {
    const uint32_t row = c >> log2_cpr;
    const uint32_t j = c & cpr_mask;
    const uint32_t t = row / num_kv_heads;
    const uint32_t h = row - t * num_kv_heads;
    const int64_t s = __ldg(slot_mapping + t);
    if (s < 0) continue;  // padding token
    if (s >= num_slots) {
      if (h == 0 && j == 0) record_error(KVP_DEVERR_SLOT, uint64_t(t));
      continue;
    }
    const int64_t blk = s >> log2_bs;
    const int64_t off = s & ((int64_t(1) << log2_bs) - 1);
    const int64_t dst = (((blk * num_kv_heads + h) << log2_bs) + off) * (int64_t(1) << log2_cpr) + j;
    const uint4 kv = __ldg(k_new + c);
    const uint4 vv = __ldg(v_new + c);
    k_cache[dst] = kv;
    v_cache[dst] = vv;
  }
}

// Virtually contiguous cache: token t's K and V rows go to position pos[t] of
// slot slots[t], i.e. row (slot * slot_tokens + pos) * Hkv + h of the
// token-major ranges. A position outside [0, cap[slot]) (the slot's mapped
// capacity) or a slot >= num_slots is skipped and recorded, so no store
// reaches an unmapped address; a negative slot is padding. Chunks as in
// reshape_and_cache_kernel: c moves chunk c % cpr of row c / cpr.
__global__ void __launch_bounds__(256) vcache_write_kernel(
    const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, uint4* __restrict__ k_base,
    uint4* __restrict__ v_base, const int32_t* __restrict__ slots, const int32_t* __restrict__ pos,
    const int32_t* __restrict__ cap, uint32_t num_chunks, uint32_t num_kv_heads, uint32_t log2_cpr,
    int32_t num_slots, int64_t slot_tokens) {
  const uint32_t stride = gridDim.x * blockDim.x;
  const uint32_t cpr_mask = (1u << log2_cpr) - 1u;
  for (uint32_t c = blockIdx.x * blockDim.x + threadIdx.x; c < num_chunks; c += stride) {
    const uint32_t row = c >> log2_cpr;
    const uint32_t j = c & cpr_mask;
    const uint32_t t = row / num_kv_heads;
    const uint32_t h = row - t * num_kv_heads;
    const int32_t s = __ldg(slots + t);
    if (s < 0) continue;  // padding token
    const int32_t p = __ldg(pos + t);
    if (s >= num_slots || p < 0 || p >= __ldg(cap + s)) {
      if (h == 0 && j == 0) record_error(KVP_DEVERR_SLOT, uint64_t(t));
      continue;
    }
    const int64_t dst = ((int64_t(s) * slot_tokens + p) * num_kv_heads + h) * (int64_t(1) << log2_cpr) + j;
    k_base[dst] = __ldg(k_new + c);
    v_base[dst] = __ldg(v_new + c);
  }
}

// One slot's capacity in the device copy, in stream order with the kernels
// that read it.
__global__ void vcache_set_cap_kernel(int32_t* cap, int32_t slot, int32_t value) {
  if (threadIdx.x == 0 && blockIdx.x == 0) cap[slot] = value;
}

// FP8 cache: the new tokens' K and V rows quantised into their slots, KV head
// h with its own scales: code = E4M3(x / scale[h]), the division correctly
// rounded in fp32, then rounded to the nearest E4M3 value (ties to even) and
// saturated to +-448. Quantised cached values are a lower-precision
// representation of the same state ["PagedAttention: KV cache memory
// management", section "PagedAttention vs KV-cache quantization vs prefix
// caching"]. k_new/v_new: [T][Hkv][D] of T; cache: [NB][Hkv][bs][D] bytes.
// Thread-iteration c writes the 16-byte chunk j = c % cpr (16 codes) of row
// (t, h) = c / cpr, cpr = D / 16.
template <typename T>
__global__ void __launch_bounds__(256) reshape_and_cache_fp8_kernel(
    const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, const int64_t* __restrict__ slot_mapping,
    const float* __restrict__ k_scale, const float* __restrict__ v_scale, uint32_t num_chunks,
    uint32_t num_kv_heads, uint32_t log2_cpr, uint32_t log2_bs, int64_t num_slots) {
  const uint32_t stride = gridDim.x * blockDim.x;
  const uint32_t cpr_mask = (1u << log2_cpr) - 1u;
  auto quantize = [](uint4 a, uint4 b, float s) {  // 16 values -> 16 codes
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f0 = Elem<T>::to_float2(w[2 * i]);
      const float2 f1 = Elem<T>::to_float2(w[2 * i + 1]);
      const uint32_t c0 = float2_to_e4m3x2(__fdiv_rn(f0.x, s), __fdiv_rn(f0.y, s));
      const uint32_t c1 = float2_to_e4m3x2(__fdiv_rn(f1.x, s), __fdiv_rn(f1.y, s));
      o[i] = c0 | (c1 << 16);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
  };
  for (uint32_t c = blockIdx.x * blockDim.x + threadIdx.x; c < num_chunks; c += stride) {
    const uint32_t row = c >> log2_cpr;
    const uint32_t j = c & cpr_mask;
    const uint32_t t = row / num_kv_heads;
    const uint32_t h = row - t * num_kv_heads;
    const int64_t s = __ldg(slot_mapping + t);
    if (s < 0) continue;  // padding token
    if (s >= num_slots) {
      if (h == 0 && j == 0) record_error(KVP_DEVERR_SLOT, uint64_t(t));
      continue;
    }
    const int64_t blk = s >> log2_bs;
    const int64_t off = s & ((int64_t(1) << log2_bs) - 1);
    const int64_t dst = (((blk * num_kv_heads + h) << log2_bs) + off) * (int64_t(1) << log2_cpr) + j;
    // source: 16 elements of T = two 16-byte vectors
    const uint4 k0 = __ldg(k_new + 2 * int64_t(c)), k1 = __ldg(k_new + 2 * int64_t(c) + 1);
    const uint4 v0 = __ldg(v_new + 2 * int64_t(c)), v1 = __ldg(v_new + 2 * int64_t(c) + 1);
    k_cache[dst] = quantize(k0, k1, __ldg(k_scale + h));
    v_cache[dst] = quantize(v0, v1, __ldg(v_scale + h));
  }
}

// Block-level copy-on-write: block dst of K and V becomes a copy of block src
// ["Your GPU was mostly empty", section "Paging's second gift: copy-on-write"].
// grid.y = pair, grid.z = 0 (K) / 1 (V); grid.x strides over the block's chunks,
// each thread keeping kCopyUnroll 16-byte loads in flight before its stores
// (destinations are distinct and never sources, so the loads may take the
// read-only path).
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* __restrict__ k_cache,
                                                          uint4* __restrict__ v_cache,
                                                          const int32_t* __restrict__ pairs,
                                                          int64_t chunks_per_block,
                                                          int32_t num_blocks) {
  const int32_t i = blockIdx.y;
  const int32_t src = __ldg(pairs + 2 * i);
  const int32_t dst = __ldg(pairs + 2 * i + 1);
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0)
      record_error(KVP_DEVERR_PAIR, uint64_t(i));
    return;
  }
  uint4* base = blockIdx.z == 0 ? k_cache : v_cache;
  const uint4* s = base + int64_t(src) * chunks_per_block;
  uint4* d = base + int64_t(dst) * chunks_per_block;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t c0 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; c0 < chunks_per_block;
       c0 += stride * kCopyUnroll) {
    uint4 r[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      const int64_t c = c0 + u * stride;
      if (c < chunks_per_block) r[u] = __ldg(s + c);
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      const int64_t c = c0 + u * stride;
      if (c < chunks_per_block) d[c] = r[u];
    }
  }
}

}  // namespace dev
}  // namespace kvp
