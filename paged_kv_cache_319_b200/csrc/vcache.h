// Internal layout of a virtually contiguous KV cache (the kv_vcache_* calls of
// kvp.h), shared by the host object (host/vcache.cpp) and the device entry
// points (kvp_device.cu).
//
// The cache of each sequence slot is one range of virtual addresses,
// token-major: token j of slot s, KV head g, element d of K lives at
//   k_base + ((s * slot_tokens + j) * num_kv_heads + g) * head_dim + d
// (V likewise from v_base). The ranges are reserved once; physical memory is
// mapped into them in chunks of the device's allocation granularity as the
// slots grow, so a sequence's keys and values stay contiguous in virtual
// memory while physical memory follows its actual length ["Your GPU was
// mostly empty", section "The tradeoff: you just wrote a virtual memory
// subsystem in userspace": keeping the cache virtually contiguous and backing
// it with on-demand physical pages through CUDA's virtual memory management].
//
// Invariant the kernels rely on: for every slot, tokens [0, cap[s] +
// kVcacheTailTokens) are mapped, so a tile that starts below cap[s] and spans
// at most kVcacheTailTokens tokens never touches an unmapped address. The
// kernels clamp each sequence's context to cap of its slot (device copy).
#pragma once

#include <cuda.h>

#include <cstddef>
#include <cstdint>
#include <vector>

// Mapped tokens a slot keeps beyond its capacity: at least the longest tile a
// kernel reads past the last valid token (128-token tensor-core tiles).
constexpr int32_t kVcacheTailTokens = 256;

struct kvp_vcache {
  int device = 0;
  int32_t num_slots = 0;
  int32_t max_tokens = 0;    // largest capacity a slot can be given
  int32_t num_kv_heads = 0;
  int32_t head_dim = 0;
  int32_t dtype = 0;
  int32_t slot_tokens = 0;   // token stride between slots: >= max_tokens + tail, whole chunks
  size_t token_bytes = 0;    // num_kv_heads * head_dim * 2
  size_t chunk_bytes = 0;    // physical mapping granularity
  size_t slot_bytes = 0;     // slot_tokens * token_bytes, a multiple of chunk_bytes
  CUdeviceptr k_base = 0, v_base = 0;
  size_t reserved_bytes = 0;  // per cache (K or V)
  // per slot, the physical chunks mapped at its start, in address order
  std::vector<std::vector<CUmemGenericAllocationHandle>> k_chunks, v_chunks;
  std::vector<CUmemGenericAllocationHandle> spare;  // unmapped chunks kept for reuse
  std::vector<int32_t> cap;   // host copy of the per-slot capacity (tokens)
  int32_t* cap_dev = nullptr; // device copy, int32 [num_slots]
  int64_t map_calls = 0, create_calls = 0;
};

// Stream-ordered update of one slot's capacity in the device copy (a one-thread
// kernel, defined with the other kernels in kvp_device.cu).
int kvp_vcache_push_cap(int32_t* cap_dev, int32_t slot, int32_t value, void* stream);
