// Host object of the virtually contiguous KV cache: reserved virtual address
// ranges per sequence slot, backed on demand by physical chunks through CUDA's
// virtual memory management (cuMemAddressReserve / cuMemCreate / cuMemMap /
// cuMemSetAccess), the alternative to block tables that keeps the paging in
// the GPU's own address translation ["Your GPU was mostly empty", section
// "The tradeoff: you just wrote a virtual memory subsystem in userspace"].
//
// Policy (the page names the idea only):
//  - a slot's capacity grows by mapping whole chunks at the end of its range;
//    it always keeps kVcacheTailTokens mapped tokens past its capacity, so a
//    kernel tile that starts inside the capacity stays inside mapped memory;
//  - shrinking (kv_vcache_trim) is explicit: the slot's capacity drops in
//    stream order, the device is synchronised, then chunks are unmapped and
//    kept as spares; a slot that a finished request leaves keeps its mapping
//    for the next request (reclamation is deferred);
//  - new chunks come from the spares first, then from cuMemCreate;
//  - every call checks first and mutates after, undoing its own mappings if a
//    driver call fails part way, so a failed call changes nothing.
// Driver entry points are fetched through the runtime
// (cudaGetDriverEntryPointByVersion), so the library needs no libcuda link.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <mutex>
#include <new>
#include <vector>

#include "../status.h"
#include "../vcache.h"

using kvp::fail;

namespace {

struct Driver {
  PFN_cuMemAddressReserve_v10020 reserve = nullptr;
  PFN_cuMemAddressFree_v10020 addr_free = nullptr;
  PFN_cuMemCreate_v10020 create = nullptr;
  PFN_cuMemRelease_v10020 release = nullptr;
  PFN_cuMemMap_v10020 map = nullptr;
  PFN_cuMemUnmap_v10020 unmap = nullptr;
  PFN_cuMemSetAccess_v10020 set_access = nullptr;
  PFN_cuMemGetAllocationGranularity_v10020 granularity = nullptr;
  bool ok = false;
};

template <typename F>
bool fetch(const char* name, F* fn) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, &p, 10020, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !p)
    return false;
  *fn = reinterpret_cast<F>(p);
  return true;
}

const Driver& drv() {
  static Driver d;
  static std::once_flag once;
  std::call_once(once, [] {
    d.ok = fetch("cuMemAddressReserve", &d.reserve) && fetch("cuMemAddressFree", &d.addr_free) &&
           fetch("cuMemCreate", &d.create) && fetch("cuMemRelease", &d.release) &&
           fetch("cuMemMap", &d.map) && fetch("cuMemUnmap", &d.unmap) &&
           fetch("cuMemSetAccess", &d.set_access) &&
           fetch("cuMemGetAllocationGranularity", &d.granularity);
  });
  return d;
}

CUmemAllocationProp chunk_prop(int device) {
  CUmemAllocationProp p{};
  p.type = CU_MEM_ALLOCATION_TYPE_PINNED;
  p.location.type = CU_MEM_LOCATION_TYPE_DEVICE;
  p.location.id = device;
  return p;
}

int64_t gcd64(int64_t a, int64_t b) {
  while (b) {
    const int64_t t = a % b;
    a = b;
    b = t;
  }
  return a;
}

// Tokens a slot can hold with `chunks` chunks mapped (the tail kept aside).
int32_t cap_of(const kvp_vcache* vc, size_t chunks) {
  const int64_t mapped = int64_t(chunks * vc->chunk_bytes / vc->token_bytes);
  return int32_t(std::max<int64_t>(0, std::min<int64_t>(vc->max_tokens, mapped - kVcacheTailTokens)));
}

// Chunks a slot needs for a capacity of `tokens`.
size_t chunks_for(const kvp_vcache* vc, int32_t tokens) {
  if (tokens <= 0) return 0;
  const size_t bytes = size_t(int64_t(tokens) + kVcacheTailTokens) * vc->token_bytes;
  return (bytes + vc->chunk_bytes - 1) / vc->chunk_bytes;
}

// Maps one chunk (a spare, else a new one) at `va`, readable and writable by
// the cache's device; on success *out holds its handle.
int map_chunk(kvp_vcache* vc, CUdeviceptr va, CUmemGenericAllocationHandle* out) {
  const Driver& d = drv();
  CUmemGenericAllocationHandle h = 0;
  bool fresh = false;
  if (!vc->spare.empty()) {
    h = vc->spare.back();
  } else {
    const CUmemAllocationProp prop = chunk_prop(vc->device);
    CUresult r = d.create(&h, vc->chunk_bytes, &prop, 0);
    if (r == CUDA_ERROR_OUT_OF_MEMORY) return fail(KVP_ERR_OOM, "kv_vcache: no device memory for a chunk");
    if (r != CUDA_SUCCESS) return fail(KVP_ERR_CUDA, "kv_vcache: cuMemCreate failed (%d)", int(r));
    fresh = true;
    ++vc->create_calls;
  }
  CUresult r = d.map(va, vc->chunk_bytes, 0, h, 0);
  if (r == CUDA_SUCCESS) {
    CUmemAccessDesc acc{};
    acc.location.type = CU_MEM_LOCATION_TYPE_DEVICE;
    acc.location.id = vc->device;
    acc.flags = CU_MEM_ACCESS_FLAGS_PROT_READWRITE;
    r = d.set_access(va, vc->chunk_bytes, &acc, 1);
    if (r != CUDA_SUCCESS) d.unmap(va, vc->chunk_bytes);
  }
  if (r != CUDA_SUCCESS) {
    if (fresh) {
      d.release(h);
    }
    return fail(KVP_ERR_CUDA, "kv_vcache: mapping a chunk failed (%d)", int(r));
  }
  if (!fresh) vc->spare.pop_back();
  ++vc->map_calls;
  *out = h;
  return KVP_OK;
}

// Unmaps the chunks of `slot` from index `keep` on (both caches) and keeps
// their handles as spares (the caller has reserved room in `spare`), or, with
// to_spare false, returns them to the driver.
void unmap_from(kvp_vcache* vc, int32_t slot, size_t keep, bool to_spare = true) {
  const Driver& d = drv();
  auto drop = [&](std::vector<CUmemGenericAllocationHandle>& v, CUdeviceptr base) {
    while (v.size() > keep) {
      const size_t i = v.size() - 1;
      d.unmap(base + size_t(slot) * vc->slot_bytes + i * vc->chunk_bytes, vc->chunk_bytes);
      if (to_spare)
        vc->spare.push_back(v[i]);
      else
        d.release(v[i]);
      v.pop_back();
    }
  };
  drop(vc->k_chunks[slot], vc->k_base);
  drop(vc->v_chunks[slot], vc->v_base);
}

void destroy_all(kvp_vcache* vc) {
  const Driver& d = drv();
  for (int32_t s = 0; s < vc->num_slots && s < int32_t(vc->k_chunks.size()); ++s)
    unmap_from(vc, s, 0, false);
  for (CUmemGenericAllocationHandle h : vc->spare) d.release(h);
  vc->spare.clear();
  if (vc->k_base) d.addr_free(vc->k_base, vc->reserved_bytes);
  if (vc->v_base) d.addr_free(vc->v_base, vc->reserved_bytes);
  if (vc->cap_dev) cudaFree(vc->cap_dev);
  vc->k_base = vc->v_base = 0;
  vc->cap_dev = nullptr;
}

int check_slot(const kvp_vcache* vc, int32_t slot, const char* who) {
  if (!vc) return fail(KVP_ERR_INVALID, "%s: NULL cache", who);
  if (slot < 0 || slot >= vc->num_slots) return fail(KVP_ERR_INVALID, "%s: slot %d out of range", who, slot);
  return KVP_OK;
}

// The calls run with the cache's device current (restored afterwards).
struct OnDevice {
  int prev = -1;
  bool ok = false;
  explicit OnDevice(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) return;
    ok = prev == dev || cudaSetDevice(dev) == cudaSuccess;
  }
  ~OnDevice() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

}  // namespace

extern "C" {

int kv_vcache_create(int32_t num_slots, int32_t max_tokens, int32_t num_kv_heads, int32_t head_dim,
                     int32_t dtype, kvp_vcache** out) {
  if (!out) return fail(KVP_ERR_INVALID, "kv_vcache_create: out is NULL");
  *out = nullptr;
  if (num_slots <= 0 || max_tokens <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return fail(KVP_ERR_INVALID, "kv_vcache_create: sizes must be positive");
  if (dtype != KVP_F16 && dtype != KVP_BF16)
    return fail(KVP_ERR_INVALID, "kv_vcache_create: dtype must be KVP_F16 or KVP_BF16");
  if (head_dim != 128) return fail(KVP_ERR_INVALID, "kv_vcache_create: head_dim must be 128");
  const Driver& d = drv();
  if (!d.ok) return fail(KVP_ERR_CUDA, "kv_vcache_create: CUDA virtual memory management is not available");
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(KVP_ERR_CUDA, "kv_vcache_create: no current device");
  auto* vc = new (std::nothrow) kvp_vcache();
  if (!vc) return fail(KVP_ERR_OOM, "kv_vcache_create: host allocation failed");
  vc->device = dev;
  vc->num_slots = num_slots;
  vc->max_tokens = max_tokens;
  vc->num_kv_heads = num_kv_heads;
  vc->head_dim = head_dim;
  vc->dtype = dtype;
  vc->token_bytes = size_t(num_kv_heads) * head_dim * 2;
  const CUmemAllocationProp prop = chunk_prop(dev);
  size_t gran = 0;
  CUresult r = d.granularity(&gran, &prop, CU_MEM_ALLOC_GRANULARITY_MINIMUM);
  if (r != CUDA_SUCCESS || gran == 0) {
    delete vc;
    return fail(KVP_ERR_CUDA, "kv_vcache_create: allocation granularity unavailable (%d)", int(r));
  }
  vc->chunk_bytes = gran;
  // slot stride: a whole number of tokens and of chunks, so no chunk spans two slots
  const int64_t tok_per_unit = int64_t(gran) / gcd64(int64_t(gran), int64_t(vc->token_bytes));
  const int64_t want = int64_t(max_tokens) + kVcacheTailTokens;
  const int64_t slot_tokens = (want + tok_per_unit - 1) / tok_per_unit * tok_per_unit;
  if (slot_tokens * num_slots >= (int64_t(1) << 31)) {
    delete vc;
    return fail(KVP_ERR_INVALID, "kv_vcache_create: too many tokens for 32-bit coordinates");
  }
  vc->slot_tokens = int32_t(slot_tokens);
  vc->slot_bytes = size_t(slot_tokens) * vc->token_bytes;
  vc->reserved_bytes = vc->slot_bytes * size_t(num_slots);
  try {
    vc->k_chunks.resize(size_t(num_slots));
    vc->v_chunks.resize(size_t(num_slots));
    vc->cap.assign(size_t(num_slots), 0);
  } catch (...) {
    delete vc;
    return fail(KVP_ERR_OOM, "kv_vcache_create: host allocation failed");
  }
  r = d.reserve(&vc->k_base, vc->reserved_bytes, gran, 0, 0);
  if (r == CUDA_SUCCESS) r = d.reserve(&vc->v_base, vc->reserved_bytes, gran, 0, 0);
  if (r != CUDA_SUCCESS) {
    destroy_all(vc);
    delete vc;
    return fail(KVP_ERR_CUDA, "kv_vcache_create: cuMemAddressReserve failed (%d)", int(r));
  }
  cudaError_t e = cudaMalloc(&vc->cap_dev, sizeof(int32_t) * size_t(num_slots));
  if (e == cudaSuccess) e = cudaMemset(vc->cap_dev, 0, sizeof(int32_t) * size_t(num_slots));
  if (e != cudaSuccess) {
    destroy_all(vc);
    delete vc;
    return fail(e == cudaErrorMemoryAllocation ? KVP_ERR_OOM : KVP_ERR_CUDA,
                "kv_vcache_create: capacity array: %s", cudaGetErrorString(e));
  }
  *out = vc;
  return KVP_OK;
}

int kv_vcache_destroy(kvp_vcache* vc) {
  if (!vc) return KVP_OK;
  OnDevice on(vc->device);
  cudaDeviceSynchronize();  // no kernel may still read the ranges being unmapped
  destroy_all(vc);
  delete vc;
  return KVP_OK;
}

int kv_vcache_reserve(kvp_vcache* vc, int32_t slot, int32_t tokens, kvp_stream_t stream) {
  int rc = check_slot(vc, slot, "kv_vcache_reserve");
  if (rc) return rc;
  if (tokens < 0 || tokens > vc->max_tokens)
    return fail(KVP_ERR_INVALID, "kv_vcache_reserve: %d tokens outside [0, %d]", tokens, vc->max_tokens);
  if (vc->cap[size_t(slot)] >= tokens) return KVP_OK;
  OnDevice on(vc->device);
  if (!on.ok) return fail(KVP_ERR_CUDA, "kv_vcache_reserve: cannot select the cache's device");
  const size_t have = vc->k_chunks[size_t(slot)].size();
  const size_t need = chunks_for(vc, tokens);
  try {
    vc->k_chunks[size_t(slot)].reserve(need);
    vc->v_chunks[size_t(slot)].reserve(need);
    vc->spare.reserve(vc->spare.size() + 2 * need);
  } catch (...) {
    return fail(KVP_ERR_OOM, "kv_vcache_reserve: host allocation failed");
  }
  for (size_t i = have; i < need; ++i) {
    const size_t off = size_t(slot) * vc->slot_bytes + i * vc->chunk_bytes;
    CUmemGenericAllocationHandle hk = 0, hv = 0;
    rc = map_chunk(vc, vc->k_base + off, &hk);
    if (!rc) {
      vc->k_chunks[size_t(slot)].push_back(hk);
      rc = map_chunk(vc, vc->v_base + off, &hv);
      if (!rc) vc->v_chunks[size_t(slot)].push_back(hv);
    }
    if (rc) {  // undo this call's mappings: nothing changes
      const std::string msg = kvp::last_error();
      // an unpaired K chunk of this index goes back first
      if (vc->k_chunks[size_t(slot)].size() > vc->v_chunks[size_t(slot)].size()) {
        drv().unmap(vc->k_base + off, vc->chunk_bytes);
        vc->spare.push_back(vc->k_chunks[size_t(slot)].back());
        vc->k_chunks[size_t(slot)].pop_back();
      }
      unmap_from(vc, slot, have);
      kvp::last_error() = msg;
      return rc;
    }
  }
  const int32_t cap = cap_of(vc, need);
  rc = kvp_vcache_push_cap(vc->cap_dev, slot, cap, stream);
  if (rc) {
    const std::string msg = kvp::last_error();
    unmap_from(vc, slot, have);
    kvp::last_error() = msg;
    return rc;
  }
  vc->cap[size_t(slot)] = cap;
  return KVP_OK;
}

int kv_vcache_reserve_batch(kvp_vcache* vc, const int32_t* slots, const int32_t* tokens,
                            int32_t n, kvp_stream_t stream) {
  if (!vc) return fail(KVP_ERR_INVALID, "kv_vcache_reserve_batch: NULL cache");
  if (n < 0) return fail(KVP_ERR_INVALID, "kv_vcache_reserve_batch: negative count");
  if (n == 0) return KVP_OK;
  if (!slots || !tokens) return fail(KVP_ERR_INVALID, "kv_vcache_reserve_batch: NULL argument");
  for (int32_t i = 0; i < n; ++i) {
    if (slots[i] < 0 || slots[i] >= vc->num_slots)
      return fail(KVP_ERR_INVALID, "kv_vcache_reserve_batch: slot %d out of range", slots[i]);
    if (tokens[i] < 0 || tokens[i] > vc->max_tokens)
      return fail(KVP_ERR_INVALID, "kv_vcache_reserve_batch: %d tokens outside [0, %d]", tokens[i],
                  vc->max_tokens);
  }
  // the slots that grow, with what they had, to undo on failure
  struct Grown {
    int32_t slot;
    size_t chunks;
    int32_t cap;
  };
  std::vector<Grown> grown;
  size_t new_chunks = 0;  // room for every chunk a rollback may return to the spares
  for (int32_t i = 0; i < n; ++i) {
    const size_t want = chunks_for(vc, tokens[i]), have = vc->k_chunks[size_t(slots[i])].size();
    if (want > have) new_chunks += 2 * (want - have);
  }
  try {
    grown.reserve(size_t(n));
    vc->spare.reserve(vc->spare.size() + new_chunks);
  } catch (...) {
    return fail(KVP_ERR_OOM, "kv_vcache_reserve_batch: host allocation failed");
  }
  for (int32_t i = 0; i < n; ++i) {
    const int32_t s = slots[i];
    if (vc->cap[size_t(s)] >= tokens[i]) continue;
    const Grown g{s, vc->k_chunks[size_t(s)].size(), vc->cap[size_t(s)]};
    const int rc = kv_vcache_reserve(vc, s, tokens[i], stream);
    if (rc) {
      const std::string msg = kvp::last_error();
      for (auto it = grown.rbegin(); it != grown.rend(); ++it) {
        kvp_vcache_push_cap(vc->cap_dev, it->slot, it->cap, stream);
        vc->cap[size_t(it->slot)] = it->cap;
        unmap_from(vc, it->slot, it->chunks);
      }
      kvp::last_error() = msg;
      return rc;
    }
    grown.push_back(g);
  }
  return KVP_OK;
}

int kv_vcache_trim(kvp_vcache* vc, int32_t slot, int32_t tokens, kvp_stream_t stream) {
  int rc = check_slot(vc, slot, "kv_vcache_trim");
  if (rc) return rc;
  if (tokens < 0) return fail(KVP_ERR_INVALID, "kv_vcache_trim: negative tokens");
  const size_t keep = chunks_for(vc, std::min(tokens, vc->max_tokens));
  if (keep >= vc->k_chunks[size_t(slot)].size()) return KVP_OK;
  OnDevice on(vc->device);
  if (!on.ok) return fail(KVP_ERR_CUDA, "kv_vcache_trim: cannot select the cache's device");
  try {
    vc->spare.reserve(vc->spare.size() + 2 * (vc->k_chunks[size_t(slot)].size() - keep));
  } catch (...) {
    return fail(KVP_ERR_OOM, "kv_vcache_trim: host allocation failed");
  }
  const int32_t cap = cap_of(vc, keep);
  rc = kvp_vcache_push_cap(vc->cap_dev, slot, cap, stream);
  if (rc) return rc;
  // every kernel that could read the chunks (on any stream) finishes first
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail(KVP_ERR_CUDA, "kv_vcache_trim: synchronize: %s", cudaGetErrorString(e));
  vc->cap[size_t(slot)] = cap;
  unmap_from(vc, slot, keep);
  return KVP_OK;
}

int kv_vcache_release_spares(kvp_vcache* vc) {
  if (!vc) return fail(KVP_ERR_INVALID, "kv_vcache_release_spares: NULL cache");
  OnDevice on(vc->device);
  for (CUmemGenericAllocationHandle h : vc->spare) drv().release(h);
  vc->spare.clear();
  return KVP_OK;
}

int kv_vcache_capacity(const kvp_vcache* vc, int32_t slot, int32_t* tokens) {
  int rc = check_slot(vc, slot, "kv_vcache_capacity");
  if (rc) return rc;
  if (!tokens) return fail(KVP_ERR_INVALID, "kv_vcache_capacity: NULL argument");
  *tokens = vc->cap[size_t(slot)];
  return KVP_OK;
}

int kv_vcache_layout(const kvp_vcache* vc, void** k_base, void** v_base, int32_t* slot_tokens) {
  if (!vc || !k_base || !v_base || !slot_tokens)
    return fail(KVP_ERR_INVALID, "kv_vcache_layout: NULL argument");
  *k_base = reinterpret_cast<void*>(vc->k_base);
  *v_base = reinterpret_cast<void*>(vc->v_base);
  *slot_tokens = vc->slot_tokens;
  return KVP_OK;
}

int kv_vcache_stats(const kvp_vcache* vc, kvp_vcache_stats* out) {
  if (!vc || !out) return fail(KVP_ERR_INVALID, "kv_vcache_stats: NULL argument");
  int64_t mapped = 0;
  for (const auto& v : vc->k_chunks) mapped += int64_t(v.size());
  for (const auto& v : vc->v_chunks) mapped += int64_t(v.size());
  out->chunk_bytes = int64_t(vc->chunk_bytes);
  out->mapped_chunks = mapped;
  out->spare_chunks = int64_t(vc->spare.size());
  out->mapped_bytes = mapped * int64_t(vc->chunk_bytes);
  out->reserved_bytes = 2 * int64_t(vc->reserved_bytes);
  out->map_calls = vc->map_calls;
  out->create_calls = vc->create_calls;
  out->slot_tokens = vc->slot_tokens;
  return KVP_OK;
}

}  // extern "C"
