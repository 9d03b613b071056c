// Device entry points of libkvp (C ABI): argument checks, TMA tensor maps,
// kernel selection by geometry, launches on the caller's stream.
//
// All device code lives in this one translation unit (the kernels are
// headers) so the device error word is a single symbol per GPU.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "kernels/cache_ops.cuh"
#include "kernels/common.cuh"
#include "kernels/decode_group.cuh"
#include "kernels/decode_simt.cuh"
#include "kernels/decode_tc.cuh"
#include "kernels/prefill_tc.cuh"
#include "pack_layout.h"
#include "status.h"
#include "vcache.h"

using kvp::fail;

// Launch shape of the CUDA-core decode kernel: warps per CTA and TMA stages per
// warp (shared memory per CTA = warps x stages x 2 tiles + merge area). The
// kernel is bound by per-warp latency more than by bytes in flight: on the
// OPT-13B geometry, 4 warps x 2 stages (67 KB, 3 CTAs = 12 warps per SM) ran
// at 190.5 us per call against 231.9 us for 4 x 3 (2 CTAs per SM). Tiles of
// 8 KB (block size 32) use half the warps to keep about 64 KB per CTA.
#ifndef KVP_SIMT_WARPS
#define KVP_SIMT_WARPS 4
#endif
#ifndef KVP_SIMT_STAGES
#define KVP_SIMT_STAGES 2
#endif
// Batches of at least this many sequences take one stage per warp (32 KiB per
// CTA, five CTAs per SM instead of three): many (sequence, head) rows give
// many CTAs, and more of them resident hide their start-up better than a
// deeper per-warp ring. LLaMA-13B churn (256 sequences): 86.1 % -> 90.0 % of
// the copy peak; the OPT-13B batch (64) keeps two stages (95.8 % against
// 94.9 % with one).
#ifndef KVP_SIMT_ONE_STAGE_SEQS
#define KVP_SIMT_ONE_STAGE_SEQS 128
#endif
// Stages of the CUDA-core kernel on an E4M3 cache (tiles of half the bytes).
// On the OPT-13B batch: 2 stages 140.4 us, 3 stages 144.4 us, 4 stages 172.1 us.
#ifndef KVP_SIMT_FP8_STAGES
#define KVP_SIMT_FP8_STAGES 2
#endif
// Grouped decode with a host plan: the tensor-core kernel's per-SM rate on
// shared blocks, in percent of the CUDA-core kernel's rate on a sequence's own
// blocks; it sets the tensor-core kernel's share of the SMs.
#ifndef KVP_GROUP_TC_RATE
#define KVP_GROUP_TC_RATE 70
#endif
// Grouped decode: the CUDA-core kernel on the sequences' own ranges. Ranges
// that average fewer than KVP_GROUP_PER_HEAD_BELOW blocks per sequence (beams,
// a block or two each) run with per-head warps (each warp one query head's
// whole range, 4 warps x 3 stages); longer ones as in the plain decode (warps
// split a range's blocks). On the OPT-13B geometry: 8 parallel samples with
// about 9 own blocks each, 70.7 us split against 74.9 us per-head; beams of
// about 1 own block, 54.3 us split against 50.1 us per-head.
#ifndef KVP_GROUP_PER_HEAD_BELOW
#define KVP_GROUP_PER_HEAD_BELOW 4
#endif
// Warps and stages of the CUDA-core kernel on longer own ranges. One stage per
// warp: an own range is a few blocks per (sequence, head), so a deeper ring
// buys little, and 32 KiB of tiles per CTA lets registers, not shared memory,
// set the CTAs per SM (four at 4 warps).
#ifndef KVP_GROUP_SPLIT_WARPS
#define KVP_GROUP_SPLIT_WARPS KVP_SIMT_WARPS
#endif
#ifndef KVP_GROUP_SPLIT_STAGES
#define KVP_GROUP_SPLIT_STAGES 1
#endif

namespace {

constexpr int kMaxDevices = 64;

int cuda_fail(cudaError_t e, const char* what) {
  return fail(KVP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

int sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 148;
  int n = cache[d].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d);
    if (n <= 0) n = 148;
    cache[d].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Raises a kernel's dynamic shared-memory limit once per (kernel, device).
template <typename K>
cudaError_t ensure_smem(K kernel, int bytes) {
  static std::mutex mu;
  static std::unordered_map<const void*, uint64_t> done;  // kernel -> device bit mask
  const int d = current_device();
  const uint64_t bit = d < 64 ? (1ull << d) : 0;
  const void* key = reinterpret_cast<const void*>(kernel);
  {
    std::lock_guard<std::mutex> g(mu);
    auto it = done.find(key);
    if (bit && it != done.end() && (it->second & bit)) return cudaSuccess;
  }
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) {
    std::lock_guard<std::mutex> g(mu);
    done[key] |= bit;
  }
  return e;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D view [rows][cols] of 2-byte elements with a {64, box_rows} box and
// 128-byte swizzle; out-of-range rows read as zeros.
int make_map(CUtensorMap* map, const void* base, int32_t dtype, uint64_t rows, uint64_t cols,
             uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(KVP_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      dtype == KVP_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KVP_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return KVP_OK;
}

// 3-D view of [rows][128] 2-byte elements as {64 dims, rows, 2 halves} (strides
// 256 and 128 bytes) with a {64, box_rows, 2} box: one load brings a whole
// (block, head) tile as [half][row][64], 128-byte swizzled.
int make_map_halves(CUtensorMap* map, const void* base, int32_t dtype, uint64_t rows,
                    uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(KVP_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {64, rows, 2};
  cuuint64_t strides[2] = {256, 128};
  cuuint32_t box[3] = {64, box_rows, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt =
      dtype == KVP_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = fn(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KVP_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (%d)", int(r));
  return KVP_OK;
}

// 2-D view [rows][128] of E4M3 codes with a {128, box_rows} box and 128-byte
// swizzle: one load brings a whole (block, head) tile of head_dim 128.
int make_map_u8(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(KVP_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KVP_ERR_CUDA, "cuTensorMapEncodeTiled (E4M3) failed (%d)", int(r));
  return KVP_OK;
}

// 4-D view of a virtually contiguous cache, {64 dims, tokens, 2 halves, KV
// heads} with strides (Hkv * 256, 128, 256) bytes, and a {64, box_tokens,
// box_halves, 1} box: one load brings box_tokens consecutive tokens of one
// head as [half][token][64], 128-byte swizzled (the paged tiles' layout).
int make_map_vcache(CUtensorMap* map, const void* base, int32_t dtype, uint64_t tokens,
                    uint32_t heads, uint32_t box_tokens, uint32_t box_halves) {
  auto fn = encode_fn();
  if (!fn) return fail(KVP_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[4] = {64, tokens, 2, heads};
  cuuint64_t strides[3] = {uint64_t(heads) * 256, 128, 256};
  cuuint32_t box[4] = {64, box_tokens, box_halves, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt =
      dtype == KVP_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = fn(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KVP_ERR_CUDA, "cuTensorMapEncodeTiled (4-D) failed (%d)", int(r));
  return KVP_OK;
}

// q of a prefill chunk as 3-D {128 dims, heads, tokens} (strides 256 and
// heads * 256 bytes) with a {64, G, 128 / G} box: 128 rows (token, head of the
// group), 128-byte swizzled, per 64-dim half.
// Prefill queries or outputs [tokens, heads, 128]: box {64 dims, G heads,
// rows / G tokens} (128 rows for a Q tile, 32 for one softmax warp's output).
int make_map_prefill_q(CUtensorMap* map, const void* base, int32_t dtype, uint32_t heads,
                       uint64_t tokens, uint32_t G, uint32_t rows) {
  auto fn = encode_fn();
  if (!fn) return fail(KVP_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {128, heads, tokens};
  cuuint64_t strides[2] = {256, uint64_t(heads) * 256};
  cuuint32_t box[3] = {64, G, rows / G};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt =
      dtype == KVP_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = fn(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KVP_ERR_CUDA, "cuTensorMapEncodeTiled (prefill q) failed (%d)", int(r));
  return KVP_OK;
}

// E4M3 decode with at least this many query heads per KV head runs on the
// tensor cores (E4M3 tiles widened in shared memory); fewer, on CUDA cores.
#ifndef KVP_FP8_TC_MIN_G
#define KVP_FP8_TC_MIN_G 2
#endif

// Prefill chunks with at least this many query rows (q_len x query heads per
// KV head, a power of two) run on the prompt-shaped kernel (128 query rows per
// tensor-core tile); shorter ones on the decode-shaped kernel, 16 columns per
// launch, which suits a few tokens per sequence.
#ifndef KVP_PREFILL_TILE_MIN_ROWS
#define KVP_PREFILL_TILE_MIN_ROWS 64
#endif

// Tokens per tile of the CUDA-core decode over a virtually contiguous cache.
#ifndef KVP_VCACHE_SIMT_TILE
#define KVP_VCACHE_SIMT_TILE 16
#endif

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int ilog2(int64_t v) {
  int l = 0;
  while ((int64_t(1) << l) < v) ++l;
  return (int64_t(1) << l) == v ? l : -1;
}

struct Workspace {
  size_t ml_bytes, acc_bytes, total;
};

Workspace ws_layout(int64_t S, int64_t Hq, int64_t D, int64_t pmax) {
  Workspace w{};
  if (pmax <= 1) return w;
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  w.ml_bytes = up(size_t(S * Hq * pmax * 2 * 4));
  w.acc_bytes = up(size_t(S * Hq * pmax * D * 4));
  w.total = w.ml_bytes + w.acc_bytes;
  return w;
}

// Grouped decode: [ml][acc][plan], with pmax + 1 slots per (sequence, head)
// (a sequence's shared prefix and its own range may each end in a partial
// partition) and the grouping plan.
struct GroupWorkspace {
  size_t ml_bytes, acc_bytes, plan_bytes, total;
};

GroupWorkspace group_ws_layout(int64_t S, int64_t Hq, int64_t D, int64_t pmax) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  GroupWorkspace w{};
  w.ml_bytes = up(size_t(S * Hq * (pmax + 1) * 2 * 4));
  w.acc_bytes = up(size_t(S * Hq * (pmax + 1) * D * 4));
  w.plan_bytes = up(size_t(kvp::grp::plan_words(S) * 4));
  w.total = w.ml_bytes + w.acc_bytes + w.plan_bytes;
  return w;
}

// ---- decode launches ----------------------------------------------------------
// programmatic: launched with programmatic stream serialisation (the grouped
// decode, after the shared-prefix kernel).
template <typename T, int D, int BS, int W = KVP_SIMT_WARPS, int NST = KVP_SIMT_STAGES,
          bool PH = false, bool F8 = false, bool VC = false>
int launch_simt(const CUtensorMap& km, const CUtensorMap& vm, const kvp::dev::DecodeArgs& a,
                cudaStream_t st, bool programmatic = false, int grid_x = 0) {
  constexpr int EB = F8 ? 1 : 2;
  constexpr int NW = (BS * D * EB >= 8192 && W > 1) ? W / 2 : W;
  using C = kvp::dev::SimtCfg<T, D, BS, NW, NST, EB>;
  auto k = kvp::dev::decode_simt_kernel<T, D, BS, NW, NST, PH, F8, VC>;
  cudaError_t e = ensure_smem(k, C::kSmemBytes);
  if (e != cudaSuccess) return cuda_fail(e, "decode (CUDA cores): smem attribute");
  dim3 grid(grid_x > 0 ? grid_x : a.pmax, PH ? (a.num_q_heads + NW - 1) / NW : a.num_q_heads,
            a.num_seqs);
  if (!programmatic) {
    k<<<grid, NW * 32, C::kSmemBytes, st>>>(km, vm, a);
  } else {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(NW * 32);
    cfg.dynamicSmemBytes = size_t(C::kSmemBytes);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k, km, vm, a);
    if (e != cudaSuccess) return cuda_fail(e, "decode (CUDA cores): launch");
  }
  e = cudaGetLastError();
  return e == cudaSuccess ? KVP_OK : cuda_fail(e, "decode (CUDA cores): launch");
}

template <typename T, int BS, int NG, int MODE = kvp::dev::tc::kPlain>
int launch_tc(const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& qm,
              const kvp::dev::DecodeArgs& a, cudaStream_t st) {
  auto k = kvp::dev::decode_tc_kernel<T, BS, NG, MODE>;
  constexpr bool f8 = MODE == kvp::dev::tc::kPlainF8;
  // context lengths of small batches are cached in shared memory
  using Cfg = kvp::dev::tc::Cfg<NG, f8>;
  const int ctx_bytes = a.num_seqs <= Cfg::kCtxCap ? 4 * a.num_seqs : 0;
  const int smem = Cfg::kSmemBytes + ctx_bytes;
  cudaError_t e = ensure_smem(k, Cfg::kSmemBytes + 4 * Cfg::kCtxCap);
  if (e != cudaSuccess) return cuda_fail(e, "decode (tensor cores): smem attribute");
  const int64_t units = int64_t(a.num_seqs) * a.num_kv_heads * a.pmax;
  const int grid = int(units < sm_count() ? units : sm_count());
  k<<<grid, f8 ? kvp::dev::tc::kThreadsF8 : kvp::dev::tc::kThreads, smem, st>>>(km, vm, qm, a, units);
  e = cudaGetLastError();
  return e == cudaSuccess ? KVP_OK : cuda_fail(e, "decode (tensor cores): launch");
}

template <typename T, int D>
int launch_reduce(const kvp::dev::DecodeArgs& a, cudaStream_t st) {
  // Programmatic dependent launch: the reduce's launch overlaps the tail of the
  // partition kernel; the kernel itself waits (griddepcontrol.wait) for it.
  cudaLaunchConfig_t cfg{};
  constexpr int HR = kvp::dev::kReduceHeads;
  const size_t smem = size_t(HR) * (a.ws_slots + 1) * 4;
  if (smem > 200u * 1024u)
    return fail(KVP_ERR_INVALID, "decode reduce: %d partitions per sequence is too many", a.ws_slots);
  if (smem > 48u * 1024u) {
    cudaError_t e = ensure_smem(kvp::dev::decode_reduce_kernel<T, D>, int(200u * 1024u));
    if (e != cudaSuccess) return cuda_fail(e, "decode reduce: smem attribute");
  }
  cfg.gridDim = dim3((a.num_q_heads + HR - 1) / HR, a.num_seqs * a.q_len);
  cfg.blockDim = dim3(HR * D);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kvp::dev::decode_reduce_kernel<T, D>, a);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? KVP_OK : cuda_fail(e, "decode reduce: launch");
}

template <typename T>
int simt_fp8_by_bs(int bs, const CUtensorMap& km, const CUtensorMap& vm,
                   const kvp::dev::DecodeArgs& a, cudaStream_t st) {
  constexpr int W = KVP_SIMT_WARPS, NST = KVP_SIMT_FP8_STAGES;
  switch (bs) {
    case 8: return launch_simt<T, 128, 8, W, NST, false, true>(km, vm, a, st);
    case 16: return launch_simt<T, 128, 16, W, NST, false, true>(km, vm, a, st);
    case 32: return launch_simt<T, 128, 32, W, NST, false, true>(km, vm, a, st);
  }
  return fail(KVP_ERR_INVALID, "block_size %d not supported", bs);
}

template <typename T, int D>
int simt_by_bs(int bs, const CUtensorMap& km, const CUtensorMap& vm, const kvp::dev::DecodeArgs& a,
               cudaStream_t st) {
  constexpr int W = KVP_SIMT_WARPS;
  if (a.num_seqs >= KVP_SIMT_ONE_STAGE_SEQS) {
    switch (bs) {
      case 8: return launch_simt<T, D, 8, W, 1>(km, vm, a, st);
      case 16: return launch_simt<T, D, 16, W, 1>(km, vm, a, st);
      case 32: return launch_simt<T, D, 32, W, 1>(km, vm, a, st);
    }
  } else {
    switch (bs) {
      case 8: return launch_simt<T, D, 8>(km, vm, a, st);
      case 16: return launch_simt<T, D, 16>(km, vm, a, st);
      case 32: return launch_simt<T, D, 32>(km, vm, a, st);
    }
  }
  return fail(KVP_ERR_INVALID, "block_size %d not supported", bs);
}

// Grouped decode, tensor-core kernel: launched right after the plan kernel
// with programmatic serialisation; its CTAs set up while the plan is built and
// wait for it (griddepcontrol.wait) before reading it.
// with_private: the kernel also takes every sequence's own range (else the
// CUDA-core kernel launched after it does).
// grid_ctas > 0 sets the grid (else one CTA per SM, at most one per unit);
// programmatic: launched right after the plan kernel, overlapping it.
template <typename T, int BS, int NG>
int launch_tc_grouped(const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& qm,
                      const kvp::dev::DecodeArgs& a, cudaStream_t st, bool with_private,
                      int grid_ctas, bool programmatic) {
  auto k = kvp::dev::decode_tc_kernel<T, BS, NG, kvp::dev::tc::kGrouped>;
  using Cfg = kvp::dev::tc::Cfg<NG>;
  // shared-memory tail: context lengths, per-sequence prefix blocks and the
  // subgroup table when they fit (S <= kPlanCap), else the context lengths alone
  auto plan_bytes = [](int S) { return 8 * S + (S / 2 + 1) * kvp::grp::kSubWords * 4; };
  const int S = a.num_seqs;
  const int ctx_bytes = S <= Cfg::kPlanCap ? plan_bytes(S) : (S <= Cfg::kCtxCap ? 4 * S : 0);
  const int tail_max = std::max(4 * Cfg::kCtxCap, plan_bytes(Cfg::kPlanCap));
  cudaError_t e = ensure_smem(k, Cfg::kSmemBytes + tail_max);
  if (e != cudaSuccess) return cuda_fail(e, "grouped decode: smem attribute");
  const int64_t units = with_private ? int64_t(a.num_seqs) * a.num_kv_heads * a.pmax : 0;
  // at most S / 2 subgroups of at most pmax shared partitions each
  const int64_t bound = std::max<int64_t>(
      1, units + int64_t(a.num_seqs / 2) * a.num_kv_heads * a.pmax);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(unsigned(grid_ctas > 0 ? grid_ctas : (bound < sm_count() ? bound : sm_count())));
  cfg.blockDim = dim3(kvp::dev::tc::kThreads);
  cfg.dynamicSmemBytes = size_t(Cfg::kSmemBytes + ctx_bytes);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = programmatic ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, k, km, vm, qm, a, units);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? KVP_OK : cuda_fail(e, "grouped decode: launch");
}

template <typename T>
int tc_grouped_dispatch(int bs, int ng, const CUtensorMap& km, const CUtensorMap& vm,
                        const CUtensorMap& qm, const kvp::dev::DecodeArgs& a, cudaStream_t st,
                        bool with_private, int grid_ctas, bool programmatic) {
  if (bs == 16)
    return ng == 8 ? launch_tc_grouped<T, 16, 8>(km, vm, qm, a, st, with_private, grid_ctas, programmatic)
                   : launch_tc_grouped<T, 16, 16>(km, vm, qm, a, st, with_private, grid_ctas, programmatic);
  return ng == 8 ? launch_tc_grouped<T, 32, 8>(km, vm, qm, a, st, with_private, grid_ctas, programmatic)
                 : launch_tc_grouped<T, 32, 16>(km, vm, qm, a, st, with_private, grid_ctas, programmatic);
}

// Packed grouped decode: one persistent tensor-core launch over units x KV heads.
template <typename T, int BS, int NG>
int launch_tc_packed(const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& qm,
                     const kvp::dev::DecodeArgs& a, int64_t units, int32_t groups, cudaStream_t st) {
  auto k = kvp::dev::decode_tc_kernel<T, BS, NG, kvp::dev::tc::kPacked>;
  using Cfg = kvp::dev::tc::Cfg<NG>;
  constexpr int kMax = 226 * 1024;
  const int ctx_bytes = a.num_seqs <= Cfg::kCtxCap ? 4 * a.num_seqs : 0;
  cudaError_t e = ensure_smem(k, kMax);
  if (e != cudaSuccess) return cuda_fail(e, "packed decode: smem attribute");
  // the group table in shared memory when it fits (the Q gather and every
  // unit read it), else read from the plan in global memory
  kvp::dev::DecodeArgs a2 = a;
  int smem = Cfg::kSmemBytes + ctx_bytes;
  const int grp_bytes = groups * kvp::pack::kGroupWords * 4;
  if (smem + grp_bytes <= kMax) {
    smem += grp_bytes;
    a2.plan_packed = 2;
  }
  const int grid = int(units < sm_count() ? units : sm_count());
  k<<<grid, kvp::dev::tc::kThreads, smem, st>>>(km, vm, qm, a2, units);
  e = cudaGetLastError();
  return e == cudaSuccess ? KVP_OK : cuda_fail(e, "packed decode: launch");
}

// Grouped decode: the CUDA-core kernel over the sequences' own ranges
// (grid_x partitions; 0: all).
int launch_own_ranges(int bs, int32_t dtype, bool per_head, const CUtensorMap& km,
                      const CUtensorMap& vm, const kvp::dev::DecodeArgs& a, cudaStream_t st,
                      bool programmatic, int grid_x) {
  using H = __half;
  using B = __nv_bfloat16;
  constexpr int W = KVP_GROUP_SPLIT_WARPS, N = KVP_GROUP_SPLIT_STAGES;
  const bool f16 = dtype == KVP_F16;
  if (per_head) {
    if (bs == 16)
      return f16 ? launch_simt<H, 128, 16, 4, 3, true>(km, vm, a, st, programmatic, grid_x)
                 : launch_simt<B, 128, 16, 4, 3, true>(km, vm, a, st, programmatic, grid_x);
    return f16 ? launch_simt<H, 128, 32, 4, 3, true>(km, vm, a, st, programmatic, grid_x)
               : launch_simt<B, 128, 32, 4, 3, true>(km, vm, a, st, programmatic, grid_x);
  }
  if (bs == 16)
    return f16 ? launch_simt<H, 128, 16, W, N>(km, vm, a, st, programmatic, grid_x)
               : launch_simt<B, 128, 16, W, N>(km, vm, a, st, programmatic, grid_x);
  return f16 ? launch_simt<H, 128, 32, W, N>(km, vm, a, st, programmatic, grid_x)
             : launch_simt<B, 128, 32, W, N>(km, vm, a, st, programmatic, grid_x);
}

// Multi-query (prefill) chunk on the tensor cores: one launch per a.q_count
// queries of every sequence.
template <typename T, int BS, int NG>
int launch_tc_mq(const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& qm,
                 const kvp::dev::DecodeArgs& a, cudaStream_t st) {
  auto k = kvp::dev::decode_tc_kernel<T, BS, NG, kvp::dev::tc::kMultiQuery>;
  using Cfg = kvp::dev::tc::Cfg<NG>;
  const int ctx_bytes = a.num_seqs <= Cfg::kCtxCap ? 4 * a.num_seqs : 0;
  cudaError_t e = ensure_smem(k, Cfg::kSmemBytes + 4 * Cfg::kCtxCap);
  if (e != cudaSuccess) return cuda_fail(e, "prefill (tensor cores): smem attribute");
  const int64_t units = int64_t(a.num_seqs) * a.num_kv_heads * a.pmax;
  const int grid = int(units < sm_count() ? units : sm_count());
  k<<<grid, kvp::dev::tc::kThreads, Cfg::kSmemBytes + ctx_bytes, st>>>(km, vm, qm, a, units);
  e = cudaGetLastError();
  return e == cudaSuccess ? KVP_OK : cuda_fail(e, "prefill (tensor cores): launch");
}

template <typename T, int BS>
int launch_prefill_tc(const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& qm,
                      const CUtensorMap& om, const kvp::dev::DecodeArgs& a, int32_t qtiles,
                      cudaStream_t st) {
  auto k = kvp::dev::prefill_tc_kernel<T, BS>;
  cudaError_t e = ensure_smem(k, kvp::dev::pf::kSmemBytes);
  if (e != cudaSuccess) return cuda_fail(e, "prefill (prompt tiles): smem attribute");
  const int64_t units = int64_t(a.num_seqs) * a.num_kv_heads * qtiles * a.pmax;
  if (units >= int64_t(kvp::dev::pf::kMaxUnits))
    return fail(KVP_ERR_INVALID, "paged_attention_prefill: %lld work units exceed the kernel's index range",
                static_cast<long long>(units));
  const int grid = int(units < sm_count() ? units : sm_count());
  k<<<grid, kvp::dev::pf::kThreads, kvp::dev::pf::kSmemBytes, st>>>(km, vm, qm, om, a, qtiles, units);
  e = cudaGetLastError();
  return e == cudaSuccess ? KVP_OK : cuda_fail(e, "prefill (prompt tiles): launch");
}

template <typename T>
int tc_mq_dispatch(int bs, int ng, const CUtensorMap& km, const CUtensorMap& vm,
                   const CUtensorMap& qm, const kvp::dev::DecodeArgs& a, cudaStream_t st) {
  if (bs == 16) return ng == 8 ? launch_tc_mq<T, 16, 8>(km, vm, qm, a, st)
                               : launch_tc_mq<T, 16, 16>(km, vm, qm, a, st);
  return ng == 8 ? launch_tc_mq<T, 32, 8>(km, vm, qm, a, st)
                 : launch_tc_mq<T, 32, 16>(km, vm, qm, a, st);
}

// E4M3 cache, grouped-query heads: the tensor-core decode with converter warps.
template <typename T>
int tc_fp8_dispatch(int bs, int G, const CUtensorMap& km, const CUtensorMap& vm,
                    const CUtensorMap& qm, const kvp::dev::DecodeArgs& a, cudaStream_t st) {
  constexpr int M = kvp::dev::tc::kPlainF8;
  const int ng = G <= 4 ? 4 : (G <= 8 ? 8 : 16);
  if (bs == 16) {
    if (ng == 4) return launch_tc<T, 16, 4, M>(km, vm, qm, a, st);
    if (ng == 8) return launch_tc<T, 16, 8, M>(km, vm, qm, a, st);
    return launch_tc<T, 16, 16, M>(km, vm, qm, a, st);
  }
  if (ng == 4) return launch_tc<T, 32, 4, M>(km, vm, qm, a, st);
  if (ng == 8) return launch_tc<T, 32, 8, M>(km, vm, qm, a, st);
  return launch_tc<T, 32, 16, M>(km, vm, qm, a, st);
}

template <typename T>
int tc_dispatch(int bs, int G, const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& qm,
                const kvp::dev::DecodeArgs& a, cudaStream_t st) {
  const int ng = G <= 4 ? 4 : (G <= 8 ? 8 : 16);
  if (bs == 16) {
    if (ng == 4) return launch_tc<T, 16, 4>(km, vm, qm, a, st);
    if (ng == 8) return launch_tc<T, 16, 8>(km, vm, qm, a, st);
    return launch_tc<T, 16, 16>(km, vm, qm, a, st);
  }
  if (ng == 4) return launch_tc<T, 32, 4>(km, vm, qm, a, st);
  if (ng == 8) return launch_tc<T, 32, 8>(km, vm, qm, a, st);
  return launch_tc<T, 32, 16>(km, vm, qm, a, st);
}

// A caller's grouping plan, checked word by word before any kernel reads it:
// counts in range, every index inside the batch and every shared prefix inside
// the block tables, members distinct and in one subgroup each, per-sequence
// prefixes equal to their subgroup's, and the header's partition counts. (A
// plan built from other tables that passes still gives wrong results; only
// its shape is checked.)
bool host_plan_fits(const int32_t* plan, int32_t S, int32_t MB, int32_t max_ctx, int32_t bs,
                    int32_t part, int mmax, int32_t pmax) {
  namespace g = kvp::grp;
  const int32_t n_sub = plan[g::kNumSub], psh = plan[g::kSharedParts], pown = plan[g::kOwnParts];
  if (n_sub < 0 || n_sub > S / 2 || psh < 0 || psh > pmax || pown < 0 || pown > pmax ||
      plan[g::kSharedBlocks] < 0 || plan[g::kOwnBlocks] < 0)
    return false;
  const int32_t cap = max_ctx / bs;  // a shared prefix is made of full blocks
  const int32_t* cblk = plan + g::kHdrWords;
  const int32_t* subs = plan + g::sub_offset(S);
  std::vector<int32_t> owner(size_t(S), -1);
  int32_t most = 0;
  for (int32_t i = 0; i < n_sub; ++i) {
    const int32_t* e = subs + int64_t(i) * g::kSubWords;
    const int32_t c = e[0], nm = e[1];
    if (c < 1 || c > cap || c > MB || nm < 2 || nm > mmax) return false;
    most = std::max(most, (c * bs + part - 1) / part);
    for (int m = 0; m < nm; ++m) {
      const int32_t s = e[4 + m];
      if (s < 0 || s >= S || owner[size_t(s)] >= 0 || cblk[s] != c) return false;
      owner[size_t(s)] = i;
    }
  }
  for (int32_t s = 0; s < S; ++s)
    if (owner[size_t(s)] < 0 && cblk[s] != 0) return false;
  return most == psh;
}

// Packed decode workspace: (m, l) and acc with one slot per chunk of the
// longest group stream, then room for a copy of the plan.
struct PackWorkspace {
  size_t ml_bytes, acc_bytes, plan_bytes, total;
};

PackWorkspace pack_ws_layout(int64_t S, int64_t Hq, int64_t D, int64_t slots, int64_t plan_words) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  PackWorkspace w{};
  w.ml_bytes = up(size_t(S * Hq * slots * 2 * 4));
  w.acc_bytes = up(size_t(S * Hq * slots * D * 4));
  w.plan_bytes = up(size_t(plan_words * 4));
  w.total = w.ml_bytes + w.acc_bytes + w.plan_bytes;
  return w;
}

// Words of a packed plan as its header gives them (header, groups, units, entries).
int64_t pack_plan_used_words(const int32_t* plan) {
  namespace pk = kvp::pack;
  return int64_t(plan[pk::kEntryOffset]) + 2 * int64_t(plan[pk::kEntries]);
}

// A caller's packed plan, checked word by word before any kernel reads it:
// header and offsets consistent, every group's members distinct sequences of
// the batch whose group word names it, every sequence in one group, every
// group's entries inside the entry table with column masks inside its columns
// and valid counts in [1, block_size], every (group, chunk) covered by exactly
// one unit record with its entries. (A plan of other tables that passes still
// gives wrong results; only its shape is checked.)
bool pack_plan_fits(const int32_t* plan, int32_t S, int32_t bs, int32_t G, int mmax) {
  namespace pk = kvp::pack;
  const int32_t ngr = plan[pk::kGroups], nu = plan[pk::kUnits], ne = plan[pk::kEntries];
  const int32_t mc = plan[pk::kMaxChunks], bpc = plan[pk::kChunkBlocks];
  if (plan[pk::kBlockSize] != bs || bpc != 512 / bs) return false;
  if (ngr < 0 || ngr > S || nu < 0 || ne < 0 || mc < 0) return false;
  if (int64_t(plan[pk::kUnitOffset]) != pk::group_offset(S) + int64_t(ngr) * pk::kGroupWords) return false;
  if (int64_t(plan[pk::kEntryOffset]) != int64_t(plan[pk::kUnitOffset]) + int64_t(nu) * pk::kUnitWords)
    return false;
  std::vector<int32_t> owner(size_t(S), -1);
  std::vector<int32_t> chunk_base(size_t(ngr) + 1, 0);
  const int32_t* ents = plan + plan[pk::kEntryOffset];
  for (int32_t g = 0; g < ngr; ++g) {
    const int32_t* e = plan + pk::group_offset(S) + int64_t(g) * pk::kGroupWords;
    const int32_t first = e[0], nm = e[1], n = e[2], ch = e[3];
    if (nm < 1 || nm > mmax || first < 0 || n < 0 || int64_t(first) + n > ne) return false;
    if (ch != (n + bpc - 1) / bpc || ch > mc) return false;
    chunk_base[size_t(g) + 1] = chunk_base[size_t(g)] + ch;
    for (int m = 0; m < nm; ++m) {
      const int32_t sq = e[4 + m];
      if (sq < 0 || sq >= S || owner[size_t(sq)] >= 0 || plan[pk::kHdrWords + sq] != g) return false;
      owner[size_t(sq)] = g;
    }
    const uint32_t cols = nm * G >= 32 ? 0xFFFFFFFFu : ((1u << (nm * G)) - 1u);
    for (int32_t i = first; i < first + n; ++i) {
      const uint32_t w = uint32_t(ents[2 * int64_t(i) + 1]);
      const int32_t valid = int32_t(w & 0xFFu);
      if (((w >> 8) & ~cols) != 0 || valid < 1 || valid > bs) return false;
    }
  }
  for (int32_t sq = 0; sq < S; ++sq)
    if (owner[size_t(sq)] < 0) return false;
  if (chunk_base[size_t(ngr)] != nu) return false;
  std::vector<char> seen(size_t(nu), 0);
  const int32_t* u = plan + plan[pk::kUnitOffset];
  for (int32_t i = 0; i < nu; ++i, u += pk::kUnitWords) {
    const int32_t g = u[0], first = u[1], n = u[2], chunk = u[3];
    if (g < 0 || g >= ngr) return false;
    const int32_t* e = plan + pk::group_offset(S) + int64_t(g) * pk::kGroupWords;
    if (chunk < 0 || chunk >= e[3] || first != e[0] + chunk * bpc ||
        n != std::min(bpc, e[2] - chunk * bpc))
      return false;
    char& sn = seen[size_t(chunk_base[size_t(g)] + chunk)];
    if (sn) return false;
    sn = 1;
  }
  return true;
}

// Argument checks of the decode entry points (fn names the caller in the
// messages); *empty is set when there is nothing to do (no sequences).
int check_decode(const char* fn, const void* q, const void* k_cache, const void* v_cache,
                 const int32_t* block_tables, const int32_t* context_lens, int32_t num_seqs,
                 int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                 int32_t num_blocks, int32_t max_blocks_per_seq, int32_t max_context_len,
                 float scale, int32_t partition_size, const void* out, int32_t dtype, bool* empty) {
  *empty = false;
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
      max_blocks_per_seq <= 0 || max_context_len < 0 || partition_size < 0)
    return fail(KVP_ERR_INVALID, "%s: bad sizes", fn);
  if (num_q_heads % num_kv_heads) return fail(KVP_ERR_INVALID, "%s: num_q_heads %% num_kv_heads != 0", fn);
  if (head_dim != 64 && head_dim != 128) return fail(KVP_ERR_INVALID, "%s: head_dim must be 64 or 128", fn);
  if (block_size != 8 && block_size != 16 && block_size != 32)
    return fail(KVP_ERR_INVALID, "%s: block_size must be 8, 16 or 32", fn);
  if (dtype != KVP_F16 && dtype != KVP_BF16) return fail(KVP_ERR_INVALID, "%s: bad dtype", fn);
  if (int64_t(max_context_len) > int64_t(max_blocks_per_seq) * block_size)
    return fail(KVP_ERR_INVALID, "%s: max_context_len > max_blocks_per_seq * block_size", fn);
  if (int64_t(num_blocks) * num_kv_heads * block_size >= (int64_t(1) << 31))
    return fail(KVP_ERR_INVALID, "%s: pool too large for 32-bit row coordinates", fn);
  if (partition_size % block_size) return fail(KVP_ERR_INVALID, "%s: partition_size must be a multiple of block_size", fn);
  if (!std::isfinite(scale)) return fail(KVP_ERR_INVALID, "%s: scale not finite", fn);
  if (num_seqs == 0) {
    *empty = true;
    return KVP_OK;
  }
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out)
    return fail(KVP_ERR_INVALID, "%s: NULL pointer", fn);
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return fail(KVP_ERR_INVALID, "%s: misaligned pointer", fn);
  return KVP_OK;
}

}  // namespace

extern "C" {

int reshape_and_cache(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                      const int64_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
                      int32_t head_dim, int32_t block_size, int32_t num_blocks, int32_t dtype,
                      kvp_stream_t stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
    return fail(KVP_ERR_INVALID, "reshape_and_cache: bad sizes");
  if (dtype != KVP_F16 && dtype != KVP_BF16) return fail(KVP_ERR_INVALID, "reshape_and_cache: bad dtype");
  const int lcpr = ilog2(head_dim / 8);
  const int lbs = ilog2(block_size);
  if (head_dim % 8 || lcpr < 0 || lbs < 0)
    return fail(KVP_ERR_INVALID, "reshape_and_cache: head_dim/8 and block_size must be powers of two");
  if (num_tokens == 0) return KVP_OK;
  if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping)
    return fail(KVP_ERR_INVALID, "reshape_and_cache: NULL pointer");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(slot_mapping, 8))
    return fail(KVP_ERR_INVALID, "reshape_and_cache: misaligned pointer");
  const int64_t chunks = int64_t(num_tokens) * num_kv_heads * (head_dim / 8);
  if (chunks >= (int64_t(1) << 31)) return fail(KVP_ERR_INVALID, "reshape_and_cache: too many tokens in one call");
  const int threads = 256;
  int64_t blocks = (chunks + threads - 1) / threads;
  const int64_t cap = int64_t(sm_count()) * 16;
  if (blocks > cap) blocks = cap;
  kvp::dev::reshape_and_cache_kernel<<<int(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), static_cast<uint4*>(k_cache),
      static_cast<uint4*>(v_cache), slot_mapping, uint32_t(chunks), uint32_t(num_kv_heads),
      uint32_t(lcpr), uint32_t(lbs), int64_t(num_blocks) * block_size);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KVP_OK : cuda_fail(e, "reshape_and_cache: launch");
}

int copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs, int32_t num_pairs,
                int32_t num_blocks, int64_t block_elems, int32_t dtype, kvp_stream_t stream) {
  if (num_pairs < 0 || num_blocks <= 0 || block_elems <= 0)
    return fail(KVP_ERR_INVALID, "copy_blocks: bad sizes");
  if (dtype != KVP_F16 && dtype != KVP_BF16 && dtype != KVP_FP8_E4M3)
    return fail(KVP_ERR_INVALID, "copy_blocks: bad dtype");
  const int64_t eb = dtype == KVP_FP8_E4M3 ? 1 : 2;
  if ((block_elems * eb) % 16) return fail(KVP_ERR_INVALID, "copy_blocks: block bytes not a multiple of 16");
  if (num_pairs == 0) return KVP_OK;
  if (num_pairs > 65535) return fail(KVP_ERR_INVALID, "copy_blocks: more than 65535 pairs in one call");
  if (!k_cache || !v_cache || !pairs) return fail(KVP_ERR_INVALID, "copy_blocks: NULL pointer");
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(pairs, 4))
    return fail(KVP_ERR_INVALID, "copy_blocks: misaligned pointer");
  const int64_t chunks = block_elems * eb / 16;
  constexpr int64_t per_cta = 256 * kvp::dev::kCopyUnroll;
  int gx = int((chunks + per_cta - 1) / per_cta);
  if (gx > 64) gx = 64;
  dim3 grid(gx, num_pairs, 2);
  kvp::dev::copy_blocks_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), pairs, chunks, num_blocks);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KVP_OK : cuda_fail(e, "copy_blocks: launch");
}

size_t kvp_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                  int32_t max_context_len, int32_t partition_size) {
  if (partition_size <= 0 || num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len <= 0)
    return 0;
  const int64_t pmax = (int64_t(max_context_len) + partition_size - 1) / partition_size;
  return ws_layout(num_seqs, num_q_heads, head_dim, pmax).total;
}

int paged_attention_decode(const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens,
                           int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                           int32_t head_dim, int32_t block_size, int32_t num_blocks,
                           int32_t max_blocks_per_seq, int32_t max_context_len, float scale,
                           int32_t partition_size, void* workspace, size_t workspace_bytes,
                           void* out, int32_t dtype, kvp_stream_t stream) {
  bool empty = false;
  const int crc = check_decode("paged_attention_decode", q, k_cache, v_cache, block_tables,
                               context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                               block_size, num_blocks, max_blocks_per_seq, max_context_len, scale,
                               partition_size, out, dtype, &empty);
  if (crc || empty) return crc;

  const int G = num_q_heads / num_kv_heads;
  const bool tensor_cores = G > 1 && G <= 16 && head_dim == 128 && (block_size == 16 || block_size == 32);
  if (tensor_cores && partition_size % 128)
    return fail(KVP_ERR_INVALID, "paged_attention_decode: grouped-query path needs partition_size %% 128 == 0");

  const int32_t ctx_cap = max_context_len > 0 ? max_context_len : 1;
  int32_t part_tokens, pmax;
  if (partition_size > 0) {
    part_tokens = partition_size;
    pmax = (ctx_cap + partition_size - 1) / partition_size;
  } else {
    part_tokens = ((ctx_cap + block_size - 1) / block_size) * block_size;
    pmax = 1;
  }
  const Workspace wl = ws_layout(num_seqs, num_q_heads, head_dim, pmax);
  if (wl.total) {
    if (!workspace || workspace_bytes < wl.total)
      return fail(KVP_ERR_INVALID, "paged_attention_decode: workspace of %zu bytes needed", wl.total);
    if (!aligned(workspace, 256)) return fail(KVP_ERR_INVALID, "paged_attention_decode: workspace not 256-byte aligned");
  }

  kvp::dev::DecodeArgs a{};
  a.q = q;
  a.out = out;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.ws_ml = wl.total ? static_cast<float*>(workspace) : nullptr;
  a.ws_acc = wl.total ? reinterpret_cast<float*>(static_cast<char*>(workspace) + wl.ml_bytes) : nullptr;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.num_blocks = num_blocks;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.max_context_len = max_context_len;
  a.part_blocks = part_tokens / block_size;
  a.part_tokens = part_tokens;
  a.pmax = pmax;
  a.ws_slots = pmax;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.q_len = 1;
  a.q_first = 0;
  a.q_count = 1;

  const uint64_t rows = uint64_t(num_blocks) * num_kv_heads * block_size;
  CUtensorMap km, vm;
  int rc;
  if (!tensor_cores && head_dim == 128) {  // CUDA-core kernel: one 3-D box per tile
    rc = make_map_halves(&km, k_cache, dtype, rows, block_size);
    if (rc) return rc;
    rc = make_map_halves(&vm, v_cache, dtype, rows, block_size);
  } else if (tensor_cores) {  // K as 2-D boxes per 64-dim half, V as one 3-D box per block
    rc = make_map(&km, k_cache, dtype, rows, head_dim, block_size);
    if (rc) return rc;
    rc = make_map_halves(&vm, v_cache, dtype, rows, block_size);
  } else {
    rc = make_map(&km, k_cache, dtype, rows, head_dim, block_size);
    if (rc) return rc;
    rc = make_map(&vm, v_cache, dtype, rows, head_dim, block_size);
  }
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  if (tensor_cores) {
    CUtensorMap qm;
    rc = make_map(&qm, q, dtype, uint64_t(num_seqs) * num_q_heads, head_dim, kvp::dev::tc::kN);
    if (rc) return rc;
    rc = dtype == KVP_F16 ? tc_dispatch<__half>(block_size, G, km, vm, qm, a, st)
                          : tc_dispatch<__nv_bfloat16>(block_size, G, km, vm, qm, a, st);
  } else if (head_dim == 128) {
    rc = dtype == KVP_F16 ? simt_by_bs<__half, 128>(block_size, km, vm, a, st)
                          : simt_by_bs<__nv_bfloat16, 128>(block_size, km, vm, a, st);
  } else {
    rc = dtype == KVP_F16 ? simt_by_bs<__half, 64>(block_size, km, vm, a, st)
                          : simt_by_bs<__nv_bfloat16, 64>(block_size, km, vm, a, st);
  }
  if (rc || pmax <= 1) return rc;
  if (head_dim == 128)
    return dtype == KVP_F16 ? launch_reduce<__half, 128>(a, st) : launch_reduce<__nv_bfloat16, 128>(a, st);
  return dtype == KVP_F16 ? launch_reduce<__half, 64>(a, st) : launch_reduce<__nv_bfloat16, 64>(a, st);
}

size_t kvp_prefill_workspace_bytes(int32_t num_seqs, int32_t q_len, int32_t num_q_heads,
                                   int32_t head_dim, int32_t max_context_len,
                                   int32_t partition_size) {
  if (q_len <= 0 || num_seqs <= 0 || int64_t(num_seqs) * q_len > 0x7FFFFFFF) return 0;
  return kvp_decode_workspace_bytes(num_seqs * q_len, num_q_heads, head_dim, max_context_len,
                                    partition_size);
}

int paged_attention_prefill(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, const int32_t* context_lens,
                            int32_t num_seqs, int32_t q_len, int32_t num_q_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                            int32_t num_blocks, int32_t max_blocks_per_seq,
                            int32_t max_context_len, float scale, int32_t partition_size,
                            void* workspace, size_t workspace_bytes, void* out, int32_t dtype,
                            kvp_stream_t stream) {
  bool empty = false;
  const int crc = check_decode("paged_attention_prefill", q, k_cache, v_cache, block_tables,
                               context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                               block_size, num_blocks, max_blocks_per_seq, max_context_len, scale,
                               partition_size, out, dtype, &empty);
  if (crc || empty) return crc;
  if (q_len < 1 || int64_t(num_seqs) * q_len > 0x7FFFFFFF)
    return fail(KVP_ERR_INVALID, "paged_attention_prefill: bad q_len");
  if (q_len == 1)
    return paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                                  num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                  max_blocks_per_seq, max_context_len, scale, partition_size,
                                  workspace, workspace_bytes, out, dtype, stream);
  const int G = num_q_heads / num_kv_heads;
  if (head_dim != 128 || (block_size != 16 && block_size != 32) || G > 16)
    return fail(KVP_ERR_INVALID,
                "paged_attention_prefill: needs head_dim 128, block_size 16 or 32, and at most 16 "
                "query heads per KV head");
  if (partition_size % 128)
    return fail(KVP_ERR_INVALID, "paged_attention_prefill: partition_size must be a multiple of 128");
  const int32_t ctx_cap = max_context_len > 0 ? max_context_len : 1;
  // prompt-shaped chunks: 128 query rows per tile (G a power of two)
  const bool prompt_tiles = (G & (G - 1)) == 0 && int64_t(q_len) * G >= KVP_PREFILL_TILE_MIN_ROWS;
  const int32_t round = prompt_tiles ? 128 : block_size;
  int32_t part_tokens, pmax;
  if (partition_size > 0) {
    part_tokens = partition_size;
    pmax = (ctx_cap + partition_size - 1) / partition_size;
  } else {
    part_tokens = ((ctx_cap + round - 1) / round) * round;
    pmax = 1;
  }
  const Workspace wl = ws_layout(int64_t(num_seqs) * q_len, num_q_heads, head_dim, pmax);
  if (wl.total) {
    if (!workspace || workspace_bytes < wl.total)
      return fail(KVP_ERR_INVALID, "paged_attention_prefill: workspace of %zu bytes needed", wl.total);
    if (!aligned(workspace, 256)) return fail(KVP_ERR_INVALID, "paged_attention_prefill: workspace not 256-byte aligned");
  }
  kvp::dev::DecodeArgs a{};
  a.q = q;
  a.out = out;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.ws_ml = wl.total ? static_cast<float*>(workspace) : nullptr;
  a.ws_acc = wl.total ? reinterpret_cast<float*>(static_cast<char*>(workspace) + wl.ml_bytes) : nullptr;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.num_blocks = num_blocks;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.max_context_len = max_context_len;
  a.part_blocks = part_tokens / block_size;
  a.part_tokens = part_tokens;
  a.pmax = pmax;
  a.ws_slots = pmax;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.q_len = q_len;
  const uint64_t rows = uint64_t(num_blocks) * num_kv_heads * block_size;
  CUtensorMap km, vm, qm;
  int rc = make_map(&km, k_cache, dtype, rows, head_dim, block_size);
  if (!rc) rc = make_map_halves(&vm, v_cache, dtype, rows, block_size);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (prompt_tiles) {
    CUtensorMap om;
    rc = make_map_prefill_q(&qm, q, dtype, uint32_t(num_q_heads), uint64_t(num_seqs) * q_len,
                            uint32_t(G), 128);
    if (!rc)
      rc = make_map_prefill_q(&om, out, dtype, uint32_t(num_q_heads), uint64_t(num_seqs) * q_len,
                              uint32_t(G), 32);
    if (rc) return rc;
    const int32_t qtiles = (q_len + 128 / G - 1) / (128 / G);
    a.q_first = 0;
    a.q_count = q_len;
    const bool f16 = dtype == KVP_F16;
    using H = __half;
    using B = __nv_bfloat16;
    if (block_size == 16)
      rc = f16 ? launch_prefill_tc<H, 16>(km, vm, qm, om, a, qtiles, st)
               : launch_prefill_tc<B, 16>(km, vm, qm, om, a, qtiles, st);
    else
      rc = f16 ? launch_prefill_tc<H, 32>(km, vm, qm, om, a, qtiles, st)
               : launch_prefill_tc<B, 32>(km, vm, qm, om, a, qtiles, st);
    if (rc || pmax <= 1) return rc;
    return f16 ? launch_reduce<H, 128>(a, st) : launch_reduce<B, 128>(a, st);
  }
  rc = make_map(&qm, q, dtype, uint64_t(num_seqs) * q_len * num_q_heads, head_dim, kvp::dev::tc::kN);
  if (rc) return rc;
  // up to 16 columns per launch: 16 / G query tokens of every sequence
  const int per_launch = std::max(1, kvp::dev::tc::kN / G);
  for (int32_t c0 = 0; c0 < q_len; c0 += per_launch) {
    a.q_first = c0;
    a.q_count = std::min(per_launch, q_len - c0);
    const int ng = a.q_count * G <= 8 ? 8 : 16;
    rc = dtype == KVP_F16 ? tc_mq_dispatch<__half>(block_size, ng, km, vm, qm, a, st)
                          : tc_mq_dispatch<__nv_bfloat16>(block_size, ng, km, vm, qm, a, st);
    if (rc) return rc;
  }
  if (pmax <= 1) return KVP_OK;
  return dtype == KVP_F16 ? launch_reduce<__half, 128>(a, st) : launch_reduce<__nv_bfloat16, 128>(a, st);
}

int reshape_and_cache_fp8(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                          const int64_t* slot_mapping, const float* k_scale, const float* v_scale,
                          int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                          int32_t block_size, int32_t num_blocks, int32_t dtype,
                          kvp_stream_t stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
    return fail(KVP_ERR_INVALID, "reshape_and_cache_fp8: bad sizes");
  if (dtype != KVP_F16 && dtype != KVP_BF16) return fail(KVP_ERR_INVALID, "reshape_and_cache_fp8: bad dtype");
  const int lcpr = ilog2(head_dim / 16);
  const int lbs = ilog2(block_size);
  if (head_dim % 16 || lcpr < 0 || lbs < 0)
    return fail(KVP_ERR_INVALID, "reshape_and_cache_fp8: head_dim/16 and block_size must be powers of two");
  if (num_tokens == 0) return KVP_OK;
  if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping || !k_scale || !v_scale)
    return fail(KVP_ERR_INVALID, "reshape_and_cache_fp8: NULL pointer");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(slot_mapping, 8) || !aligned(k_scale, 4) || !aligned(v_scale, 4))
    return fail(KVP_ERR_INVALID, "reshape_and_cache_fp8: misaligned pointer");
  const int64_t chunks = int64_t(num_tokens) * num_kv_heads * (head_dim / 16);
  if (chunks >= (int64_t(1) << 31))
    return fail(KVP_ERR_INVALID, "reshape_and_cache_fp8: too many tokens in one call");
  const int threads = 256;
  int64_t blocks = (chunks + threads - 1) / threads;
  const int64_t cap = int64_t(sm_count()) * 16;
  if (blocks > cap) blocks = cap;
  auto k = dtype == KVP_F16 ? kvp::dev::reshape_and_cache_fp8_kernel<__half>
                            : kvp::dev::reshape_and_cache_fp8_kernel<__nv_bfloat16>;
  k<<<int(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), static_cast<uint4*>(k_cache),
      static_cast<uint4*>(v_cache), slot_mapping, k_scale, v_scale, uint32_t(chunks),
      uint32_t(num_kv_heads), uint32_t(lcpr), uint32_t(lbs), int64_t(num_blocks) * block_size);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KVP_OK : cuda_fail(e, "reshape_and_cache_fp8: launch");
}

int paged_attention_decode_fp8(const void* q, const void* k_cache, const void* v_cache,
                               const float* k_scale, const float* v_scale,
                               const int32_t* block_tables, const int32_t* context_lens,
                               int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                               int32_t head_dim, int32_t block_size, int32_t num_blocks,
                               int32_t max_blocks_per_seq, int32_t max_context_len, float scale,
                               int32_t partition_size, void* workspace, size_t workspace_bytes,
                               void* out, int32_t dtype, kvp_stream_t stream) {
  bool empty = false;
  const int crc = check_decode("paged_attention_decode_fp8", q, k_cache, v_cache, block_tables,
                               context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                               block_size, num_blocks, max_blocks_per_seq, max_context_len, scale,
                               partition_size, out, dtype, &empty);
  if (crc || empty) return crc;
  if (head_dim != 128) return fail(KVP_ERR_INVALID, "paged_attention_decode_fp8: head_dim must be 128");
  if (!k_scale || !v_scale) return fail(KVP_ERR_INVALID, "paged_attention_decode_fp8: NULL scales");
  if (!aligned(k_scale, 4) || !aligned(v_scale, 4))
    return fail(KVP_ERR_INVALID, "paged_attention_decode_fp8: misaligned scales");
  const int32_t ctx_cap = max_context_len > 0 ? max_context_len : 1;
  int32_t part_tokens, pmax;
  if (partition_size > 0) {
    part_tokens = partition_size;
    pmax = (ctx_cap + partition_size - 1) / partition_size;
  } else {
    part_tokens = ((ctx_cap + block_size - 1) / block_size) * block_size;
    pmax = 1;
  }
  const Workspace wl = ws_layout(num_seqs, num_q_heads, head_dim, pmax);
  if (wl.total) {
    if (!workspace || workspace_bytes < wl.total)
      return fail(KVP_ERR_INVALID, "paged_attention_decode_fp8: workspace of %zu bytes needed", wl.total);
    if (!aligned(workspace, 256))
      return fail(KVP_ERR_INVALID, "paged_attention_decode_fp8: workspace not 256-byte aligned");
  }
  kvp::dev::DecodeArgs a{};
  a.q = q;
  a.out = out;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.ws_ml = wl.total ? static_cast<float*>(workspace) : nullptr;
  a.ws_acc = wl.total ? reinterpret_cast<float*>(static_cast<char*>(workspace) + wl.ml_bytes) : nullptr;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.num_blocks = num_blocks;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.max_context_len = max_context_len;
  a.part_blocks = part_tokens / block_size;
  a.part_tokens = part_tokens;
  a.pmax = pmax;
  a.ws_slots = pmax;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.q_len = 1;
  a.q_first = 0;
  a.q_count = 1;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  const uint64_t rows = uint64_t(num_blocks) * num_kv_heads * block_size;
  CUtensorMap km, vm;
  int rc = make_map_u8(&km, k_cache, rows, block_size);
  if (!rc) rc = make_map_u8(&vm, v_cache, rows, block_size);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G = num_q_heads / num_kv_heads;
  if (G >= KVP_FP8_TC_MIN_G && G <= 16 && (block_size == 16 || block_size == 32)) {
    // grouped-query heads: one widened tile serves the group's heads on the tensor cores
    CUtensorMap qm;
    rc = make_map(&qm, q, dtype, uint64_t(num_seqs) * num_q_heads, head_dim, kvp::dev::tc::kN);
    if (rc) return rc;
    rc = dtype == KVP_F16 ? tc_fp8_dispatch<__half>(block_size, G, km, vm, qm, a, st)
                          : tc_fp8_dispatch<__nv_bfloat16>(block_size, G, km, vm, qm, a, st);
  } else {
    rc = dtype == KVP_F16 ? simt_fp8_by_bs<__half>(block_size, km, vm, a, st)
                          : simt_fp8_by_bs<__nv_bfloat16>(block_size, km, vm, a, st);
  }
  if (rc || pmax <= 1) return rc;
  return dtype == KVP_F16 ? launch_reduce<__half, 128>(a, st) : launch_reduce<__nv_bfloat16, 128>(a, st);
}

size_t kvp_decode_grouped_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                          int32_t max_context_len, int32_t partition_size) {
  if (partition_size <= 0 || num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len < 0)
    return 0;
  const int64_t ctx = max_context_len > 0 ? max_context_len : 1;
  const int64_t pmax = (ctx + partition_size - 1) / partition_size;
  // covers paged_attention_decode's own layout too (pmax slots, no plan)
  return group_ws_layout(num_seqs, num_q_heads, head_dim, pmax).total;
}

int paged_attention_decode_grouped(const void* q, const void* k_cache, const void* v_cache,
                                   const int32_t* block_tables, const int32_t* context_lens,
                                   int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                   int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                   int32_t max_blocks_per_seq, int32_t max_context_len, float scale,
                                   int32_t partition_size, const int32_t* host_plan,
                                   const int32_t* device_plan, void* workspace,
                                   size_t workspace_bytes, void* out, int32_t dtype,
                                   kvp_stream_t stream) {
  bool empty = false;
  const int crc = check_decode("paged_attention_decode_grouped", q, k_cache, v_cache, block_tables,
                               context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                               block_size, num_blocks, max_blocks_per_seq, max_context_len, scale,
                               partition_size, out, dtype, &empty);
  if (crc || empty) return crc;
  // Columns of the tensor-core contraction: 8 for one query head per KV head
  // (up to 8 members per subgroup), else 16 (16 / G members).
  const int G = num_q_heads / num_kv_heads;
  const int ng = kvp::grp::plan_columns(G);
  const int mmax = kvp::grp::members_per_subgroup(G);
  const bool grouped = head_dim == 128 && (block_size == 16 || block_size == 32) && G <= 16 &&
                       mmax >= 2 && partition_size > 0 && partition_size % 128 == 0 &&
                       num_seqs <= kvp::grp::kMaxSeqs && max_context_len > 0;
  if (!grouped)
    return paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                                  num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                  max_blocks_per_seq, max_context_len, scale, partition_size,
                                  workspace, workspace_bytes, out, dtype, stream);

  const int32_t pmax = (max_context_len + partition_size - 1) / partition_size;
  const GroupWorkspace wl = group_ws_layout(num_seqs, num_q_heads, head_dim, pmax);
  if (!workspace || workspace_bytes < wl.total)
    return fail(KVP_ERR_INVALID, "paged_attention_decode_grouped: workspace of %zu bytes needed", wl.total);
  if (!aligned(workspace, 256))
    return fail(KVP_ERR_INVALID, "paged_attention_decode_grouped: workspace not 256-byte aligned");

  if (device_plan && !host_plan)
    return fail(KVP_ERR_INVALID, "paged_attention_decode_grouped: device_plan needs host_plan");
  if (device_plan && !aligned(device_plan, 4))
    return fail(KVP_ERR_INVALID, "paged_attention_decode_grouped: misaligned device_plan");
  char* ws = static_cast<char*>(workspace);
  int32_t* plan = device_plan ? const_cast<int32_t*>(device_plan)
                              : reinterpret_cast<int32_t*>(ws + wl.ml_bytes + wl.acc_bytes);
  kvp::dev::DecodeArgs a{};
  a.q = q;
  a.out = out;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.ws_ml = reinterpret_cast<float*>(ws);
  a.ws_acc = reinterpret_cast<float*>(ws + wl.ml_bytes);
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.num_blocks = num_blocks;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.max_context_len = max_context_len;
  a.part_blocks = partition_size / block_size;
  a.part_tokens = partition_size;
  a.pmax = pmax;
  a.ws_slots = pmax + 1;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.q_len = 1;
  a.q_first = 0;
  a.q_count = 1;
  a.plan = plan;

  // One query head per KV head: the CUDA-core kernel takes the sequences' own
  // ranges (short, many: its independent per-warp pipelines suit them); with
  // grouped-query heads the tensor-core kernel takes both.
  const bool simt_private = G == 1;
  const uint64_t rows = uint64_t(num_blocks) * num_kv_heads * block_size;
  // tensor cores: K as 2-D boxes, V as 3-D boxes; CUDA cores: both 3-D
  CUtensorMap km, vm3, qm, km3;
  int rc = make_map(&km, k_cache, dtype, rows, head_dim, block_size);
  if (!rc) rc = make_map_halves(&vm3, v_cache, dtype, rows, block_size);
  if (!rc) rc = make_map(&qm, q, dtype, uint64_t(num_seqs) * num_q_heads, head_dim, kvp::dev::tc::kN);
  if (!rc && simt_private) rc = make_map_halves(&km3, k_cache, dtype, rows, block_size);
  if (rc) return rc;
  const CUtensorMap& vm = vm3;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  using namespace kvp::dev;
  const int sms = sm_count();
  bool after_kernel = false;  // the tensor-core kernel precedes the CUDA-core one
  if (host_plan) {
    // 1. the caller's plan (host memory) into the workspace; its header sizes
    // the launches: the tensor-core kernel gets a share of the SMs by the
    // estimated times of the shared blocks and of the sequences' own blocks,
    // and the CUDA-core kernel, launched right after it, the rest
    namespace g = kvp::grp;
    const int32_t n_sub = host_plan[g::kNumSub], psh = host_plan[g::kSharedParts];
    const int32_t pown = host_plan[g::kOwnParts];
    const int32_t sblk = host_plan[g::kSharedBlocks], oblk = host_plan[g::kOwnBlocks];
    if (!host_plan_fits(host_plan, num_seqs, max_blocks_per_seq, max_context_len, block_size,
                        partition_size, mmax, pmax))
      return fail(KVP_ERR_INVALID, "paged_attention_decode_grouped: host_plan does not fit this batch");
    if (!device_plan) {
      cudaError_t e = cudaMemcpyAsync(plan, host_plan, size_t(g::plan_words(num_seqs)) * 4,
                                      cudaMemcpyHostToDevice, st);
      if (e != cudaSuccess) return cuda_fail(e, "grouped decode: plan copy");
    }
    if (simt_private) {
      const int64_t shared_units = int64_t(n_sub) * psh * num_kv_heads;
      if (shared_units > 0) {
        const double ts = double(sblk) * 100.0 / KVP_GROUP_TC_RATE, to = double(oblk);
        int64_t grid = std::llround(sms * ts / (ts + to));
        grid = std::max<int64_t>(1, std::min<int64_t>(grid, std::min<int64_t>(sms, shared_units)));
        rc = dtype == KVP_F16
                 ? tc_grouped_dispatch<__half>(block_size, ng, km, vm, qm, a, st, false, int(grid), false)
                 : tc_grouped_dispatch<__nv_bfloat16>(block_size, ng, km, vm, qm, a, st, false, int(grid), false);
        if (rc) return rc;
        after_kernel = true;
      }
      if (pown > 0) {
        const bool per_head = int64_t(oblk) < int64_t(KVP_GROUP_PER_HEAD_BELOW) * num_seqs;
        rc = launch_own_ranges(block_size, dtype, per_head, km3, vm3, a, st, after_kernel, pown);
        if (rc) return rc;
      }
    } else {
      const int64_t units = int64_t(num_seqs) * num_kv_heads * pmax + int64_t(n_sub) * psh * num_kv_heads;
      const int grid = int(std::max<int64_t>(1, std::min<int64_t>(units, sms)));
      rc = dtype == KVP_F16
               ? tc_grouped_dispatch<__half>(block_size, ng, km, vm, qm, a, st, true, grid, false)
               : tc_grouped_dispatch<__nv_bfloat16>(block_size, ng, km, vm, qm, a, st, true, grid, false);
      if (rc) return rc;
    }
  } else {
    // 1. the plan (one CTA)
    cudaError_t e = ensure_smem(group_plan_kernel, int(kvp::grp::plan_smem_bytes(kvp::grp::kMaxSeqs)));
    if (e != cudaSuccess) return cuda_fail(e, "grouped decode: plan smem attribute");
    group_plan_kernel<<<1, kvp::grp::plan_threads(kvp::grp::sort_len(num_seqs)),
                        kvp::grp::plan_smem_bytes(num_seqs), st>>>(
        block_tables, context_lens, num_seqs, max_blocks_per_seq, max_context_len, block_size,
        partition_size, mmax, num_blocks, plan);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "grouped decode: plan launch");
    // 2. shared prefixes once per subgroup (and, with grouped-query heads, every
    // sequence's own range) on the tensor cores, overlapping the plan kernel
    rc = dtype == KVP_F16
             ? tc_grouped_dispatch<__half>(block_size, ng, km, vm, qm, a, st, !simt_private, 0, true)
             : tc_grouped_dispatch<__nv_bfloat16>(block_size, ng, km, vm, qm, a, st, !simt_private, 0, true);
    if (rc) return rc;
    // 2b. every sequence's own range on the CUDA cores, overlapping the tail of 2
    if (simt_private) {
      rc = launch_own_ranges(block_size, dtype, false, km3, vm3, a, st, true, 0);
      if (rc) return rc;
    }
  }
  // 3. the log-sum-exp merge of every row
  return dtype == KVP_F16 ? launch_reduce<__half, 128>(a, st) : launch_reduce<__nv_bfloat16, 128>(a, st);
}

int reshape_and_cache_vcache(const void* k_new, const void* v_new, kvp_vcache* vc,
                             const int32_t* slots, const int32_t* positions, int32_t num_tokens,
                             kvp_stream_t stream) {
  if (!vc) return fail(KVP_ERR_INVALID, "reshape_and_cache_vcache: NULL cache");
  if (num_tokens < 0) return fail(KVP_ERR_INVALID, "reshape_and_cache_vcache: bad sizes");
  if (num_tokens == 0) return KVP_OK;
  if (!k_new || !v_new || !slots || !positions)
    return fail(KVP_ERR_INVALID, "reshape_and_cache_vcache: NULL pointer");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(slots, 4) || !aligned(positions, 4))
    return fail(KVP_ERR_INVALID, "reshape_and_cache_vcache: misaligned pointer");
  const int lcpr = ilog2(vc->head_dim / 8);
  const int64_t chunks = int64_t(num_tokens) * vc->num_kv_heads * (vc->head_dim / 8);
  if (lcpr < 0 || chunks >= (int64_t(1) << 31))
    return fail(KVP_ERR_INVALID, "reshape_and_cache_vcache: too many tokens in one call");
  const int threads = 256;
  int64_t blocks = (chunks + threads - 1) / threads;
  const int64_t cap = int64_t(sm_count()) * 16;
  if (blocks > cap) blocks = cap;
  kvp::dev::vcache_write_kernel<<<int(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
      reinterpret_cast<uint4*>(vc->k_base), reinterpret_cast<uint4*>(vc->v_base), slots, positions,
      vc->cap_dev, uint32_t(chunks), uint32_t(vc->num_kv_heads), uint32_t(lcpr), vc->num_slots,
      int64_t(vc->slot_tokens));
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KVP_OK : cuda_fail(e, "reshape_and_cache_vcache: launch");
}

int attention_decode_vcache(const void* q, const kvp_vcache* vc, const int32_t* seq_slots,
                            const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                            int32_t max_context_len, float scale, int32_t partition_size,
                            void* workspace, size_t workspace_bytes, void* out,
                            kvp_stream_t stream) {
  if (!vc) return fail(KVP_ERR_INVALID, "attention_decode_vcache: NULL cache");
  const int32_t Hkv = vc->num_kv_heads, D = vc->head_dim, dtype = vc->dtype;
  if (num_seqs < 0 || num_q_heads <= 0 || max_context_len < 0 || partition_size < 0)
    return fail(KVP_ERR_INVALID, "attention_decode_vcache: bad sizes");
  if (num_q_heads % Hkv) return fail(KVP_ERR_INVALID, "attention_decode_vcache: num_q_heads %% num_kv_heads != 0");
  if (max_context_len > vc->max_tokens)
    return fail(KVP_ERR_INVALID, "attention_decode_vcache: max_context_len > the cache's max_tokens");
  if (!std::isfinite(scale)) return fail(KVP_ERR_INVALID, "attention_decode_vcache: scale not finite");
  if (num_seqs == 0) return KVP_OK;
  if (!q || !seq_slots || !context_lens || !out)
    return fail(KVP_ERR_INVALID, "attention_decode_vcache: NULL pointer");
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(seq_slots, 4) || !aligned(context_lens, 4))
    return fail(KVP_ERR_INVALID, "attention_decode_vcache: misaligned pointer");
  const int G = num_q_heads / Hkv;
  if (G > 16) return fail(KVP_ERR_INVALID, "attention_decode_vcache: more than 16 query heads per KV head");
  const bool tensor_cores = G > 1;
  constexpr int kSimtTile = KVP_VCACHE_SIMT_TILE;
  const int tile = tensor_cores ? kvp::dev::tc::kTileTok : kSimtTile;
  if (partition_size % tile)
    return fail(KVP_ERR_INVALID, "attention_decode_vcache: partition_size must be a multiple of %d", tile);
  const int32_t ctx_cap = max_context_len > 0 ? max_context_len : 1;
  int32_t part_tokens, pmax;
  if (partition_size > 0) {
    part_tokens = partition_size;
    pmax = (ctx_cap + partition_size - 1) / partition_size;
  } else {
    part_tokens = ((ctx_cap + tile - 1) / tile) * tile;
    pmax = 1;
  }
  const Workspace wl = ws_layout(num_seqs, num_q_heads, D, pmax);
  if (wl.total) {
    if (!workspace || workspace_bytes < wl.total)
      return fail(KVP_ERR_INVALID, "attention_decode_vcache: workspace of %zu bytes needed", wl.total);
    if (!aligned(workspace, 256)) return fail(KVP_ERR_INVALID, "attention_decode_vcache: workspace not 256-byte aligned");
  }
  kvp::dev::DecodeArgs a{};
  a.q = q;
  a.out = out;
  a.block_tables = nullptr;
  a.context_lens = context_lens;
  a.ws_ml = wl.total ? static_cast<float*>(workspace) : nullptr;
  a.ws_acc = wl.total ? reinterpret_cast<float*>(static_cast<char*>(workspace) + wl.ml_bytes) : nullptr;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = Hkv;
  a.num_blocks = 1;
  a.max_blocks_per_seq = 1;
  a.max_context_len = max_context_len;
  a.part_blocks = part_tokens / tile;
  a.part_tokens = part_tokens;
  a.pmax = pmax;
  a.ws_slots = pmax;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.q_len = 1;
  a.q_first = 0;
  a.q_count = 1;
  a.vc_seq_slots = seq_slots;
  a.vc_cap = vc->cap_dev;
  a.vc_slot_tokens = vc->slot_tokens;
  a.vc_num_slots = vc->num_slots;
  const uint64_t tokens = uint64_t(vc->num_slots) * uint64_t(vc->slot_tokens);
  const void* kb = reinterpret_cast<const void*>(vc->k_base);
  const void* vb = reinterpret_cast<const void*>(vc->v_base);
  CUtensorMap km, vm;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc;
  if (tensor_cores) {
    rc = make_map_vcache(&km, kb, dtype, tokens, uint32_t(Hkv), kvp::dev::tc::kTileTok, 1);
    if (!rc) rc = make_map_vcache(&vm, vb, dtype, tokens, uint32_t(Hkv), kvp::dev::tc::kTileTok, 2);
    CUtensorMap qm;
    if (!rc) rc = make_map(&qm, q, dtype, uint64_t(num_seqs) * num_q_heads, D, kvp::dev::tc::kN);
    if (rc) return rc;
    constexpr int M = kvp::dev::tc::kContig, TT = kvp::dev::tc::kTileTok;
    using H = __half;
    using B = __nv_bfloat16;
    const bool f16 = dtype == KVP_F16;
    if (G <= 4)
      rc = f16 ? launch_tc<H, TT, 4, M>(km, vm, qm, a, st) : launch_tc<B, TT, 4, M>(km, vm, qm, a, st);
    else if (G <= 8)
      rc = f16 ? launch_tc<H, TT, 8, M>(km, vm, qm, a, st) : launch_tc<B, TT, 8, M>(km, vm, qm, a, st);
    else
      rc = f16 ? launch_tc<H, TT, 16, M>(km, vm, qm, a, st) : launch_tc<B, TT, 16, M>(km, vm, qm, a, st);
  } else {
    rc = make_map_vcache(&km, kb, dtype, tokens, uint32_t(Hkv), kSimtTile, 2);
    if (!rc) rc = make_map_vcache(&vm, vb, dtype, tokens, uint32_t(Hkv), kSimtTile, 2);
    if (rc) return rc;
    // the paged decode's shapes, by the same batch-size rule, so the A/B compares like with like
    constexpr int W = KVP_SIMT_WARPS, N = KVP_SIMT_STAGES;
    const bool f16 = dtype == KVP_F16;
    if (num_seqs >= KVP_SIMT_ONE_STAGE_SEQS)
      rc = f16 ? launch_simt<__half, 128, kSimtTile, W, 1, false, false, true>(km, vm, a, st)
               : launch_simt<__nv_bfloat16, 128, kSimtTile, W, 1, false, false, true>(km, vm, a, st);
    else
      rc = f16 ? launch_simt<__half, 128, kSimtTile, W, N, false, false, true>(km, vm, a, st)
               : launch_simt<__nv_bfloat16, 128, kSimtTile, W, N, false, false, true>(km, vm, a, st);
  }
  if (rc || pmax <= 1) return rc;
  return dtype == KVP_F16 ? launch_reduce<__half, 128>(a, st) : launch_reduce<__nv_bfloat16, 128>(a, st);
}

size_t kvp_decode_packed_workspace_bytes(const int32_t* host_plan, int32_t num_seqs,
                                         int32_t num_q_heads, int32_t head_dim) {
  if (!host_plan || num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0) return 0;
  const int64_t slots = std::max<int32_t>(1, host_plan[kvp::pack::kMaxChunks]);
  return pack_ws_layout(num_seqs, num_q_heads, head_dim, slots, pack_plan_used_words(host_plan)).total;
}

int paged_attention_decode_packed(const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* context_lens, int32_t num_seqs,
                                  int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                  int32_t block_size, int32_t num_blocks, int32_t max_context_len,
                                  float scale, const int32_t* host_plan, const int32_t* device_plan,
                                  void* workspace, size_t workspace_bytes, void* out,
                                  int32_t dtype, kvp_stream_t stream) {
  const char* fn = "paged_attention_decode_packed";
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 || max_context_len < 0)
    return fail(KVP_ERR_INVALID, "%s: bad sizes", fn);
  if (num_q_heads % num_kv_heads) return fail(KVP_ERR_INVALID, "%s: num_q_heads %% num_kv_heads != 0", fn);
  const int G = num_q_heads / num_kv_heads;
  if (head_dim != 128 || (block_size != 16 && block_size != 32) || G > 16)
    return fail(KVP_ERR_INVALID, "%s: needs head_dim 128, block_size 16 or 32, at most 16 query heads per KV head", fn);
  if (dtype != KVP_F16 && dtype != KVP_BF16) return fail(KVP_ERR_INVALID, "%s: bad dtype", fn);
  if (num_seqs > kvp::grp::kMaxSeqs) return fail(KVP_ERR_INVALID, "%s: more than %d sequences", fn, kvp::grp::kMaxSeqs);
  if (int64_t(num_blocks) * num_kv_heads * block_size >= (int64_t(1) << 31))
    return fail(KVP_ERR_INVALID, "%s: pool too large for 32-bit row coordinates", fn);
  if (!std::isfinite(scale)) return fail(KVP_ERR_INVALID, "%s: scale not finite", fn);
  if (num_seqs == 0) return KVP_OK;
  if (!q || !k_cache || !v_cache || !context_lens || !out || !host_plan || !workspace)
    return fail(KVP_ERR_INVALID, "%s: NULL pointer", fn);
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(context_lens, 4) || !aligned(workspace, 256) || (device_plan && !aligned(device_plan, 4)))
    return fail(KVP_ERR_INVALID, "%s: misaligned pointer", fn);
  const int mmax = kvp::grp::members_per_subgroup(G);
  if (!pack_plan_fits(host_plan, num_seqs, block_size, G, mmax))
    return fail(KVP_ERR_INVALID, "%s: host_plan does not fit this batch", fn);
  const int64_t plan_words = pack_plan_used_words(host_plan);
  const int32_t slots = std::max<int32_t>(1, host_plan[kvp::pack::kMaxChunks]);
  const PackWorkspace wl = pack_ws_layout(num_seqs, num_q_heads, head_dim, slots, plan_words);
  if (workspace_bytes < wl.total)
    return fail(KVP_ERR_INVALID, "%s: workspace of %zu bytes needed", fn, wl.total);
  char* ws = static_cast<char*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* plan = device_plan ? const_cast<int32_t*>(device_plan)
                              : reinterpret_cast<int32_t*>(ws + wl.ml_bytes + wl.acc_bytes);
  if (!device_plan) {
    cudaError_t e = cudaMemcpyAsync(plan, host_plan, size_t(plan_words) * 4, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "packed decode: plan copy");
  }
  kvp::dev::DecodeArgs a{};
  a.q = q;
  a.out = out;
  a.block_tables = nullptr;
  a.context_lens = context_lens;
  a.ws_ml = reinterpret_cast<float*>(ws);
  a.ws_acc = reinterpret_cast<float*>(ws + wl.ml_bytes);
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.num_blocks = num_blocks;
  a.max_blocks_per_seq = 1;
  a.max_context_len = max_context_len;
  a.part_tokens = 512;
  a.part_blocks = 512 / block_size;
  a.pmax = 1;
  a.ws_slots = slots;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.q_len = 1;
  a.q_first = 0;
  a.q_count = 1;
  a.plan = plan;
  a.plan_packed = 1;
  const uint64_t rows = uint64_t(num_blocks) * num_kv_heads * block_size;
  CUtensorMap km, vm, qm;
  int rc = make_map(&km, k_cache, dtype, rows, head_dim, block_size);
  if (!rc) rc = make_map_halves(&vm, v_cache, dtype, rows, block_size);
  if (!rc) rc = make_map(&qm, q, dtype, uint64_t(num_seqs) * num_q_heads, head_dim, kvp::dev::tc::kN);
  if (rc) return rc;
  const int64_t units = int64_t(host_plan[kvp::pack::kUnits]) * num_kv_heads;
  const int32_t ngroups = host_plan[kvp::pack::kGroups];
  if (units > 0) {
    const int ng = kvp::grp::plan_columns(G);
    const bool f16 = dtype == KVP_F16;
    using H = __half;
    using B = __nv_bfloat16;
    if (block_size == 16)
      rc = ng == 8 ? (f16 ? launch_tc_packed<H, 16, 8>(km, vm, qm, a, units, ngroups, st)
                          : launch_tc_packed<B, 16, 8>(km, vm, qm, a, units, ngroups, st))
                   : (f16 ? launch_tc_packed<H, 16, 16>(km, vm, qm, a, units, ngroups, st)
                          : launch_tc_packed<B, 16, 16>(km, vm, qm, a, units, ngroups, st));
    else
      rc = ng == 8 ? (f16 ? launch_tc_packed<H, 32, 8>(km, vm, qm, a, units, ngroups, st)
                          : launch_tc_packed<B, 32, 8>(km, vm, qm, a, units, ngroups, st))
                   : (f16 ? launch_tc_packed<H, 32, 16>(km, vm, qm, a, units, ngroups, st)
                          : launch_tc_packed<B, 32, 16>(km, vm, qm, a, units, ngroups, st));
    if (rc) return rc;
  }
  // the log-sum-exp merge of every row (a sequence of no tokens gets zeros)
  return dtype == KVP_F16 ? launch_reduce<__half, 128>(a, st) : launch_reduce<__nv_bfloat16, 128>(a, st);
}

}  // extern "C"

int kvp_vcache_push_cap(int32_t* cap_dev, int32_t slot, int32_t value, void* stream) {
  kvp::dev::vcache_set_cap_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(cap_dev, slot, value);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KVP_OK : cuda_fail(e, "kv_vcache: capacity update");
}

// One thread waits, with the decode kernels' bounded wait, for a phase of an
// mbarrier that nothing arrives on: the wait runs out and records a status.
__global__ void selftest_bounded_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    kvp::dev::mbar_init(&bar, 1);
    kvp::dev::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) kvp::dev::mbar_wait(&bar, 0, 0xFFFFu, limit_ns);
}

extern "C" {

int kvp_selftest_bounded_wait(int32_t limit_ms, kvp_stream_t stream) {
  if (limit_ms < 1 || limit_ms > 2000)
    return fail(KVP_ERR_INVALID, "kvp_selftest_bounded_wait: limit_ms must be in [1, 2000]");
  selftest_bounded_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      uint64_t(limit_ms) * 1000000ull);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KVP_OK : cuda_fail(e, "kvp_selftest_bounded_wait: launch");
}

int kvp_check_device_error(kvp_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "kvp_check_device_error: stream synchronize");
  unsigned long long v = 0;
  e = cudaMemcpyFromSymbol(&v, kvp::dev::g_error_word, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "kvp_check_device_error: read");
  if (v == 0) return KVP_OK;
  const unsigned long long zero = 0;
  e = cudaMemcpyToSymbol(kvp::dev::g_error_word, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "kvp_check_device_error: clear");
  const unsigned kind = unsigned(v >> 56);
  const unsigned long long payload = v & ((1ull << 56) - 1);
  static const char* names[] = {"none", "slot out of range (token index)",
                                "block table entry out of range (seq << 32 | logical block)",
                                "context length out of range (sequence)",
                                "copy pair out of range (pair index)", "bounded wait timed out (site)"};
  const char* name = kind < 6 ? names[kind] : "unknown";
  if (kind == kvp::dev::KVP_DEVERR_TIMEOUT)
    return fail(KVP_ERR_CUDA, "device: %s 0x%llx", name, payload);
  return fail(KVP_ERR_BOUNDS, "device: %s %llu", name, payload);
}

}  // extern "C"

// ---- decode for callers that cannot allocate device memory ------------------------
// The split-context scratch of paged_attention_decode_noalloc: one static array
// in this module, so every GPU that loads the library holds it until exit. Host
// code must not pass the symbol itself to a kernel (on the host it names a
// host-side stand-in); its device address is looked up once per device below.
static __device__ __align__(256) unsigned char g_static_decode_scratch[KVP_STATIC_SCRATCH_BYTES];

namespace {

// The static scratch's device address, per device, with the context it was
// taken in: a device reset (cudaDeviceReset) or a thread bound to another
// context makes a cached address stale, so a call whose current context
// differs looks the address up again.
struct ScratchAddr {
  CUcontext ctx;
  void* ptr;
};
std::mutex g_static_scratch_mu;
ScratchAddr g_static_scratch[kMaxDevices] = {};

CUcontext current_context() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of the static scratch in the current context. The lookup
// (cudaGetSymbolAddress, with the device current) runs on the first call per
// device and context; it may load the module, which a stream capture does not
// allow, so a lookup while `stream` is capturing is refused.
int static_scratch_address(cudaStream_t stream, void** out) {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return fail(KVP_ERR_INVALID, "device index %d out of range", d);
  std::lock_guard<std::mutex> g(g_static_scratch_mu);
  ScratchAddr& slot = g_static_scratch[d];
  const CUcontext ctx = current_context();
  if (slot.ptr && ctx && slot.ctx == ctx) {
    *out = slot.ptr;
    return KVP_OK;
  }
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs != cudaStreamCaptureStatusNone)
    return fail(KVP_ERR_INVALID,
                "paged_attention_decode_noalloc: the first call on a device (and the first after "
                "a device reset) looks up the static scratch and must come before any stream "
                "capture");
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_static_decode_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "paged_attention_decode_noalloc: scratch address");
  slot.ptr = p;
  slot.ctx = current_context();
  *out = p;
  return KVP_OK;
}

}  // namespace

extern "C" int paged_attention_decode_noalloc(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t num_blocks, int32_t max_blocks_per_seq,
    int32_t max_context_len, float scale, int32_t partition_size, void* out, int32_t dtype,
    kvp_stream_t stream) {
  const size_t need = kvp_decode_workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len,
                                                 partition_size);
  if (need > size_t(KVP_STATIC_SCRATCH_BYTES))
    return fail(KVP_ERR_INVALID,
                "paged_attention_decode_noalloc: this batch needs %zu bytes of split-context "
                "scratch; the static area holds %zu (use paged_attention_decode with a workspace)",
                need, size_t(KVP_STATIC_SCRATCH_BYTES));
  void* ws = nullptr;
  if (need > 0) {
    const int rc = static_scratch_address(static_cast<cudaStream_t>(stream), &ws);
    if (rc) return rc;
  }
  return paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                                num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                max_blocks_per_seq, max_context_len, scale, partition_size, ws,
                                need > 0 ? size_t(KVP_STATIC_SCRATCH_BYTES) : 0, out, dtype, stream);
}
