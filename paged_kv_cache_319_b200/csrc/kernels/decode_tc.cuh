// Paged decode attention for grouped-query heads on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory).
//
// What it computes is the same as the CUDA-core kernel: for sequence s and
// query head h with KV head g = h / G, softmax(scale * q K^T) V over the keys
// and values found through the block table ["vLLM and PagedAttention",
// section "Architecture, step by step", step 3]. With G query heads sharing a
// KV head, QK^T and PV are small dense contractions, so they run as MMAs with
// the token axis as the 128-row M dimension (operands swapped):
//
//   S^T [128 tokens x N] = K_tile [128 x 128 dims] . Q_g^T [128 dims x N]
//   O^T [128 dims x N]  += V_tile^T [128 dims x 128 tokens] . P^T [128 x N]
//
// with N = 16 columns (the G real heads; the rest are ignored).
//
// Structure: a persistent CTA per SM walks its share of work units
// (sequence, KV head, partition); a unit is cut into chunks of up to 512
// tokens (4 M-tiles). Warp roles:
//   warp 0  producer: TMA loads (128-byte swizzle) of Q (per unit) and of
//           K then V tiles (per chunk) into a 5-stage ring of 32 KiB stages;
//           a stage is 128 tokens = 128 / block_size cache blocks: a K block
//           lands as two 2-D boxes at its rows of the stage's two 64-dim
//           regions (the QK MMA's 128 token rows need one 8-row stride), a V
//           block as one 3-D box [half][rows][64] that PV reads in place.
//   warp 1  MMA issuer (one thread) and tensor-memory owner: per chunk, QK^T
//           into a double-buffered S region, then PV into a double-buffered O
//           region; tcgen05.commit releases ring stages and signals softmax.
//   warps 2-5  softmax and epilogue (thread = TMEM lane = token row for S,
//           head-dim row for O): chunk max per head, p = 2^(s - m) rounded to
//           the input type into a shared-memory P^T buffer, then the chunk's
//           O is merged into fp32 registers by the log-sum-exp rule; the unit
//           ends by writing the normalised output or (m, l, acc) for the
//           split-context reduce.
// The exponent sum l is accumulated from the same rounded p that the MMA
// uses, so the weights stay a normalised average.
#pragma once

#include <type_traits>

#include "../pack_layout.h"
#include "common.cuh"
#include "decode_group.cuh"
#include "decode_simt.cuh"

namespace kvp {
namespace dev {

static_assert(grp::kHdrWords == kPlanSeqWord, "plan layout");

namespace tc {

// kPlainF8: kPlain over an E4M3 cache (codes widened to the query type in
// shared memory by four converter warps; scales per KV head).
enum Mode : int { kPlain = 0, kGrouped = 1, kMultiQuery = 2, kContig = 3, kPacked = 4, kPlainF8 = 5 };

constexpr int kD = 128;             // head_dim
constexpr int kN = 16;              // MMA N (query heads of a group, padded)
constexpr int kTileTok = 128;       // MMA M: tokens per tile
// Tiles per chunk (the unit of the softmax pipeline) and ring stages are
// compile-time tunables; defaults: 4 tiles (512 tokens), 5 stages.
#ifndef KVP_TC_CHUNK_TILES
#define KVP_TC_CHUNK_TILES 4
#endif
constexpr int kChunkTiles = KVP_TC_CHUNK_TILES;  // tiles per chunk
constexpr int kChunkTok = kTileTok * kChunkTiles;
constexpr int kStageBytes = kTileTok * kD * 2;       // 32 KiB
constexpr int kRegionBytes = kTileTok * 128;         // 16 KiB: 64 dims of 128 tokens
constexpr int kQBytes = kN * kD * 2;                 // 4 KiB
constexpr int kTmemCols = 256;
constexpr int kSCol = 0;                             // S buffers: [0, 128)
constexpr int kOCol = 128;                           // O buffers: [128, 128 + 2 * kNPV)
constexpr int kThreads = 192;
constexpr int kThreadsF8 = 320;          // + four converter warps (E4M3 cache)
constexpr int kCodeBytes = 128 * 128;    // 16 KiB: E4M3 codes of one 128-token tile
constexpr int kSoftmaxThreads = 128;
// Batches of up to Cfg<NG>::kCtxCap sequences (at most kCtxCacheMax) keep their
// context lengths in shared memory, so no warp role waits on a global load when
// it moves to a new unit.
constexpr int kCtxCacheMax = 4096;

// Layout for a group width NG (query heads per KV head, padded to 4, 8 or 16).
// P^T holds p split into a high part and a low part, both in the input type
// (columns [0, NG) and [NG, 2 NG)): the PV MMA multiplies V by hi + lo, which
// carries p to about 16 significant bits instead of the 8 of one bf16.
// P^T is the MMA's B operand in the MN-major layout without swizzle: the 8
// columns [8g, 8g + 8) of a token are 16 contiguous bytes, tokens follow each
// other every 16 bytes, and column groups are kPSbo bytes apart. A softmax
// thread owns one token, so it writes its columns with 16-byte stores, and a
// warp's 32 tokens fill 512 contiguous bytes.
template <int NG, bool F8 = false>
struct Cfg {
  static constexpr int kNPV = 2 * NG <= 16 ? 16 : 32;  // N of the PV MMA
#ifndef KVP_TC_STAGES
#define KVP_TC_STAGES 5
#endif
  // groups of 16 need a P^T twice as wide, which costs one stage. An E4M3
  // cache keeps its loads in flight as codes (4 stages of 16 KiB, 3 for groups
  // of 16) besides 3 widened stages (measured on the long-context GQA batch:
  // 3 + 4 and 4 + 3 626 us, 2 + 6 677 us, 4 + 2 725 us, 5 + 1 1261 us).
  static constexpr int kStages = F8 ? 3 : (NG <= 8 ? KVP_TC_STAGES : KVP_TC_STAGES - 1);
  static constexpr int kCodeStages = F8 ? (NG <= 8 ? 4 : 3) : 0;
  static constexpr int kPBytes = kChunkTok * kNPV * 2;
  static constexpr int kPSbo = kChunkTok * 16;          // bytes between 8-column groups of P^T
  static constexpr int kOffRing = 0;
  static constexpr int kOffCodes = kOffRing + kStages * kStageBytes;
  static constexpr int kOffQ = kOffCodes + kCodeStages * kCodeBytes;
  static constexpr int kOffP = kOffQ + 2 * kQBytes;
  static constexpr int kOffBar = kOffP + 2 * kPBytes;
  static constexpr int kNumBars = 2 * kStages + 2 * 10 + 2 * kCodeStages;
  static constexpr int kOffRed = kOffBar + kNumBars * 8;     // [2 halves][4 warps][kN] maxima
  static constexpr int kOffRedL = kOffRed + 2 * 4 * kN * 4;  // [2 halves][4 warps][kN] sums
  static constexpr int kOffTmemPtr = kOffRedL + 2 * 4 * kN * 4;
  static constexpr int kOffTags = kOffTmemPtr + 16;          // E4M3: K / V / end per code stage
  static constexpr int kOffCtx = kOffTags + 32;              // cached context lengths
  static constexpr int kSmemBytes = 1024 + kOffCtx;          // + 4 bytes per cached length
  static constexpr int kCtxCap =
      (226 * 1024 - kSmemBytes) / 4 < kCtxCacheMax ? (226 * 1024 - kSmemBytes) / 4 : kCtxCacheMax;
  // Grouped decode: batches of up to kPlanCap sequences keep their context
  // lengths and the grouping plan (per-sequence prefix blocks, subgroup table)
  // in shared memory: 48 bytes per sequence + 80.
  static constexpr int kPlanCap = (226 * 1024 - kSmemBytes - 80) / 48;
  static_assert(kStages >= 2, "ring stages");
  static_assert(kCodeStages <= 8, "a tag per code stage in 32 bytes");
  static_assert(kCtxCap >= 0, "shared memory budget");
  static_assert(kOCol + 2 * kNPV <= kTmemCols, "tensor memory budget");
};

// 2^x by the PTX instruction ex2.approx.ftz.f32. For p = 2^(s - m) with
// s <= m, flushing a subnormal result to zero drops only weights below 2^-126
// of the chunk's largest, far under the resolution of p in fp16 or bf16.
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// tcgen05 instruction descriptor, kind::f16, fp32 accumulate, M = 128.
__host__ __device__ constexpr uint32_t idesc_f16(uint32_t ab_fmt, uint32_t a_mn, uint32_t b_mn,
                                                 uint32_t n) {
  return (1u << 4) | (ab_fmt << 7) | (ab_fmt << 10) | (a_mn << 15) | (b_mn << 16) |
         ((n >> 3) << 17) | (uint32_t(kTileTok >> 4) << 24);
}

// Shared-memory matrix descriptor (sm_100 format, version 1).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (uint64_t(layout) << 61);
}
constexpr uint32_t kLayoutNone = 0;
constexpr uint32_t kLayoutSw128 = 2;

template <int NG>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[NG]) {
  uint32_t r[NG];
  if constexpr (NG == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr)
                 : "memory");
  } else if constexpr (NG == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
  } else if constexpr (NG == 32) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
  } else {
    static_assert(NG == 16, "4, 8, 16 or 32 columns");

    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
  }
#pragma unroll
  for (int j = 0; j < NG; ++j) v[j] = __uint_as_float(r[j]);
}

// Work unit u -> (s, p, g) over S x pmax x Hkv with the KV head fastest, so the
// CTAs running at the same time read different heads of each block (different
// offsets inside the blocks, spread over the HBM channels) rather than one head
// of many blocks.
struct Unit {
  int32_t s, g, p;
  int32_t tok_begin, tok_end;  // token range of the unit
  int32_t ctx;                 // tokens of the block-table row s that the unit may read
  int32_t nparts;
  int32_t sg;                  // grouped decode: subgroup of a shared-prefix unit, else -1
  int32_t slot;                // workspace slot of the unit's partial
  int32_t vbase;               // virtually contiguous cache: token coordinate of the slot
  int32_t e0;                  // packed decode: the chunk's first entry
};

// Context length of sequence s as the tensor-core kernel reads it (VC: over a
// virtually contiguous cache, clamped to the slot's capacity).
template <bool VC>
__device__ __forceinline__ int32_t ctx_of(const DecodeArgs& a, int32_t s, bool report) {
  if constexpr (VC) return seq_ctx(a, s, report);
  return load_ctx(a, s, report);
}

// ctx_sm: the batch's clamped context lengths in shared memory, or null.
template <bool VC = false>
__device__ __forceinline__ bool decode_unit(const DecodeArgs& a, int64_t u, Unit& w,
                                            const int32_t* ctx_sm) {
  const int64_t per_seq = int64_t(a.pmax) * a.num_kv_heads;
  w.s = int32_t(u / per_seq);
  const int32_t rem = int32_t(u - int64_t(w.s) * per_seq);
  w.p = rem / a.num_kv_heads;
  w.g = rem - w.p * a.num_kv_heads;
  w.ctx = ctx_sm ? ctx_sm[w.s] : ctx_of<VC>(a, w.s, w.g == 0 && w.p == 0);
  w.vbase = VC ? vc_base(a, w.s) : 0;
  w.nparts = (w.ctx + a.part_tokens - 1) / a.part_tokens;
  if (w.p > 0 && w.p >= w.nparts) return false;  // empty (p == 0 always runs)
  w.tok_begin = w.p * a.part_tokens;
  w.tok_end = min(w.ctx, w.tok_begin + a.part_tokens);
  if (a.q_len > 1) {  // multi-query: no query of the launch sees a token from vis_end on
    const int32_t vis_end = w.ctx - a.q_len + a.q_first + a.q_count;
    if (w.tok_end > vis_end) w.tok_end = vis_end;
    if (w.p > 0 && w.tok_end <= w.tok_begin) return false;
  }
  if (w.tok_end < w.tok_begin) w.tok_end = w.tok_begin;
  w.sg = -1;
  w.slot = w.p;
  return true;
}

// Grouped decode: units [0, shared_units) are (subgroup, partition of the
// shared prefix, KV head), the rest (sequence, partition of the sequence's
// own range from block c on, KV head); KV head fastest in both.
struct GroupHdr {
  int64_t shared_units;
  int32_t psh;          // most shared partitions of any subgroup
  const int32_t* cblk;  // per sequence: shared-prefix blocks
  const int32_t* subs;  // subgroup table (packed decode: the group table)
  bool in_smem;         // cblk and subs point at the CTA's shared-memory copy
  const int32_t* units; // packed decode: the unit table
  const int32_t* ents;  // packed decode: the entries
  bool ldg;             // global plan words read through the read-only path (packed decode:
                        // the plan was written before the launch)
};

__device__ __forceinline__ int32_t plan_at(const GroupHdr& gh, const int32_t* p) {
  return gh.in_smem ? *p : (gh.ldg ? __ldg(p) : ld_relaxed_gpu(p));
}
__device__ __forceinline__ const int32_t* sub_entry(const GroupHdr& gh, int32_t sg) {
  return gh.subs + int64_t(sg) * grp::kSubWords;
}

template <int BS>
__device__ __forceinline__ bool decode_unit_grp(const DecodeArgs& a, int64_t u, Unit& w,
                                                const int32_t* ctx_sm, const GroupHdr& gh) {
  if (u < gh.shared_units) {
    const int64_t per = int64_t(gh.psh) * a.num_kv_heads;
    w.sg = int32_t(u / per);
    const int32_t rem = int32_t(u - int64_t(w.sg) * per);
    w.p = rem / a.num_kv_heads;
    w.g = rem - w.p * a.num_kv_heads;
    const int32_t* e = sub_entry(gh, w.sg);
    const int32_t shared = plan_at(gh, e) * BS;
    w.tok_begin = w.p * a.part_tokens;
    if (w.tok_begin >= shared) return false;
    w.tok_end = min(shared, w.tok_begin + a.part_tokens);
    w.s = plan_at(gh, e + 4);  // every member holds the same blocks here
    w.ctx = shared;
    w.vbase = 0;
    w.nparts = 0;
    w.slot = w.p;
    return true;
  }
  u -= gh.shared_units;
  const int64_t per_seq = int64_t(a.pmax) * a.num_kv_heads;
  w.s = int32_t(u / per_seq);
  const int32_t rem = int32_t(u - int64_t(w.s) * per_seq);
  w.p = rem / a.num_kv_heads;
  w.g = rem - w.p * a.num_kv_heads;
  w.ctx = ctx_sm ? ctx_sm[w.s] : load_ctx(a, w.s, w.g == 0 && w.p == 0);
  w.vbase = 0;
  const int32_t shared = plan_at(gh, gh.cblk + w.s) * BS;
  w.tok_begin = shared + w.p * a.part_tokens;
  if (w.tok_begin >= w.ctx) return false;
  w.tok_end = min(w.ctx, w.tok_begin + a.part_tokens);
  w.nparts = 0;
  w.sg = -1;
  w.slot = (shared + a.part_tokens - 1) / a.part_tokens + w.p;
  return true;
}

// Packed decode: unit u is (unit record u / Hkv, KV head u % Hkv); its tokens
// are the blocks of one chunk of its group's stream (n * BS token rows, which
// the entries' column masks and valid counts qualify).
template <int BS>
__device__ __forceinline__ bool decode_unit_pack(const DecodeArgs& a, int64_t u, Unit& w,
                                                 const GroupHdr& gh) {
  const int64_t ui = u / a.num_kv_heads;
  w.g = int32_t(u - ui * a.num_kv_heads);
  const int32_t* ur = gh.units + ui * pack::kUnitWords;
  w.sg = __ldg(ur + 0);
  w.e0 = __ldg(ur + 1);
  const int32_t n = __ldg(ur + 2);
  w.slot = __ldg(ur + 3);
  w.p = w.slot;
  w.tok_begin = 0;
  w.tok_end = n * BS;
  w.ctx = n * BS;
  w.s = plan_at(gh, gh.subs + int64_t(w.sg) * pack::kGroupWords + 4);
  w.nparts = 0;
  w.vbase = 0;
  return n > 0;
}

__device__ __forceinline__ int32_t chunks_of(const Unit& w) {
  return (w.tok_end - w.tok_begin + kChunkTok - 1) / kChunkTok;
}
__device__ __forceinline__ int32_t tiles_of(const Unit& w, int32_t c) {
  const int32_t c0 = w.tok_begin + c * kChunkTok;
  const int32_t c1 = min(w.tok_end, c0 + kChunkTok);
  return (c1 - c0 + kTileTok - 1) / kTileTok;
}

// The chunks a persistent CTA processes, in order: its units blockIdx.x,
// blockIdx.x + gridDim.x, ... (empty partitions and units without tokens
// skipped), each cut into chunks of up to kChunkTok tokens. Every warp role
// walks the same stream.
template <int MODE, int BS>
struct ChunkStream {
  static constexpr bool GRP = MODE == kGrouped;
  static constexpr bool PK = MODE == kPacked;
  int64_t u, stride, num_units;
  const int32_t* ctx_sm;
  GroupHdr gh;
  Unit w;
  int32_t c, nch;
  bool valid;

  __device__ __forceinline__ void init(const DecodeArgs& a, int64_t first, int64_t step,
                                       int64_t n, const int32_t* ctx_cache, const GroupHdr& g) {
    ctx_sm = ctx_cache;
    gh = g;
    stride = step;
    num_units = n;
    u = first - step;
    c = 0;
    nch = 0;
    valid = true;
    next_unit(a);
  }
  __device__ __forceinline__ void next_unit(const DecodeArgs& a) {
    for (u += stride; u < num_units; u += stride) {
      const bool has = PK    ? decode_unit_pack<BS>(a, u, w, gh)
                       : GRP ? decode_unit_grp<BS>(a, u, w, ctx_sm, gh)
                             : decode_unit<BS == kTileTok>(a, u, w, ctx_sm);
      if (has && (nch = chunks_of(w)) > 0) {
        c = 0;
        return;
      }
    }
    valid = false;
  }
  __device__ __forceinline__ void advance(const DecodeArgs& a) {
    if (++c >= nch) next_unit(a);
  }
  __device__ __forceinline__ int32_t tiles() const { return tiles_of(w, c); }
  __device__ __forceinline__ bool first() const { return c == 0; }
  __device__ __forceinline__ bool last() const { return c == nch - 1; }
};

}  // namespace tc

// MODE tc::kContig: decode over a virtually contiguous cache (a.vc_* set,
// BS = 128): a tile is 128 consecutive tokens of the sequence's slot, loaded
// as one 4-D box per 64-dim half of K and one for V at the computed token
// coordinate, with no block table. MODE tc::kPlain: decode. MODE tc::kGrouped: grouped decode (a.plan set;
// launched after the plan kernel with programmatic serialisation); num_units
// then counts the per-sequence units (0 when the CUDA-core kernel takes them)
// and the shared-prefix units are read from the plan. MODE tc::kMultiQuery:
// a chunk of a.q_count query tokens per sequence (tokens a.q_first.. of an
// a.q_len-token chunk, rows s * q_len + i of q and out), causal within the
// chunk: column j is query a.q_first + j / G at head g * G + j % G and sees
// the tokens before ctx - q_len + q_first + j / G + 1.
template <typename T, int BS, int NG, int MODE>
__global__ void __launch_bounds__(MODE == tc::kPlainF8 ? tc::kThreadsF8 : tc::kThreads, 1) decode_tc_kernel(
    const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
    const __grid_constant__ CUtensorMap qmap, const DecodeArgs a, int64_t num_units) {
  using namespace tc;
  constexpr bool GRP = MODE == kGrouped;
  constexpr bool MQ = MODE == kMultiQuery;
  constexpr bool VC = MODE == kContig;
  constexpr bool PK = MODE == kPacked;
  constexpr bool F8 = MODE == kPlainF8;
  static_assert(VC ? BS == kTileTok : (BS == 16 || BS == 32), "block_size 16 or 32");
  using L = tc::Cfg<NG, F8>;
  constexpr int kStages = L::kStages;
  constexpr int kPBytes = L::kPBytes;
  constexpr int kNPV = L::kNPV;
  constexpr int kBlocksPerTile = kTileTok / BS;
  // the MMA operand type: T, except over an E4M3 cache, whose codes widen to
  // fp16 in one instruction per pair (a bf16 q is converted to fp16 in shared
  // memory, exactly for |q| in [2^-14, 65504]); outputs stay in T
  using TM = typename std::conditional<F8, __half, T>::type;
  constexpr bool kQToHalf = F8 && !std::is_same<T, __half>::value;
  constexpr uint32_t kFmt = std::is_same<TM, __half>::value ? 0u : 1u;
  // A = K (K-major), B = Q (K-major), N = 16
  constexpr uint32_t kIdescQK = idesc_f16(kFmt, 0, 0, kN);
  // A = V^T (MN-major), B = P^T (K-major, hi and lo rows), N = kNPV
  constexpr uint32_t kIdescPV = idesc_f16(kFmt, 1, 1, kNPV);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint8_t* ring = smem + L::kOffRing;
  uint8_t* qbuf = smem + L::kOffQ;
  uint8_t* pbuf = smem + L::kOffP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* full = bars;                   // [kStages]
  uint64_t* empty = bars + kStages;        // [kStages]
  uint64_t* q_full = empty + kStages;      // [2]
  uint64_t* q_empty = q_full + 2;          // [2]
  uint64_t* s_full = q_empty + 2;          // [2]
  uint64_t* s_free = s_full + 2;           // [2]
  uint64_t* p_full = s_free + 2;           // [2]
  uint64_t* p_free = p_full + 2;           // [2]
  uint64_t* o_full = p_free + 2;           // [2]
  uint64_t* o_free = o_full + 2;           // [2]
  uint64_t* red_bar = o_free + 2;          // [2] chunk maxima of the 4 softmax warps
  uint64_t* lred_bar = red_bar + 2;        // [2] unit sums of the 4 softmax warps
  // E4M3 cache: code stages filled by TMA (cfull) and handed back by the four
  // converter warps once read (cempty); a widened ring stage's full barrier
  // counts the converter warps' writes instead of TMA bytes
  uint64_t* cfull = lred_bar + 2;               // [kCodeStages]
  uint64_t* cempty = cfull + L::kCodeStages;    // [kCodeStages]
  uint8_t* codes = smem + L::kOffCodes;
  int32_t* ctags = reinterpret_cast<int32_t*>(smem + L::kOffTags);
  float* red = reinterpret_cast<float*>(smem + L::kOffRed);
  float* redl = reinterpret_cast<float*>(smem + L::kOffRedL);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + L::kOffTmemPtr);
  int32_t* ctx_cache = reinterpret_cast<int32_t*>(smem + L::kOffCtx);
  const int32_t* ctx_sm = a.num_seqs <= L::kCtxCap ? ctx_cache : nullptr;
  // grouped decode: plan copy after the context lengths (when it fits)
  const bool plan_sm = GRP && a.num_seqs <= L::kPlanCap;
  if (ctx_sm) {
    for (int i = threadIdx.x; i < a.num_seqs; i += blockDim.x)
      ctx_cache[i] = tc::ctx_of<VC>(a, i, blockIdx.x == 0);  // clamped; out-of-range reported once
  }
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // the split-context reduce waits for this grid to complete; in the grouped
  // decode the trigger comes after the wait for the plan (below)
  if constexpr (!GRP) pdl_trigger();

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], F8 ? 4 : 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < L::kCodeStages; ++i) {
      mbar_init(&cfull[i], 1);
      mbar_init(&cempty[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&p_free[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], 4);
      mbar_init(&red_bar[i], 4);
      mbar_init(&lred_bar[i], 4);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  // P^T buffers start as zeros (rows of padded heads are never written).
  for (int i = threadIdx.x; i < 2 * kPBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(pbuf)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(tmem_ptr, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_ptr;

  const int32_t G = a.num_q_heads / a.num_kv_heads;
  // the coordinate of a tile past the tensor (read as zeros): paged rows, or
  // the virtually contiguous cache's tokens
  const int32_t rows_total = VC ? a.vc_num_slots * a.vc_slot_tokens : a.num_blocks * a.num_kv_heads * BS;
  tc::GroupHdr gh{0, 0, nullptr, nullptr, false};
  if constexpr (GRP) {
    pdl_wait();  // the plan kernel has completed and its writes are visible
    // The kernel launched next (the CUDA-core kernel for the sequences' own
    // ranges, or the reduce) may start once every CTA is past this point, so
    // it may read the plan without a wait of its own.
    pdl_trigger();
    const int32_t n_sub = ld_relaxed_gpu(a.plan + grp::kNumSub);
    gh.psh = ld_relaxed_gpu(a.plan + grp::kSharedParts);
    gh.shared_units = int64_t(n_sub) * gh.psh * a.num_kv_heads;
    num_units += gh.shared_units;
    const int32_t* g_cblk = a.plan + kPlanSeqWord;
    const int32_t* g_subs = a.plan + grp::sub_offset(a.num_seqs);
    if (plan_sm) {
      int32_t* c_sm = ctx_cache + a.num_seqs;
      int32_t* s_sm = c_sm + a.num_seqs;
      for (int i = threadIdx.x; i < a.num_seqs; i += blockDim.x) c_sm[i] = ld_relaxed_gpu(g_cblk + i);
      for (int i = threadIdx.x; i < n_sub * grp::kSubWords; i += blockDim.x)
        s_sm[i] = ld_relaxed_gpu(g_subs + i);
      __syncthreads();
      gh.cblk = c_sm;
      gh.subs = s_sm;
      gh.in_smem = true;
    } else {
      gh.cblk = g_cblk;
      gh.subs = g_subs;
    }
  }

  if constexpr (PK) {  // the packed plan: uploaded before the launch, read-only here
    const int32_t* g_subs = a.plan + pack::group_offset(a.num_seqs);
    gh.units = a.plan + __ldg(a.plan + pack::kUnitOffset);
    gh.ents = a.plan + __ldg(a.plan + pack::kEntryOffset);
    gh.ldg = true;
    if (a.plan_packed == 2) {  // the launch made room for the group table after the lengths
      int32_t* s_sm = ctx_cache + (ctx_sm ? a.num_seqs : 0);
      const int32_t n = __ldg(a.plan + pack::kGroups) * pack::kGroupWords;
      for (int i = threadIdx.x; i < n; i += blockDim.x) s_sm[i] = __ldg(g_subs + i);
      __syncthreads();
      gh.subs = s_sm;
      gh.in_smem = true;
    } else {
      gh.subs = g_subs;
    }
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Ring order: K tiles of chunk 0, then for every chunk i: K tiles of chunk
    // i + 1, V tiles of chunk i (the keys run one chunk ahead of the values).
    if (lane == 0) {
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
      prefetch_tensormap(&qmap);
    }
    const uint64_t pol_kv = l2_policy_kv();
    const uint64_t pol_q = l2_policy_evict_last();
    uint32_t ctr = 0;   // ring tiles issued
    uint32_t ucnt = 0;  // units started
    bool ok = true;
    // Lane j's block of a chunk (one chunk = 512 / BS <= 32 blocks): its table
    // entry is loaded a chunk ahead (chunk_id, not waited on) and turned into a
    // TMA row, range-checked, when the chunk's tiles are issued (id_row).
    auto lane_has_block = [&](const tc::ChunkStream<MODE, BS>& cs, int32_t& bidx) {
      const tc::Unit& w = cs.w;
      bidx = (w.tok_begin + cs.c * kChunkTok) / BS + lane;
      return lane < cs.tiles() * kBlocksPerTile && bidx < (w.ctx + BS - 1) / BS;
    };
    auto chunk_id = [&](const tc::ChunkStream<MODE, BS>& cs) -> int32_t {
      int32_t bidx;
      if (!lane_has_block(cs, bidx)) return -1;
      if constexpr (VC) return 0;  // no table: the coordinate is computed
      if constexpr (PK) return __ldg(gh.ents + 2 * (int64_t(cs.w.e0) + bidx));
      return __ldg(a.block_tables + int64_t(cs.w.s) * a.max_blocks_per_seq + bidx);
    };
    auto id_row = [&](const tc::ChunkStream<MODE, BS>& cs, int32_t id) -> int32_t {
      int32_t bidx;
      if (!lane_has_block(cs, bidx)) return rows_total;  // past the sequence: zeros
      if constexpr (VC) return cs.w.vbase + bidx * kTileTok;  // inside the slot's capacity
      if (id < 0 || id >= a.num_blocks) {
        record_error(KVP_DEVERR_BLOCK_ID, (uint64_t(cs.w.s) << 32) | uint32_t(bidx));
        return rows_total;
      }
      return (id * a.num_kv_heads + cs.w.g) * BS;
    };
    // Key tiles: two 2-D boxes per block (its rows of each 64-dim region of the
    // stage). Value tiles: one 3-D box per block ([half][BS rows][64], 256 * BS
    // bytes at block j's offset), which the PV descriptors read in place.
    auto load_tiles = [&](const CUtensorMap* map, int32_t row, int32_t head, int32_t ntile,
                          bool values) {
      for (int32_t t = 0; t < ntile && ok; ++t, ++ctr) {
        if constexpr (F8) {
          // E4M3: one 2-D box {128 codes, BS rows} per block into a code stage,
          // tagged K or V for the converter warps
          const uint32_t cs = ctr % L::kCodeStages;
          if (lane == 0) {
            ok = mbar_wait(&cempty[cs], ((ctr / L::kCodeStages) & 1u) ^ 1u, 0x7f01u);
            if (ok) {
              ctags[cs] = values ? 1 : 0;
              mbar_arrive_expect_tx(&cfull[cs], kCodeBytes);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          const int j = lane - t * kBlocksPerTile;
          if (j >= 0 && j < kBlocksPerTile)
            tma_load_2d(codes + cs * kCodeBytes + j * BS * 128, map, &cfull[cs], 0, row, pol_kv);
          __syncwarp();
          continue;
        }
        const uint32_t st = ctr % kStages;
        if (lane == 0) {
          ok = mbar_wait(&empty[st], ((ctr / kStages) & 1u) ^ 1u, 0x7200u);
          if (ok) mbar_arrive_expect_tx(&full[st], kStageBytes);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        const int j = lane - t * kBlocksPerTile;  // block j of this tile
        if (VC && j == 0) {
          // one box {64, 128 tokens, halves, 1 head}: K one per 64-dim region, V both halves
          uint8_t* dst = ring + st * kStageBytes;
          if (values) {
            tma_load_4d(dst, map, &full[st], 0, row, 0, head, pol_kv);
          } else {
            tma_load_4d(dst, map, &full[st], 0, row, 0, head, pol_kv);
            tma_load_4d(dst + kRegionBytes, map, &full[st], 0, row, 1, head, pol_kv);
          }
        } else if (!VC && j >= 0 && j < kBlocksPerTile) {
          if (values) {
            tma_load_3d(ring + st * kStageBytes + j * BS * 256, map, &full[st], 0, row, 0, pol_kv);
          } else {
            uint8_t* dst = ring + st * kStageBytes + j * BS * 128;
            tma_load_2d(dst, map, &full[st], 0, row, pol_kv);
            tma_load_2d(dst + kRegionBytes, map, &full[st], 64, row, pol_kv);
          }
        }
        __syncwarp();
      }
    };
    // Shared-prefix units (grouped decode): column j of Q is query head
    // g * G + j % G of member j / G. The warp loads a unit's rows into
    // registers one iteration ahead and stores them in the 128-byte-swizzled
    // layout a TMA load would produce (16-byte chunk c of row j at
    // (c ^ (j & 7)) * 16) before the previous unit's value tiles, since the MMA
    // needs this Q before it frees the ring stages those wait for.
    constexpr int kQChunksPerLane = kN * 16 / 32;
    auto is_gather = [&](const tc::ChunkStream<MODE, BS>& cs) {
      return cs.valid && cs.first() && ((GRP && cs.w.sg >= 0) || MQ || PK);
    };
    auto gather_q = [&](const tc::ChunkStream<MODE, BS>& cs, uint4 (&v)[kQChunksPerLane]) {
      const int32_t* e = (GRP || PK) ? tc::sub_entry(gh, cs.w.sg) : nullptr;
      const int32_t ncol = (GRP || PK) ? tc::plan_at(gh, e + 1) * G : a.q_count * G;
#pragma unroll
      for (int i = 0; i < kQChunksPerLane; ++i) {
        const int idx = lane + 32 * i;
        const int j = idx >> 4, ch = idx & 15;
        v[i] = make_uint4(0, 0, 0, 0);
        if (j < ncol) {
          const int32_t m = j / G;  // member (grouped) or query token (multi-query)
          const int64_t seq_row = (GRP || PK) ? int64_t(tc::plan_at(gh, e + 4 + m))
                                      : int64_t(cs.w.s) * a.q_len + a.q_first + m;
          const int64_t qrow = seq_row * a.num_q_heads + cs.w.g * G + (j - m * G);
          v[i] = __ldg(reinterpret_cast<const uint4*>(static_cast<const T*>(a.q) + qrow * kD) + ch);
        }
      }
    };
    tc::ChunkStream<MODE, BS> cur;
    cur.init(a, blockIdx.x, gridDim.x, num_units, ctx_sm, gh);
    int32_t pend_row = rows_total, pend_tiles = 0, pend_head = 0;
    bool have_pend = false;
    int32_t id = cur.valid ? chunk_id(cur) : -1;
    uint4 qv[kQChunksPerLane];
    if (is_gather(cur)) gather_q(cur, qv);
    while (cur.valid && ok) {
      // the next chunk's block ids (and a grouped unit's Q rows) are loaded now
      // and used one iteration later
      tc::ChunkStream<MODE, BS> nxt = cur;
      nxt.advance(a);
      // (packed decode: the next unit's block ids and Q rows hang on its unit
      // record, a global load, so they are loaded after this chunk's tiles are
      // issued)
      int32_t id_next = -1;
      uint4 qn[kQChunksPerLane];
      const bool gather_next = is_gather(nxt);
      if constexpr (!PK) {
        id_next = nxt.valid ? chunk_id(nxt) : -1;
        if (gather_next) gather_q(nxt, qn);
      }
      const int32_t row = id_row(cur, id);
      const int32_t nt = cur.tiles();
      // A unit's Q goes in before its key tiles (gathered rows were loaded an
      // iteration ago), so the MMA can start on the first key tile that lands.
      const bool gather = is_gather(cur);
      if (cur.first() && ok) {
        const uint32_t qb = ucnt & 1u;
        if (lane == 0) ok = mbar_wait(&q_empty[qb], ((ucnt >> 1) & 1u) ^ 1u, 0x7100u);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (gather) {
          uint8_t* qdst = qbuf + qb * kQBytes;
#pragma unroll
          for (int i = 0; i < kQChunksPerLane; ++i) {
            const int idx = lane + 32 * i;
            const int j = idx >> 4, ch = idx & 15;
            *reinterpret_cast<uint4*>(qdst + (ch >> 3) * (kN * 128) + j * 128 +
                                      (((ch & 7) ^ (j & 7)) << 4)) = qv[i];
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&q_full[qb]);
        } else if (lane == 0) {
          mbar_arrive_expect_tx(&q_full[qb], kQBytes);
          const int32_t qrow = cur.w.s * a.num_q_heads + cur.w.g * G;
          tma_load_2d(qbuf + qb * kQBytes, &qmap, &q_full[qb], 0, qrow, pol_q);
          tma_load_2d(qbuf + qb * kQBytes + kN * 128, &qmap, &q_full[qb], 64, qrow, pol_q);
        }
        ++ucnt;
      }
      if (ok) load_tiles(&kmap, row, cur.w.g, nt, false);
      if (have_pend && ok) load_tiles(&vmap, pend_row, pend_head, pend_tiles, true);
      if constexpr (PK) {
        id_next = nxt.valid ? chunk_id(nxt) : -1;
        if (gather_next) gather_q(nxt, qn);
      }
      pend_row = row;
      pend_head = cur.w.g;
      pend_tiles = nt;
      have_pend = true;
      id = id_next;
      if (gather_next) {
#pragma unroll
        for (int i = 0; i < kQChunksPerLane; ++i) qv[i] = qn[i];
      }
      cur = nxt;
    }
    if (have_pend && ok) load_tiles(&vmap, pend_row, pend_head, pend_tiles, true);
    if constexpr (F8) {
      // the end of the stream for the converter warps: a code stage tagged 2
      if (ok && lane == 0) {
        const uint32_t cs = ctr % L::kCodeStages;
        ok = mbar_wait(&cempty[cs], ((ctr / L::kCodeStages) & 1u) ^ 1u, 0x7f02u);
        if (ok) {
          ctags[cs] = 2;
          mbar_arrive(&cfull[cs]);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (!ok) {
      atomicExch(&abort_flag, 1);
      if (lane == 0) {  // drain the loads that may still be in flight
        if constexpr (F8) {
          for (uint32_t i = ctr > L::kCodeStages ? ctr - L::kCodeStages : 0; i < ctr; ++i)
            mbar_wait(&cfull[i % L::kCodeStages], (i / L::kCodeStages) & 1u, 0x7f05u);
        } else {
          for (uint32_t i = ctr > kStages ? ctr - kStages : 0; i < ctr; ++i)
            mbar_wait(&full[i % kStages], (i / kStages) & 1u, 0x7300u);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Issue order: S^T of chunk i + 1 before O^T of chunk i, so the tensor
    // cores and the loads of the next keys run while chunk i's softmax runs.
    uint32_t ctr = 0, ucnt = 0, cc = 0;
    bool ok = true;
    uint32_t q_addr = 0, qb = 0;
    auto qk = [&](uint32_t b, uint32_t use, int32_t ntile) {  // lane 0
      ok = mbar_wait(&s_free[b], (use & 1u) ^ 1u, 0x7500u);
      tc_fence_after();
      for (int32_t t = 0; t < ntile && ok; ++t, ++ctr) {
        const uint32_t st = ctr % kStages;
        ok = mbar_wait(&full[st], (ctr / kStages) & 1u, 0x7600u);
        if (!ok) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(ring + st * kStageBytes);
        const uint32_t d_tmem = tmem_base + kSCol + b * (kChunkTiles * kN) + t * kN;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kRegionBytes + (kk & 3) * 32;
          const uint32_t qoff = (kk >> 2) * (kN * 128) + (kk & 3) * 32;
          umma_f16_ss(d_tmem, smem_desc(k_addr + off, 16, 1024, kLayoutSw128),
                      smem_desc(q_addr + qoff, 16, 1024, kLayoutSw128), kIdescQK, kk > 0);
        }
        umma_commit(&empty[st]);
      }
      if (ok) umma_commit(&s_full[b]);
    };
    // O^T += V^T P^T for a chunk, run by the whole warp: lane 0 waits and
    // issues; in the chunk's last tile the lanes first zero the V rows of
    // tokens past the end of the sequence (rows >= zero_from), which hold
    // whatever the pool had there: p is 0 for them, but 0 * inf is NaN.
    // Packed decode: nv is the valid tokens of this lane's block of the chunk
    // (lane j holds block j); rows past them (a member's last block) are zeroed
    // the same way.
    auto pv = [&](uint32_t b, uint32_t use, int32_t ntile, int32_t zero_from, int32_t nv) {
      if (lane == 0) {
        ok = mbar_wait(&p_full[b], use & 1u, 0x7700u);
        if (ok) ok = mbar_wait(&o_free[b], (use & 1u) ^ 1u, 0x7800u);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      tc_fence_after();
      const uint32_t p_addr = smem_u32(pbuf + b * kPBytes);
      const uint32_t o_tmem = tmem_base + kOCol + b * kNPV;
      for (int32_t t = 0; t < ntile && ok; ++t, ++ctr) {
        const uint32_t st = ctr % kStages;
        if (lane == 0) ok = mbar_wait(&full[st], (ctr / kStages) & 1u, 0x7900u);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        if (t == ntile - 1 && zero_from < kTileTok) {
          uint8_t* tile = ring + st * kStageBytes;
          for (int row = zero_from + lane; row < kTileTok; row += 32) {
            // token row of block row / BS: [half][BS rows][128 bytes]
            uint8_t* r0 = tile + (row / BS) * (BS * 256) + (row % BS) * 128;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              reinterpret_cast<uint4*>(r0)[q] = make_uint4(0, 0, 0, 0);
              reinterpret_cast<uint4*>(r0 + BS * 128)[q] = make_uint4(0, 0, 0, 0);
            }
          }
          fence_proxy_async_smem();
        }
        if constexpr (PK) {
          const int jb = lane - t * kBlocksPerTile;  // this lane's block within the tile
          if (jb >= 0 && jb < kBlocksPerTile && nv < BS) {
            uint8_t* tile = ring + st * kStageBytes;
            for (int rr = nv; rr < BS; ++rr) {
              uint8_t* r0 = tile + jb * (BS * 256) + rr * 128;
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                reinterpret_cast<uint4*>(r0)[q] = make_uint4(0, 0, 0, 0);
                reinterpret_cast<uint4*>(r0 + BS * 128)[q] = make_uint4(0, 0, 0, 0);
              }
            }
            fence_proxy_async_smem();
          }
        }
        __syncwarp();
        if (lane == 0) {
          tc_fence_after();
          const uint32_t v_addr = smem_u32(ring + st * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < kTileTok / 16; ++kk) {
            const uint32_t pk = (t * kTileTok + kk * 16) * 16;
            // V^T, MN-major: tokens kk*16.. of block (kk*16)/BS; the two 64-dim
            // halves BS*128 bytes apart (LBO), 8-token groups 1024 apart (SBO)
            const uint32_t va = v_addr + ((kk * 16) / BS) * (BS * 256) + ((kk * 16) % BS) * 128;
            umma_f16_ss(o_tmem, smem_desc(va, BS * 128, 1024, kLayoutSw128),
                        smem_desc(p_addr + pk, 128, L::kPSbo, kLayoutNone), kIdescPV,
                        (t > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[st]);
        }
        __syncwarp();
      }
      if (ok && lane == 0) {
        umma_commit(&o_full[b]);
        umma_commit(&p_free[b]);
      }
    };
    tc::ChunkStream<MODE, BS> cur;
    cur.init(a, blockIdx.x, gridDim.x, num_units, ctx_sm, gh);
    uint32_t pend_b = 0, pend_use = 0;
    int32_t pend_tiles = 0, pend_zero = kTileTok, pend_nv = BS;
    bool have_pend = false;
    int32_t nv_cur = BS;  // packed decode: valid tokens of this lane's block of the chunk
    if constexpr (PK) {
      if (cur.valid && lane < (cur.w.ctx + BS - 1) / BS)
        nv_cur = __ldg(gh.ents + 2 * (int64_t(cur.w.e0) + lane) + 1) & 0xFF;
    }
    while (cur.valid && ok) {
      const uint32_t b = cc & 1u, use = cc >> 1;
      const int32_t nt = cur.tiles();
      // packed decode: the next unit is decoded now (its plan loads overlap this
      // chunk), and nv_cur, this lane's block's valid tokens, was loaded a unit ago
      tc::ChunkStream<MODE, BS> nxt;
      int32_t nv_next = BS;
      if constexpr (PK) {
        nxt = cur;
        nxt.advance(a);
        if (nxt.valid && lane < (nxt.w.ctx + BS - 1) / BS)
          nv_next = __ldg(gh.ents + 2 * (int64_t(nxt.w.e0) + lane) + 1) & 0xFF;
      }
      if constexpr (kQToHalf) {
        // a unit's bf16 Q tile, once landed, becomes fp16 in place (the whole warp)
        if (cur.first()) {
          const uint32_t qbc = ucnt & 1u;
          if (lane == 0) ok = mbar_wait(&q_full[qbc], (ucnt >> 1) & 1u, 0x7f06u);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          uint4* qv = reinterpret_cast<uint4*>(qbuf + qbc * kQBytes);
#pragma unroll
          for (int i = 0; i < kQBytes / 16 / 32; ++i) {
            uint4 v = qv[lane + 32 * i];
            uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = Elem<T>::to_float2(w[e]);
              w[e] = Elem<__half>::pack2(f.x, f.y);
            }
            qv[lane + 32 * i] = make_uint4(w[0], w[1], w[2], w[3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
      }
      if (lane == 0) {
        if (cur.first()) {
          qb = ucnt & 1u;
          ok = mbar_wait(&q_full[qb], (ucnt >> 1) & 1u, 0x7400u);
          q_addr = smem_u32(qbuf + qb * kQBytes);
        }
        if (ok) qk(b, use, nt);
        if (ok && cur.last()) umma_commit(&q_empty[qb]);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ctr = __shfl_sync(0xffffffffu, ctr, 0);  // qk advanced the ring on lane 0 only
      if (ok && have_pend) pv(pend_b, pend_use, pend_tiles, pend_zero, pend_nv);
      pend_nv = nv_cur;
      if (cur.first()) ++ucnt;
      // valid tokens in this chunk's last tile; rows from there on are zeroed
      const int32_t ctok0 = cur.w.tok_begin + cur.c * kChunkTok;
      const int32_t nvalid = min(cur.w.tok_end, ctok0 + kChunkTok) - ctok0;
      pend_zero = nvalid - (nt - 1) * kTileTok;
      pend_b = b;
      pend_use = use;
      pend_tiles = nt;
      have_pend = true;
      ++cc;
      if constexpr (PK) {
        cur = nxt;
        nv_cur = nv_next;
      } else {
        cur.advance(a);
      }
    }
    if (ok && have_pend) pv(pend_b, pend_use, pend_tiles, pend_zero, pend_nv);
    if (!ok) atomicExch(&abort_flag, 1);
  } else if (F8 && warp >= 6) {
    // ------------------------------------------------------------ E4M3 converters
    // Item k of the stream (the producer's order): code stage k % kCodeStages
    // into ring stage k % kStages, widened exactly to fp16 (cvt.rn.f16x2.e4m3x2,
    // two codes per instruction; NaN codes stay NaN) in the layout the TMA would
    // have produced for a 16-bit cache:
    // keys as two 64-dim regions of 128 rows, values per block as [half][BS
    // rows][64] (128-byte swizzle on both). The four warps share each item:
    // thread ct takes 16 codes (dims 16c .. 16c + 15, c = ct % 8) of token rows
    // ct / 8 + 16u, reads them all, hands the code stage back, then writes.
    const int ct = threadIdx.x - 6 * 32;  // 0 .. 127
    const int c = ct & 7;
    bool ok = true;
    for (uint32_t k = 0;; ++k) {
      const uint32_t cs = k % L::kCodeStages;
      const uint32_t st = k % kStages;
      if (lane == 0) ok = mbar_wait(&cfull[cs], (k / L::kCodeStages) & 1u, 0x7f03u);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const int32_t tag = ctags[cs];
      if (tag == 2) break;  // end of the stream
      const uint8_t* src = codes + cs * kCodeBytes;
      uint4 wv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int row = (ct >> 3) + 16 * u;
        wv[u] = *reinterpret_cast<const uint4*>(src + row * 128 + ((c ^ (row & 7)) << 4));
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&cempty[cs]);  // releases this warp's reads
        ok = mbar_wait(&empty[st], ((k / kStages) & 1u) ^ 1u, 0x7f04u);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      uint8_t* dst = ring + st * kStageBytes;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int row = (ct >> 3) + 16 * u;
        const uint32_t cw[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
        uint32_t h[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          h[2 * e] = e4m3x2_to_x2<TM>(cw[e] & 0xFFFFu);
          h[2 * e + 1] = e4m3x2_to_x2<TM>(cw[e] >> 16);
        }
        uint8_t* base;
        int sw;
        if (tag == 0) {  // key row: region c / 4, row `row`
          base = dst + (c >> 2) * kRegionBytes + row * 128;
          sw = row & 7;
        } else {  // value row: block row / BS, half c / 4, row row % BS
          const int jb = row / BS, ib = row % BS;
          base = dst + jb * BS * 256 + (c >> 2) * BS * 128 + ib * 128;
          sw = ib & 7;
        }
        // 16-byte chunks ch, ch + 1 of the 128-byte row. A 16-byte store is served
        // eight lanes at a time, and lanes c and c + 4 (same row, other region)
        // would meet at the same bank positions: lanes of the second region store
        // chunk ch + 1 first, so each group of eight covers all 32 banks once.
        const int ch = 2 * (c & 3);
        const bool sec = c >= 4;
        const uint4 d0 = make_uint4(h[0], h[1], h[2], h[3]);
        const uint4 d1 = make_uint4(h[4], h[5], h[6], h[7]);
        *reinterpret_cast<uint4*>(base + (((ch + (sec ? 1 : 0)) ^ sw) << 4)) = sec ? d1 : d0;
        *reinterpret_cast<uint4*>(base + (((ch + (sec ? 0 : 1)) ^ sw) << 4)) = sec ? d0 : d1;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[st]);
    }
    if (!ok) atomicExch(&abort_flag, 1);
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // All waits here are bounded mbarrier waits made warp-uniform; the four
    // warps exchange maxima and sums through shared memory guarded by count-4
    // mbarriers on alternating halves (no unbounded named barriers). Order per
    // chunk i: p of chunk i, then the merge of chunk i - 1's O (and the
    // epilogue of its unit when it was the unit's last chunk).
    const int quarter = warp & 3;          // TMEM lanes 32*quarter .. +31
    const int r = quarter * 32 + lane;     // token row (S) / head-dim row (O)
    const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
    const int wi = warp - 2;               // softmax warp index 0..3
    auto wait_all = [&](uint64_t* bar, uint32_t parity, uint32_t where) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, where)) != 0;
    };
    int32_t col_q[NG];  // multi-query: the query token of column j within the launch
#pragma unroll
    for (int j = 0; j < NG; ++j) col_q[j] = j / G;
    // Units without tokens (context length 0) attend to nothing: zero rows
    // (written by the reduce in the grouped decode).
    for (int64_t u = blockIdx.x; !GRP && !PK && u < num_units; u += gridDim.x) {
      tc::Unit w;
      if (!tc::decode_unit<VC>(a, u, w, ctx_sm) || tc::chunks_of(w) > 0) continue;
      const int32_t nq = MQ ? a.q_count : 1;
      for (int i = 0; i < nq; ++i) {
        const int64_t row = MQ ? int64_t(w.s) * a.q_len + a.q_first + i : int64_t(w.s);
        for (int j = 0; j < G; ++j)
          static_cast<uint16_t*>(a.out)[(row * a.num_q_heads + w.g * G + j) * kD + r] = 0;
      }
    }
    float acc[NG], m_run[NG], l_thr[NG];
#pragma unroll
    for (int j = 0; j < NG; ++j) {
      acc[j] = 0.f;
      m_run[j] = -INFINITY;
      l_thr[j] = 0.f;
    }
    // The chunk whose O is merged one step later.
    tc::Unit pw{};
    uint32_t pb_ = 0, puse = 0;
    bool plast = false, have_pend = false;
    float pmax_[NG], psum_[NG];
    uint32_t cc = 0, ucnt = 0;
    bool ok = true;

    auto merge = [&]() {  // merge the pending chunk; epilogue when it ends its unit
      ok = wait_all(&o_full[pb_], puse & 1u, 0x7d00u);
      if (!ok) return;
      tc_fence_after();
      float ov2[2 * NG];  // [hi columns | lo columns]
      tmem_ld_cols<2 * NG>(tmem_base + lane_addr + kOCol + pb_ * kNPV, ov2);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[pb_]);
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        const float ov = ov2[j] + ov2[NG + j];
        const float mn = fmaxf(m_run[j], pmax_[j]);
        const float fo = m_run[j] == -INFINITY ? 0.f : exp2f(m_run[j] - mn);
        const float fc = pmax_[j] == -INFINITY ? 0.f : exp2f(pmax_[j] - mn);
        acc[j] = acc[j] * fo + ov * fc;
        l_thr[j] = l_thr[j] * fo + psum_[j] * fc;
        m_run[j] = mn;
      }
      if (!plast) return;
      // ---- unit epilogue: l over all 128 rows, then write
      const uint32_t ub = ucnt & 1u;
      float* rl = redl + ub * 4 * kN;
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        float v = l_thr[j];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) rl[wi * kN + j] = v;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&lred_bar[ub]);
      ok = wait_all(&lred_bar[ub], (ucnt >> 1) & 1u, 0x7e00u);
      ++ucnt;
      if (!ok) return;
      const int32_t h0 = pw.g * G;
      // E4M3: O was accumulated on codes; the value scale of the KV head applies
      const float vsc = F8 ? __ldg(a.v_scale + pw.g) : 1.f;
      // grouped decode: a shared-prefix unit's columns are its members' heads
      const int32_t* ge = ((GRP && pw.sg >= 0) || PK) ? tc::sub_entry(gh, pw.sg) : nullptr;
      const int32_t ncol = ge ? tc::plan_at(gh, ge + 1) * G : (MQ ? a.q_count * G : G);
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        const float Lj = (rl[j] + rl[kN + j]) + (rl[2 * kN + j] + rl[3 * kN + j]);
        if (j < ncol) {
          int64_t row_sh = int64_t(pw.s) * a.num_q_heads + h0 + j;
          if (ge) {
            const int32_t m = j / G;
            row_sh = int64_t(tc::plan_at(gh, ge + 4 + m)) * a.num_q_heads + h0 + (j - m * G);
          } else if (MQ) {
            const int32_t i = col_q[j];
            row_sh = (int64_t(pw.s) * a.q_len + a.q_first + i) * a.num_q_heads + h0 + (j - i * G);
          }
          if (!GRP && !PK && pw.nparts <= 1) {
            const float y = Lj > 0.f ? acc[j] * vsc / Lj : 0.f;
            static_cast<uint16_t*>(a.out)[row_sh * kD + r] = Elem<T>::from_float(y);
          } else {
            a.ws_acc[(row_sh * a.ws_slots + pw.slot) * kD + r] = acc[j] * vsc;
            if (r == 0) {
              a.ws_ml[(row_sh * a.ws_slots + pw.slot) * 2 + 0] = m_run[j];
              a.ws_ml[(row_sh * a.ws_slots + pw.slot) * 2 + 1] = Lj;
            }
          }
        }
        acc[j] = 0.f;
        m_run[j] = -INFINITY;
        l_thr[j] = 0.f;
      }
    };

    // packed decode: per tile of a unit, the columns that take this thread's
    // token row (its block's column mask, none past the block's valid tokens)
    auto row_masks = [&](const tc::ChunkStream<MODE, BS>& cs, uint32_t (&m)[kChunkTiles]) {
      const int32_t nblk = cs.valid ? (cs.w.ctx + BS - 1) / BS : 0;
#pragma unroll
      for (int t = 0; t < kChunkTiles; ++t) {
        const int32_t blk = t * kBlocksPerTile + r / BS;
        m[t] = 0;
        if (blk < nblk) {
          const uint32_t wd = uint32_t(__ldg(gh.ents + 2 * (int64_t(cs.w.e0) + blk) + 1));
          m[t] = (r % BS) < int32_t(wd & 0xFFu) ? (wd >> 8) : 0u;
        }
      }
    };
    tc::ChunkStream<MODE, BS> cur;
    cur.init(a, blockIdx.x, gridDim.x, num_units, ctx_sm, gh);
    uint32_t pm[kChunkTiles];
#pragma unroll
    for (int t = 0; t < kChunkTiles; ++t) pm[t] = 0xFFFFFFFFu;
    if constexpr (PK) row_masks(cur, pm);
    while (cur.valid && ok) {
      const uint32_t b = cc & 1u;
      const uint32_t use = cc >> 1;
      const int32_t ntile = cur.tiles();
      // packed decode: the next unit is decoded now and its row masks loaded (the
      // loads overlap this chunk); pm holds this unit's, loaded a unit ago
      tc::ChunkStream<MODE, BS> nxt;
      uint32_t pm_next[kChunkTiles];
      if constexpr (PK) {
        nxt = cur;
        nxt.advance(a);
        row_masks(nxt, pm_next);
      }
      const int32_t ctok0 = cur.w.tok_begin + cur.c * kChunkTok;
      const int32_t ctok1 = min(cur.w.tok_end, ctok0 + kChunkTok);
      // ---- scores of this thread's tokens (row r of each tile)
      ok = wait_all(&s_full[b], use & 1u, 0x7a00u);
      if (!ok) break;
      tc_fence_after();
      float sv[kChunkTiles][NG];
#pragma unroll
      for (int t = 0; t < kChunkTiles; ++t) {
        if (t < ntile) {
          tmem_ld_cols<NG>(tmem_base + lane_addr + kSCol + b * (kChunkTiles * kN) + t * kN, sv[t]);
        } else {
#pragma unroll
          for (int j = 0; j < NG; ++j) sv[t][j] = -INFINITY;
        }
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[b]);
      float cmax[NG];
#pragma unroll
      for (int j = 0; j < NG; ++j) cmax[j] = -INFINITY;
      // multi-query: column j sees the tokens before lim0 + j / G
      const int32_t lim0 = MQ ? cur.w.ctx - a.q_len + a.q_first + 1 : 0;
      // E4M3: the scores were taken on codes; the key scale of the KV head joins
      // the softmax scale
      const float sc_log2 = F8 ? a.scale_log2 * __ldg(a.k_scale + cur.w.g) : a.scale_log2;
#pragma unroll
      for (int t = 0; t < kChunkTiles; ++t) {
        const int32_t tok = ctok0 + t * kTileTok + r;
        const bool valid = t < ntile && tok < ctok1;
#pragma unroll
        for (int j = 0; j < NG; ++j) {
          const bool vis = valid && (!MQ || tok < lim0 + col_q[j]) && (!PK || ((pm[t] >> j) & 1u));
          sv[t][j] = vis ? sv[t][j] * sc_log2 : -INFINITY;
          cmax[j] = fmaxf(cmax[j], sv[t][j]);
        }
      }
      float* redm = red + b * 4 * kN;
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        cmax[j] = warp_max(cmax[j]);
        if (lane == 0) redm[wi * kN + j] = cmax[j];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_bar[b]);
      ok = wait_all(&red_bar[b], use & 1u, 0x7a80u);
      if (!ok) break;
#pragma unroll
      for (int j = 0; j < NG; ++j)
        cmax[j] = fmaxf(fmaxf(redm[j], redm[kN + j]), fmaxf(redm[2 * kN + j], redm[3 * kN + j]));
      // ---- p = 2^(s - m) as hi + lo parts in the input type, into P^T
      ok = wait_all(&p_free[b], (use & 1u) ^ 1u, 0x7b00u);
      if (!ok) break;
      uint8_t* pbuf_b = pbuf + b * kPBytes;
      float psum[NG];
#pragma unroll
      for (int j = 0; j < NG; ++j) psum[j] = 0.f;
#pragma unroll
      for (int t = 0; t < kChunkTiles; ++t) {
        if (t < ntile) {
          const int tok = t * kTileTok + r;  // token within the chunk
          uint8_t* prow = pbuf_b + tok * 16;
          // p of columns [j0, j0 + 2n) as packed hi and lo pairs
          auto p_pairs = [&](int j0, uint32_t* hw, uint32_t* lw, int n) {
#pragma unroll
            for (int i = 0; i < n; ++i) {
              const int j = j0 + 2 * i;
              const float p0 = sv[t][j] == -INFINITY ? 0.f : ex2_ftz(sv[t][j] - cmax[j]);
              const float p1 = sv[t][j + 1] == -INFINITY ? 0.f : ex2_ftz(sv[t][j + 1] - cmax[j + 1]);
              hw[i] = Elem<TM>::pack2(p0, p1);
              const float2 hf = Elem<TM>::to_float2(hw[i]);
              lw[i] = Elem<TM>::pack2(p0 - hf.x, p1 - hf.y);
              const float2 lf = Elem<TM>::to_float2(lw[i]);
              psum[j] += hf.x + lf.x;
              psum[j + 1] += hf.y + lf.y;
            }
          };
          if constexpr (NG == 4) {  // hi and lo share one 8-column group
            uint32_t hw[2], lw[2];
            p_pairs(0, hw, lw, 2);
            *reinterpret_cast<uint4*>(prow) = make_uint4(hw[0], hw[1], lw[0], lw[1]);
          } else {
#pragma unroll
            for (int g = 0; g < NG / 8; ++g) {
              uint32_t hw[4], lw[4];
              p_pairs(8 * g, hw, lw, 4);
              *reinterpret_cast<uint4*>(prow + g * L::kPSbo) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
              *reinterpret_cast<uint4*>(prow + (NG / 8 + g) * L::kPSbo) =
                  make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
      if (!ok) break;
      // ---- merge the previous chunk's O, now that this chunk's P is out
      if (have_pend) {
        merge();
        if (!ok) break;
      }
      pw = cur.w;
      pb_ = b;
      puse = use;
      plast = cur.last();
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        pmax_[j] = cmax[j];
        psum_[j] = psum[j];
      }
      have_pend = true;
      ++cc;
      if constexpr (PK) {
        cur = nxt;
#pragma unroll
        for (int t = 0; t < kChunkTiles; ++t) pm[t] = pm_next[t];
      } else {
        cur.advance(a);
      }
    }
    if (ok && have_pend) merge();
    if (!ok) atomicExch(&abort_flag, 1);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace dev
}  // namespace kvp
