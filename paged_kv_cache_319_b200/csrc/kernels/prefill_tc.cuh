// Paged prefill attention for prompts: 128 query rows per tensor-core tile.
//
// What it computes is paged_attention_prefill's definition: query i of the
// T-token chunk of sequence s sits at position ctx - T + i and attends to the
// keys and values of tokens j <= ctx - T + i, found through the block table
// ["PagedAttention: KV cache memory management", section "A request
// lifecycle": prefill creates the cache state the decode steps extend; "vLLM
// and PagedAttention", section "Architecture, step by step", step 3].
//
// Shape: a work unit is (sequence, KV head, query tile, partition). Its 128
// MMA rows are 128 / G query tokens x the G query heads of the KV head (row r
// = token r / G, head r % G), so one load of a key tile serves every head of
// the group. Per tile of 128 keys:
//
//   S [128 rows x 128 keys]  = Q [128 x 128 dims] . K^T            (TMEM)
//   O [128 rows x 128 dims] += P [128 x 128 keys] . V [128 x 128]  (TMEM)
//
// with P held, for bf16 inputs, as a high and a low part (the product V.(hi +
// lo) carries p to about 16 significant bits, as the decode kernel does); for
// fp16 inputs one part of 11 significant bits suffices (on causal 512-token
// prompts of N(0, 1) data the output moves by at most 3.8e-4 against exact p).
//
// Warp roles (192 threads, one CTA per SM, persistent over units):
//   warp 0     producer: TMA loads of Q (a 3-D box {64 dims, G heads, 128 / G
//              tokens} per 64-dim half) and of K then V tiles (the decode
//              kernel's per-block boxes) into a 3-stage ring, in the order
//              the MMAs take them (K of tile t, then V of tile t - 2).
//   warp 1     MMA issuer and TMEM owner: QK of tile t, then PV of tile t - 2,
//              and a unit's last two PVs at its end; S is double-buffered, O
//              double-buffered by unit.
//   warps 2-5  softmax and epilogue, thread = TMEM lane = row: per tile a
//              masked row max (causal: key j visible to the row's position),
//              p = 2^(s - m) into shared memory, and at a unit's end the
//              normalised row (or its partial for the split-context reduce).
//              fp16 inputs: P is double-buffered (the softmax of tile n + 1
//              runs while PV of tile n does) and a unit's epilogue waits
//              until after the next tile's softmax; bf16: one buffer of hi +
//              lo, epilogue at once.
// The running maximum m of a row moves only when a tile's maximum exceeds it
// by more than 8 (log2 units); O and l are then rescaled in TMEM, once the
// previous PV has completed, so p <= 2^8 and (m, l, O) stay a consistent
// partial.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "decode_simt.cuh"
#include "decode_tc.cuh"

namespace kvp {
namespace dev {
namespace pf {

constexpr int kD = 128;
constexpr int kRows = 128;            // MMA M: query rows per tile
constexpr int kKeys = 128;            // MMA N of QK: keys per tile
constexpr int kTileBytes = 128 * 128 * 2;  // 32 KiB: a Q, K, V or P tile
constexpr int kRegion = 16 * 1024;         // one 64-dim (or 64-key) half of a tile
constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kSCol = 0;               // S buffers: columns [0, 256)
constexpr int kOCol = 256;             // O buffers: columns [256, 512)
// The running maximum moves when a tile's maximum exceeds it by more than this
// (log2 units), so every p is at most 2^kLazy.
constexpr float kLazy = 8.f;

// shared memory (offsets from a 1024-byte aligned base)
constexpr int kOffQ = 0;                                // 2 Q buffers
constexpr int kOffRing = kOffQ + 2 * kTileBytes;        // kStages K/V stages
constexpr int kOffPHi = kOffRing + kStages * kTileBytes;
constexpr int kOffPLo = kOffPHi + kTileBytes;
constexpr int kOffBar = kOffPLo + kTileBytes;
constexpr int kNumBars = 2 * kStages + 2 * 7;
constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = 1024 + kOffTmemPtr + 16;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

struct Unit {
  int32_t s, g, p;
  int32_t q0, nq;            // first query token of the tile, tokens in it
  int32_t ctx;
  int32_t k_begin, k_end;    // keys of the unit
  int32_t ntiles;
  bool to_ws;                // partial to the workspace (the sequence is split)
};

// Units are ordered (sequence, KV head, query tile, partition), so the tiles
// of one (sequence, head) run at about the same time and share their key and
// value tiles through L2. CTAs take units round-robin; the query tiles of a
// (sequence, head) are rotated by the round in which its first unit is dealt,
// so a CTA meets every query tile in turn (a causal prompt's tile qt has qt + 1
// key tiles; without the rotation a grid that is a multiple of the tile count
// would hand each CTA one tile index throughout). Unit indices are below
// kMaxUnits (the host's bound), so the arithmetic is 32-bit.
constexpr uint32_t kMaxUnits = 0x7FF00000u;
__device__ __forceinline__ void unit_at(const DecodeArgs& a, uint32_t u, uint32_t G, uint32_t qtiles,
                                        const int32_t* ctx_sm, Unit& w) {
  const int32_t tq = kRows / int32_t(G);
  const uint32_t pmax = uint32_t(a.pmax);
  const uint32_t per_head = qtiles * pmax;
  const uint32_t head_unit = u / per_head;  // (sequence, KV head)
  const uint32_t within = u - head_unit * per_head;
  const uint32_t rot = ((head_unit * per_head) / gridDim.x) % qtiles;
  w.p = int32_t(within % pmax);
  const int32_t qt = int32_t(qtiles - 1 - (within / pmax + rot) % qtiles);
  w.g = int32_t(head_unit % uint32_t(a.num_kv_heads));
  w.s = int32_t(head_unit / uint32_t(a.num_kv_heads));
  w.ctx = ctx_sm ? ctx_sm[w.s] : load_ctx(a, w.s, w.g == 0 && qt == 0 && w.p == 0);
  w.q0 = qt * tq;
  w.nq = min(tq, a.q_len - w.q0);
  const int32_t vis_end = w.ctx - a.q_len + w.q0 + w.nq;  // keys any row of the tile sees
  w.k_begin = w.p * a.part_tokens;
  w.k_end = min(w.k_begin + a.part_tokens, vis_end);
  w.ntiles = w.k_end > w.k_begin ? (w.k_end - w.k_begin + kKeys - 1) / kKeys : 0;
  w.to_ws = w.ctx > a.part_tokens;
}

// Units with at least one key tile, in a CTA's order: blockIdx.x, + gridDim.x,
// ... A unit without one is passed to on_empty as the stream steps over it.
struct UnitStream {
  uint32_t u, stride, n;
  uint32_t G, qtiles;
  const int32_t* ctx_sm;
  Unit w;
  bool valid;
  template <typename F>
  __device__ __forceinline__ void init(const DecodeArgs& a, int32_t G_, int32_t qtiles_,
                                       int64_t num_units, const int32_t* ctx_cache, F on_empty) {
    G = uint32_t(G_);
    qtiles = uint32_t(qtiles_);
    n = uint32_t(num_units);
    ctx_sm = ctx_cache;
    stride = gridDim.x;
    u = blockIdx.x;
    seek(a, on_empty);
  }
  __device__ __forceinline__ void init(const DecodeArgs& a, int32_t G_, int32_t qtiles_,
                                       int64_t num_units, const int32_t* ctx_cache) {
    init(a, G_, qtiles_, num_units, ctx_cache, [](const Unit&) {});
  }
  template <typename F>
  __device__ __forceinline__ void next(const DecodeArgs& a, F on_empty) {
    u += stride;
    seek(a, on_empty);
  }
  __device__ __forceinline__ void next(const DecodeArgs& a) { next(a, [](const Unit&) {}); }
  template <typename F>
  __device__ __forceinline__ void seek(const DecodeArgs& a, F on_empty) {
    for (; u < n; u += stride) {
      unit_at(a, u, G, qtiles, ctx_sm, w);
      if (w.ntiles > 0) {
        valid = true;
        return;
      }
      on_empty(w);
    }
    valid = false;
  }
};

__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

// Two fp32 lanes in one 64-bit register: packed FMA and add (each lane rounds
// as its scalar instruction does).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

}  // namespace pf

// q map: 3-D {128 dims, num_q_heads, num_seqs * q_len} with a {64, G, 128 / G}
// box, o map the same over the output with a {64, G, 32 / G} box (each softmax
// warp stores its 32 rows of an unsplit unit through it); K map 2-D {128, rows} with a {64, BS} box; V map 3-D halves {64, rows,
// 2} with a {64, BS, 2} box (the decode kernel's maps). num_units = num_seqs
// x num_kv_heads x query tiles x a.pmax.
template <typename T, int BS>
__global__ void __launch_bounds__(pf::kThreads, 1) prefill_tc_kernel(
    const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap omap,
    const DecodeArgs a, int32_t qtiles, int64_t num_units) {
  using namespace pf;
  static_assert(BS == 16 || BS == 32, "block_size 16 or 32");
  constexpr int kBlocksPerTile = kKeys / BS;
  constexpr uint32_t kFmt = std::is_same<T, __half>::value ? 0u : 1u;
  constexpr bool kLo = !std::is_same<T, __half>::value;  // p's low part (bf16 inputs)
  constexpr uint32_t kIdescQK = tc::idesc_f16(kFmt, 0, 0, kKeys);  // Q, K both K-major
  constexpr uint32_t kIdescPV = tc::idesc_f16(kFmt, 0, 1, kD);     // P K-major, V MN-major

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint8_t* qbuf = smem + kOffQ;
  uint8_t* ring = smem + kOffRing;
  uint8_t* phi = smem + kOffPHi;
  uint8_t* plo = smem + kOffPLo;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = bars;                 // [kStages]
  uint64_t* empty = full + kStages;      // [kStages]
  uint64_t* q_full = empty + kStages;    // [2]
  uint64_t* q_empty = q_full + 2;        // [2]
  uint64_t* s_full = q_empty + 2;        // [2]
  uint64_t* s_free = s_full + 2;         // [2]
  uint64_t* o_free = s_free + 2;         // [2]
  // P buffer b (fp16: tile parity; bf16: always 0): p_full[b] completes when the
  // softmax has written it, p_free[b] when the PV that read it has completed.
  // Each barrier is at most one phase ahead of its waiter: a buffer is written
  // again only after its previous PV has been waited for.
  uint64_t* p_full = o_free + 2;         // [2]
  uint64_t* p_free = p_full + 2;         // [2]
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + kOffTmemPtr);
  __shared__ int abort_flag;
  const int32_t* ctx_sm = nullptr;  // context lengths are read per unit (L1-resident)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_trigger();  // the split-context reduce waits for this grid to complete
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&o_free[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&p_free[i], 1);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_ptr, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_ptr;
  const int32_t G = a.num_q_heads / a.num_kv_heads;
  const int32_t rows_total = a.num_blocks * a.num_kv_heads * BS;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
      prefetch_tensormap(&qmap);
      prefetch_tensormap(&omap);
    }
    const uint64_t pol_kv = l2_policy_evict_normal();  // a key tile serves every query tile
    const uint64_t pol_q = l2_policy_evict_first();
    uint32_t ctr = 0, ucnt = 0;
    bool ok = true;
    // lane j < kBlocksPerTile: the TMA row of block j of a tile (table loaded
    // one tile ahead)
    auto tile_id = [&](const Unit& w, int32_t t) -> int32_t {
      const int32_t k0 = w.k_begin + t * kKeys;
      const int32_t bidx = k0 / BS + lane;
      if (lane >= kBlocksPerTile || bidx * BS >= w.k_end) return -2;  // past the unit: zeros
      return __ldg(a.block_tables + int64_t(w.s) * a.max_blocks_per_seq + bidx);
    };
    auto id_row = [&](const Unit& w, int32_t t, int32_t id) -> int32_t {
      if (id == -2) return rows_total;
      if (id < 0 || id >= a.num_blocks) {
        const int32_t bidx = (w.k_begin + t * kKeys) / BS + lane;
        record_error(KVP_DEVERR_BLOCK_ID, (uint64_t(w.s) << 32) | uint32_t(bidx));
        return rows_total;
      }
      return (id * a.num_kv_heads + w.g) * BS;
    };
    auto load_tile = [&](const CUtensorMap* map, int32_t row, bool values) {
      const uint32_t st = ctr % kStages;
      if (lane == 0) {
        ok = mbar_wait(&empty[st], ((ctr / kStages) & 1u) ^ 1u, 0x8100u);
        if (ok) mbar_arrive_expect_tx(&full[st], kTileBytes);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok && lane < kBlocksPerTile) {
        if (values) {
          tma_load_3d(ring + st * kTileBytes + lane * BS * 256, map, &full[st], 0, row, 0, pol_kv);
        } else {
          uint8_t* dst = ring + st * kTileBytes + lane * BS * 128;
          tma_load_2d(dst, map, &full[st], 0, row, pol_kv);
          tma_load_2d(dst + kRegion, map, &full[st], 64, row, pol_kv);
        }
      }
      __syncwarp();
      ++ctr;
    };
    UnitStream cur;
    cur.init(a, G, qtiles, num_units, ctx_sm);
    uint32_t n = 0;                               // tiles of the CTA's stream so far
    int32_t v_row[2] = {rows_total, rows_total};  // rows of tiles n - 2 and n - 1
    while (cur.valid && ok) {
      const Unit w = cur.w;
      UnitStream nxt = cur;  // the next unit, decoded now (its loads overlap this one)
      nxt.next(a);
      // Q of the unit
      const uint32_t qb = ucnt & 1u;
      if (lane == 0) {
        ok = mbar_wait(&q_empty[qb], ((ucnt >> 1) & 1u) ^ 1u, 0x8200u);
        if (ok) {
          mbar_arrive_expect_tx(&q_full[qb], kTileBytes);
          const int32_t z = w.s * a.q_len + w.q0;
          tma_load_3d(qbuf + qb * kTileBytes, &qmap, &q_full[qb], 0, w.g * G, z, pol_q);
          tma_load_3d(qbuf + qb * kTileBytes + kRegion, &qmap, &q_full[qb], 64, w.g * G, z, pol_q);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ++ucnt;
      int32_t id = ok ? tile_id(w, 0) : -2;
      for (int32_t t = 0; t < w.ntiles && ok; ++t, ++n) {
        const int32_t id_next = t + 1 < w.ntiles ? tile_id(w, t + 1) : -2;
        const int32_t row = id_row(w, t, id);
        load_tile(&kmap, row, false);                          // K of tile n
        if (ok && n >= 2) load_tile(&vmap, v_row[n & 1], true);  // V of tile n - 2
        v_row[n & 1] = row;
        id = id_next;
      }
      cur = nxt;
    }
    // V of the stream's last two tiles
    for (uint32_t k = n < 2 ? 0u : n - 2; k < n && ok; ++k) load_tile(&vmap, v_row[k & 1], true);
    if (!ok) {
      atomicExch(&abort_flag, 1);
      if (lane == 0)
        for (uint32_t i = ctr > kStages ? ctr - kStages : 0; i < ctr; ++i)
          mbar_wait(&full[i % kStages], (i / kStages) & 1u, 0x8300u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Order over the CTA's stream of tiles (units one after another): QK(n),
    // then PV(n - 2), both waiting for the softmax of tile n - 2, and the last
    // two PVs at the end: S of a tile never waits behind a PV or a unit
    // boundary.
    uint32_t ctr = 0, ucnt = 0, n = 0;
    bool ok = true;
    struct Pend {
      uint32_t ob, ucnt;
      int32_t zero_from;
      bool first;
    } pend[2] = {};
    // O[ob] (+)= (P_hi + P_lo) . V for the pending tile; the warp zeroes the V
    // rows of tokens past the context (they hold whatever the pool had there;
    // p is 0 for them, but 0 * inf is NaN).
    auto pv = [&](const Pend& pd, uint32_t tile_n) {
      const uint32_t pb = kLo ? 0u : (tile_n & 1u);          // P buffer of the tile
      const uint32_t pphase = kLo ? tile_n : (tile_n >> 1);  // its use count
      if (lane == 0) {
        ok = mbar_wait(&p_full[pb], pphase & 1u, 0x8700u);
        if (ok && pd.first) ok = mbar_wait(&o_free[pd.ob], ((pd.ucnt >> 1) & 1u) ^ 1u, 0x8800u);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) return;
      const uint32_t st = ctr % kStages;
      if (lane == 0) ok = mbar_wait(&full[st], (ctr / kStages) & 1u, 0x8900u);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) return;
      tc_fence_after();
      uint8_t* tile = ring + st * kTileBytes;
      if (pd.zero_from < kKeys) {
        for (int row = pd.zero_from + lane; row < kKeys; row += 32) {
          uint8_t* r0 = tile + (row / BS) * (BS * 256) + (row % BS) * 128;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            reinterpret_cast<uint4*>(r0)[q] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4*>(r0 + BS * 128)[q] = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) {
        tc_fence_after();
        const uint32_t v_addr = smem_u32(tile);
        const uint32_t o_tmem = tmem_base + kOCol + pd.ob * kD;
#pragma unroll
        for (int part = 0; part < (kLo ? 2 : 1); ++part) {
          // bf16: the hi and lo parts; fp16: one part, buffer by tile parity
          const uint32_t p_addr =
              smem_u32(kLo ? (part == 0 ? phi : plo) : ((tile_n & 1u) ? plo : phi));
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk) {
            const uint32_t pa = p_addr + (kk >> 2) * kRegion + (kk & 3) * 32;
            const uint32_t va = v_addr + ((kk * 16) / BS) * (BS * 256) + ((kk * 16) % BS) * 128;
            umma_f16_ss(o_tmem, tc::smem_desc(pa, 16, 1024, tc::kLayoutSw128),
                        tc::smem_desc(va, BS * 128, 1024, tc::kLayoutSw128), kIdescPV,
                        (!pd.first || part > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[st]);
        umma_commit(&p_free[pb]);
      }
      __syncwarp();
      ++ctr;
    };
    UnitStream cur;
    cur.init(a, G, qtiles, num_units, ctx_sm);
    while (cur.valid && ok) {
      const Unit w = cur.w;
      UnitStream nxt = cur;
      nxt.next(a);
      const uint32_t qb = ucnt & 1u;
      if (lane == 0) ok = mbar_wait(&q_full[qb], (ucnt >> 1) & 1u, 0x8400u);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      const uint32_t q_addr = smem_u32(qbuf + qb * kTileBytes);
      for (int32_t t = 0; t < w.ntiles && ok; ++t, ++n) {
        // S[n & 1] = Q . K^T of tile n
        const uint32_t sb = n & 1u;
        if (lane == 0) {
          ok = mbar_wait(&s_free[sb], ((n >> 1) & 1u) ^ 1u, 0x8500u);
          const uint32_t st = ctr % kStages;
          if (ok) ok = mbar_wait(&full[st], (ctr / kStages) & 1u, 0x8600u);
          if (ok) {
            tc_fence_after();
            const uint32_t k_addr = smem_u32(ring + st * kTileBytes);
            const uint32_t d_tmem = tmem_base + kSCol + sb * kKeys;
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
              const uint32_t off = (kk >> 2) * kRegion + (kk & 3) * 32;
              // A = Q (rows), B = K (keys): S row r = query row r's scores
              umma_f16_ss(d_tmem, tc::smem_desc(q_addr + off, 16, 1024, tc::kLayoutSw128),
                          tc::smem_desc(k_addr + off, 16, 1024, tc::kLayoutSw128), kIdescQK,
                          kk > 0);
            }
            umma_commit(&empty[st]);
            umma_commit(&s_full[sb]);
            if (t == w.ntiles - 1) umma_commit(&q_empty[qb]);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        ++ctr;
        if (!ok) break;
        if (n >= 2) pv(pend[n & 1], n - 2);  // PV of tile n - 2
        const int32_t k0 = w.k_begin + t * kKeys;
        pend[n & 1].ob = ucnt & 1u;
        pend[n & 1].ucnt = ucnt;
        pend[n & 1].first = t == 0;
        pend[n & 1].zero_from = w.ctx - k0;
      }
      ++ucnt;
      cur = nxt;
    }
    // the last two PVs
    for (uint32_t k = n < 2 ? 0u : n - 2; k < n && ok; ++k) pv(pend[k & 1], k);
    if (!ok) atomicExch(&abort_flag, 1);
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row of the tile = TMEM lane
    const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
    auto wait_all = [&](uint64_t* bar, uint32_t parity, uint32_t where) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, where)) != 0;
    };
    // Rows of query tiles that see no key (a context shorter than its chunk)
    // in a sequence that is not split: zero output rows, as the stream steps
    // over their units.
    auto zero_rows = [&](const Unit& w) {
      if (w.to_ws || w.p > 0 || r / G >= w.nq) return;
      const int64_t row = (int64_t(w.s) * a.q_len + w.q0 + r / G) * a.num_q_heads + w.g * G + r % G;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<T*>(a.out) + row * kD);
#pragma unroll
      for (int c = 0; c < kD * 2 / 16; ++c) dst[c] = make_uint4(0, 0, 0, 0);
    };
    uint32_t n = 0, ucnt = 0;
    uint32_t seen[2] = {0, 0};  // phases of p_free[b] consumed
    // P buffer that this warp's last output store may still be reading
    const uint8_t* store_src = nullptr;
    bool ok = true;
    // waits until the PV of tile k has completed (and with it every earlier
    // MMA), consuming its buffer's phases in order
    auto wait_pv = [&](uint32_t k) {
      const uint32_t b = kLo ? 0u : (k & 1u);
      const uint32_t ph = kLo ? k : (k >> 1);
      while (ok && seen[b] <= ph) {
        ok = wait_all(&p_free[b], seen[b] & 1u, 0x8b00u);
        ++seen[b];
      }
    };
    // ---- epilogue of unit w (last tile nl, O buffer ob): the normalised rows,
    // or the partial (m, l, O) of a split sequence, once PV(nl) has completed
    auto epilogue = [&](const Unit& w, float m_ref, float l, uint32_t nl, uint32_t ob) {
      wait_pv(nl);
      if (!ok) return;
      tc_fence_after();
      const int32_t ti = r / G;  // query token of the row within the tile
      const bool row_live = ti < w.nq;
      const uint32_t o_taddr = tmem_base + lane_addr + kOCol + ob * kD;
      const int64_t qrow = (int64_t(w.s) * a.q_len + w.q0 + ti) * a.num_q_heads + w.g * G + r % G;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      // an unsplit unit's rows go out through the P buffer of tile nl (its PV
      // has completed) and one TMA store per 64-dim half, when every row of
      // the warp is a token of the chunk
      const int32_t tw = 32 / G;  // tokens of the warp's rows
      const bool staged = !w.to_ws && (quarter + 1) * tw <= w.nq;
      uint8_t* stage = kLo ? phi : ((nl & 1u) ? plo : phi);
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        float ov[32];
        tc::tmem_ld_cols<32>(o_taddr + c * 32, ov);
        tmem_ld_wait();
        if (c == kD / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&o_free[ob]);
        }
        if (staged) {
          // dims c*32 .. +32 of row r: four 16-byte chunks of region c / 2
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = (c & 1) * 4 + q;
            const uint32_t off = (c >> 1) * kRegion + r * 128 + ((chunk ^ (r & 7)) << 4);
            *reinterpret_cast<uint4*>(stage + off) =
                make_uint4(Elem<T>::pack2(ov[8 * q] * inv, ov[8 * q + 1] * inv),
                           Elem<T>::pack2(ov[8 * q + 2] * inv, ov[8 * q + 3] * inv),
                           Elem<T>::pack2(ov[8 * q + 4] * inv, ov[8 * q + 5] * inv),
                           Elem<T>::pack2(ov[8 * q + 6] * inv, ov[8 * q + 7] * inv));
          }
          continue;
        }
        if (!row_live) continue;
        if (!w.to_ws) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<T*>(a.out) + qrow * kD + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(Elem<T>::pack2(ov[8 * q] * inv, ov[8 * q + 1] * inv),
                                Elem<T>::pack2(ov[8 * q + 2] * inv, ov[8 * q + 3] * inv),
                                Elem<T>::pack2(ov[8 * q + 4] * inv, ov[8 * q + 5] * inv),
                                Elem<T>::pack2(ov[8 * q + 6] * inv, ov[8 * q + 7] * inv));
        } else {
          float4* dst = reinterpret_cast<float4*>(a.ws_acc + (qrow * a.ws_slots + w.p) * kD + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(ov[4 * q], ov[4 * q + 1], ov[4 * q + 2], ov[4 * q + 3]);
        }
      }
      if (row_live && w.to_ws) {
        a.ws_ml[(qrow * a.ws_slots + w.p) * 2 + 0] = m_ref;
        a.ws_ml[(qrow * a.ws_slots + w.p) * 2 + 1] = l;
      }
      if (staged) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const uint8_t* src = stage + quarter * 32 * 128;
          const int32_t z = w.s * a.q_len + w.q0 + quarter * tw;
          tma_store_3d(&omap, src, 0, w.g * G, z);
          tma_store_3d(&omap, src + kRegion, 64, w.g * G, z);
          bulk_commit();
        }
        store_src = stage;
      }
    };
    // fp16: a unit's epilogue runs after the softmax of the next tile, by which
    // time its last PV has completed (the P buffer of tile nl + 1 is the other
    // one); bf16 P fills both buffers, so its epilogue runs at once.
    struct Deferred {
      Unit w;
      float m, l;
      uint32_t nl, ob;
      bool valid;
    } dfr{};
    UnitStream cur;
    cur.init(a, G, qtiles, num_units, ctx_sm, zero_rows);
    while (cur.valid && ok) {
      const Unit w = cur.w;
      UnitStream nxt = cur;
      nxt.next(a, zero_rows);
      const int32_t ti = r / G;  // query token of the row within the tile
      const int32_t pos = w.ctx - a.q_len + w.q0 + ti;   // the row sees keys j <= pos
      const int32_t lim = min(pos + 1, w.k_end);          // exclusive end of its keys here
      float m_ref = -INFINITY, l = 0.f;
      const uint32_t ob = ucnt & 1u;
      const uint32_t o_taddr = tmem_base + lane_addr + kOCol + ob * kD;
      for (int32_t t = 0; t < w.ntiles && ok; ++t, ++n) {
        const uint32_t sb = n & 1u;
        const int32_t k0 = w.k_begin + t * kKeys;
        ok = wait_all(&s_full[sb], (n >> 1) & 1u, 0x8a00u);
        if (!ok) break;
        tc_fence_after();
        const uint32_t s_taddr = tmem_base + lane_addr + kSCol + sb * kKeys;
        // every row of the warp sees the whole tile (all but the diagonal tiles):
        // no per-key masks
        const bool full = __all_sync(0xffffffffu, k0 + kKeys <= lim);
        // pass 1: the row's largest score over the tile (keys it sees), scaled
        // once (scaling by a positive factor commutes with the max, rounding
        // included)
        float mx = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < kKeys / 32; ++c) {
          float sv[32];
          tc::tmem_ld_cols<32>(s_taddr + c * 32, sv);
          tmem_ld_wait();
          float m0 = -INFINITY, m1 = -INFINITY;
          if (full) {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              m0 = fmaxf(m0, sv[e]);
              m1 = fmaxf(m1, sv[e + 1]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              if (k0 + c * 32 + e < lim) m0 = fmaxf(m0, sv[e]);
              if (k0 + c * 32 + e + 1 < lim) m1 = fmaxf(m1, sv[e + 1]);
            }
          }
          mx = fmaxf(mx, fmaxf(m0, m1));
        }
        mx *= a.scale_log2;
        // the running maximum moves only by more than kLazy
        float factor = 1.f;
        bool need = false;
        if (mx > -INFINITY) {
          if (m_ref == -INFINITY) {
            m_ref = mx;  // nothing accumulated for this row yet (its p were 0)
          } else if (mx > m_ref + kLazy) {
            factor = exp2f(m_ref - mx);
            m_ref = mx;
            need = true;
          }
        }
        // P's buffer is free once the PV that last read it has completed (one
        // buffer: the previous tile's; two: the one before)
        if (kLo ? n >= 1 : n >= 2) wait_pv(kLo ? n - 1 : n - 2);
        if (!ok) break;
        if (__any_sync(0xffffffffu, need) && t > 0) {
          wait_pv(n - 1);  // O holds every PV of the unit so far
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < kD / 32; ++c) {
            float ov[32];
            tc::tmem_ld_cols<32>(o_taddr + c * 32, ov);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] *= factor;
            tmem_st_x32(o_taddr + c * 32, ov);
          }
          tmem_st_wait();
        }
        l *= factor;
        // pass 2: p = 2^(s - m) (bf16: as hi + lo parts) into P (row r, 128-byte
        // swizzle); l sums p in fp32 (pairs of lanes per instruction)
        const float nm = -m_ref;
        const uint64_t scale2 = f2_pack(a.scale_log2, a.scale_log2);
        const uint64_t nm2 = f2_pack(nm, nm);
        uint8_t* pdst = kLo ? phi : ((n & 1u) ? plo : phi);
        if (store_src == pdst) {  // the warp's output rows staged there have been read
          if (lane == 0) bulk_wait_read();
          __syncwarp();
          store_src = nullptr;
        }
#pragma unroll 1
        for (int c = 0; c < kKeys / 32; ++c) {
          float sv[32];
          tc::tmem_ld_cols<32>(s_taddr + c * 32, sv);
          tmem_ld_wait();
          uint32_t hw[16], lw[16];
          uint64_t l2 = f2_pack(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int j = k0 + c * 32 + e;
            const float2 x = f2_unpack(f2_fma(f2_pack(sv[e], sv[e + 1]), scale2, nm2));
            float p0 = tc::ex2_ftz(x.x);
            float p1 = tc::ex2_ftz(x.y);
            if (!full) {  // keys the row does not see (select, not multiply: NaN scores)
              p0 = j < lim ? p0 : 0.f;
              p1 = j + 1 < lim ? p1 : 0.f;
            }
            hw[e / 2] = Elem<T>::pack2(p0, p1);
            if constexpr (kLo) {
              const float2 hf = Elem<T>::to_float2(hw[e / 2]);
              lw[e / 2] = Elem<T>::pack2(p0 - hf.x, p1 - hf.y);
            }
            l2 = f2_add(l2, f2_pack(p0, p1));
          }
          const float2 lp = f2_unpack(l2);
          l += lp.x + lp.y;
          // keys c*32 .. +32 of row r: four 16-byte chunks of region c / 2
          const int region = c >> 1;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = (c & 1) * 4 + q;  // 16-byte chunk within the 128-byte row
            const uint32_t off = region * kRegion + r * 128 + ((chunk ^ (r & 7)) << 4);
            *reinterpret_cast<uint4*>(pdst + off) =
                make_uint4(hw[4 * q], hw[4 * q + 1], hw[4 * q + 2], hw[4 * q + 3]);
            if constexpr (kLo)
              *reinterpret_cast<uint4*>(plo + off) =
                  make_uint4(lw[4 * q], lw[4 * q + 1], lw[4 * q + 2], lw[4 * q + 3]);
          }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&s_free[sb]);
          mbar_arrive(&p_full[kLo ? 0u : (n & 1u)]);
        }
        if (!kLo && dfr.valid) {
          epilogue(dfr.w, dfr.m, dfr.l, dfr.nl, dfr.ob);
          dfr.valid = false;
          if (!ok) break;
        }
        if (t == w.ntiles - 1) {
          if (kLo) {
            epilogue(w, m_ref, l, n, ob);
          } else {
            dfr.w = w;
            dfr.m = m_ref;
            dfr.l = l;
            dfr.nl = n;
            dfr.ob = ob;
            dfr.valid = true;
          }
        }
      }
      ++ucnt;
      cur = nxt;
    }
    if (ok && dfr.valid) epilogue(dfr.w, dfr.m, dfr.l, dfr.nl, dfr.ob);
    if (lane == 0) bulk_wait_all();  // the warp's output stores have completed
    if (!ok) atomicExch(&abort_flag, 1);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace dev
}  // namespace kvp
