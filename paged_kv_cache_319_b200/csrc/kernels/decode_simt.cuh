// Paged decode attention on the CUDA cores, one CTA per (partition, query
// head, sequence), and the log-sum-exp merge of split partitions.
//
// What it computes: for sequence s and query head h (KV head g = h / G), the
// keys and values of tokens j < ctx are found through the block table -
// physical block block_tables[s][j / bs], slot j % bs - and the output is
// softmax(scale * q K^T) V, the same result as over a contiguous cache ["vLLM
// and PagedAttention", section "Architecture, step by step", step 3; "Your
// GPU was mostly empty", section "The OS already solved this in the 1960s"].
//
// How: each warp of the CTA owns every NW-th block of the partition and runs
// its own TMA pipeline of NST stages: one elected lane issues two tensor loads
// (K tile, V tile: block_size rows x head_dim, 128-byte swizzled; for 128 dims
// one 3-D box {64 dims, rows, 2 halves} each, so a tile costs one TMA
// operation) per block onto the stage's mbarrier. A (block, KV head) tile is one contiguous
// block_size * head_dim run of the cache, so every load is one dense 2-4 KiB
// burst. The warp keeps a running max m, a per-lane exponent sum and an fp32
// accumulator (online softmax in the log2 domain, q pre-scaled by
// scale * log2 e). QK: two lanes per key row, 16-byte swizzled reads (no
// bank conflicts), one shuffle to join the halves; row max by a single
// integer max-reduction. PV: each lane owns head_dim / 32 output dims and
// broadcasts p by shuffle. At the end the warps merge through shared memory
// and the CTA writes either the normalised output or, for split sequences,
// (m, l, acc) to the workspace.
#pragma once

#include <math.h>

#include "../pack_layout.h"
#include "common.cuh"

namespace kvp {
namespace dev {

// Grouped decode: word of the plan where the per-sequence shared-prefix block
// counts start (the plan's layout is described in decode_group.cuh).
constexpr int kPlanSeqWord = 8;

struct DecodeArgs {
  const void* q;                // [S][Hq][D]
  void* out;                    // [S][Hq][D]
  const int32_t* block_tables;  // [S][max_blocks_per_seq]
  const int32_t* context_lens;  // [S]
  float* ws_ml;                 // [S][Hq][ws_slots][2] = (m in log2 units, l)
  float* ws_acc;                // [S][Hq][ws_slots][D], unnormalised
  int32_t num_seqs;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t num_blocks;
  int32_t max_blocks_per_seq;
  int32_t max_context_len;
  int32_t part_blocks;  // partition length in blocks (whole context when unsplit)
  int32_t part_tokens;  // part_blocks * block_size
  int32_t pmax;         // partitions per (sequence, head) in the grid
  int32_t ws_slots;     // partial slots per (sequence, head) in the workspace
  float scale_log2;     // scale * log2(e)
  // Multi-query (prefill) chunks: q and out hold q_len rows per sequence; a
  // launch takes queries [q_first, q_first + q_count) of each. Decode: 1, 0, 1.
  int32_t q_len, q_first, q_count;
  // Grouped decode only (null otherwise): the grouping plan of
  // decode_group.cuh. Every (sequence, head) then has ceil(c * bs / P) slots
  // for its shared prefix followed by the slots of its own range, and the
  // reduce writes every output row.
  const int32_t* plan;
  // FP8 cache only (null otherwise): per KV head, the scales of the E4M3 keys
  // and values (a cached code c of head g stands for value(c) * scale[g]).
  const float* k_scale;
  const float* v_scale;
  // Virtually contiguous cache only (null otherwise): the slot of each
  // sequence and each slot's mapped capacity; a tile of sequence s starting at
  // token j has the token coordinate vc_seq_slots[s] * vc_slot_tokens + j.
  const int32_t* vc_seq_slots;
  const int32_t* vc_cap;
  int32_t vc_slot_tokens;
  int32_t vc_num_slots;
  // Packed grouped decode: `plan` is a packed plan (pack_layout.h); every
  // (sequence, head) has one partial per chunk of its group's block stream.
  int32_t plan_packed;
};

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// Clamped context length of sequence s (records out-of-range values once).
__device__ __forceinline__ int32_t load_ctx(const DecodeArgs& a, int32_t s, bool report) {
  int32_t ctx = __ldg(a.context_lens + s);
  if (ctx < 0 || ctx > a.max_context_len) {
    if (report) record_error(KVP_DEVERR_CTX, uint64_t(s));
    ctx = ctx < 0 ? 0 : a.max_context_len;
  }
  return ctx;
}

// Context length of sequence s as every kernel of a call reads it: clamped as
// by load_ctx and, over a virtually contiguous cache, to the mapped capacity
// of the sequence's slot (a slot out of range reads nothing), so no tile ever
// reaches an unmapped address.
__device__ __forceinline__ int32_t seq_ctx(const DecodeArgs& a, int32_t s, bool report) {
  int32_t ctx = load_ctx(a, s, report);
  if (a.vc_cap) {
    const int32_t slot = __ldg(a.vc_seq_slots + s);
    if (slot < 0 || slot >= a.vc_num_slots) {
      if (report) record_error(KVP_DEVERR_BLOCK_ID, (uint64_t(s) << 32) | 0xFFFFFFFFu);
      return 0;
    }
    const int32_t cap = __ldg(a.vc_cap + slot);
    if (ctx > cap) {
      if (report) record_error(KVP_DEVERR_CTX, uint64_t(s));
      ctx = cap;
    }
  }
  return ctx;
}

// Token coordinate of the first token of sequence s's slot (virtually
// contiguous cache; 0 for a slot out of range, whose context is 0).
__device__ __forceinline__ int32_t vc_base(const DecodeArgs& a, int32_t s) {
  const int32_t slot = __ldg(a.vc_seq_slots + s);
  return (slot >= 0 && slot < a.vc_num_slots) ? slot * a.vc_slot_tokens : 0;
}

// EB: bytes per cached element (2: fp16 / bf16; 1: E4M3).
template <typename T, int D, int BS, int NW, int NST, int EB = 2>
struct SimtCfg {
  static constexpr int kRegions = D * EB / 128;    // 128-byte row regions (1 or 2)
  static constexpr int kTileBytes = BS * D * EB;   // one (block, KV head) tile
  static constexpr int kChunksPerRow = D / 8;      // 16-byte chunks per row
  static constexpr int kChunksPerLane = kChunksPerRow / 2;
  static constexpr int kPasses = (BS + 15) / 16;   // 16 rows per QK pass
  static constexpr int kDimsPerLane = D / 32;
  static constexpr int kTileArea = NW * NST * 2 * kTileBytes;
  static constexpr int kBarArea = NW * NST * 8;
  static constexpr int kMergeArea = NW * (D + 2) * 4;
  static constexpr int kSmemBytes = 1024 + kTileArea + kBarArea + kMergeArea;
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(BS == 8 || BS == 16 || BS == 32, "block_size 8, 16 or 32");
  static_assert(NST >= 1 && NST <= 32, "stages");
  static_assert(EB == 2 || D == 128, "E4M3 caches: head_dim 128 (one 128-byte row)");
};

// Per-lane shapes of a (block, KV head) tile in the CUDA-core kernels.
template <int D, int BS>
struct TileShape {
  static constexpr int kChunksPerLane = D / 16;  // 16-byte chunks of q / a key row per lane
  static constexpr int kPasses = (BS + 15) / 16;  // 16 key rows per QK pass
  static constexpr int kDimsPerLane = D / 32;     // output dims per lane
};

// Folds one tile of keys and values ([region][row][64], 128-byte swizzled,
// rows r < nvalid valid) into a warp's online-softmax state (log2 domain):
// running max m_run, per-lane exponent sum l_lane (lanes 0..15), and the
// lane's kDimsPerLane output dims acc. qf: the lane's half of q, pre-scaled.
// QK: two lanes per key row, swizzled 16-byte shared loads, one shuffle; row
// max by one integer max-reduction; PV: p broadcast by shuffle.
template <typename T, int D, int BS>
__device__ __forceinline__ void simt_tile(const uint8_t* kt, const uint8_t* vt, int32_t nvalid,
                                          const float (&qf)[TileShape<D, BS>::kChunksPerLane * 8],
                                          float& m_run, float& l_lane,
                                          float (&acc)[TileShape<D, BS>::kDimsPerLane], int lane) {
  using TC_ = TileShape<D, BS>;
  const int part = lane >> 4;
  // ---- scores: row r = pass * 16 + (lane & 15), half `part` of its chunks
  float sc[TC_::kPasses];
#pragma unroll
  for (int ps = 0; ps < TC_::kPasses; ++ps) {
    const int r = ps * 16 + (lane & 15);
    float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
    if (r < BS) {
#pragma unroll
      for (int c = 0; c < TC_::kChunksPerLane; ++c) {
        const int lc = part * TC_::kChunksPerLane + c;
        const int region = lc >> 3;
        const int cc = lc & 7;
        const uint4 kv = *reinterpret_cast<const uint4*>(kt + region * BS * 128 + r * 128 +
                                                         ((cc ^ (r & 7)) << 4));
        const float2 f0 = Elem<T>::to_float2(kv.x);
        const float2 f1 = Elem<T>::to_float2(kv.y);
        const float2 f2 = Elem<T>::to_float2(kv.z);
        const float2 f3 = Elem<T>::to_float2(kv.w);
        d0 = fmaf(qf[c * 8 + 0], f0.x, d0);
        d1 = fmaf(qf[c * 8 + 1], f0.y, d1);
        d2 = fmaf(qf[c * 8 + 2], f1.x, d2);
        d3 = fmaf(qf[c * 8 + 3], f1.y, d3);
        d0 = fmaf(qf[c * 8 + 4], f2.x, d0);
        d1 = fmaf(qf[c * 8 + 5], f2.y, d1);
        d2 = fmaf(qf[c * 8 + 6], f3.x, d2);
        d3 = fmaf(qf[c * 8 + 7], f3.y, d3);
      }
    }
    float dot = (d0 + d1) + (d2 + d3);
    dot += __shfl_xor_sync(0xffffffffu, dot, 16);
    sc[ps] = r < nvalid ? dot : -INFINITY;
  }

  // ---- online softmax update (log2 domain)
  float tmax = sc[0];
#pragma unroll
  for (int ps = 1; ps < TC_::kPasses; ++ps) tmax = fmaxf(tmax, sc[ps]);
  tmax = warp_max(tmax);
  const float m_new = fmaxf(m_run, tmax);
  const float alpha = m_run == -INFINITY ? 0.f : exp2f(m_run - m_new);
  float pr[TC_::kPasses];
  float psum = 0.f;
#pragma unroll
  for (int ps = 0; ps < TC_::kPasses; ++ps) {
    pr[ps] = sc[ps] == -INFINITY ? 0.f : exp2f(sc[ps] - m_new);
    psum += pr[ps];
  }
  l_lane = l_lane * alpha + (lane < 16 ? psum : 0.f);
#pragma unroll
  for (int e = 0; e < TC_::kDimsPerLane; ++e) acc[e] *= alpha;
  m_run = m_new;

  // ---- acc += p V: lane owns dims [lane * kDimsPerLane, +kDimsPerLane)
  {
    constexpr int DPL = TC_::kDimsPerLane;
    const int d0 = lane * DPL;
    const int region = d0 >> 6;
    const int cc = (d0 & 63) >> 3;
    const int pos = d0 & 7;
#pragma unroll
    for (int r = 0; r < BS; ++r) {
      const float pv = __shfl_sync(0xffffffffu, pr[r >> 4], r & 15);
      if (r < nvalid) {
        const uint8_t* src = vt + region * BS * 128 + r * 128 + ((cc ^ (r & 7)) << 4) + pos * 2;
        if constexpr (DPL == 4) {
          const uint2 v = *reinterpret_cast<const uint2*>(src);
          const float2 f0 = Elem<T>::to_float2(v.x);
          const float2 f1 = Elem<T>::to_float2(v.y);
          acc[0] = fmaf(pv, f0.x, acc[0]);
          acc[1] = fmaf(pv, f0.y, acc[1]);
          acc[2] = fmaf(pv, f1.x, acc[2]);
          acc[3] = fmaf(pv, f1.y, acc[3]);
        } else {
          const uint32_t v = *reinterpret_cast<const uint32_t*>(src);
          const float2 f0 = Elem<T>::to_float2(v);
          acc[0] = fmaf(pv, f0.x, acc[0]);
          acc[1] = fmaf(pv, f0.y, acc[1]);
        }
      }
    }
  }
}

// simt_tile for an E4M3 cache (head_dim 128: a tile row is 128 codes, one
// 128-byte swizzled region). Same lanes and steps as simt_tile: a QK lane
// covers 64 dims of its key row as four 16-byte chunks of 16 codes; a PV lane
// owns 4 output dims (4 codes of each value row). Codes convert exactly to
// fp16 (cvt.rn.f16x2.e4m3x2, two per instruction). With half the bytes of a
// 16-bit cache per token the kernel is bound by instructions, not HBM, so the
// QK products of an fp16 q take the fp16 keys directly in sm_100's mixed-
// precision fma (fp16 x fp16 + fp32; the products are exact in fp32), with
// the scales applied to the dot. On the OPT-13B batch this took the call from
// 142 us (keys widened to fp32 first) to 118 us; widening by shifts and masks
// instead of cvt was slower (167 us). A bf16 q uses fp32 FMAs for the QK
// products. The PV products take p rounded to fp16 (p <= 1, relative error
// at most 2^-12) and the fp16 codes in the same mixed-precision fma; the value
// scale is applied by the caller to the finished accumulator.
#ifndef KVP_FP8_MIXED
#define KVP_FP8_MIXED 1  // 0: widen fp16 keys to fp32 for the QK products as well
#endif
// d0 += lo(q2) * lo(k2), d1 += hi(q2) * hi(k2): fp16 products accumulated in
// fp32 by sm_100's mixed-precision fma (no conversion of k to fp32).
__device__ __forceinline__ void fma2_f16_f32(float& d0, float& d1, uint32_t q2, uint32_t k2) {
  asm("{\n\t.reg .f16 ql, qh, kl, kh;\n\t"
      "mov.b32 {ql, qh}, %2;\n\t"
      "mov.b32 {kl, kh}, %3;\n\t"
      "fma.rn.f32.f16 %0, ql, kl, %0;\n\t"
      "fma.rn.f32.f16 %1, qh, kh, %1;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "r"(q2), "r"(k2));
}

// acc[0..3] += p * v[0..3] for four E4M3 codes of a value row (bytes of v4,
// lowest first): the codes widen exactly to fp16 (two per cvt) and meet p,
// rounded once to fp16, in the mixed-precision fma with fp32 accumulation.
__device__ __forceinline__ void fma4_p16_e4m3(float (&acc)[4], uint32_t p16, uint32_t v4) {
  uint32_t k01, k23;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(k01) : "h"(static_cast<uint16_t>(v4)));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(k23) : "h"(static_cast<uint16_t>(v4 >> 16)));
  asm("{\n\t.reg .f16 p, pz, a, b, c, d;\n\t"
      "mov.b32 {p, pz}, %4;\n\t"
      "mov.b32 {a, b}, %5;\n\t"
      "mov.b32 {c, d}, %6;\n\t"
      "fma.rn.f32.f16 %0, p, a, %0;\n\t"
      "fma.rn.f32.f16 %1, p, b, %1;\n\t"
      "fma.rn.f32.f16 %2, p, c, %2;\n\t"
      "fma.rn.f32.f16 %3, p, d, %3;\n\t}"
      : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3])
      : "r"(p16), "r"(k01), "r"(k23));
}

// MX: q is fp16 and arrives as 32 packed pairs in qh (qf unused), unscaled; the
// score is dot * q_mul.
template <int BS, bool MX = false>
__device__ __forceinline__ void simt_tile_fp8(const uint8_t* kt, const uint8_t* vt, int32_t nvalid,
                                              const float (&qf)[64], const uint32_t (&qh)[32],
                                              float q_mul, float& m_run, float& l_lane,
                                              float (&acc)[4], int lane) {
  constexpr int kPasses = (BS + 15) / 16;
  const int part = lane >> 4;
  float sc[kPasses];
#pragma unroll
  for (int ps = 0; ps < kPasses; ++ps) {
    const int r = ps * 16 + (lane & 15);
    float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
    if (r < BS) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int lc = part * 4 + c;  // 16-byte chunk of the row: dims lc * 16 ..
        const uint4 kv = *reinterpret_cast<const uint4*>(kt + r * 128 + ((lc ^ (r & 7)) << 4));
        const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if constexpr (MX) {
            uint32_t k01, k23;
            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(k01) : "h"(static_cast<uint16_t>(w[e])));
            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(k23) : "h"(static_cast<uint16_t>(w[e] >> 16)));
            fma2_f16_f32(d0, d1, qh[c * 8 + 2 * e], k01);
            fma2_f16_f32(d2, d3, qh[c * 8 + 2 * e + 1], k23);
          } else {
            const float2 f0 = e4m3x2_to_float2(w[e]);
            const float2 f1 = e4m3x2_to_float2(w[e] >> 16);
            d0 = fmaf(qf[c * 16 + 4 * e + 0], f0.x, d0);
            d1 = fmaf(qf[c * 16 + 4 * e + 1], f0.y, d1);
            d2 = fmaf(qf[c * 16 + 4 * e + 2], f1.x, d2);
            d3 = fmaf(qf[c * 16 + 4 * e + 3], f1.y, d3);
          }
        }
      }
    }
    float dot = (d0 + d1) + (d2 + d3);
    if constexpr (MX) dot *= q_mul;
    dot += __shfl_xor_sync(0xffffffffu, dot, 16);
    sc[ps] = r < nvalid ? dot : -INFINITY;
  }
  float tmax = sc[0];
#pragma unroll
  for (int ps = 1; ps < kPasses; ++ps) tmax = fmaxf(tmax, sc[ps]);
  tmax = warp_max(tmax);
  const float m_new = fmaxf(m_run, tmax);
  const float alpha = m_run == -INFINITY ? 0.f : exp2f(m_run - m_new);
  uint32_t p16[kPasses];  // p in fp16 (p <= 1) for the value products; l sums it in fp32
  float psum = 0.f;
#pragma unroll
  for (int ps = 0; ps < kPasses; ++ps) {
    const float p = sc[ps] == -INFINITY ? 0.f : exp2f(sc[ps] - m_new);
    p16[ps] = __half_as_ushort(__float2half_rn(p));
    psum += p;
  }
  l_lane = l_lane * alpha + (lane < 16 ? psum : 0.f);
#pragma unroll
  for (int e = 0; e < 4; ++e) acc[e] *= alpha;
  m_run = m_new;
  // acc += p V: dims lane * 4 .. + 3 are bytes (lane & 3) * 4 .. of chunk lane / 4
  const int cc = lane >> 2;
  const int pos = (lane & 3) * 4;
#pragma unroll
  for (int r = 0; r < BS; ++r) {
    const uint32_t pv = __shfl_sync(0xffffffffu, p16[r >> 4], r & 15);
    if (r < nvalid)
      fma4_p16_e4m3(acc, pv,
                    *reinterpret_cast<const uint32_t*>(vt + r * 128 + ((cc ^ (r & 7)) << 4) + pos));
  }
}

// PH (per-head warps): grid (partition, ceil(Hq / NW), sequence); warp w takes
// query head blockIdx.y * NW + w over the whole partition and writes its own
// partial, with no merge across warps. For short ranges (a few blocks per
// (sequence, head)), where splitting a range over the warps would leave each
// warp one or two blocks, this keeps every warp's pipeline busy.
// F8: the cache holds E4M3 codes (a.k_scale / a.v_scale set; head_dim 128);
// q and out stay in T.
// VC: a virtually contiguous cache (a.vc_* set; head_dim 128): a tile is BS
// consecutive tokens of the sequence's slot, one 4-D box {64 dims, BS tokens,
// 2 halves, 1 head} at the computed token coordinate, in place of a block
// table lookup; everything else is the paged kernel's.
template <typename T, int D, int BS, int NW, int NST, bool PH = false, bool F8 = false,
          bool VC = false>
__global__ void __launch_bounds__(NW * 32) decode_simt_kernel(
    const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
    const DecodeArgs a) {
  using C = SimtCfg<T, D, BS, NW, NST, F8 ? 1 : 2>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint8_t* tiles = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kTileArea);
  float* mg_m = reinterpret_cast<float*>(smem + C::kTileArea + C::kBarArea);
  float* mg_l = mg_m + NW;
  float* mg_acc = mg_l + NW;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int p = blockIdx.x;
  const int h = PH ? int(blockIdx.y) * NW + warp : int(blockIdx.y);
  const int s = blockIdx.z;

  // The split-context reduce may be scheduled as soon as every CTA of this grid
  // has started; it waits for this grid to complete before reading partials.
  pdl_trigger();
  // Grouped decode: this kernel attends to each sequence's own blocks, from
  // the end of its shared prefix on, and was launched while the shared-prefix
  // kernel ahead of it may still run (every CTA of that kernel had passed its
  // wait for the plan). One CTA waits for that kernel, so this grid completes
  // after it and the reduce's wait covers both.
  const bool grouped = a.plan != nullptr;
  if (grouped && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) pdl_wait();
  if (PH && h >= a.num_q_heads) return;  // a warp past the last head (no CTA-wide sync follows)
  // the plan word and the context length are loaded together
  int32_t b_first = grouped ? ld_relaxed_gpu(a.plan + kPlanSeqWord + s) : 0;
  const int32_t ctx = seq_ctx(a, s, p == 0 && blockIdx.y == 0 && threadIdx.x == 0);
  const int32_t nblk = (ctx + BS - 1) / BS;
  int32_t slot = p;
  if (grouped) slot = (b_first + a.part_blocks - 1) / a.part_blocks + p;  // after the shared slots
  const int32_t b0 = b_first + p * a.part_blocks;
  // empty partition (p == 0 always writes its row, except in the grouped decode)
  if ((p > 0 || grouped) && b0 >= nblk) return;
  const int32_t b1 = min(nblk, b0 + a.part_blocks);
  // partials go to the workspace for split sequences and in the grouped decode
  const bool to_ws = grouped || nblk > a.part_blocks;
  const int32_t g = h / (a.num_q_heads / a.num_kv_heads);
  const int32_t* table = a.block_tables + int64_t(s) * a.max_blocks_per_seq;

  // Blocks of this warp: b0 + warp + NW * i, i < nw (PH: b0 + i, i < span).
  const int32_t span = b1 - b0;
  constexpr int kStride = PH ? 1 : NW;
  const int32_t wfirst = PH ? 0 : warp;
  const int32_t nw = span > wfirst ? (span - wfirst + kStride - 1) / kStride : 0;

  uint64_t* my_bars = bars + warp * NST;
  uint8_t* my_tiles = tiles + size_t(warp) * NST * 2 * C::kTileBytes;
  if (lane == 0) {
    for (int i = 0; i < NST; ++i) mbar_init(&my_bars[i], 1);
    fence_mbar_init();
  }
  if (lane == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  __syncwarp();

  const uint64_t policy = l2_policy_kv();
  const int32_t rows_total = a.num_blocks * a.num_kv_heads * BS;

  // Register cache of 32 block ids: lane l holds id of index base + l (a
  // virtually contiguous cache has no ids: the tile coordinate is computed).
  int32_t id_base = 0;
  int32_t my_id = -1;
  const int32_t tok_base = VC ? vc_base(a, s) : 0;
  auto load_ids = [&](int32_t base) {
    if constexpr (!VC) {
      const int32_t idx = base + lane;
      my_id = idx < nw ? __ldg(table + b0 + wfirst + kStride * idx) : -1;
    }
  };
  load_ids(0);

  auto issue = [&](int32_t i, int32_t id) {  // lane 0 only
    const int stage = i % NST;
    uint8_t* kt = my_tiles + size_t(stage) * 2 * C::kTileBytes;
    uint8_t* vt = kt + C::kTileBytes;
    if constexpr (VC) {
      // tokens [j, j + BS) of the slot, all inside its mapped range (j < ctx <= cap)
      const int32_t tok = tok_base + (b0 + wfirst + kStride * i) * BS;
      mbar_arrive_expect_tx(&my_bars[stage], 2 * C::kTileBytes);
      tma_load_4d(kt, &kmap, &my_bars[stage], 0, tok, 0, g, policy);
      tma_load_4d(vt, &vmap, &my_bars[stage], 0, tok, 0, g, policy);
      return;
    }
    int32_t row;
    if (id < 0 || id >= a.num_blocks) {
      record_error(KVP_DEVERR_BLOCK_ID, (uint64_t(s) << 32) | uint32_t(b0 + wfirst + kStride * i));
      row = rows_total;  // out of the tensor: the load fills zeros
    } else {
      row = (id * a.num_kv_heads + g) * BS;
    }
    mbar_arrive_expect_tx(&my_bars[stage], 2 * C::kTileBytes);
    if constexpr (F8) {
      // one 2-D box {128 codes, BS rows} per tile: smem [row][128]
      tma_load_2d(kt, &kmap, &my_bars[stage], 0, row, policy);
      tma_load_2d(vt, &vmap, &my_bars[stage], 0, row, policy);
    } else if constexpr (C::kRegions == 2) {
      // one 3-D box {64 dims, BS rows, 2 halves} per tile: smem [half][row][64]
      tma_load_3d(kt, &kmap, &my_bars[stage], 0, row, 0, policy);
      tma_load_3d(vt, &vmap, &my_bars[stage], 0, row, 0, policy);
    } else {
      tma_load_2d(kt, &kmap, &my_bars[stage], 0, row, policy);
      tma_load_2d(vt, &vmap, &my_bars[stage], 0, row, policy);
    }
  };

  {
    const int npro = nw < NST ? nw : NST;
    for (int i = 0; i < npro; ++i) {
      const int32_t id = __shfl_sync(0xffffffffu, my_id, i);
      if (lane == 0) issue(i, id);
    }
  }

  // q of this head, pre-scaled: lane part (lane >> 4) covers chunks
  // [part * kChunksPerLane, (part + 1) * kChunksPerLane) of the row.
  const int part = lane >> 4;
  float qf[C::kChunksPerLane * 8];
  float q_mul = a.scale_log2;
  if constexpr (F8) q_mul *= __ldg(a.k_scale + g);
  constexpr bool kMixed = F8 && KVP_FP8_MIXED && std::is_same<T, __half>::value;
  uint32_t qh[32];  // kMixed: this lane's 64 dims of q as fp16 pairs
  if constexpr (kMixed) {
    const uint4* qrow = reinterpret_cast<const uint4*>(static_cast<const T*>(a.q) +
                                                       (int64_t(s) * a.num_q_heads + h) * D);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 v = __ldg(qrow + part * 8 + c);
      qh[4 * c] = v.x;
      qh[4 * c + 1] = v.y;
      qh[4 * c + 2] = v.z;
      qh[4 * c + 3] = v.w;
    }
  } else {
    const uint4* qrow = reinterpret_cast<const uint4*>(static_cast<const T*>(a.q) +
                                                       (int64_t(s) * a.num_q_heads + h) * D);
#pragma unroll
    for (int c = 0; c < C::kChunksPerLane; ++c) {
      const uint4 v = __ldg(qrow + part * C::kChunksPerLane + c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = Elem<T>::to_float2(w[e]);
        qf[c * 8 + 2 * e] = f.x * q_mul;
        qf[c * 8 + 2 * e + 1] = f.y * q_mul;
      }
    }
  }

  float m_run = -INFINITY;
  float l_lane = 0.f;
  float acc[C::kDimsPerLane];
#pragma unroll
  for (int e = 0; e < C::kDimsPerLane; ++e) acc[e] = 0.f;

  bool aborted = false;
  int32_t i_fail = 0;
  for (int32_t i = 0; i < nw; ++i) {
    const int stage = i % NST;
    const uint32_t phase = uint32_t(i / NST) & 1u;
    if (!__all_sync(0xffffffffu, mbar_wait(&my_bars[stage], phase, 0x5100u + stage))) {
      aborted = true;
      i_fail = i;
      break;
    }
    const uint8_t* kt = my_tiles + size_t(stage) * 2 * C::kTileBytes;
    const uint8_t* vt = kt + C::kTileBytes;
    const int32_t tok0 = (b0 + wfirst + kStride * i) * BS;
    const int32_t nvalid = min(BS, ctx - tok0);

    if constexpr (F8) {
      simt_tile_fp8<BS, kMixed>(kt, vt, nvalid, qf, qh, q_mul, m_run, l_lane, acc, lane);
    } else {
      simt_tile<T, D, BS>(kt, vt, nvalid, qf, m_run, l_lane, acc, lane);
    }

    // ---- refill this stage with block i + NST
    const int32_t nxt = i + NST;
    if (nxt < nw && nxt >= id_base + 32) {
      id_base += 32;
      load_ids(id_base);
    }
    const int32_t id = __shfl_sync(0xffffffffu, my_id, (nxt - id_base) & 31);
    __syncwarp();
    if (lane == 0 && nxt < nw) {
      fence_proxy_async_smem();
      issue(nxt, id);
    }
  }

  if constexpr (F8) {  // the values' scale, once, on the finished sums
    const float vs = __ldg(a.v_scale + g);
#pragma unroll
    for (int e = 0; e < C::kDimsPerLane; ++e) acc[e] *= vs;
  }
  if (aborted) {
    // Drain this warp's loads still in flight before the CTA exits.
    if (lane == 0) {
      for (int32_t i = i_fail; i < nw && i < i_fail + NST; ++i)
        mbar_wait(&my_bars[i % NST], uint32_t(i / NST) & 1u, 0x5200u);
    }
    m_run = -INFINITY;
  }

  if constexpr (PH) {
    // ---- this warp's partial (no merge across warps)
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) l_lane += __shfl_xor_sync(0xffffffffu, l_lane, o);
    const float L = __shfl_sync(0xffffffffu, l_lane, 0);
    const int64_t row_sh = int64_t(s) * a.num_q_heads + h;
#pragma unroll
    for (int e = 0; e < C::kDimsPerLane; ++e) {
      const int t = lane * C::kDimsPerLane + e;
      if (!to_ws) {
        const float y = (L > 0.f && !aborted) ? acc[e] / L : 0.f;
        static_cast<uint16_t*>(a.out)[row_sh * D + t] = Elem<T>::from_float(y);
      } else {
        a.ws_acc[(row_sh * a.ws_slots + slot) * D + t] = acc[e];
      }
    }
    if (to_ws && lane == 0) {
      a.ws_ml[(row_sh * a.ws_slots + slot) * 2 + 0] = aborted ? -INFINITY : m_run;
      a.ws_ml[(row_sh * a.ws_slots + slot) * 2 + 1] = aborted ? 0.f : L;
    }
  } else {
    // ---- merge the warps
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) l_lane += __shfl_xor_sync(0xffffffffu, l_lane, o);
    if (lane == 0) {
      mg_m[warp] = m_run;
      mg_l[warp] = l_lane;
    }
#pragma unroll
    for (int e = 0; e < C::kDimsPerLane; ++e) mg_acc[warp * D + lane * C::kDimsPerLane + e] = acc[e];
    const int any_abort = __syncthreads_or(aborted ? 1 : 0);

    const int64_t row_sh = int64_t(s) * a.num_q_heads + h;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mg_m[w]);
    float wgt[NW];
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      wgt[w] = (mg_m[w] == -INFINITY || M == -INFINITY) ? 0.f : exp2f(mg_m[w] - M);
      L += mg_l[w] * wgt[w];
    }
    for (int t = threadIdx.x; t < D; t += NW * 32) {
      float o = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) o = fmaf(mg_acc[w * D + t], wgt[w], o);
      if (!to_ws) {
        const float y = (L > 0.f && !any_abort) ? o / L : 0.f;
        static_cast<uint16_t*>(a.out)[row_sh * D + t] = Elem<T>::from_float(y);
      } else {
        a.ws_acc[(row_sh * a.ws_slots + slot) * D + t] = o;
      }
    }
    if (to_ws && threadIdx.x == 0) {
      a.ws_ml[(row_sh * a.ws_slots + slot) * 2 + 0] = any_abort ? -INFINITY : M;
      a.ws_ml[(row_sh * a.ws_slots + slot) * 2 + 1] = any_abort ? 0.f : L;
    }
  }
}

// Log-sum-exp merge of the partitions of split sequences: M = max_p m_p,
// L = sum_p l_p 2^(m_p - M), out = sum_p 2^(m_p - M) acc_p / L.
// grid (ceil(Hq / kReduceHeads), S * q_len), kReduceHeads * D threads: a CTA
// merges kReduceHeads heads of one row (a sequence, or one query row of a
// multi-query chunk), thread (i, t) output dim t of head i
// (few CTAs, so that they are resident, waiting, while the partition kernels
// run). Sequences with a single partition were written by the partition
// kernel and are skipped, except in the grouped decode, where this kernel
// writes every row (a row without tokens is zero).
#ifndef KVP_REDUCE_HEADS
#define KVP_REDUCE_HEADS 4
#endif
constexpr int kReduceHeads = KVP_REDUCE_HEADS;

template <typename T, int D>
__global__ void __launch_bounds__(kReduceHeads * D) decode_reduce_kernel(const DecodeArgs a) {
  extern __shared__ float wsh[];  // [kReduceHeads][ws_slots] weights, then [kReduceHeads] sums
  // The context length and the plan words are the call's inputs, not pass 1's
  // outputs: they are read before the wait for pass 1, so only the partials'
  // loads follow it.
  const int h0 = blockIdx.x * kReduceHeads;
  const int row = blockIdx.y;          // a sequence, or one of its q_len query rows
  const int s = row / a.q_len;
  const int i = threadIdx.x / D, t = threadIdx.x % D;
  const int32_t ctx = seq_ctx(a, s, false);
  int32_t nparts;
  if (a.plan && a.plan_packed) {  // packed: one slot per chunk of the sequence's group
    const int32_t gid = a.plan[pack::kHdrWords + s];
    nparts = a.plan[pack::group_offset(a.num_seqs) + int64_t(gid) * pack::kGroupWords + 3];
    if (nparts > a.ws_slots) {
      if (threadIdx.x == 0 && blockIdx.x == 0) record_error(KVP_DEVERR_CTX, uint64_t(s));
      nparts = a.ws_slots;
    }
  } else if (a.plan) {  // grouped: shared-prefix slots, then the sequence's own
    const int32_t shared = a.plan[kPlanSeqWord + s] * (a.part_tokens / a.part_blocks);
    nparts = (shared + a.part_tokens - 1) / a.part_tokens +
             (ctx > shared ? (ctx - shared + a.part_tokens - 1) / a.part_tokens : 0);
    if (nparts > a.ws_slots) {  // a prefix longer than the context: a plan of other tables
      if (threadIdx.x == 0 && blockIdx.x == 0) record_error(KVP_DEVERR_CTX, uint64_t(s));
      nparts = a.ws_slots;
    }
  } else {
    nparts = (ctx + a.part_tokens - 1) / a.part_tokens;
    if (nparts > 1 && a.q_len > 1) {  // query row i of a chunk sees ctx - q_len + i + 1 tokens
      const int32_t vis = min(ctx, max(0, ctx - a.q_len + row % a.q_len + 1));
      nparts = (vis + a.part_tokens - 1) / a.part_tokens;
    }
  }
  // every CTA waits, so that the grid completes only after the partition kernel
  pdl_wait();  // launched programmatically: the partition kernel must be complete
  if (!a.plan && (ctx + a.part_tokens - 1) / a.part_tokens <= 1) return;  // pass 1 wrote the output
  const bool head = h0 + i < a.num_q_heads;
  const int64_t row_sh = int64_t(row) * a.num_q_heads + h0 + i;
  float* lsh = wsh + kReduceHeads * a.ws_slots;
  if (head && t < 32) {  // the weights of head h0 + i, by its first warp: lane p takes
                         // partitions p, p + 32, ... (their loads go out together)
    const float* ml = a.ws_ml + row_sh * a.ws_slots * 2;
    float M = -INFINITY;
    for (int p = t; p < nparts; p += 32) M = fmaxf(M, ml[2 * p]);
    M = warp_max(M);
    float L = 0.f;
    for (int p = t; p < nparts; p += 32) {
      const float w = (ml[2 * p] == -INFINITY || M == -INFINITY) ? 0.f : exp2f(ml[2 * p] - M);
      wsh[i * a.ws_slots + p] = w;
      L += ml[2 * p + 1] * w;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (t == 0) lsh[i] = L;
  }
  __syncthreads();
  if (!head) return;
  const float* acc = a.ws_acc + row_sh * a.ws_slots * D;
  float o = 0.f;
  for (int p = 0; p < nparts; ++p) o = fmaf(acc[int64_t(p) * D + t], wsh[i * a.ws_slots + p], o);
  const float L = lsh[i];
  const float y = L > 0.f ? o / L : 0.f;
  static_cast<uint16_t*>(a.out)[row_sh * D + t] = Elem<T>::from_float(y);
}

}  // namespace dev
}  // namespace kvp
