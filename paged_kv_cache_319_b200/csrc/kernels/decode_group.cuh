// The grouping plan of the grouped decode, built on the GPU: the rule and
// the plan's layout are in group_layout.h (the host planner,
// host/group_plan.cpp, builds the same plan word for word). One CTA sorts
// the batch's (first block id, sequence) keys (bitonic sort in shared memory),
// finds the runs of equal keys and their subgroups with prefix scans, and
// compares the members' block tables, one warp per subgroup.
#pragma once

#include "common.cuh"
#include "group_layout.h"

namespace kvp {
namespace grp {

constexpr int kMaxThreads = 1024;

// Sort length: a power of two >= S (and >= 2).
KVP_HD constexpr int sort_len(int S) {
  int n = 2;
  while (n < S) n <<= 1;
  return n;
}
// at least 8 warps: one warp per subgroup compares block tables
KVP_HD constexpr int plan_threads(int N) {
  return N < 256 ? 256 : (N > kMaxThreads ? kMaxThreads : N);
}
// Shared memory of the plan kernel: sort keys, three scan arrays, per-sequence
// context and subgroup, per-subgroup head position, size and prefix.
KVP_HD constexpr size_t plan_smem_bytes(int S) {
  return size_t(sort_len(S)) * (8 + 3 * 4) + size_t(S) * 2 * 4 + size_t(S / 2 + 1) * 3 * 4;
}

}  // namespace grp

namespace dev {

// One CTA. tables: [S][MB]; lens: [S] (clamped to [0, max_ctx] as the decode
// kernels do); plan: grp::plan_words(S) words.
__global__ void __launch_bounds__(grp::kMaxThreads, 1) group_plan_kernel(
    const int32_t* __restrict__ tables, const int32_t* __restrict__ lens, int32_t S, int32_t MB,
    int32_t max_ctx, int32_t bs, int32_t part_tokens, int32_t mmax, int32_t num_blocks,
    int32_t* __restrict__ plan) {
  constexpr int kEPT = grp::kMaxSeqs / grp::kMaxThreads;  // sort elements per thread, at most
  extern __shared__ __align__(16) uint8_t psm[];
  const int N = grp::sort_len(S);
  uint64_t* key = reinterpret_cast<uint64_t*>(psm);  // (first block id << 32) | sequence
  int32_t* run_lo = reinterpret_cast<int32_t*>(key + N);
  int32_t* run_hi = run_lo + N;
  int32_t* heads = run_hi + N;
  int32_t* ctxs = heads + N;
  int32_t* sub_of = ctxs + S;
  int32_t* sub_head = sub_of + S;
  int32_t* sub_nm = sub_head + (S / 2 + 1);
  int32_t* sub_c = sub_nm + (S / 2 + 1);
  __shared__ int32_t psh_sh, pown_sh, shared_blk_sh, own_blk_sh;

  // the decode kernel launched after this one prepares while this one runs
  pdl_trigger();
  const int tid = threadIdx.x, nt = blockDim.x;
  constexpr uint32_t kNoKey = 0xFFFFFFFFu;
  if (tid == 0) {
    psh_sh = 0;
    pown_sh = 0;
    shared_blk_sh = 0;
    own_blk_sh = 0;
  }
  for (int i = tid; i < N; i += nt) {
    uint64_t k = ~0ull;
    if (i < S) {
      int32_t ctx = __ldg(lens + i);
      ctx = ctx < 0 ? 0 : (ctx > max_ctx ? max_ctx : ctx);
      ctxs[i] = ctx;
      sub_of[i] = -1;
      uint32_t hk = kNoKey;
      if (ctx >= bs) {
        const int32_t id = __ldg(tables + int64_t(i) * MB);
        if (id >= 0 && id < num_blocks) hk = uint32_t(id);
      }
      k = (uint64_t(hk) << 32) | uint32_t(i);
    }
    key[i] = k;
  }
  __syncthreads();

  // ---- bitonic sort of the N keys, ascending
  for (int k = 2; k <= N; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < N; i += nt) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t x = key[i], y = key[ixj];
          if ((x > y) == ((i & k) == 0)) {
            key[i] = y;
            key[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  auto hk_at = [&](int i) { return uint32_t(key[i] >> 32); };

  // ---- bounds of each run of equal keys: prefix max of run starts, suffix
  // min of run ends (Hillis-Steele scans, kEPT elements per thread)
  for (int i = tid; i < N; i += nt) {
    run_lo[i] = (i == 0 || hk_at(i) != hk_at(i - 1)) ? i : 0;
    run_hi[i] = (i == N - 1 || hk_at(i) != hk_at(i + 1)) ? i : N;
  }
  __syncthreads();
  for (int off = 1; off < N; off <<= 1) {
    int32_t lo[kEPT], hi[kEPT];
#pragma unroll
    for (int e = 0; e < kEPT; ++e) {
      const int i = tid + e * nt;
      if (i < N) {
        lo[e] = run_lo[i];
        if (i >= off) lo[e] = max(lo[e], run_lo[i - off]);
        hi[e] = run_hi[i];
        if (i + off < N) hi[e] = min(hi[e], run_hi[i + off]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < kEPT; ++e) {
      const int i = tid + e * nt;
      if (i < N) {
        run_lo[i] = lo[e];
        run_hi[i] = hi[e];
      }
    }
    __syncthreads();
  }

  // ---- subgroup heads (first member of each subgroup of >= 2), numbered in
  // sorted order by an inclusive prefix sum
  auto sub_size = [&](int i) {  // members of the subgroup that sorted position i heads or joins
    const int n = run_hi[i] - run_lo[i] + 1;
    const int first = run_lo[i] + ((i - run_lo[i]) / mmax) * mmax;
    return min(mmax, n - (first - run_lo[i]));
  };
  for (int i = tid; i < N; i += nt) {
    int32_t f = 0;
    if (hk_at(i) != kNoKey && (i - run_lo[i]) % mmax == 0 && sub_size(i) >= 2) f = 1;
    heads[i] = f;
  }
  __syncthreads();
  for (int off = 1; off < N; off <<= 1) {
    int32_t v[kEPT];
#pragma unroll
    for (int e = 0; e < kEPT; ++e) {
      const int i = tid + e * nt;
      if (i < N) v[e] = heads[i] + (i >= off ? heads[i - off] : 0);
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < kEPT; ++e) {
      const int i = tid + e * nt;
      if (i < N) heads[i] = v[e];
    }
    __syncthreads();
  }
  const int32_t n_sub = heads[N - 1];
  int32_t* subs = plan + grp::sub_offset(S);
  for (int i = tid; i < N; i += nt) {
    if (hk_at(i) == kNoKey) continue;
    const int first = run_lo[i] + ((i - run_lo[i]) / mmax) * mmax;
    const int nm = sub_size(i);
    if (nm < 2) continue;
    const int sg = heads[first] - 1;
    const int32_t s = int32_t(uint32_t(key[i]));
    subs[int64_t(sg) * grp::kSubWords + 4 + (i - first)] = s;
    sub_of[s] = sg;
    if (i == first) {
      sub_head[sg] = first;
      sub_nm[sg] = nm;
    }
  }
  __syncthreads();

  // ---- shared prefix of each subgroup: one warp per subgroup compares the
  // members' block-table entries 32 at a time
  const int warp = tid >> 5, lane = tid & 31, nwarps = nt >> 5;
  for (int sg = warp; sg < n_sub; sg += nwarps) {
    const int first = sub_head[sg];
    const int nm = sub_nm[sg];
    int32_t cmax = 0x7FFFFFFF;
    for (int m = 0; m < nm; ++m) cmax = min(cmax, ctxs[uint32_t(key[first + m])] / bs);
    const int64_t row0 = int64_t(uint32_t(key[first])) * MB;
    int32_t c = cmax;
    int64_t rows[grp::kMaxMembers];
#pragma unroll
    for (int m = 0; m < grp::kMaxMembers; ++m)
      rows[m] = m < nm ? int64_t(uint32_t(key[first + m])) * MB : row0;
    for (int32_t base = 0; base < cmax; base += 32) {
      const int32_t j = base + lane;
      bool diff = false;
      if (j < cmax) {
        // all members' entries are loaded before any is compared
        int32_t id[grp::kMaxMembers];
#pragma unroll
        for (int m = 0; m < grp::kMaxMembers; ++m) id[m] = m < nm ? __ldg(tables + rows[m] + j) : 0;
#pragma unroll
        for (int m = 1; m < grp::kMaxMembers; ++m) diff |= m < nm && id[m] != id[0];
      }
      const uint32_t b = __ballot_sync(0xffffffffu, diff);
      if (b) {
        c = base + __ffs(b) - 1;
        break;
      }
    }
    if (lane == 0) {
      sub_c[sg] = c;
      int32_t* e = subs + int64_t(sg) * grp::kSubWords;
      e[0] = c;
      e[1] = nm;
      e[2] = 0;
      e[3] = 0;
      atomicMax(&psh_sh, (c * bs + part_tokens - 1) / part_tokens);
      atomicAdd(&shared_blk_sh, c);
    }
  }
  __syncthreads();
  for (int s = tid; s < S; s += nt) {
    const int32_t c = sub_of[s] >= 0 ? sub_c[sub_of[s]] : 0;
    plan[grp::kHdrWords + s] = c;
    const int32_t own = ctxs[s] - c * bs;  // tokens of the sequence's own range
    if (own > 0) {
      atomicMax(&pown_sh, (own + part_tokens - 1) / part_tokens);
      atomicAdd(&own_blk_sh, (own + bs - 1) / bs);
    }
  }
  __syncthreads();
  if (tid == 0) {
    plan[grp::kNumSub] = n_sub;
    plan[grp::kSharedParts] = psh_sh;
    plan[grp::kOwnParts] = pown_sh;
    plan[grp::kSharedBlocks] = shared_blk_sh;
    plan[grp::kOwnBlocks] = own_blk_sh;
#pragma unroll
    for (int i = 5; i < grp::kHdrWords; ++i) plan[i] = 0;
  }
}

}  // namespace dev
}  // namespace kvp
