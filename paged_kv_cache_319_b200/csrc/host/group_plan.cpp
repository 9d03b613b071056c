// Host planner of the grouped decode: builds, from a batch's host-side block
// tables and context lengths, the grouping plan that the GPU plan kernel would
// build (same rule, same words; the rule and the layout are in
// group_layout.h). A caller that assembles its block tables on the host, as
// the block pool does, passes this plan to paged_attention_decode_grouped and
// saves the GPU the plan kernel; the plan's totals also let the call split the
// GPU between the shared-prefix and per-sequence kernels.

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <vector>

#include "../group_layout.h"
#include "../status.h"

using kvp::fail;

extern "C" {

size_t kvp_decode_group_plan_words(int32_t num_seqs) {
  return num_seqs > 0 ? size_t(kvp::grp::plan_words(num_seqs)) : 0;
}

int kv_decode_group_plan(const int32_t* block_tables, const int32_t* context_lens,
                         int32_t num_seqs, int32_t max_blocks_per_seq, int32_t max_context_len,
                         int32_t block_size, int32_t partition_size, int32_t num_q_heads,
                         int32_t num_kv_heads, int32_t num_blocks, int32_t* plan,
                         size_t plan_words) {
  namespace g = kvp::grp;
  if (num_seqs <= 0 || num_seqs > g::kMaxSeqs || max_blocks_per_seq <= 0 || max_context_len < 0 ||
      block_size <= 0 || partition_size <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
      num_blocks <= 0 || num_q_heads % num_kv_heads)
    return fail(KVP_ERR_INVALID, "kv_decode_group_plan: bad sizes");
  if (partition_size % block_size)
    return fail(KVP_ERR_INVALID, "kv_decode_group_plan: partition_size must be a multiple of block_size");
  if (int64_t(max_context_len) > int64_t(max_blocks_per_seq) * block_size)
    return fail(KVP_ERR_INVALID, "kv_decode_group_plan: max_context_len > max_blocks_per_seq * block_size");
  if (!block_tables || !context_lens || !plan) return fail(KVP_ERR_INVALID, "kv_decode_group_plan: NULL pointer");
  const int64_t S = num_seqs;
  if (plan_words < size_t(g::plan_words(S)))
    return fail(KVP_ERR_INVALID, "kv_decode_group_plan: plan needs %lld words",
                static_cast<long long>(g::plan_words(S)));
  const int mmax = g::members_per_subgroup(num_q_heads / num_kv_heads);
  const int64_t MB = max_blocks_per_seq;
  const int32_t bs = block_size, part = partition_size;
  std::memset(plan, 0, sizeof(int32_t) * size_t(g::plan_words(S)));

  // keys: (first block id << 32) | sequence; sequences that cannot share sort last
  constexpr uint32_t kNoKey = 0xFFFFFFFFu;
  std::vector<int32_t> ctx(static_cast<size_t>(S));
  std::vector<uint64_t> key(static_cast<size_t>(S));
  for (int64_t s = 0; s < S; ++s) {
    int32_t c = context_lens[s];
    c = c < 0 ? 0 : (c > max_context_len ? max_context_len : c);
    ctx[size_t(s)] = c;
    uint32_t hk = kNoKey;
    if (c >= bs) {
      const int32_t id = block_tables[s * MB];
      if (id >= 0 && id < num_blocks) hk = uint32_t(id);
    }
    key[size_t(s)] = (uint64_t(hk) << 32) | uint32_t(s);
  }
  std::sort(key.begin(), key.end());

  int32_t n_sub = 0, shared_parts = 0, shared_blocks = 0;
  int32_t* cblk = plan + g::kHdrWords;
  int32_t* subs = plan + g::sub_offset(S);
  for (int64_t lo = 0; lo < S;) {
    const uint32_t hk = uint32_t(key[size_t(lo)] >> 32);
    int64_t hi = lo + 1;
    while (hi < S && uint32_t(key[size_t(hi)] >> 32) == hk) ++hi;
    if (hk != kNoKey) {
      for (int64_t first = lo; first < hi; first += mmax) {
        const int nm = int(std::min<int64_t>(mmax, hi - first));
        if (nm < 2) continue;
        int32_t* e = subs + int64_t(n_sub) * g::kSubWords;
        int32_t cmax = 0x7FFFFFFF;
        for (int m = 0; m < nm; ++m) {
          const int32_t s = int32_t(uint32_t(key[size_t(first + m)]));
          e[4 + m] = s;
          cmax = std::min(cmax, ctx[size_t(s)] / bs);
        }
        const int32_t* row0 = block_tables + int64_t(e[4]) * MB;
        int32_t c = 0;
        for (; c < cmax; ++c) {
          bool same = true;
          for (int m = 1; m < nm && same; ++m) same = block_tables[int64_t(e[4 + m]) * MB + c] == row0[c];
          if (!same) break;
        }
        e[0] = c;
        e[1] = nm;
        for (int m = 0; m < nm; ++m) cblk[e[4 + m]] = c;
        shared_parts = std::max(shared_parts, (c * bs + part - 1) / part);
        shared_blocks += c;
        ++n_sub;
      }
    }
    lo = hi;
  }
  int32_t own_parts = 0, own_blocks = 0;
  for (int64_t s = 0; s < S; ++s) {
    const int32_t own = ctx[size_t(s)] - cblk[s] * bs;
    if (own > 0) {
      own_parts = std::max(own_parts, (own + part - 1) / part);
      own_blocks += (own + bs - 1) / bs;
    }
  }
  plan[g::kNumSub] = n_sub;
  plan[g::kSharedParts] = shared_parts;
  plan[g::kOwnParts] = own_parts;
  plan[g::kSharedBlocks] = shared_blocks;
  plan[g::kOwnBlocks] = own_blocks;
  return KVP_OK;
}

}  // extern "C"

// ---- packed plan ---------------------------------------------------------------
// The grouping rule above, then one block stream per group (shared prefix,
// then each member's own blocks) cut into chunks; layout in pack_layout.h.

#include "../pack_layout.h"

extern "C" {

size_t kvp_decode_pack_plan_words(int32_t num_seqs, int32_t max_blocks_per_seq) {
  if (num_seqs <= 0 || max_blocks_per_seq <= 0) return 0;
  return size_t(kvp::pack::plan_words_bound(num_seqs, max_blocks_per_seq));
}

int kv_decode_pack_plan(const int32_t* block_tables, const int32_t* context_lens,
                        int32_t num_seqs, int32_t max_blocks_per_seq, int32_t max_context_len,
                        int32_t block_size, int32_t num_q_heads, int32_t num_kv_heads,
                        int32_t num_blocks, int32_t* plan, size_t plan_words) {
  namespace g = kvp::grp;
  namespace pk = kvp::pack;
  if (num_seqs <= 0 || num_seqs > g::kMaxSeqs || max_blocks_per_seq <= 0 || max_context_len < 0 ||
      num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 || num_q_heads % num_kv_heads)
    return fail(KVP_ERR_INVALID, "kv_decode_pack_plan: bad sizes");
  if (block_size != 16 && block_size != 32)
    return fail(KVP_ERR_INVALID, "kv_decode_pack_plan: block_size must be 16 or 32");
  if (int64_t(max_context_len) > int64_t(max_blocks_per_seq) * block_size)
    return fail(KVP_ERR_INVALID, "kv_decode_pack_plan: max_context_len > max_blocks_per_seq * block_size");
  if (!block_tables || !context_lens || !plan) return fail(KVP_ERR_INVALID, "kv_decode_pack_plan: NULL pointer");
  const int64_t S = num_seqs, MB = max_blocks_per_seq;
  if (plan_words < size_t(pk::plan_words_bound(S, MB)))
    return fail(KVP_ERR_INVALID, "kv_decode_pack_plan: plan needs %lld words",
                static_cast<long long>(pk::plan_words_bound(S, MB)));
  const int G = num_q_heads / num_kv_heads;
  const int mmax = g::members_per_subgroup(G);
  if (G > g::kMaxMembers || g::plan_columns(G) < G)
    return fail(KVP_ERR_INVALID, "kv_decode_pack_plan: more than 16 query heads per KV head");
  const int32_t bs = block_size;
  const int32_t bpc = 512 / bs;  // blocks per chunk: the tensor-core kernel's 512-token chunk

  std::vector<int32_t> ctx(static_cast<size_t>(S));
  std::vector<uint64_t> key(static_cast<size_t>(S));
  constexpr uint32_t kNoKey = 0xFFFFFFFFu;
  for (int64_t s = 0; s < S; ++s) {
    int32_t c = context_lens[s];
    c = c < 0 ? 0 : (c > max_context_len ? max_context_len : c);
    ctx[size_t(s)] = c;
    uint32_t hk = kNoKey;
    if (c >= bs) {
      const int32_t id = block_tables[s * MB];
      if (id >= 0 && id < num_blocks) hk = uint32_t(id);
    }
    key[size_t(s)] = (uint64_t(hk) << 32) | uint32_t(s);
  }
  std::sort(key.begin(), key.end());

  // groups: {shared prefix c, members}; subgroups of the rule, then singletons
  struct Grp {
    int32_t c, nm;
    int32_t seq[g::kMaxMembers];
  };
  std::vector<Grp> groups;
  std::vector<char> grouped(static_cast<size_t>(S), 0);
  groups.reserve(size_t(S));
  for (int64_t lo = 0; lo < S;) {
    const uint32_t hk = uint32_t(key[size_t(lo)] >> 32);
    int64_t hi = lo + 1;
    while (hi < S && uint32_t(key[size_t(hi)] >> 32) == hk) ++hi;
    if (hk != kNoKey) {
      for (int64_t first = lo; first < hi; first += mmax) {
        const int nm = int(std::min<int64_t>(mmax, hi - first));
        if (nm < 2) continue;
        Grp gr{};
        gr.nm = nm;
        int32_t cmax = 0x7FFFFFFF;
        for (int m = 0; m < nm; ++m) {
          gr.seq[m] = int32_t(uint32_t(key[size_t(first + m)]));
          cmax = std::min(cmax, ctx[size_t(gr.seq[m])] / bs);
          grouped[size_t(gr.seq[m])] = 1;
        }
        const int32_t* row0 = block_tables + int64_t(gr.seq[0]) * MB;
        int32_t c = 0;
        for (; c < cmax; ++c) {
          bool same = true;
          for (int m = 1; m < nm && same; ++m) same = block_tables[int64_t(gr.seq[m]) * MB + c] == row0[c];
          if (!same) break;
        }
        gr.c = c;
        groups.push_back(gr);
      }
    }
    lo = hi;
  }
  for (int64_t s = 0; s < S; ++s)
    if (!grouped[size_t(s)]) {
      Grp gr{};
      gr.c = 0;
      gr.nm = 1;
      gr.seq[0] = int32_t(s);
      groups.push_back(gr);
    }

  // streams, entries and units
  const int64_t ngr = int64_t(groups.size());
  const int64_t unit_off = pk::group_offset(S) + ngr * pk::kGroupWords;
  std::vector<int32_t> ent;  // (id, mask << 8 | valid) pairs
  struct Unit {
    int32_t group, first, n, chunk;
  };
  std::vector<Unit> units;
  ent.reserve(size_t(2 * S * MB));
  units.reserve(size_t(S * MB));
  std::memset(plan, 0, sizeof(int32_t) * size_t(pk::group_offset(S) + ngr * pk::kGroupWords));
  int32_t max_chunks = 0;
  for (int64_t gi = 0; gi < ngr; ++gi) {
    const Grp& gr = groups[size_t(gi)];
    const int32_t first = int32_t(ent.size() / 2);
    const uint32_t cols_all = gr.nm * G >= 32 ? 0xFFFFFFFFu : ((1u << (gr.nm * G)) - 1u);
    for (int32_t b = 0; b < gr.c; ++b) {  // the shared prefix: full blocks, every member
      ent.push_back(block_tables[int64_t(gr.seq[0]) * MB + b]);
      ent.push_back(int32_t((cols_all << 8) | uint32_t(bs)));
    }
    for (int m = 0; m < gr.nm; ++m) {  // each member's own blocks
      const int32_t s = gr.seq[m];
      const int32_t nblk = (ctx[size_t(s)] + bs - 1) / bs;
      const uint32_t cols = ((1u << G) - 1u) << (m * G);
      for (int32_t b = gr.c; b < nblk; ++b) {
        const int32_t valid = std::min(bs, ctx[size_t(s)] - b * bs);
        ent.push_back(block_tables[int64_t(s) * MB + b]);
        ent.push_back(int32_t((cols << 8) | uint32_t(valid)));
      }
    }
    const int32_t n = int32_t(ent.size() / 2) - first;
    const int32_t chunks = (n + bpc - 1) / bpc;
    max_chunks = std::max(max_chunks, chunks);
    int32_t* e = plan + pk::group_offset(S) + gi * pk::kGroupWords;
    e[0] = first;
    e[1] = gr.nm;
    e[2] = n;
    e[3] = chunks;
    for (int m = 0; m < gr.nm; ++m) {
      e[4 + m] = gr.seq[m];
      plan[pk::kHdrWords + gr.seq[m]] = int32_t(gi);
    }
    for (int32_t ch = 0; ch < chunks; ++ch)
      units.push_back(Unit{int32_t(gi), first + ch * bpc, std::min(bpc, n - ch * bpc), ch});
  }
  // longest units first, so the last to start are short
  std::stable_sort(units.begin(), units.end(), [](const Unit& x, const Unit& y) { return x.n > y.n; });
  const int64_t ent_off = unit_off + int64_t(units.size()) * pk::kUnitWords;
  int32_t* u = plan + unit_off;
  for (const Unit& x : units) {
    u[0] = x.group;
    u[1] = x.first;
    u[2] = x.n;
    u[3] = x.chunk;
    u += pk::kUnitWords;
  }
  std::memcpy(plan + ent_off, ent.data(), sizeof(int32_t) * ent.size());
  plan[pk::kGroups] = int32_t(ngr);
  plan[pk::kUnits] = int32_t(units.size());
  plan[pk::kEntries] = int32_t(ent.size() / 2);
  plan[pk::kMaxChunks] = max_chunks;
  plan[pk::kBlockSize] = bs;
  plan[pk::kChunkBlocks] = bpc;
  plan[pk::kUnitOffset] = int32_t(unit_off);
  plan[pk::kEntryOffset] = int32_t(ent_off);
  return KVP_OK;
}

}  // extern "C"
