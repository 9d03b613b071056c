// Host-side paged KV block pool: free list, per-sequence block tables,
// reference counts, copy-on-write queue.
//
// Method: fixed-size blocks taken only when a sequence grows into them, a
// block table per sequence ["Your GPU was mostly empty", section "The OS
// already solved this in the 1960s"; "vLLM and PagedAttention", section
// "Architecture, step by step", steps 1-2]; sharing by reference count with a
// copy only when a sequence writes into a shared block ["Your GPU was mostly
// empty", section "Paging's second gift: copy-on-write"]; blocks no sequence
// references go back to the shared pool ["PagedAttention: KV cache memory
// management", section "A request lifecycle: allocation, growth, sharing and
// release"].
//
// Policy (the pages leave it open; fixed here so placement is reproducible):
// the free list is a LIFO stack seeded with the caller's order (first pop =
// free_order[0]); release walks a table in logical order and pushes blocks
// that reach zero; copy-on-write fires only on a write into a partly filled
// last block whose count is > 1, and the writer gets the new block.
//
// Every mutating call first checks that it can succeed (block need vs free
// count, ids), then mutates, so a failed call changes nothing.
//
// Prefix caching across requests (off unless kv_pool_set_prefix_caching turns
// it on): full blocks keep the keys and values of a token prefix that a later
// request with the same prefix reuses ["PagedAttention: KV cache memory
// management", section "PagedAttention vs KV-cache quantization vs prefix
// caching"; sharing across requests: "vLLM and PagedAttention", section "Key
// claims from the paper"]. Policy: a block that fills during
// kv_seq_append_tokens is registered under the key (registration number of
// the block before it, or -1; its token ids), unless the key is taken, the
// block is registered or the block before it is not; registration numbers
// are never reused, so a key names one exact token prefix. kv_seq_create_prefixed
// attaches the longest run of leading registered blocks that ends before the
// prompt's last token. A registered block whose count reaches zero becomes
// evictable (the blocks of one release from the last logical one to the
// first) instead of free; a new block comes from the free stack, else from
// evicting the evictable block released longest ago.

#include <cstdint>
#include <cstring>
#include <iterator>
#include <list>
#include <new>
#include <unordered_map>
#include <utility>
#include <vector>

#include "../status.h"

// Room for `extra` more elements, growing the capacity at least twofold, so a
// vector that gains a few elements per call is not copied on every call.
template <typename V>
static void reserve_more(V& v, size_t extra) {
  const size_t want = v.size() + extra;
  if (v.capacity() < want) v.reserve(want > 2 * v.capacity() ? want : 2 * v.capacity());
}

struct kvp_pool {
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  int32_t num_kv_heads = 0;
  int32_t head_dim = 0;
  int32_t dtype = 0;
  std::vector<int32_t> free_stack;  // back() is the next block handed out
  std::vector<int32_t> rc;
  struct Seq {
    std::vector<int32_t> table;
    int32_t len = 0;
    // prefix caching: the token ids appended so far, while every append gave them
    std::vector<int32_t> tokens;
    bool tracked = true;
    uint64_t batch_mark = 0;  // epoch of the last batch append that listed this sequence
  };
  std::unordered_map<int64_t, Seq> seqs;
  std::vector<std::pair<int32_t, int32_t>> pending;  // (src, dst) copy-on-write pairs
  int64_t next_seq = 0;
  int64_t cow_total = 0;
  // batch appends: an epoch per call (duplicates found in one pass), per block
  // the reference count left after the batch's earlier copies (-1: untouched),
  // and the blocks whose entry a call set, so it can put them back
  uint64_t batch_epoch = 0;
  std::vector<int32_t> rc_seen;
  std::vector<int32_t> rc_touched;
  std::vector<Seq*> batch_ptrs;

  // ---- prefix caching
  struct KeyHash {
    size_t operator()(const std::vector<int64_t>& k) const noexcept {
      uint64_t h = 1469598103934665603ull;  // FNV-1a over the words
      for (int64_t w : k) {
        h ^= uint64_t(w);
        h *= 1099511628211ull;
      }
      return size_t(h);
    }
  };
  bool prefix_caching = false;
  std::unordered_map<std::vector<int64_t>, int32_t, KeyHash> block_of;  // key -> block
  std::vector<std::vector<int64_t>> key_of;   // per block: its key, empty if unregistered
  std::vector<int64_t> reg_of;                // per block: registration number, -1 if none
  int64_t next_reg = 0;
  std::list<int32_t> evictable;               // front: evicted next
  std::vector<std::list<int32_t>::iterator> evict_pos;
  std::vector<char> in_evict;
  int64_t hit_tokens = 0;

  int64_t available() const { return int64_t(free_stack.size()) + int64_t(evictable.size()); }

  // A block for a new table entry: the free stack first, else the evictable
  // block released longest ago (its key dropped).
  int32_t take_block() {
    if (!free_stack.empty()) {
      const int32_t b = free_stack.back();
      free_stack.pop_back();
      return b;
    }
    const int32_t b = evictable.front();
    evictable.pop_front();
    in_evict[b] = 0;
    block_of.erase(key_of[b]);
    key_of[b].clear();
    key_of[b].shrink_to_fit();
    reg_of[b] = -1;
    return b;
  }

  // Block bi of s has just filled: register it (policy above). Registration is
  // a cache, so a host allocation failure here only skips it.
  void maybe_register(const Seq& s, int32_t bi) {
    const int32_t blk = s.table[bi];
    if (reg_of[blk] >= 0) return;
    const int64_t parent = bi == 0 ? -1 : reg_of[s.table[bi - 1]];
    if (bi > 0 && parent < 0) return;
    try {
      std::vector<int64_t> key;
      key.reserve(size_t(block_size) + 1);
      key.push_back(parent);
      for (int32_t i = 0; i < block_size; ++i) key.push_back(s.tokens[size_t(bi) * block_size + i]);
      if (block_of.count(key)) return;
      key_of[blk] = key;
      block_of.emplace(std::move(key), blk);
      reg_of[blk] = next_reg++;
    } catch (...) {
      key_of[blk].clear();
    }
  }

  // Drops one reference of each block of a released table (logical order);
  // blocks reaching zero go to the free stack, or become evictable if
  // registered. Everything that allocates happens first (it may throw), then
  // the pool changes without allocating.
  void drop_table(const std::vector<int32_t>& table) {
    std::list<int32_t> newly;  // the blocks to become evictable, last logical block first
    for (int32_t b : table)
      if (rc[b] == 1 && prefix_caching && reg_of[b] >= 0) newly.push_front(b);
    free_stack.reserve(free_stack.size() + table.size());
    for (int32_t b : table) {
      if (--rc[b] != 0) continue;
      if (!(prefix_caching && reg_of[b] >= 0)) free_stack.push_back(b);
    }
    if (newly.empty()) return;
    for (int32_t b : newly) in_evict[b] = 1;
    auto first = newly.begin();  // stays valid: splice moves the nodes
    evictable.splice(evictable.end(), newly);
    for (auto it = first; it != evictable.end(); ++it) evict_pos[*it] = it;
  }

  Seq* find(int64_t id) {
    auto it = seqs.find(id);
    return it == seqs.end() ? nullptr : &it->second;
  }
  const Seq* find(int64_t id) const {
    auto it = seqs.find(id);
    return it == seqs.end() ? nullptr : &it->second;
  }

  static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

  // Blocks an append of n tokens to s takes, given the last block's count.
  int64_t need_for(const Seq& s, int32_t n, int32_t last_rc) const {
    int64_t need = ceil_div(int64_t(s.len) + n, block_size) - ceil_div(s.len, block_size);
    if (n > 0 && s.len % block_size != 0 && last_rc > 1) need += 1;
    return need;
  }

  // Appends n tokens (their ids, or null if unknown); the caller has checked
  // that free and evictable blocks suffice and reserved s.tokens when given.
  void append_unchecked(Seq& s, int32_t n, int64_t* slots, const int32_t* ids = nullptr) {
    const bool track = prefix_caching && s.tracked && ids;
    if (prefix_caching && !ids) {  // later tokens unknown: no more registrations
      s.tracked = false;
      s.tokens.clear();
    }
    for (int32_t i = 0; i < n; ++i) {
      const int32_t pos = s.len;
      if (pos % block_size == 0) {
        const int32_t b = take_block();
        rc[b] = 1;
        s.table.push_back(b);
      } else if (rc[s.table.back()] > 1) {
        const int32_t src = s.table.back();
        const int32_t dst = take_block();
        pending.emplace_back(src, dst);
        ++cow_total;
        rc[src] -= 1;
        rc[dst] = 1;
        s.table.back() = dst;
      }
      slots[i] = int64_t(s.table[pos / block_size]) * block_size + pos % block_size;
      s.len = pos + 1;
      if (track) {
        s.tokens.push_back(ids[i]);
        if (s.len % block_size == 0) maybe_register(s, pos / block_size);
      }
    }
  }
};

namespace kvp {
std::string& last_error() {
  static thread_local std::string msg;
  return msg;
}
}  // namespace kvp

using kvp::fail;

extern "C" {

const char* kvp_last_error_message(void) { return kvp::last_error().c_str(); }

const char* kvp_version(void) { return "libkvp 0.1.0 (sm_100a)"; }

int64_t kvp_kv_bytes_per_token(int64_t hidden, int64_t layers, int64_t elem_bytes) {
  return 2 * hidden * layers * elem_bytes;
}

int kv_pool_create(int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                   int32_t head_dim, int32_t dtype, const int32_t* free_order, kvp_pool** out) {
  if (!out) return fail(KVP_ERR_INVALID, "kv_pool_create: out is NULL");
  if (num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return fail(KVP_ERR_INVALID, "kv_pool_create: sizes must be positive");
  if (dtype != KVP_F16 && dtype != KVP_BF16 && dtype != KVP_FP8_E4M3)
    return fail(KVP_ERR_INVALID, "kv_pool_create: dtype must be KVP_F16, KVP_BF16 or KVP_FP8_E4M3");
  if (int64_t(num_blocks) * block_size > (int64_t(1) << 40))
    return fail(KVP_ERR_INVALID, "kv_pool_create: pool too large");
  kvp_pool* p = new (std::nothrow) kvp_pool();
  if (!p) return fail(KVP_ERR_OOM, "kv_pool_create: host allocation failed");
  try {
    p->num_blocks = num_blocks;
    p->block_size = block_size;
    p->num_kv_heads = num_kv_heads;
    p->head_dim = head_dim;
    p->dtype = dtype;
    p->rc.assign(num_blocks, 0);
    p->rc_seen.assign(num_blocks, -1);
    p->free_stack.resize(num_blocks);
    p->key_of.resize(num_blocks);
    p->reg_of.assign(num_blocks, -1);
    p->evict_pos.resize(num_blocks);
    p->in_evict.assign(num_blocks, 0);
    if (free_order) {
      std::vector<char> seen(num_blocks, 0);
      for (int32_t i = 0; i < num_blocks; ++i) {
        const int32_t b = free_order[i];
        if (b < 0 || b >= num_blocks || seen[b]) {
          delete p;
          return fail(KVP_ERR_INVALID, "kv_pool_create: free_order is not a permutation");
        }
        seen[b] = 1;
      }
    }
    for (int32_t i = 0; i < num_blocks; ++i)
      p->free_stack[num_blocks - 1 - i] = free_order ? free_order[i] : i;
  } catch (...) {
    delete p;
    return fail(KVP_ERR_OOM, "kv_pool_create: host allocation failed");
  }
  *out = p;
  return KVP_OK;
}

int kv_pool_destroy(kvp_pool* pool) {
  delete pool;
  return KVP_OK;
}

int kv_pool_num_free(const kvp_pool* pool, int32_t* n) {
  if (!pool || !n) return fail(KVP_ERR_INVALID, "kv_pool_num_free: NULL argument");
  *n = int32_t(pool->free_stack.size());
  return KVP_OK;
}

int kv_pool_free_list(const kvp_pool* pool, int32_t* out, int32_t cap, int32_t* n) {
  if (!pool || !n) return fail(KVP_ERR_INVALID, "kv_pool_free_list: NULL argument");
  const int32_t cnt = int32_t(pool->free_stack.size());
  *n = cnt;
  if (cap < cnt || (cnt && !out)) return fail(KVP_ERR_CAPACITY, "kv_pool_free_list: cap %d < %d", cap, cnt);
  for (int32_t i = 0; i < cnt; ++i) out[i] = pool->free_stack[cnt - 1 - i];
  return KVP_OK;
}

int kv_pool_refcount(const kvp_pool* pool, int32_t block, int32_t* rc) {
  if (!pool || !rc) return fail(KVP_ERR_INVALID, "kv_pool_refcount: NULL argument");
  if (block < 0 || block >= pool->num_blocks)
    return fail(KVP_ERR_INVALID, "kv_pool_refcount: block %d out of range", block);
  *rc = pool->rc[block];
  return KVP_OK;
}

int kv_pool_refcounts(const kvp_pool* pool, int32_t* out, int32_t cap) {
  if (!pool || !out) return fail(KVP_ERR_INVALID, "kv_pool_refcounts: NULL argument");
  if (cap < pool->num_blocks) return fail(KVP_ERR_CAPACITY, "kv_pool_refcounts: cap too small");
  std::memcpy(out, pool->rc.data(), sizeof(int32_t) * pool->num_blocks);
  return KVP_OK;
}

int kv_pool_stats(const kvp_pool* pool, kvp_pool_stats* out) {
  if (!pool || !out) return fail(KVP_ERR_INVALID, "kv_pool_stats: NULL argument");
  kvp_pool_stats s{};
  s.num_blocks = pool->num_blocks;
  s.num_free = int64_t(pool->free_stack.size());
  for (int32_t c : pool->rc) {
    s.num_used += c > 0;
    s.num_shared += c > 1;
  }
  for (const auto& kv : pool->seqs)
    s.waste_slots += int64_t(kv.second.table.size()) * pool->block_size - kv.second.len;
  s.cow_copies_total = pool->cow_total;
  s.num_seqs = int64_t(pool->seqs.size());
  *out = s;
  return KVP_OK;
}

int kv_seq_create(kvp_pool* pool, int64_t* seq_id) {
  if (!pool || !seq_id) return fail(KVP_ERR_INVALID, "kv_seq_create: NULL argument");
  try {
    pool->seqs.emplace(pool->next_seq, kvp_pool::Seq{});
  } catch (...) {
    return fail(KVP_ERR_OOM, "kv_seq_create: host allocation failed");
  }
  *seq_id = pool->next_seq++;
  return KVP_OK;
}

int kv_seq_append(kvp_pool* pool, int64_t seq, int32_t n_tokens, int64_t* slots_out) {
  if (!pool) return fail(KVP_ERR_INVALID, "kv_seq_append: NULL pool");
  kvp_pool::Seq* s = pool->find(seq);
  if (!s) return fail(KVP_ERR_NO_SEQ, "kv_seq_append: no live sequence %lld", (long long)seq);
  if (n_tokens < 0) return fail(KVP_ERR_INVALID, "kv_seq_append: n_tokens < 0");
  if (n_tokens > 0 && !slots_out) return fail(KVP_ERR_INVALID, "kv_seq_append: slots_out is NULL");
  if (int64_t(s->len) + n_tokens > INT32_MAX) return fail(KVP_ERR_INVALID, "kv_seq_append: length overflow");
  const int32_t last_rc = s->table.empty() ? 0 : pool->rc[s->table.back()];
  const int64_t need = pool->need_for(*s, n_tokens, last_rc);
  if (need > pool->available())
    return fail(KVP_ERR_OOM, "kv_seq_append: need %lld blocks, %lld free or evictable",
                (long long)need, (long long)pool->available());
  try {
    reserve_more(s->table, size_t(need));
    reserve_more(pool->pending, 1);
  } catch (...) {
    return fail(KVP_ERR_OOM, "kv_seq_append: host allocation failed");
  }
  pool->append_unchecked(*s, n_tokens, slots_out);
  return KVP_OK;
}

int kv_seq_append_tokens(kvp_pool* pool, int64_t seq, const int32_t* tokens, int32_t n_tokens,
                         int64_t* slots_out) {
  if (!pool) return fail(KVP_ERR_INVALID, "kv_seq_append_tokens: NULL pool");
  kvp_pool::Seq* s = pool->find(seq);
  if (!s) return fail(KVP_ERR_NO_SEQ, "kv_seq_append_tokens: no live sequence %lld", (long long)seq);
  if (n_tokens < 0) return fail(KVP_ERR_INVALID, "kv_seq_append_tokens: n_tokens < 0");
  if (n_tokens > 0 && (!slots_out || !tokens))
    return fail(KVP_ERR_INVALID, "kv_seq_append_tokens: NULL argument");
  if (int64_t(s->len) + n_tokens > INT32_MAX)
    return fail(KVP_ERR_INVALID, "kv_seq_append_tokens: length overflow");
  const int32_t last_rc = s->table.empty() ? 0 : pool->rc[s->table.back()];
  const int64_t need = pool->need_for(*s, n_tokens, last_rc);
  if (need > pool->available())
    return fail(KVP_ERR_OOM, "kv_seq_append_tokens: need %lld blocks, %lld free or evictable",
                (long long)need, (long long)pool->available());
  try {
    reserve_more(s->table, size_t(need));
    reserve_more(pool->pending, 1);
    if (pool->prefix_caching && s->tracked) reserve_more(s->tokens, size_t(n_tokens));
  } catch (...) {
    return fail(KVP_ERR_OOM, "kv_seq_append_tokens: host allocation failed");
  }
  static const int32_t kNone = 0;
  pool->append_unchecked(*s, n_tokens, slots_out, tokens ? tokens : &kNone);
  return KVP_OK;
}

int kv_pool_set_prefix_caching(kvp_pool* pool, int32_t enable) {
  if (!pool) return fail(KVP_ERR_INVALID, "kv_pool_set_prefix_caching: NULL pool");
  if (enable) {
    if (!pool->prefix_caching && !pool->seqs.empty())
      return fail(KVP_ERR_INVALID, "kv_pool_set_prefix_caching: turn it on while no sequence is live");
    pool->prefix_caching = true;
    return KVP_OK;
  }
  // off: every registration is dropped; evictable blocks become free (front first)
  try {
    pool->free_stack.reserve(pool->free_stack.size() + pool->evictable.size());
  } catch (...) {
    return fail(KVP_ERR_OOM, "kv_pool_set_prefix_caching: host allocation failed");
  }
  for (int32_t b : pool->evictable) {
    pool->free_stack.push_back(b);
    pool->in_evict[b] = 0;
  }
  pool->evictable.clear();
  pool->block_of.clear();
  for (int32_t b = 0; b < pool->num_blocks; ++b) {
    pool->key_of[b].clear();
    pool->reg_of[b] = -1;
  }
  for (auto& kv : pool->seqs) {
    kv.second.tracked = false;
    kv.second.tokens.clear();
  }
  pool->prefix_caching = false;
  return KVP_OK;
}

int kv_seq_create_prefixed(kvp_pool* pool, const int32_t* tokens, int32_t n_tokens, int64_t* seq_id,
                           int32_t* cached_tokens) {
  if (!pool || !seq_id || !cached_tokens)
    return fail(KVP_ERR_INVALID, "kv_seq_create_prefixed: NULL argument");
  if (n_tokens < 0 || (n_tokens > 0 && !tokens))
    return fail(KVP_ERR_INVALID, "kv_seq_create_prefixed: bad tokens");
  if (!pool->prefix_caching) return fail(KVP_ERR_INVALID, "kv_seq_create_prefixed: prefix caching is off");
  const int32_t bs = pool->block_size;
  kvp_pool::Seq s;
  try {
    std::vector<int64_t> key(size_t(bs) + 1);
    int64_t parent = -1;
    for (int32_t i = 0; int64_t(i + 1) * bs <= int64_t(n_tokens) - 1; ++i) {
      key[0] = parent;
      for (int32_t j = 0; j < bs; ++j) key[size_t(j) + 1] = tokens[int64_t(i) * bs + j];
      auto it = pool->block_of.find(key);
      if (it == pool->block_of.end()) break;
      s.table.push_back(it->second);
      parent = pool->reg_of[it->second];
    }
    s.len = int32_t(s.table.size()) * bs;
    s.tokens.assign(tokens, tokens + s.len);
    pool->seqs.emplace(pool->next_seq, std::move(s));
  } catch (...) {
    return fail(KVP_ERR_OOM, "kv_seq_create_prefixed: host allocation failed");
  }
  const kvp_pool::Seq& made = pool->seqs[pool->next_seq];
  for (int32_t b : made.table) {
    if (pool->rc[b] == 0 && pool->in_evict[b]) {
      pool->evictable.erase(pool->evict_pos[b]);
      pool->in_evict[b] = 0;
    }
    pool->rc[b] += 1;
  }
  pool->hit_tokens += made.len;
  *cached_tokens = made.len;
  *seq_id = pool->next_seq++;
  return KVP_OK;
}

int kv_pool_evictable_list(const kvp_pool* pool, int32_t* out, int32_t cap, int32_t* n) {
  if (!pool || !n) return fail(KVP_ERR_INVALID, "kv_pool_evictable_list: NULL argument");
  const int32_t cnt = int32_t(pool->evictable.size());
  *n = cnt;
  if (cap < cnt || (cnt && !out))
    return fail(KVP_ERR_CAPACITY, "kv_pool_evictable_list: cap %d < %d", cap, cnt);
  int32_t i = 0;
  for (int32_t b : pool->evictable) out[i++] = b;
  return KVP_OK;
}

int kv_pool_prefix_stats(const kvp_pool* pool, int64_t* registered, int64_t* evictable,
                         int64_t* hit_tokens) {
  if (!pool || !registered || !evictable || !hit_tokens)
    return fail(KVP_ERR_INVALID, "kv_pool_prefix_stats: NULL argument");
  *registered = int64_t(pool->block_of.size());
  *evictable = int64_t(pool->evictable.size());
  *hit_tokens = pool->hit_tokens;
  return KVP_OK;
}

// kv_seq_append_batch and kv_seq_append_tokens_batch: one check of the whole
// batch's block need, then the appends in order (ids: null, or n_each token
// ids per sequence).
static int append_batch_impl(kvp_pool* pool, const int64_t* seqs, int32_t num_seqs, int32_t n_each,
                             const int32_t* ids, int64_t* slots_out, const char* who) {
  if (!pool) return fail(KVP_ERR_INVALID, "%s: NULL pool", who);
  if (num_seqs < 0 || n_each < 0) return fail(KVP_ERR_INVALID, "%s: negative size", who);
  if (num_seqs == 0 || n_each == 0) return KVP_OK;
  if (!seqs || !slots_out) return fail(KVP_ERR_INVALID, "%s: NULL argument", who);
  // Exact block need of the whole batch: a copy-on-write by an earlier
  // sequence lowers the count a later sharer of the same last block sees.
  // Linear in the batch: sequences are marked with this call's epoch, and the
  // lowered counts live in the pool's per-block scratch, reset on every exit.
  try {
    reserve_more(pool->batch_ptrs, size_t(num_seqs));
    reserve_more(pool->rc_touched, size_t(num_seqs));
  } catch (...) {
    return fail(KVP_ERR_OOM, "%s: host allocation failed", who);
  }
  pool->batch_ptrs.clear();
  pool->rc_touched.clear();
  struct Restore {
    kvp_pool* p;
    ~Restore() {
      for (int32_t b : p->rc_touched) p->rc_seen[b] = -1;
      p->rc_touched.clear();
    }
  } restore{pool};
  const uint64_t epoch = ++pool->batch_epoch;
  int64_t need = 0;
  for (int32_t i = 0; i < num_seqs; ++i) {
    kvp_pool::Seq* s = pool->find(seqs[i]);
    if (!s) return fail(KVP_ERR_NO_SEQ, "%s: no live sequence %lld", who, (long long)seqs[i]);
    if (s->batch_mark == epoch) return fail(KVP_ERR_INVALID, "%s: duplicate sequence", who);
    s->batch_mark = epoch;
    pool->batch_ptrs.push_back(s);
    if (int64_t(s->len) + n_each > INT32_MAX) return fail(KVP_ERR_INVALID, "%s: overflow", who);
    int32_t last_rc = 0;
    if (!s->table.empty()) {
      const int32_t last = s->table.back();
      const int32_t seen = pool->rc_seen[last];
      last_rc = seen >= 0 ? seen : pool->rc[last];
      if (s->len % pool->block_size != 0 && last_rc > 1) {
        if (seen < 0) pool->rc_touched.push_back(last);
        pool->rc_seen[last] = last_rc - 1;
      }
    }
    need += pool->need_for(*s, n_each, last_rc);
  }
  if (need > pool->available())
    return fail(KVP_ERR_OOM, "%s: need %lld blocks, %lld free or evictable", who, (long long)need,
                (long long)pool->available());
  std::vector<kvp_pool::Seq*>& ptrs = pool->batch_ptrs;
  try {
    for (int32_t i = 0; i < num_seqs; ++i) {
      reserve_more(ptrs[i]->table, size_t(n_each / pool->block_size + 2));
      if (ids && pool->prefix_caching && ptrs[i]->tracked) reserve_more(ptrs[i]->tokens, size_t(n_each));
    }
    reserve_more(pool->pending, size_t(num_seqs));
  } catch (...) {
    return fail(KVP_ERR_OOM, "%s: host allocation failed", who);
  }
  for (int32_t i = 0; i < num_seqs; ++i)
    pool->append_unchecked(*ptrs[i], n_each, slots_out + int64_t(i) * n_each,
                           ids ? ids + int64_t(i) * n_each : nullptr);
  return KVP_OK;
}

int kv_seq_append_batch(kvp_pool* pool, const int64_t* seqs, int32_t num_seqs, int32_t n_each,
                        int64_t* slots_out) {
  return append_batch_impl(pool, seqs, num_seqs, n_each, nullptr, slots_out, "kv_seq_append_batch");
}

int kv_seq_append_tokens_batch(kvp_pool* pool, const int64_t* seqs, int32_t num_seqs,
                               int32_t n_each, const int32_t* tokens, int64_t* slots_out) {
  if (num_seqs > 0 && n_each > 0 && !tokens)
    return fail(KVP_ERR_INVALID, "kv_seq_append_tokens_batch: NULL tokens");
  return append_batch_impl(pool, seqs, num_seqs, n_each, tokens, slots_out,
                           "kv_seq_append_tokens_batch");
}

int kv_seq_fork(kvp_pool* pool, int64_t parent, int64_t* child) {
  if (!pool || !child) return fail(KVP_ERR_INVALID, "kv_seq_fork: NULL argument");
  const kvp_pool::Seq* p = pool->find(parent);
  if (!p) return fail(KVP_ERR_NO_SEQ, "kv_seq_fork: no live sequence %lld", (long long)parent);
  try {
    kvp_pool::Seq c = *p;
    pool->seqs.emplace(pool->next_seq, std::move(c));
  } catch (...) {
    return fail(KVP_ERR_OOM, "kv_seq_fork: host allocation failed");
  }
  for (int32_t b : pool->seqs[pool->next_seq].table) pool->rc[b] += 1;
  *child = pool->next_seq++;
  return KVP_OK;
}

int kv_seq_release(kvp_pool* pool, int64_t seq) {
  if (!pool) return fail(KVP_ERR_INVALID, "kv_seq_release: NULL pool");
  auto it = pool->seqs.find(seq);
  if (it == pool->seqs.end()) return fail(KVP_ERR_NO_SEQ, "kv_seq_release: no live sequence %lld", (long long)seq);
  try {
    pool->drop_table(it->second.table);
  } catch (...) {
    return fail(KVP_ERR_OOM, "kv_seq_release: host allocation failed");
  }
  pool->seqs.erase(it);
  return KVP_OK;
}

int kv_seq_len(const kvp_pool* pool, int64_t seq, int32_t* len) {
  if (!pool || !len) return fail(KVP_ERR_INVALID, "kv_seq_len: NULL argument");
  const kvp_pool::Seq* s = pool->find(seq);
  if (!s) return fail(KVP_ERR_NO_SEQ, "kv_seq_len: no live sequence %lld", (long long)seq);
  *len = s->len;
  return KVP_OK;
}

int kv_seq_block_table(const kvp_pool* pool, int64_t seq, int32_t* out, int32_t cap, int32_t* n) {
  if (!pool || !n) return fail(KVP_ERR_INVALID, "kv_seq_block_table: NULL argument");
  const kvp_pool::Seq* s = pool->find(seq);
  if (!s) return fail(KVP_ERR_NO_SEQ, "kv_seq_block_table: no live sequence %lld", (long long)seq);
  const int32_t cnt = int32_t(s->table.size());
  *n = cnt;
  if (cap < cnt || (cnt && !out)) return fail(KVP_ERR_CAPACITY, "kv_seq_block_table: cap %d < %d", cap, cnt);
  if (cnt) std::memcpy(out, s->table.data(), sizeof(int32_t) * cnt);
  return KVP_OK;
}

static int copy_pairs_out(const kvp_pool* pool, int32_t* pairs, int32_t cap, int32_t* n,
                          const char* who) {
  if (!pool || !n) return fail(KVP_ERR_INVALID, "%s: NULL argument", who);
  const int32_t cnt = int32_t(pool->pending.size());
  *n = cnt;
  if (cap < cnt || (cnt && !pairs)) return fail(KVP_ERR_CAPACITY, "%s: cap %d < %d", who, cap, cnt);
  for (int32_t i = 0; i < cnt; ++i) {
    pairs[2 * i] = pool->pending[i].first;
    pairs[2 * i + 1] = pool->pending[i].second;
  }
  return KVP_OK;
}

int kv_pool_take_copies(kvp_pool* pool, int32_t* pairs, int32_t cap, int32_t* n) {
  const int rc = copy_pairs_out(pool, pairs, cap, n, "kv_pool_take_copies");
  if (rc == KVP_OK) pool->pending.clear();
  return rc;
}

int kv_pool_pending_copies(const kvp_pool* pool, int32_t* pairs, int32_t cap, int32_t* n) {
  return copy_pairs_out(pool, pairs, cap, n, "kv_pool_pending_copies");
}

int kv_build_batch(const kvp_pool* pool, const int64_t* seqs, int32_t num_seqs, int32_t max_blocks,
                   int32_t* block_tables, int32_t* context_lens) {
  if (!pool) return fail(KVP_ERR_INVALID, "kv_build_batch: NULL pool");
  if (num_seqs < 0 || max_blocks < 0) return fail(KVP_ERR_INVALID, "kv_build_batch: negative size");
  if (num_seqs == 0) return KVP_OK;
  if (!seqs || !context_lens || (max_blocks && !block_tables))
    return fail(KVP_ERR_INVALID, "kv_build_batch: NULL argument");
  for (int32_t i = 0; i < num_seqs; ++i) {
    const kvp_pool::Seq* s = pool->find(seqs[i]);
    if (!s) return fail(KVP_ERR_NO_SEQ, "kv_build_batch: no live sequence %lld", (long long)seqs[i]);
    if (int32_t(s->table.size()) > max_blocks)
      return fail(KVP_ERR_CAPACITY, "kv_build_batch: table of %lld has %zu > %d blocks",
                  (long long)seqs[i], s->table.size(), max_blocks);
  }
  for (int32_t i = 0; i < num_seqs; ++i) {
    const kvp_pool::Seq* s = pool->find(seqs[i]);
    int32_t* row = block_tables + int64_t(i) * max_blocks;
    const int32_t cnt = int32_t(s->table.size());
    if (cnt) std::memcpy(row, s->table.data(), sizeof(int32_t) * cnt);
    for (int32_t j = cnt; j < max_blocks; ++j) row[j] = -1;
    context_lens[i] = s->len;
  }
  return KVP_OK;
}

}  // extern "C"
