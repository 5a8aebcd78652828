// Host block allocator of libpkv.
//
// Bookkeeping from "PagedAttention：让 KV cache 按需生长" (hs-black.github.io):
//   per request a block table, a written length and a state; per physical block
//   a refcount (live requests holding it, not tokens); a free queue; optionally
//   a cached set of released full blocks (section
//   "引用计数管理“谁还在读”，长度管理“哪里能写”").  Allocation happens before any
//   visible change and fails without touching the old mapping (section
//   "先确保分配成功，再改变可见状态"); capacity is checked per request before a step
//   publishes its tables (section "三个空闲块，四个请求同时跨边界"); a release drops
//   one reference per block and returns blocks that reach zero (section
//   "请求结束，块就能交给下一位"); active + cached + free == pool always holds
//   (section "占用率只有 70%，为什么请求还是进不来？").
//
// Readings where the page is silent: the free queue is FIFO (allocate from the
// head, release to the tail in logical block order); requests of one append are
// served in the given order, each all or nothing; a sharer that sees
// refcount > 1 copies the valid n % B slots, the last holder writes in place;
// the cached set (off by default) holds released full blocks oldest first and
// is evicted only when the free queue is empty.
//
// Storage: a ring buffer of capacity num_blocks for the free queue, another
// for the cached set (a block is in at most one of them), a refcount array and
// a hash map from request id to its table.  Every operation costs O(blocks it
// touches); nothing here touches the device.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "../../include/pkv.h"

namespace {

struct Ring {
  std::vector<int32_t> buf;
  int64_t head = 0;  // index of the oldest element
  int64_t size = 0;
  void init(int64_t cap) { buf.assign(static_cast<size_t>(std::max<int64_t>(cap, 1)), -1); }
  int64_t cap() const { return static_cast<int64_t>(buf.size()); }
  void push_back(int32_t b) {
    buf[static_cast<size_t>((head + size) % cap())] = b;
    ++size;
  }
  int32_t pop_front() {
    int32_t b = buf[static_cast<size_t>(head)];
    head = (head + 1) % cap();
    --size;
    return b;
  }
  int32_t at(int64_t i) const { return buf[static_cast<size_t>((head + i) % cap())]; }
};

// Cached set: blocks in release order (oldest first) with O(1) removal of
// any member, as a prefix hit takes a block from the middle.
struct LinkedSet {
  std::vector<int32_t> prev, next;
  int32_t head = -1, tail = -1;
  int64_t size = 0;
  void init(int64_t n) {
    prev.assign(static_cast<size_t>(n), -1);
    next.assign(static_cast<size_t>(n), -1);
  }
  void push_back(int32_t b) {
    prev[static_cast<size_t>(b)] = tail;
    next[static_cast<size_t>(b)] = -1;
    if (tail >= 0) next[static_cast<size_t>(tail)] = b; else head = b;
    tail = b;
    ++size;
  }
  void remove(int32_t b) {
    const int32_t p = prev[static_cast<size_t>(b)], n = next[static_cast<size_t>(b)];
    if (p >= 0) next[static_cast<size_t>(p)] = n; else head = n;
    if (n >= 0) prev[static_cast<size_t>(n)] = p; else tail = p;
    prev[static_cast<size_t>(b)] = next[static_cast<size_t>(b)] = -1;
    --size;
  }
  int32_t pop_front() {
    const int32_t b = head;
    remove(b);
    return b;
  }
};

struct Seq {
  std::vector<int32_t> table;
  int32_t length = 0;
};

}  // namespace

struct pkv_alloc {
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  bool cache = false;
  Ring free_q;
  LinkedSet cached;
  std::vector<int32_t> ref;
  std::vector<char> in_cached;       // block is a member of the cached set
  std::vector<uint64_t> key_of;      // content key of a keyed block
  std::vector<char> has_key;
  std::unordered_map<uint64_t, int32_t> block_of;
  std::unordered_map<int32_t, Seq> seqs;
  int64_t active = 0;  // blocks with refcount > 0
  pkv_stats ctr{};
  int32_t fault_alloc_fail = 0;
  int32_t fault_skip_release = 0;

  int64_t available() const { return free_q.size + (cache ? cached.size : 0); }

  // A fault-injected allocation failure looks exactly like an empty pool.
  bool can_take(int64_t n) {
    if (fault_alloc_fail > 0) return false;
    return available() >= n;
  }

  void drop_key(int32_t b) {
    if (has_key[static_cast<size_t>(b)]) {
      block_of.erase(key_of[static_cast<size_t>(b)]);
      has_key[static_cast<size_t>(b)] = 0;
    }
  }

  int32_t take() {
    int32_t b;
    if (free_q.size > 0) {
      b = free_q.pop_front();
    } else {
      b = cached.pop_front();
      in_cached[static_cast<size_t>(b)] = 0;
      drop_key(b);  // eviction forgets the content
      ++ctr.evictions;
    }
    ref[static_cast<size_t>(b)] = 1;
    ++active;
    ++ctr.allocs;
    return b;
  }

  void consume_alloc_fault() {
    if (fault_alloc_fail > 0) --fault_alloc_fail;
  }
};

extern "C" {

pkv_alloc* pkv_alloc_create(int32_t num_blocks, int32_t block_size,
                            const int32_t* initial_free_order, int32_t enable_cache) {
  if (num_blocks < 0 || block_size <= 0) return nullptr;
  pkv_alloc* a = new (std::nothrow) pkv_alloc();
  if (!a) return nullptr;
  try {
    a->num_blocks = num_blocks;
    a->block_size = block_size;
    a->cache = enable_cache != 0;
    a->free_q.init(num_blocks);
    a->cached.init(num_blocks);
    a->ref.assign(static_cast<size_t>(num_blocks), 0);
    a->in_cached.assign(static_cast<size_t>(num_blocks), 0);
    a->key_of.assign(static_cast<size_t>(num_blocks), 0);
    a->has_key.assign(static_cast<size_t>(num_blocks), 0);
    if (initial_free_order) {
      std::vector<char> seen(static_cast<size_t>(num_blocks), 0);
      for (int32_t i = 0; i < num_blocks; ++i) {
        int32_t b = initial_free_order[i];
        if (b < 0 || b >= num_blocks || seen[static_cast<size_t>(b)]) {
          delete a;
          return nullptr;
        }
        seen[static_cast<size_t>(b)] = 1;
        a->free_q.push_back(b);
      }
    } else {
      for (int32_t i = 0; i < num_blocks; ++i) a->free_q.push_back(i);
    }
  } catch (...) {
    delete a;
    return nullptr;
  }
  a->ctr.pool = num_blocks;
  return a;
}

void pkv_alloc_destroy(pkv_alloc* a) { delete a; }

int pkv_alloc_add_seq(pkv_alloc* a, int32_t seq_id, int32_t n_tokens) {
  if (!a || seq_id < 0 || n_tokens < 0) return PKV_ERR_INVALID;
  if (a->seqs.count(seq_id)) return PKV_ERR_INVALID;
  int64_t need = (static_cast<int64_t>(n_tokens) + a->block_size - 1) / a->block_size;
  if (need > 0 && !a->can_take(need)) {
    a->consume_alloc_fault();
    ++a->ctr.alloc_failures;
    return PKV_ERR_NO_BLOCKS;
  }
  try {
    Seq s;
    s.table.reserve(static_cast<size_t>(need));
    for (int64_t i = 0; i < need; ++i) s.table.push_back(a->take());
    s.length = n_tokens;
    a->seqs.emplace(seq_id, std::move(s));
  } catch (...) {
    return PKV_ERR_INVALID;
  }
  return PKV_OK;
}

int pkv_alloc_fork(pkv_alloc* a, int32_t parent, int32_t child) {
  if (!a || child < 0) return PKV_ERR_INVALID;
  auto it = a->seqs.find(parent);
  if (it == a->seqs.end() || a->seqs.count(child)) return PKV_ERR_INVALID;
  try {
    Seq c = it->second;  // copy table and length
    for (int32_t b : c.table) a->ref[static_cast<size_t>(b)] += 1;
    a->seqs.emplace(child, std::move(c));
  } catch (...) {
    return PKV_ERR_INVALID;
  }
  return PKV_OK;
}

int pkv_alloc_append(pkv_alloc* a, const int32_t* seq_ids, int32_t n, int32_t* status_out,
                     int32_t* copies_out, int32_t* n_copies_out) {
  if (!a || n < 0 || (n > 0 && (!seq_ids || !status_out || !copies_out)) || !n_copies_out)
    return PKV_ERR_INVALID;
  // Validate everything before changing anything.
  std::vector<Seq*> rows(static_cast<size_t>(n));
  {
    std::unordered_set<int32_t> seen;
    seen.reserve(static_cast<size_t>(n) * 2 + 1);
    for (int32_t i = 0; i < n; ++i) {
      auto it = a->seqs.find(seq_ids[i]);
      if (it == a->seqs.end() || !seen.insert(seq_ids[i]).second) return PKV_ERR_INVALID;
      rows[static_cast<size_t>(i)] = &it->second;
    }
  }
  const int32_t B = a->block_size;
  int32_t ncopy = 0;
  bool all_ok = true;
  for (int32_t i = 0; i < n; ++i) {
    Seq& s = *rows[static_cast<size_t>(i)];
    const int32_t len = s.length;
    if (len % B == 0) {
      if (!a->can_take(1)) {
        a->consume_alloc_fault();
        ++a->ctr.alloc_failures;
        status_out[i] = PKV_ERR_NO_BLOCKS;
        all_ok = false;
        continue;
      }
      s.table.push_back(a->take());
    } else {
      const int32_t tail = s.table.back();
      if (a->ref[static_cast<size_t>(tail)] > 1) {
        if (!a->can_take(1)) {
          a->consume_alloc_fault();
          ++a->ctr.alloc_failures;
          status_out[i] = PKV_ERR_NO_BLOCKS;
          all_ok = false;
          continue;
        }
        const int32_t nb = a->take();
        copies_out[3 * ncopy + 0] = tail;
        copies_out[3 * ncopy + 1] = nb;
        copies_out[3 * ncopy + 2] = len % B;
        ++ncopy;
        a->ref[static_cast<size_t>(tail)] -= 1;  // stays >= 1: another request holds it
        s.table.back() = nb;
        ++a->ctr.cow_copies;
      }
    }
    s.length = len + 1;
    status_out[i] = PKV_OK;
  }
  *n_copies_out = ncopy;
  return all_ok ? PKV_OK : PKV_ERR_NO_BLOCKS;
}

int pkv_alloc_free_seq(pkv_alloc* a, int32_t seq_id) {
  if (!a) return PKV_ERR_INVALID;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_ERR_INVALID;
  if (a->fault_skip_release > 0) {
    // Injected leak: the request disappears but its references stay.
    --a->fault_skip_release;
    a->seqs.erase(it);
    return PKV_OK;
  }
  const Seq& s = it->second;
  const int32_t B = a->block_size;
  const size_t last = s.table.empty() ? 0 : s.table.size() - 1;
  for (size_t i = 0; i < s.table.size(); ++i) {
    const int32_t b = s.table[i];
    int32_t& r = a->ref[static_cast<size_t>(b)];
    r -= 1;
    if (r == 0) {
      --a->active;
      ++a->ctr.frees;
      const bool full = i < last || (s.length > 0 && s.length % B == 0);
      if (a->cache && full) {
        a->cached.push_back(b);  // keeps its content key until evicted
        a->in_cached[static_cast<size_t>(b)] = 1;
      } else {
        a->free_q.push_back(b);
        a->drop_key(b);
      }
    }
  }
  a->seqs.erase(it);
  return PKV_OK;
}

int pkv_alloc_get_table(const pkv_alloc* a, int32_t seq_id, int32_t* out, int32_t cap,
                        int32_t* len, int32_t* n_tokens) {
  if (!a) return PKV_ERR_INVALID;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_ERR_INVALID;
  const Seq& s = it->second;
  const int32_t nb = static_cast<int32_t>(s.table.size());
  if (len) *len = nb;
  if (n_tokens) *n_tokens = s.length;
  if (out) {
    if (cap < nb) return PKV_ERR_INVALID;
    if (nb) std::memcpy(out, s.table.data(), sizeof(int32_t) * static_cast<size_t>(nb));
  }
  return PKV_OK;
}

int pkv_alloc_fill_tables(const pkv_alloc* a, const int32_t* seq_ids, int32_t n,
                          int32_t* tables_out, int32_t max_blocks_per_seq, int32_t pad,
                          int32_t* seq_lens_out) {
  if (!a || n < 0 || max_blocks_per_seq < 0) return PKV_ERR_INVALID;
  if (n > 0 && (!seq_ids || !tables_out || !seq_lens_out)) return PKV_ERR_INVALID;
  std::vector<const Seq*> rows(static_cast<size_t>(n));
  for (int32_t i = 0; i < n; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end()) return PKV_ERR_INVALID;
    if (static_cast<int64_t>(it->second.table.size()) > max_blocks_per_seq) return PKV_ERR_INVALID;
    rows[static_cast<size_t>(i)] = &it->second;
  }
  for (int32_t i = 0; i < n; ++i) {
    const Seq& s = *rows[static_cast<size_t>(i)];
    int32_t* row = tables_out + static_cast<int64_t>(i) * max_blocks_per_seq;
    const int32_t nb = static_cast<int32_t>(s.table.size());
    if (nb) std::memcpy(row, s.table.data(), sizeof(int32_t) * static_cast<size_t>(nb));
    for (int32_t j = nb; j < max_blocks_per_seq; ++j) row[j] = pad;
    seq_lens_out[i] = s.length;
  }
  return PKV_OK;
}

int pkv_alloc_stats(const pkv_alloc* a, pkv_stats* out) {
  if (!a || !out) return PKV_ERR_INVALID;
  *out = a->ctr;
  out->pool = a->num_blocks;
  out->active = a->active;
  out->cached = a->cached.size;
  out->free = a->free_q.size;
  out->seqs = static_cast<int64_t>(a->seqs.size());
  return PKV_OK;
}

int pkv_alloc_check(const pkv_alloc* a) {
  if (!a) return PKV_ERR_INVALID;
  const size_t N = static_cast<size_t>(a->num_blocks);
  if (a->active + a->cached.size + a->free_q.size != a->num_blocks) return PKV_ERR_INVALID;
  std::vector<int32_t> recount(N, 0);
  for (const auto& kv : a->seqs) {
    const Seq& s = kv.second;
    const int64_t need = (static_cast<int64_t>(s.length) + a->block_size - 1) / a->block_size;
    if (static_cast<int64_t>(s.table.size()) != need) return PKV_ERR_INVALID;
    for (int32_t b : s.table) {
      if (b < 0 || static_cast<size_t>(b) >= N) return PKV_ERR_INVALID;
      recount[static_cast<size_t>(b)] += 1;
    }
  }
  int64_t active = 0;
  for (size_t b = 0; b < N; ++b) {
    if (recount[b] != a->ref[b]) return PKV_ERR_INVALID;
    if (a->ref[b] > 0) ++active;
  }
  if (active != a->active) return PKV_ERR_INVALID;
  std::vector<char> idle(N, 0);
  for (int64_t i = 0; i < a->free_q.size; ++i) {
    const int32_t b = a->free_q.at(i);
    if (idle[static_cast<size_t>(b)] || a->ref[static_cast<size_t>(b)] != 0) return PKV_ERR_INVALID;
    idle[static_cast<size_t>(b)] = 1;
  }
  int64_t n_cached = 0;
  for (int32_t b = a->cached.head; b >= 0; b = a->cached.next[static_cast<size_t>(b)]) {
    if (++n_cached > a->num_blocks) return PKV_ERR_INVALID;  // a cycle
    if (idle[static_cast<size_t>(b)] || a->ref[static_cast<size_t>(b)] != 0 ||
        !a->in_cached[static_cast<size_t>(b)])
      return PKV_ERR_INVALID;
    idle[static_cast<size_t>(b)] = 1;
  }
  if (n_cached != a->cached.size) return PKV_ERR_INVALID;
  size_t keyed = 0;
  for (size_t b = 0; b < N; ++b) {
    if (!a->has_key[b]) continue;
    ++keyed;
    auto it = a->block_of.find(a->key_of[b]);
    if (it == a->block_of.end() || it->second != static_cast<int32_t>(b)) return PKV_ERR_INVALID;
  }
  if (keyed != a->block_of.size()) return PKV_ERR_INVALID;
  for (int64_t i = 0; i < a->free_q.size; ++i)
    if (a->has_key[static_cast<size_t>(a->free_q.at(i))]) return PKV_ERR_INVALID;
  return PKV_OK;
}

int pkv_alloc_dump(const pkv_alloc* a, int32_t* refcounts, int32_t* free_order, int32_t* n_free,
                   int32_t* cached_order, int32_t* n_cached) {
  if (!a) return PKV_ERR_INVALID;
  if (refcounts && a->num_blocks)
    std::memcpy(refcounts, a->ref.data(), sizeof(int32_t) * static_cast<size_t>(a->num_blocks));
  if (free_order)
    for (int64_t i = 0; i < a->free_q.size; ++i) free_order[i] = a->free_q.at(i);
  if (n_free) *n_free = static_cast<int32_t>(a->free_q.size);
  if (cached_order) {
    int64_t i = 0;
    for (int32_t b = a->cached.head; b >= 0; b = a->cached.next[static_cast<size_t>(b)]) cached_order[i++] = b;
  }
  if (n_cached) *n_cached = static_cast<int32_t>(a->cached.size);
  return PKV_OK;
}

int pkv_alloc_set_block_key(pkv_alloc* a, int32_t seq_id, int32_t logical_block, uint64_t key) {
  if (!a) return PKV_ERR_INVALID;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_ERR_INVALID;
  const Seq& s = it->second;
  if (logical_block < 0 ||
      (static_cast<int64_t>(logical_block) + 1) * a->block_size > s.length)
    return PKV_ERR_INVALID;  // only full blocks are shareable
  const int32_t b = s.table[static_cast<size_t>(logical_block)];
  auto owner = a->block_of.find(key);
  if (owner != a->block_of.end() && owner->second != b) return PKV_ERR_INVALID;
  if (a->has_key[static_cast<size_t>(b)] && a->key_of[static_cast<size_t>(b)] != key) return PKV_ERR_INVALID;
  try {
    a->block_of[key] = b;
  } catch (...) {
    return PKV_ERR_INVALID;
  }
  a->key_of[static_cast<size_t>(b)] = key;
  a->has_key[static_cast<size_t>(b)] = 1;
  return PKV_OK;
}

int pkv_alloc_add_seq_prefix(pkv_alloc* a, int32_t seq_id, int32_t n_tokens, const uint64_t* keys,
                             int32_t n_keys, int32_t* n_hit) {
  if (!a || seq_id < 0 || n_tokens < 0 || n_keys < 0 || (n_keys > 0 && !keys)) return PKV_ERR_INVALID;
  if (a->seqs.count(seq_id)) return PKV_ERR_INVALID;
  if (static_cast<int64_t>(n_keys) * a->block_size > n_tokens) return PKV_ERR_INVALID;
  std::vector<int32_t> hits;
  int64_t revived = 0;
  for (int32_t i = 0; i < n_keys; ++i) {
    auto it = a->block_of.find(keys[i]);
    if (it == a->block_of.end()) break;
    hits.push_back(it->second);
    if (a->ref[static_cast<size_t>(it->second)] == 0) ++revived;
  }
  const int64_t need = (static_cast<int64_t>(n_tokens) + a->block_size - 1) / a->block_size -
                       static_cast<int64_t>(hits.size());
  const int64_t avail = a->available() - (a->cache ? revived : 0);
  if (need > 0 && (a->fault_alloc_fail > 0 || need > avail)) {
    a->consume_alloc_fault();
    ++a->ctr.alloc_failures;
    if (n_hit) *n_hit = 0;
    return PKV_ERR_NO_BLOCKS;
  }
  try {
    Seq s;
    s.table.reserve(hits.size() + static_cast<size_t>(need));
    for (int32_t b : hits) {
      int32_t& r = a->ref[static_cast<size_t>(b)];
      if (r == 0) {  // a cached block comes back to active
        a->cached.remove(b);
        a->in_cached[static_cast<size_t>(b)] = 0;
        ++a->active;
      }
      r += 1;
      s.table.push_back(b);
    }
    for (int64_t i = 0; i < need; ++i) s.table.push_back(a->take());
    s.length = n_tokens;
    a->seqs.emplace(seq_id, std::move(s));
  } catch (...) {
    return PKV_ERR_INVALID;
  }
  a->ctr.prefix_hits += static_cast<int64_t>(hits.size());
  if (n_hit) *n_hit = static_cast<int32_t>(hits.size());
  return PKV_OK;
}

int pkv_alloc_inject_fault(pkv_alloc* a, int32_t kind, int32_t count) {
  if (!a || count < 0) return PKV_ERR_INVALID;
  switch (kind) {
    case PKV_FAULT_NONE:
      a->fault_alloc_fail = 0;
      a->fault_skip_release = 0;
      return PKV_OK;
    case PKV_FAULT_ALLOC_FAIL:
      a->fault_alloc_fail = count;
      return PKV_OK;
    case PKV_FAULT_SKIP_RELEASE:
      a->fault_skip_release = count;
      return PKV_OK;
    default:
      return PKV_ERR_INVALID;
  }
}

}  // extern "C"
