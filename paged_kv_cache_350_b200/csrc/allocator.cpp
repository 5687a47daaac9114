// Host block allocator with reference counts for a paged KV pool.
//
// Blocks are handed out on demand, one when the previous is full ("PagedAttention"
// concept card, 带来的能力; "什么是 LLM 中的分页注意力", 使用分页注意力).  A fork shares
// every block and raises its refcount; a block returns to the free list when its count
// reaches 0; before a sequence writes into a partial block it still shares, the block
// is copied (copy on write) so the sibling's prefix stays intact ("深入解析
// PagedAttention", 核心创新 / 多序列共享; concept card, 实现要点).  The exact policy
// (LIFO free list, splitmix64 Fisher-Yates shuffle, when a copy happens) is stated in
// include/pa.h.  Every failing call leaves the state unchanged, a failed host allocation
// included: each entry point allocates (reserves) all it needs before it changes
// anything, and returns PA_ERR_HOST_MEMORY instead of letting std::bad_alloc cross the
// C ABI.

#include <algorithm>
#include <cstring>
#include <memory>
#include <new>
#include <stdexcept>
#include <unordered_map>
#include <vector>

#include "pa.h"

namespace {

struct Seq {
  std::vector<int32_t> table;
  int64_t ntok = 0;
  uint64_t mark = 0;  // epoch of the batch call that last listed it (duplicate check)
};

// Room for one more table entry, grown geometrically.  Capacity only: no allocator
// state changes, so a call may do this before it knows it will succeed.
void reserve_one(Seq& s) {
  if (s.table.size() == s.table.capacity())
    s.table.reserve(s.table.size() < 8 ? 8 : 2 * s.table.size());
}

// splitmix64 (Steele, Lea & Flood, OOPSLA 2014).
struct SplitMix64 {
  uint64_t state;
  uint64_t next() {
    uint64_t z = (state += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
};

}  // namespace

struct pa_allocator {
  int num_blocks = 0;
  int block_size = 0;
  std::vector<int32_t> free_stack;  // back() is popped first
  std::vector<int32_t> ref;
  std::unordered_map<int64_t, Seq> seqs;
  uint64_t epoch = 0;  // one per batch call: marks the sequences it has listed

  int32_t pop() {
    int32_t b = free_stack.back();
    free_stack.pop_back();
    ref[b] = 1;
    return b;
  }
};

namespace {

bool init_from_order(pa_allocator* a, int num_blocks, int block_size,
                     const std::vector<int32_t>& pop_order) {
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->ref.assign(num_blocks, 0);
  a->free_stack.assign(pop_order.rbegin(), pop_order.rend());
  return true;
}

// The entry points' bodies: a failed host allocation (std::bad_alloc, or a size the
// containers cannot hold) becomes PA_ERR_HOST_MEMORY instead of crossing the C ABI.
template <class F>
pa_status guarded(F&& body) {
  try {
    return body();
  } catch (const std::bad_alloc&) {
    return PA_ERR_HOST_MEMORY;
  } catch (const std::length_error&) {
    return PA_ERR_HOST_MEMORY;
  }
}

pa_status create_impl(int num_blocks, int block_size, uint64_t shuffle_seed, pa_allocator** out) {
  if (!out || num_blocks <= 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
  std::vector<int32_t> order(num_blocks);
  for (int i = 0; i < num_blocks; ++i) order[i] = i;
  if (shuffle_seed != 0) {
    SplitMix64 rng{shuffle_seed};
    for (int i = num_blocks - 1; i > 0; --i) {
      int j = static_cast<int>(rng.next() % static_cast<uint64_t>(i + 1));
      std::swap(order[i], order[j]);
    }
  }
  std::unique_ptr<pa_allocator> a(new pa_allocator());
  init_from_order(a.get(), num_blocks, block_size, order);
  *out = a.release();
  return PA_OK;
}

pa_status create_ordered_impl(int num_blocks, int block_size, const int32_t* pop_order,
                              pa_allocator** out) {
  if (!out || !pop_order || num_blocks <= 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
  std::vector<int32_t> order(pop_order, pop_order + num_blocks);
  std::vector<char> seen(num_blocks, 0);
  for (int32_t b : order) {
    if (b < 0 || b >= num_blocks || seen[b]) return PA_ERR_INVALID_ARG;
    seen[b] = 1;
  }
  std::unique_ptr<pa_allocator> a(new pa_allocator());
  init_from_order(a.get(), num_blocks, block_size, order);
  *out = a.release();
  return PA_OK;
}

pa_status add_seq_impl(pa_allocator* a, int64_t seq_id, int num_tokens) {
  if (!a || num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (a->seqs.count(seq_id)) return PA_ERR_EXISTS;
  int64_t need = (static_cast<int64_t>(num_tokens) + a->block_size - 1) / a->block_size;
  if (need > static_cast<int64_t>(a->free_stack.size())) return PA_ERR_OUT_OF_BLOCKS;
  // allocate the map node and the table first; only then take blocks
  auto ins = a->seqs.emplace(seq_id, Seq());
  Seq& s = ins.first->second;
  try {
    s.table.reserve(need + 1);
  } catch (...) {
    a->seqs.erase(ins.first);
    throw;
  }
  for (int64_t i = 0; i < need; ++i) s.table.push_back(a->pop());
  s.ntok = num_tokens;
  return PA_OK;
}

pa_status fork_impl(pa_allocator* a, int64_t parent_id, int64_t child_id) {
  if (!a) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(parent_id);
  if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
  if (a->seqs.count(child_id)) return PA_ERR_EXISTS;
  Seq child = it->second;  // copy before emplace (rehash may move the parent)
  auto ins = a->seqs.emplace(child_id, std::move(child));
  for (int32_t b : ins.first->second.table) a->ref[b] += 1;
  return PA_OK;
}

// The table must have room for one more entry (reserved by the caller), so nothing here
// allocates.
void append_one(pa_allocator* a, Seq& s, int64_t* slot, int32_t* src, int32_t* dst) {
  const int bs = a->block_size;
  const int off = static_cast<int>(s.ntok % bs);
  int32_t phys;
  *src = -1;
  *dst = -1;
  if (off == 0) {
    phys = a->pop();
    s.table.push_back(phys);
  } else {
    int32_t last = s.table.back();
    if (a->ref[last] > 1) {
      phys = a->pop();
      a->ref[last] -= 1;
      s.table.back() = phys;
      *src = last;
      *dst = phys;
    } else {
      phys = last;
    }
  }
  s.ntok += 1;
  *slot = static_cast<int64_t>(phys) * bs + off;
}

pa_status append_slot_impl(pa_allocator* a, int64_t seq_id, int64_t* slot, int32_t* cow_src,
                           int32_t* cow_dst) {
  if (!a || !slot || !cow_src || !cow_dst) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
  Seq& s = it->second;
  const bool needs_block =
      (s.ntok % a->block_size == 0) || (a->ref[s.table.back()] > 1);
  if (needs_block && a->free_stack.empty()) return PA_ERR_OUT_OF_BLOCKS;
  if (s.ntok % a->block_size == 0) reserve_one(s);
  append_one(a, s, slot, cow_src, cow_dst);
  return PA_OK;
}

pa_status append_slots_impl(pa_allocator* a, const int64_t* seq_ids, int n,
                            int64_t* slot_mapping, int32_t* cow_pairs, int* n_pairs) {
  if (!a || n < 0 || (n > 0 && (!seq_ids || !slot_mapping || !cow_pairs)) || !n_pairs)
    return PA_ERR_INVALID_ARG;
  // Dry run: resolve every sequence, reject duplicates, and count the fresh blocks the
  // batch takes, replaying the refcount drops of earlier copies in the same batch.
  std::vector<Seq*> rows(n);
  std::unordered_map<int32_t, int> dropped;
  const uint64_t epoch = ++a->epoch;
  int64_t need = 0;
  for (int i = 0; i < n; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
    Seq& s = it->second;
    if (s.mark == epoch) return PA_ERR_INVALID_ARG;  // listed twice
    s.mark = epoch;
    rows[i] = &s;
    if (s.ntok % a->block_size == 0) {
      need += 1;
      reserve_one(s);
    } else {
      int32_t last = s.table.back();
      auto d = dropped.find(last);
      int drop = d == dropped.end() ? 0 : d->second;
      if (a->ref[last] - drop > 1) {
        need += 1;
        dropped[last] = drop + 1;
      }
    }
  }
  if (need > static_cast<int64_t>(a->free_stack.size())) return PA_ERR_OUT_OF_BLOCKS;
  int np = 0;
  for (int i = 0; i < n; ++i) {
    int32_t src, dst;
    append_one(a, *rows[i], &slot_mapping[i], &src, &dst);
    if (src >= 0) {
      cow_pairs[2 * np] = src;
      cow_pairs[2 * np + 1] = dst;
      ++np;
    }
  }
  *n_pairs = np;
  return PA_OK;
}

// free_stack holds every block at creation, so its capacity covers all pushes: freeing
// never allocates.
pa_status free_seq_impl(pa_allocator* a, int64_t seq_id) {
  if (!a) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
  for (int32_t b : it->second.table) {
    if (--a->ref[b] == 0) a->free_stack.push_back(b);
  }
  a->seqs.erase(it);
  return PA_OK;
}

pa_status truncate_impl(pa_allocator* a, int64_t seq_id, int num_tokens) {
  if (!a || num_tokens < 0) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
  Seq& s = it->second;
  if (num_tokens > s.ntok) return PA_ERR_INVALID_ARG;
  const size_t keep = (static_cast<size_t>(num_tokens) + a->block_size - 1) / a->block_size;
  for (size_t j = keep; j < s.table.size(); ++j) {
    const int32_t b = s.table[j];
    if (--a->ref[b] == 0) a->free_stack.push_back(b);
  }
  s.table.resize(keep);
  s.ntok = num_tokens;
  return PA_OK;
}

pa_status beam_select_impl(pa_allocator* a, const int64_t* seq_ids, const int32_t* parent_idx,
                           int n) {
  if (!a || n < 0 || (n > 0 && (!seq_ids || !parent_idx))) return PA_ERR_INVALID_ARG;
  std::vector<Seq*> rows(n);
  const uint64_t epoch = ++a->epoch;
  for (int i = 0; i < n; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
    if (it->second.mark == epoch) return PA_ERR_INVALID_ARG;  // listed twice
    it->second.mark = epoch;
    if (parent_idx[i] < 0 || parent_idx[i] >= n) return PA_ERR_INVALID_ARG;
    rows[i] = &it->second;
  }
  std::vector<Seq> next(n);
  for (int i = 0; i < n; ++i) next[i] = *rows[parent_idx[i]];  // every copy before any change
  for (int i = 0; i < n; ++i)
    for (int32_t b : next[i].table) a->ref[b] += 1;
  for (int i = 0; i < n; ++i) {
    for (int32_t b : rows[i]->table)
      if (--a->ref[b] == 0) a->free_stack.push_back(b);
  }
  for (int i = 0; i < n; ++i) *rows[i] = std::move(next[i]);
  return PA_OK;
}

pa_status prefix_groups_impl(const pa_allocator* a, const int64_t* seq_ids, int n,
                             int max_members, int align_tokens, int32_t* group_of,
                             int32_t* group_prefix, int32_t* group_members, int* ngroups) {
  if (!a || n < 0 || max_members < 1 || align_tokens < 1 || !ngroups ||
      (n > 0 && (!seq_ids || !group_of || !group_prefix || !group_members)))
    return PA_ERR_INVALID_ARG;
  std::vector<const Seq*> rows(n);
  for (int i = 0; i < n; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
    rows[i] = &it->second;
    group_of[i] = -1;
  }
  // rows by first block, in batch order (first-appearance order of the blocks)
  std::vector<int32_t> firsts;
  std::unordered_map<int32_t, std::vector<int>> buckets;
  for (int i = 0; i < n; ++i) {
    if (rows[i]->table.empty()) continue;
    const int32_t f = rows[i]->table[0];
    auto& v = buckets[f];
    if (v.empty()) firsts.push_back(f);
    v.push_back(i);
  }
  int ng = 0;
  for (int32_t f : firsts) {
    const std::vector<int>& v = buckets[f];
    for (size_t c0 = 0; c0 < v.size(); c0 += max_members) {
      const size_t c1 = std::min(v.size(), c0 + static_cast<size_t>(max_members));
      if (c1 - c0 < 2) continue;
      size_t k = rows[v[c0]]->table.size();
      int64_t shortest = rows[v[c0]]->ntok;
      for (size_t m = c0 + 1; m < c1; ++m) {
        const Seq& s = *rows[v[m]];
        size_t j = 0;
        while (j < k && j < s.table.size() && s.table[j] == rows[v[c0]]->table[j]) ++j;
        k = j;
        shortest = std::min<int64_t>(shortest, s.ntok);
      }
      int64_t prefix = std::min<int64_t>(static_cast<int64_t>(k) * a->block_size, shortest);
      prefix -= prefix % align_tokens;
      if (prefix <= 0) continue;
      group_prefix[ng] = static_cast<int32_t>(prefix);
      for (int m = 0; m < max_members; ++m) {
        const size_t idx = c0 + m;
        group_members[static_cast<size_t>(ng) * max_members + m] = idx < c1 ? v[idx] : -1;
        if (idx < c1) group_of[v[idx]] = ng;
      }
      ++ng;
    }
  }
  *ngroups = ng;
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_alloc_create(int num_blocks, int block_size, uint64_t shuffle_seed,
                          pa_allocator** out) {
  return guarded([&] { return create_impl(num_blocks, block_size, shuffle_seed, out); });
}

pa_status pa_alloc_create_ordered(int num_blocks, int block_size, const int32_t* pop_order,
                                  pa_allocator** out) {
  return guarded([&] { return create_ordered_impl(num_blocks, block_size, pop_order, out); });
}

void pa_alloc_destroy(pa_allocator* a) { delete a; }

pa_status pa_alloc_add_seq(pa_allocator* a, int64_t seq_id, int num_tokens) {
  return guarded([&] { return add_seq_impl(a, seq_id, num_tokens); });
}

pa_status pa_alloc_fork(pa_allocator* a, int64_t parent_id, int64_t child_id) {
  return guarded([&] { return fork_impl(a, parent_id, child_id); });
}

pa_status pa_alloc_append_slot(pa_allocator* a, int64_t seq_id, int64_t* slot,
                               int32_t* cow_src, int32_t* cow_dst) {
  return guarded([&] { return append_slot_impl(a, seq_id, slot, cow_src, cow_dst); });
}

pa_status pa_alloc_append_slots(pa_allocator* a, const int64_t* seq_ids, int n,
                                int64_t* slot_mapping, int32_t* cow_pairs, int* n_pairs) {
  return guarded(
      [&] { return append_slots_impl(a, seq_ids, n, slot_mapping, cow_pairs, n_pairs); });
}

pa_status pa_alloc_free_seq(pa_allocator* a, int64_t seq_id) {
  return guarded([&] { return free_seq_impl(a, seq_id); });
}

pa_status pa_alloc_truncate(pa_allocator* a, int64_t seq_id, int num_tokens) {
  return guarded([&] { return truncate_impl(a, seq_id, num_tokens); });
}

pa_status pa_alloc_beam_select(pa_allocator* a, const int64_t* seq_ids, const int32_t* parent_idx,
                               int n) {
  return guarded([&] { return beam_select_impl(a, seq_ids, parent_idx, n); });
}

pa_status pa_alloc_prefix_groups(const pa_allocator* a, const int64_t* seq_ids, int n,
                                 int max_members, int align_tokens, int32_t* group_of,
                                 int32_t* group_prefix, int32_t* group_members, int* ngroups) {
  return guarded([&] {
    return prefix_groups_impl(a, seq_ids, n, max_members, align_tokens, group_of, group_prefix,
                              group_members, ngroups);
  });
}

pa_status pa_alloc_block_table(const pa_allocator* a, int64_t seq_id, int32_t* out, int cap,
                               int* n, int* num_tokens) {
  if (!a || !n || !num_tokens || cap < 0 || (cap > 0 && !out)) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
  const Seq& s = it->second;
  int len = static_cast<int>(s.table.size());
  int m = std::min(len, cap);
  if (m > 0) std::memcpy(out, s.table.data(), sizeof(int32_t) * m);
  *n = len;
  *num_tokens = static_cast<int>(s.ntok);
  return PA_OK;
}

pa_status pa_alloc_block_tables(const pa_allocator* a, const int64_t* seq_ids, int n,
                                int32_t* block_tables, int max_blocks, int32_t* seq_lens) {
  return guarded([&]() -> pa_status {
    if (!a || n < 0 || max_blocks <= 0 ||
        (n > 0 && (!seq_ids || !block_tables || !seq_lens)))
      return PA_ERR_INVALID_ARG;
    std::vector<const Seq*> rows(n);
    for (int i = 0; i < n; ++i) {
      auto it = a->seqs.find(seq_ids[i]);
      if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
      if (static_cast<int>(it->second.table.size()) > max_blocks) return PA_ERR_INVALID_ARG;
      rows[i] = &it->second;
    }
    for (int i = 0; i < n; ++i) {
      const Seq& s = *rows[i];
      int32_t* row = block_tables + static_cast<int64_t>(i) * max_blocks;
      int len = static_cast<int>(s.table.size());
      if (len) std::memcpy(row, s.table.data(), sizeof(int32_t) * len);
      for (int j = len; j < max_blocks; ++j) row[j] = -1;
      seq_lens[i] = static_cast<int32_t>(s.ntok);
    }
    return PA_OK;
  });
}

// Whether every listed sequence exists and still has a table of at most max_blocks entries
// after one more token (the decode-step pipeline checks this before it appends, so that a
// step it cannot describe changes no state).
pa_status pa_alloc_check_append_fits(const pa_allocator* a, const int64_t* seq_ids, int n,
                                     int max_blocks) {
  if (!a || n < 0 || max_blocks <= 0 || (n > 0 && !seq_ids)) return PA_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
    const int64_t blocks = (it->second.ntok + 1 + a->block_size - 1) / a->block_size;
    if (blocks > max_blocks) return PA_ERR_INVALID_ARG;
  }
  return PA_OK;
}

pa_status pa_alloc_seq_slots(const pa_allocator* a, int64_t seq_id, int64_t* slots, int cap,
                             int* n) {
  if (!a || !n || cap < 0 || (cap > 0 && !slots)) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_NOT_FOUND;
  const Seq& s = it->second;
  const int bs = a->block_size;
  const int ntok = static_cast<int>(s.ntok);
  const int m = std::min(ntok, cap);
  for (int t = 0; t < m; ++t)
    slots[t] = static_cast<int64_t>(s.table[t / bs]) * bs + t % bs;
  *n = ntok;
  return PA_OK;
}

int pa_alloc_refcount(const pa_allocator* a, int32_t block) {
  if (!a || block < 0 || block >= a->num_blocks) return -1;
  return a->ref[block];
}

int pa_alloc_num_free(const pa_allocator* a) {
  return a ? static_cast<int>(a->free_stack.size()) : -1;
}

int64_t pa_alloc_internal_waste_slots(const pa_allocator* a) {
  if (!a) return -1;
  int64_t w = 0;
  for (const auto& kv : a->seqs)
    w += static_cast<int64_t>(kv.second.table.size()) * a->block_size - kv.second.ntok;
  return w;
}

int pa_alloc_free_list(const pa_allocator* a, int32_t* out, int cap) {
  if (!a) return -1;
  int len = static_cast<int>(a->free_stack.size());
  int m = std::min(len, cap);
  if (m > 0 && out) std::memcpy(out, a->free_stack.data(), sizeof(int32_t) * m);
  return len;
}

}  // extern "C"
