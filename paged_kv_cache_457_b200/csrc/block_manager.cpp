// Host-side page pool for the paged KV cache: free lists, per-page reference
// counts, copy-on-write of shared partly filled pages, swap plans and the
// per-step tables of a continuous batch.  The behaviour (and the readings of
// the pages behind it) is stated in include/pa_block_manager.h.
//
// Failure atomicity: every entry point first checks and plans (the only place
// that may allocate host memory), then mutates; the mutation phase cannot
// fail, because free lists are reserved for the whole pool up front and page
// tables are reserved before pages are taken.
#include "pa_block_manager.h"

#include <algorithm>
#include <cstdint>
#include <limits>
#include <mutex>
#include <new>
#include <unordered_map>
#include <unordered_set>
#include <vector>

struct pa_block_manager {
  struct Pool {
    std::vector<int32_t> refs;       // references held on each page
    std::vector<int32_t> free_list;  // stack: back() is handed out next

    explicit Pool(int64_t n) : refs(static_cast<size_t>(n), 0) {
      free_list.reserve(static_cast<size_t>(n));
      for (int64_t i = n - 1; i >= 0; --i) free_list.push_back(static_cast<int32_t>(i));
    }
    int64_t size() const { return static_cast<int64_t>(refs.size()); }
    int64_t num_free() const { return static_cast<int64_t>(free_list.size()); }
    int32_t take() {  // caller checked num_free() > 0; the page starts with no reference
      const int32_t b = free_list.back();
      free_list.pop_back();
      return b;
    }
    void unref(int32_t b) {
      if (--refs[static_cast<size_t>(b)] == 0) free_list.push_back(b);
    }
  };

  struct Seq {
    std::vector<int32_t> table;  // page ids in the pool the sequence is in
    int64_t tokens = 0;
    bool host = false;
  };

  int64_t block_size;
  Pool dev, host;
  std::unordered_map<int64_t, Seq> seqs;
  mutable std::mutex mu;

  pa_block_manager(int32_t bs, int64_t nd, int64_t nh) : block_size(bs), dev(nd), host(nh) {}

  int64_t pages_for(int64_t tokens) const { return (tokens + block_size - 1) / block_size; }

  // Whether appending one token to `s` needs a fresh device page, given the
  // references `extra_dropped` that earlier appends of the same step already
  // took off its last page.
  bool append_needs_page(const Seq &s, int32_t extra_dropped) const {
    if (s.tokens % block_size == 0) return true;
    return dev.refs[static_cast<size_t>(s.table.back())] - extra_dropped > 1;
  }

  // The mutation half of an append; the caller checked that a page is free
  // if one is needed and reserved room in s.table.
  void append(Seq &s, int64_t *slot, int64_t *src, int64_t *dst) {
    const int64_t row = s.tokens % block_size;
    *src = *dst = -1;
    if (row == 0) {
      const int32_t b = dev.take();
      dev.refs[static_cast<size_t>(b)] = 1;
      s.table.push_back(b);
    } else {
      const int32_t last = s.table.back();
      if (dev.refs[static_cast<size_t>(last)] > 1) {  // shared and partly full: private copy first
        const int32_t b = dev.take();
        dev.refs[static_cast<size_t>(b)] = 1;
        --dev.refs[static_cast<size_t>(last)];  // stays >= 1: other sequences still name it
        s.table.back() = b;
        *src = last;
        *dst = b;
      }
    }
    *slot = static_cast<int64_t>(s.table.back()) * block_size + row;
    ++s.tokens;
  }

  // Plan of a step in which sequence i brings new_tokens[i] >= 0 tokens: the fresh device pages and the
  // copy-on-write pairs its appends will take (simulating the references that earlier copies of the same
  // step drop from shared last pages) and the token total.  Tables longer than table_stride fail with
  // PA_BM_ERR_CAPACITY.  A const member: planning cannot change the pool.
  int plan_step(const int64_t *ids, const int64_t *new_tokens, int64_t n, int64_t table_stride, int64_t *pages,
                int64_t *copies, int64_t *total) const {
    std::unordered_set<int64_t> seen;
    std::unordered_map<int32_t, int32_t> dropped;
    const int64_t int32_max = std::numeric_limits<int32_t>::max();
    *pages = *copies = *total = 0;
    for (int64_t i = 0; i < n; ++i) {
      const auto it = seqs.find(ids[i]);
      if (it == seqs.end()) return PA_BM_ERR_UNKNOWN;
      const Seq &s = it->second;
      if (s.host) return PA_BM_ERR_STATE;
      if (!seen.insert(ids[i]).second) return PA_BM_ERR_ARG;
      const int64_t add = new_tokens[i];
      if (add < 0 || add > int32_max - s.tokens || add > int32_max - *total) return PA_BM_ERR_ARG;
      *total += add;
      if (add > 0) {
        const bool fresh_row = s.tokens % block_size == 0;
        if (!fresh_row && append_needs_page(s, dropped[s.table.back()])) {  // private copy of the last page
          ++*pages;
          ++*copies;
          ++dropped[s.table.back()];
        }
        *pages += pages_for(s.tokens + add) - pages_for(s.tokens);
      }
      if (pages_for(s.tokens + add) > table_stride) return PA_BM_ERR_CAPACITY;
    }
    return PA_BM_OK;
  }

  // Moves whole sequences from pool `from` to pool `to` (see swap_out / swap_in).
  int move(const int64_t *ids, int64_t n, bool to_host, int64_t *mapping, int64_t capacity, int64_t *num_pairs) {
    if (n < 0 || (n > 0 && !ids) || !num_pairs || capacity < 0 || (capacity > 0 && !mapping)) return PA_BM_ERR_ARG;
    Pool &from = to_host ? dev : host;
    Pool &to = to_host ? host : dev;
    std::vector<Seq *> list;
    list.reserve(static_cast<size_t>(n));
    std::unordered_set<int64_t> seen;
    std::unordered_map<int32_t, int32_t> remap;  // page in `from` -> index of its pair
    std::vector<int32_t> order;                   // pages of `from` in first-seen order
    for (int64_t i = 0; i < n; ++i) {
      auto it = seqs.find(ids[i]);
      if (it == seqs.end()) return PA_BM_ERR_UNKNOWN;
      if (it->second.host == to_host) return PA_BM_ERR_STATE;
      if (!seen.insert(ids[i]).second) return PA_BM_ERR_ARG;
      list.push_back(&it->second);
      for (int32_t b : it->second.table)
        if (remap.emplace(b, static_cast<int32_t>(order.size())).second) order.push_back(b);
    }
    const int64_t need = static_cast<int64_t>(order.size());
    *num_pairs = need;
    if (need > to.num_free()) return PA_BM_ERR_NO_SPACE;
    if (need > capacity) return PA_BM_ERR_CAPACITY;
    // Mutation: no allocation below.
    std::vector<int32_t> target(order.size());
    for (size_t k = 0; k < order.size(); ++k) {
      target[k] = to.take();
      mapping[2 * k] = order[k];
      mapping[2 * k + 1] = target[k];
    }
    for (Seq *s : list) {
      for (int32_t &b : s->table) {
        const int32_t t = target[static_cast<size_t>(remap.find(b)->second)];
        ++to.refs[static_cast<size_t>(t)];
        from.unref(b);
        b = t;
      }
      s->host = to_host;
    }
    return PA_BM_OK;
  }
};

namespace {

template <class F>
int guarded(pa_block_manager *bm, F &&f) {
  if (!bm) return PA_BM_ERR_ARG;
  try {
    std::lock_guard<std::mutex> g(bm->mu);
    return f();
  } catch (const std::bad_alloc &) {
    return PA_BM_ERR_HOST_MEMORY;
  }
}

template <class F>
int guarded_const(const pa_block_manager *bm, F &&f) {
  if (!bm) return PA_BM_ERR_ARG;
  std::lock_guard<std::mutex> g(bm->mu);
  return f();
}

}  // namespace

extern "C" {

pa_block_manager *pa_bm_create(int32_t block_size, int64_t num_device_blocks, int64_t num_host_blocks) {
  const int64_t max_id = std::numeric_limits<int32_t>::max();
  if (block_size <= 0 || num_device_blocks < 0 || num_host_blocks < 0 || num_device_blocks > max_id ||
      num_host_blocks > max_id)
    return nullptr;
  try {
    return new pa_block_manager(block_size, num_device_blocks, num_host_blocks);
  } catch (const std::bad_alloc &) {
    return nullptr;
  }
}

void pa_bm_destroy(pa_block_manager *bm) { delete bm; }

int64_t pa_bm_num_free_device_blocks(const pa_block_manager *bm) {
  if (!bm) return PA_BM_ERR_ARG;
  std::lock_guard<std::mutex> g(bm->mu);
  return bm->dev.num_free();
}

int64_t pa_bm_num_free_host_blocks(const pa_block_manager *bm) {
  if (!bm) return PA_BM_ERR_ARG;
  std::lock_guard<std::mutex> g(bm->mu);
  return bm->host.num_free();
}

int32_t pa_bm_ref_count(const pa_block_manager *bm, int32_t host_pool, int64_t block) {
  if (!bm) return -1;
  std::lock_guard<std::mutex> g(bm->mu);
  const auto &p = host_pool ? bm->host : bm->dev;
  if (block < 0 || block >= p.size()) return -1;
  return p.refs[static_cast<size_t>(block)];
}

int pa_bm_add_sequence(pa_block_manager *bm, int64_t seq_id, int64_t num_tokens) {
  return guarded(bm, [&] {
    if (num_tokens < 0) return PA_BM_ERR_ARG;
    if (bm->seqs.count(seq_id)) return PA_BM_ERR_EXISTS;
    const int64_t need = bm->pages_for(num_tokens);
    if (need > bm->dev.num_free()) return PA_BM_ERR_NO_SPACE;
    pa_block_manager::Seq s;
    s.table.reserve(static_cast<size_t>(need));
    s.tokens = num_tokens;
    auto it = bm->seqs.emplace(seq_id, std::move(s)).first;  // may throw: nothing taken yet
    for (int64_t i = 0; i < need; ++i) {
      const int32_t b = bm->dev.take();
      bm->dev.refs[static_cast<size_t>(b)] = 1;
      it->second.table.push_back(b);
    }
    return PA_BM_OK;
  });
}

int pa_bm_fork(pa_block_manager *bm, int64_t parent_id, int64_t child_id) {
  return guarded(bm, [&] {
    auto it = bm->seqs.find(parent_id);
    if (it == bm->seqs.end()) return PA_BM_ERR_UNKNOWN;
    if (it->second.host) return PA_BM_ERR_STATE;
    if (bm->seqs.count(child_id)) return PA_BM_ERR_EXISTS;
    pa_block_manager::Seq child = it->second;
    auto c = bm->seqs.emplace(child_id, std::move(child)).first;
    for (int32_t b : c->second.table) ++bm->dev.refs[static_cast<size_t>(b)];
    return PA_BM_OK;
  });
}

int pa_bm_free_sequence(pa_block_manager *bm, int64_t seq_id) {
  return guarded(bm, [&] {
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PA_BM_ERR_UNKNOWN;
    auto &pool = it->second.host ? bm->host : bm->dev;
    for (int32_t b : it->second.table) pool.unref(b);
    bm->seqs.erase(it);
    return PA_BM_OK;
  });
}

int64_t pa_bm_num_tokens(const pa_block_manager *bm, int64_t seq_id) {
  if (!bm) return PA_BM_ERR_ARG;
  std::lock_guard<std::mutex> g(bm->mu);
  auto it = bm->seqs.find(seq_id);
  return it == bm->seqs.end() ? PA_BM_ERR_UNKNOWN : it->second.tokens;
}

int pa_bm_is_swapped(const pa_block_manager *bm, int64_t seq_id) {
  return guarded_const(bm, [&] {
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? PA_BM_ERR_UNKNOWN : (it->second.host ? 1 : 0);
  });
}

int pa_bm_block_table(const pa_block_manager *bm, int64_t seq_id, int32_t *table, int64_t capacity,
                      int64_t *num_blocks) {
  return guarded_const(bm, [&] {
    if (!num_blocks || capacity < 0 || (capacity > 0 && !table)) return PA_BM_ERR_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PA_BM_ERR_UNKNOWN;
    const auto &t = it->second.table;
    *num_blocks = static_cast<int64_t>(t.size());
    if (static_cast<int64_t>(t.size()) > capacity) return PA_BM_ERR_CAPACITY;
    std::copy(t.begin(), t.end(), table);
    return PA_BM_OK;
  });
}

int pa_bm_slots(const pa_block_manager *bm, int64_t seq_id, int64_t first, int64_t count, int64_t *slots) {
  return guarded_const(bm, [&] {
    if (first < 0 || count < 0 || (count > 0 && !slots)) return PA_BM_ERR_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PA_BM_ERR_UNKNOWN;
    const auto &s = it->second;
    if (s.host) return PA_BM_ERR_STATE;
    if (count > s.tokens - first) return PA_BM_ERR_ARG;
    for (int64_t i = 0; i < count; ++i) {
      const int64_t tok = first + i;
      slots[i] = static_cast<int64_t>(s.table[static_cast<size_t>(tok / bm->block_size)]) * bm->block_size +
                 tok % bm->block_size;
    }
    return PA_BM_OK;
  });
}

int pa_bm_append_slot(pa_block_manager *bm, int64_t seq_id, int64_t *slot, int64_t *copy_src, int64_t *copy_dst) {
  return guarded(bm, [&] {
    if (!slot || !copy_src || !copy_dst) return PA_BM_ERR_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PA_BM_ERR_UNKNOWN;
    auto &s = it->second;
    if (s.host) return PA_BM_ERR_STATE;
    if (bm->append_needs_page(s, 0) && bm->dev.num_free() < 1) return PA_BM_ERR_NO_SPACE;
    s.table.reserve(s.table.size() + 1);
    bm->append(s, slot, copy_src, copy_dst);
    return PA_BM_OK;
  });
}

int pa_bm_build_decode_step(pa_block_manager *bm, const int64_t *seq_ids, int64_t num_seqs, int64_t table_stride,
                            int32_t *block_tables, int32_t *context_lens, int64_t *slot_mapping,
                            int64_t *copy_pairs, int64_t copy_capacity, int64_t *num_copies) {
  return guarded(bm, [&] {
    if (num_seqs < 0 || table_stride < 0 || copy_capacity < 0 || !num_copies) return PA_BM_ERR_ARG;
    if (num_seqs > 0 && (!seq_ids || !context_lens || !slot_mapping || (table_stride > 0 && !block_tables)))
      return PA_BM_ERR_ARG;
    // Plan: which appends need a page or a copy, simulating the references
    // that earlier appends of this step drop from shared last pages.
    std::vector<pa_block_manager::Seq *> list;
    list.reserve(static_cast<size_t>(num_seqs));
    std::unordered_set<int64_t> seen;
    std::unordered_map<int32_t, int32_t> dropped;
    int64_t pages = 0, copies = 0;
    for (int64_t i = 0; i < num_seqs; ++i) {
      auto it = bm->seqs.find(seq_ids[i]);
      if (it == bm->seqs.end()) return PA_BM_ERR_UNKNOWN;
      auto &s = it->second;
      if (s.host) return PA_BM_ERR_STATE;
      if (!seen.insert(seq_ids[i]).second) return PA_BM_ERR_ARG;
      if (s.tokens >= std::numeric_limits<int32_t>::max()) return PA_BM_ERR_ARG;  // context_lens is int32
      const bool fresh_row = s.tokens % bm->block_size == 0;
      const int32_t extra = fresh_row ? 0 : dropped[s.table.back()];
      if (bm->append_needs_page(s, extra)) {
        ++pages;
        if (!fresh_row) {
          ++copies;
          ++dropped[s.table.back()];
        }
      }
      const int64_t len = static_cast<int64_t>(s.table.size()) + (fresh_row ? 1 : 0);
      if (len > table_stride) return PA_BM_ERR_CAPACITY;
      list.push_back(&s);
    }
    *num_copies = copies;
    if (pages > bm->dev.num_free()) return PA_BM_ERR_NO_SPACE;
    if (copies > copy_capacity || (copies > 0 && !copy_pairs)) return PA_BM_ERR_CAPACITY;
    for (auto *s : list) s->table.reserve(s->table.size() + 1);
    // Mutation: cannot fail from here on.
    int64_t c = 0;
    for (int64_t i = 0; i < num_seqs; ++i) {
      auto &s = *list[static_cast<size_t>(i)];
      int64_t src, dst;
      bm->append(s, &slot_mapping[i], &src, &dst);
      if (src >= 0) {
        copy_pairs[2 * c] = src;
        copy_pairs[2 * c + 1] = dst;
        ++c;
      }
      context_lens[i] = static_cast<int32_t>(s.tokens);
      int32_t *row = block_tables + i * table_stride;
      const int64_t n = static_cast<int64_t>(s.table.size());
      std::copy(s.table.begin(), s.table.end(), row);
      std::fill(row + n, row + table_stride, -1);
    }
    return PA_BM_OK;
  });
}

int pa_bm_build_prefill_step(pa_block_manager *bm, const int64_t *seq_ids, const int64_t *new_tokens,
                             int64_t num_seqs, int64_t table_stride, int32_t *block_tables, int32_t *query_start,
                             int32_t *context_lens, int64_t *slot_mapping, int64_t slot_capacity,
                             int64_t *copy_pairs, int64_t copy_capacity, int64_t *num_copies) {
  return guarded(bm, [&] {
    if (num_seqs < 0 || table_stride < 0 || slot_capacity < 0 || copy_capacity < 0 || !num_copies || !query_start)
      return PA_BM_ERR_ARG;
    if (num_seqs > 0 && (!seq_ids || !new_tokens || !context_lens || (table_stride > 0 && !block_tables)))
      return PA_BM_ERR_ARG;
    int64_t pages = 0, copies = 0, total = 0;
    const int rc = bm->plan_step(seq_ids, new_tokens, num_seqs, table_stride, &pages, &copies, &total);
    if (rc != PA_BM_OK) return rc;
    *num_copies = copies;
    if (pages > bm->dev.num_free()) return PA_BM_ERR_NO_SPACE;
    if (total > slot_capacity || (total > 0 && !slot_mapping)) return PA_BM_ERR_CAPACITY;
    if (copies > copy_capacity || (copies > 0 && !copy_pairs)) return PA_BM_ERR_CAPACITY;
    // the planned sequences (all present: planning checked every id)
    std::vector<pa_block_manager::Seq *> list;
    list.reserve(static_cast<size_t>(num_seqs));
    for (int64_t i = 0; i < num_seqs; ++i) list.push_back(&bm->seqs.find(seq_ids[i])->second);
    for (int64_t i = 0; i < num_seqs; ++i) {
      auto *s = list[static_cast<size_t>(i)];
      s->table.reserve(static_cast<size_t>(bm->pages_for(s->tokens + new_tokens[i])));
    }
    // Mutation: cannot fail from here on.
    int64_t c = 0, row = 0;
    query_start[0] = 0;
    for (int64_t i = 0; i < num_seqs; ++i) {
      auto &s = *list[static_cast<size_t>(i)];
      for (int64_t k = 0; k < new_tokens[i]; ++k, ++row) {
        int64_t src, dst;
        bm->append(s, &slot_mapping[row], &src, &dst);
        if (src >= 0) {
          copy_pairs[2 * c] = src;
          copy_pairs[2 * c + 1] = dst;
          ++c;
        }
      }
      query_start[i + 1] = static_cast<int32_t>(row);
      context_lens[i] = static_cast<int32_t>(s.tokens);
      int32_t *trow = block_tables + i * table_stride;
      const int64_t nb = static_cast<int64_t>(s.table.size());
      std::copy(s.table.begin(), s.table.end(), trow);
      std::fill(trow + nb, trow + table_stride, -1);
    }
    return PA_BM_OK;
  });
}

int pa_bm_step_needs(const pa_block_manager *bm, const int64_t *seq_ids, const int64_t *new_tokens, int64_t num_seqs,
                     int64_t *pages, int64_t *copies) {
  if (!bm) return PA_BM_ERR_ARG;
  try {
    std::lock_guard<std::mutex> g(bm->mu);
    if (num_seqs < 0 || !pages || !copies || (num_seqs > 0 && (!seq_ids || !new_tokens))) return PA_BM_ERR_ARG;
    int64_t total = 0;
    return bm->plan_step(seq_ids, new_tokens, num_seqs, std::numeric_limits<int64_t>::max(), pages, copies, &total);
  } catch (const std::bad_alloc &) {
    return PA_BM_ERR_HOST_MEMORY;
  }
}

int pa_bm_swap_out(pa_block_manager *bm, const int64_t *seq_ids, int64_t num_seqs, int64_t *mapping,
                   int64_t capacity, int64_t *num_pairs) {
  return guarded(bm, [&] { return bm->move(seq_ids, num_seqs, true, mapping, capacity, num_pairs); });
}

int pa_bm_swap_in(pa_block_manager *bm, const int64_t *seq_ids, int64_t num_seqs, int64_t *mapping,
                  int64_t capacity, int64_t *num_pairs) {
  return guarded(bm, [&] { return bm->move(seq_ids, num_seqs, false, mapping, capacity, num_pairs); });
}

}  // extern "C"
