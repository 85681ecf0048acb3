// Host block allocator: LIFO free list, per-block reference counts, per
// request block tables, prefix sharing by fork and copy-on-write on append.
//
// "Paged attention in LLMs": a request takes a fixed-size block when it
// needs one, from wherever space is free ("The fix: stop demanding one
// continuous run"); a block table per request records where each block
// sits ("Keeping track: the block table"); requests with a common prefix
// point their tables at the same physical blocks ("Sharing blocks").  The
// quiz page "PagedAttention (vLLM)": blocks go back as a request ends, and
// beams copy a shared block on write (comparison table).
//
// Every append is all-or-nothing: mutations go through a journal that is
// rolled back when the free list runs dry.
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa_internal.h"

struct pa_alloc {
  struct Seq {
    std::vector<int32_t> table;
    int64_t len = 0;
  };
  int num_blocks = 0;
  int block_size = 0;
  std::vector<int32_t> free_stack;  // top = back()
  std::vector<int32_t> refcount;
  std::unordered_map<int64_t, Seq> seqs;

  // ---- journal of one append call
  enum Kind : int8_t { kPop, kRef, kPush, kSetLast, kLen };
  struct Entry {
    Kind kind;
    int32_t block;  // kPop: popped block; kRef: block; kSetLast: old last entry
    int64_t old;    // kRef: old count; kLen: old length
    Seq* seq;
  };
  std::vector<Entry> journal;

  bool pop(int32_t* out) {
    if (free_stack.empty()) return false;
    *out = free_stack.back();
    free_stack.pop_back();
    journal.push_back({kPop, *out, 0, nullptr});
    return true;
  }
  void set_ref(int32_t block, int32_t value) {
    journal.push_back({kRef, block, refcount[block], nullptr});
    refcount[block] = value;
  }
  void rollback() {
    for (auto it = journal.rbegin(); it != journal.rend(); ++it) {
      switch (it->kind) {
        case kPop: free_stack.push_back(it->block); break;
        case kRef: refcount[it->block] = static_cast<int32_t>(it->old); break;
        case kPush: it->seq->table.pop_back(); break;
        case kSetLast: it->seq->table.back() = it->block; break;
        case kLen: it->seq->len = it->old; break;
      }
    }
    journal.clear();
  }

  // One token onto `s`.  Returns false when a block was needed and none is
  // free (the caller rolls back).
  bool append_one(Seq* s, int64_t* slot, std::vector<int32_t>* cow) {
    const int64_t pos = s->len;
    const int offset = static_cast<int>(pos % block_size);
    int32_t block;
    if (offset == 0) {
      if (!pop(&block)) return false;
      set_ref(block, 1);
      s->table.push_back(block);
      journal.push_back({kPush, 0, 0, s});
    } else {
      block = s->table.back();
      if (refcount[block] > 1) {
        int32_t fresh;
        if (!pop(&fresh)) return false;
        cow->push_back(block);
        cow->push_back(fresh);
        set_ref(block, refcount[block] - 1);
        set_ref(fresh, 1);
        journal.push_back({kSetLast, block, 0, s});
        s->table.back() = fresh;
        block = fresh;
      }
    }
    *slot = static_cast<int64_t>(block) * block_size + offset;
    journal.push_back({kLen, 0, s->len, s});
    s->len = pos + 1;
    return true;
  }
};

namespace {

int append_impl(pa_alloc* a, const int64_t* seq_ids, int num_seqs, int tokens_each,
                int64_t* slots_out, int32_t* cow_out, int cow_cap, int* num_cow_out) {
  using pa::fail;
  if (a == nullptr || num_cow_out == nullptr)
    return fail(PA_ERR_INVALID, "pa_alloc_append: NULL handle or num_cow_out");
  if (num_seqs < 0 || tokens_each < 0 || cow_cap < 0)
    return fail(PA_ERR_INVALID, "pa_alloc_append: negative count");
  if (num_seqs > 0 && seq_ids == nullptr)
    return fail(PA_ERR_INVALID, "pa_alloc_append: NULL seq_ids");
  const int64_t total = static_cast<int64_t>(num_seqs) * tokens_each;
  if (total > 0 && slots_out == nullptr) return fail(PA_ERR_INVALID, "pa_alloc_append: NULL slots_out");
  std::vector<pa_alloc::Seq*> targets(num_seqs);
  for (int i = 0; i < num_seqs; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end())
      return fail(PA_ERR_NOT_FOUND, "pa_alloc_append: unknown sequence %lld",
                  static_cast<long long>(seq_ids[i]));
    targets[i] = &it->second;
  }
  a->journal.clear();
  std::vector<int32_t> cow;
  int64_t k = 0;
  for (int i = 0; i < num_seqs; ++i) {
    for (int t = 0; t < tokens_each; ++t, ++k) {
      if (!a->append_one(targets[i], slots_out + k, &cow)) {
        a->rollback();
        return fail(PA_ERR_OOM, "pa_alloc_append: out of blocks (%zu free at the start)",
                    a->free_stack.size());
      }
    }
  }
  const int ncow = static_cast<int>(cow.size() / 2);
  if (ncow > cow_cap || (ncow > 0 && cow_out == nullptr)) {
    a->rollback();
    return fail(PA_ERR_INVALID, "pa_alloc_append: %d copy-on-write pairs, room for %d", ncow,
                cow_cap);
  }
  if (ncow > 0) std::memcpy(cow_out, cow.data(), cow.size() * sizeof(int32_t));
  *num_cow_out = ncow;
  a->journal.clear();
  return PA_OK;
}

}  // namespace

extern "C" {

int pa_alloc_create(int num_blocks, int block_size, const int32_t* initial_order, pa_alloc** out) {
  using pa::fail;
  if (out == nullptr) return fail(PA_ERR_INVALID, "pa_alloc_create: NULL out");
  *out = nullptr;
  if (num_blocks <= 0 || block_size <= 0)
    return fail(PA_ERR_INVALID, "pa_alloc_create: num_blocks and block_size must be positive");
  pa_alloc* a = new (std::nothrow) pa_alloc();
  if (a == nullptr) return fail(PA_ERR_OOM, "pa_alloc_create: host allocation failed");
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->refcount.assign(num_blocks, 0);
  a->free_stack.resize(num_blocks);
  if (initial_order != nullptr) {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      const int32_t blk = initial_order[i];
      if (blk < 0 || blk >= num_blocks || seen[blk]) {
        delete a;
        return fail(PA_ERR_INVALID, "pa_alloc_create: initial_order is not a permutation");
      }
      seen[blk] = 1;
      a->free_stack[num_blocks - 1 - i] = blk;  // first entry on top
    }
  } else {
    for (int i = 0; i < num_blocks; ++i) a->free_stack[num_blocks - 1 - i] = i;
  }
  *out = a;
  return PA_OK;
}

int pa_alloc_destroy(pa_alloc* a) {
  delete a;
  return PA_OK;
}

int pa_alloc_add_seq(pa_alloc* a, int64_t seq_id) {
  if (a == nullptr) return pa::fail(PA_ERR_INVALID, "pa_alloc_add_seq: NULL handle");
  if (a->seqs.count(seq_id))
    return pa::fail(PA_ERR_EXISTS, "pa_alloc_add_seq: sequence %lld exists", static_cast<long long>(seq_id));
  a->seqs.emplace(seq_id, pa_alloc::Seq());
  return PA_OK;
}

int pa_alloc_fork(pa_alloc* a, int64_t parent, int64_t child) {
  if (a == nullptr) return pa::fail(PA_ERR_INVALID, "pa_alloc_fork: NULL handle");
  auto it = a->seqs.find(parent);
  if (it == a->seqs.end())
    return pa::fail(PA_ERR_NOT_FOUND, "pa_alloc_fork: unknown parent %lld", static_cast<long long>(parent));
  if (a->seqs.count(child))
    return pa::fail(PA_ERR_EXISTS, "pa_alloc_fork: child %lld exists", static_cast<long long>(child));
  pa_alloc::Seq copy = it->second;
  for (int32_t blk : copy.table) ++a->refcount[blk];
  a->seqs.emplace(child, std::move(copy));
  return PA_OK;
}

int pa_alloc_append(pa_alloc* a, int64_t seq_id, int num_tokens, int64_t* slots_out,
                    int32_t* cow_pairs_out, int cow_cap, int* num_cow_out) {
  return append_impl(a, &seq_id, 1, num_tokens, slots_out, cow_pairs_out, cow_cap, num_cow_out);
}

int pa_alloc_append_batch(pa_alloc* a, const int64_t* seq_ids, int num_seqs, int tokens_each,
                          int64_t* slots_out, int32_t* cow_pairs_out, int cow_cap,
                          int* num_cow_out) {
  return append_impl(a, seq_ids, num_seqs, tokens_each, slots_out, cow_pairs_out, cow_cap,
                     num_cow_out);
}

int pa_alloc_free_seq(pa_alloc* a, int64_t seq_id) {
  if (a == nullptr) return pa::fail(PA_ERR_INVALID, "pa_alloc_free_seq: NULL handle");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end())
    return pa::fail(PA_ERR_NOT_FOUND, "pa_alloc_free_seq: unknown sequence %lld", static_cast<long long>(seq_id));
  for (int32_t blk : it->second.table)
    if (--a->refcount[blk] == 0) a->free_stack.push_back(blk);
  a->seqs.erase(it);
  return PA_OK;
}

int pa_alloc_num_free(const pa_alloc* a, int* out) {
  if (a == nullptr || out == nullptr) return pa::fail(PA_ERR_INVALID, "pa_alloc_num_free: NULL argument");
  *out = static_cast<int>(a->free_stack.size());
  return PA_OK;
}

int pa_alloc_seq_len(const pa_alloc* a, int64_t seq_id, int* out) {
  if (a == nullptr || out == nullptr) return pa::fail(PA_ERR_INVALID, "pa_alloc_seq_len: NULL argument");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end())
    return pa::fail(PA_ERR_NOT_FOUND, "pa_alloc_seq_len: unknown sequence %lld", static_cast<long long>(seq_id));
  *out = static_cast<int>(it->second.len);
  return PA_OK;
}

int pa_alloc_refcount(const pa_alloc* a, int block, int* out) {
  if (a == nullptr || out == nullptr) return pa::fail(PA_ERR_INVALID, "pa_alloc_refcount: NULL argument");
  if (block < 0 || block >= a->num_blocks)
    return pa::fail(PA_ERR_INVALID, "pa_alloc_refcount: block %d outside [0, %d)", block, a->num_blocks);
  *out = a->refcount[block];
  return PA_OK;
}

int pa_alloc_block_table(const pa_alloc* a, int64_t seq_id, int32_t* out, int cap, int* n_out) {
  if (a == nullptr || n_out == nullptr) return pa::fail(PA_ERR_INVALID, "pa_alloc_block_table: NULL argument");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end())
    return pa::fail(PA_ERR_NOT_FOUND, "pa_alloc_block_table: unknown sequence %lld", static_cast<long long>(seq_id));
  const auto& t = it->second.table;
  if (static_cast<int64_t>(t.size()) > cap || (!t.empty() && out == nullptr))
    return pa::fail(PA_ERR_INVALID, "pa_alloc_block_table: table of %zu entries, room for %d", t.size(), cap);
  if (!t.empty()) std::memcpy(out, t.data(), t.size() * sizeof(int32_t));
  *n_out = static_cast<int>(t.size());
  return PA_OK;
}

int pa_alloc_block_tables(const pa_alloc* a, const int64_t* seq_ids, int num_seqs,
                          int max_blocks_per_seq, int32_t* tables_out, int32_t* seq_lens_out) {
  if (a == nullptr || (num_seqs > 0 && (seq_ids == nullptr || tables_out == nullptr || seq_lens_out == nullptr)))
    return pa::fail(PA_ERR_INVALID, "pa_alloc_block_tables: NULL argument");
  if (num_seqs < 0 || max_blocks_per_seq <= 0)
    return pa::fail(PA_ERR_INVALID, "pa_alloc_block_tables: bad sizes");
  for (int i = 0; i < num_seqs; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end())
      return pa::fail(PA_ERR_NOT_FOUND, "pa_alloc_block_tables: unknown sequence %lld",
                      static_cast<long long>(seq_ids[i]));
    const auto& t = it->second.table;
    if (static_cast<int64_t>(t.size()) > max_blocks_per_seq)
      return pa::fail(PA_ERR_INVALID, "pa_alloc_block_tables: table of %zu entries, row of %d",
                      t.size(), max_blocks_per_seq);
  }
  for (int i = 0; i < num_seqs; ++i) {
    const auto& s = a->seqs.find(seq_ids[i])->second;
    int32_t* row = tables_out + static_cast<int64_t>(i) * max_blocks_per_seq;
    if (!s.table.empty()) std::memcpy(row, s.table.data(), s.table.size() * sizeof(int32_t));
    std::memset(row + s.table.size(), 0, (max_blocks_per_seq - s.table.size()) * sizeof(int32_t));
    seq_lens_out[i] = static_cast<int32_t>(s.len);
  }
  return PA_OK;
}

int pa_alloc_stats(const pa_alloc* a, int64_t* stats_out) {
  if (a == nullptr || stats_out == nullptr) return pa::fail(PA_ERR_INVALID, "pa_alloc_stats: NULL argument");
  int64_t tokens = 0, logical = 0;
  for (const auto& kv : a->seqs) {
    tokens += kv.second.len;
    logical += static_cast<int64_t>(kv.second.table.size()) * a->block_size;
  }
  const int64_t free_blocks = static_cast<int64_t>(a->free_stack.size());
  stats_out[0] = tokens;
  stats_out[1] = logical;
  stats_out[2] = a->num_blocks - free_blocks;
  stats_out[3] = static_cast<int64_t>(a->seqs.size());
  stats_out[4] = free_blocks;
  return PA_OK;
}

int pa_alloc_dump(const pa_alloc* a, int32_t* free_list_out, int* num_free_out,
                  int32_t* refcounts_out) {
  if (a == nullptr || free_list_out == nullptr || num_free_out == nullptr || refcounts_out == nullptr)
    return pa::fail(PA_ERR_INVALID, "pa_alloc_dump: NULL argument");
  const size_t nf = a->free_stack.size();
  for (size_t i = 0; i < nf; ++i) free_list_out[i] = a->free_stack[nf - 1 - i];
  *num_free_out = static_cast<int>(nf);
  std::memcpy(refcounts_out, a->refcount.data(), a->refcount.size() * sizeof(int32_t));
  return PA_OK;
}

}  // extern "C"
