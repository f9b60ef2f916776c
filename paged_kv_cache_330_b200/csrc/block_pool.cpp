// Host block pool: the Block / BlockTable bookkeeping of the page
// "Nano-vLLM-Ascend: lightweight LLM inference framework for Ascend NPU",
// section 2.1 (16-token blocks, logical -> physical block map per sequence,
// a reference count per block), with the single-pool allocator role of
// BlockAllocator from "Ascend NPU LLM inference optimisation: the vLLM-Ascend
// approach", section 2.1, and block sharing across sequences (same page,
// section 4).
//
// The pool is pure host bookkeeping over block ids; the K/V bytes live in the
// caller's device tensors.  Every operation checks first and mutates second,
// so a failed call leaves the pool unchanged.

#include <algorithm>
#include <cstdint>
#include <unordered_map>
#include <vector>

#include "paged_attn.h"

// The free list is a ring of num_blocks entries allocated once at creation: a block is in it at most once,
// so handing blocks out and taking them back never allocates, and an operation cannot fail half-way.
struct FreeRing {
  std::vector<int32_t> slot;
  size_t head = 0, count = 0;
  size_t size() const { return count; }
  int32_t pop_front() {
    const int32_t b = slot[head];
    head = (head + 1) % slot.size();
    --count;
    return b;
  }
  void push_back(int32_t b) {
    slot[(head + count) % slot.size()] = b;
    ++count;
  }
};

struct pa_pool {
  int num_blocks = 0;
  int block_size = 0;
  FreeRing free_list;                   // head = next block handed out
  std::vector<int32_t> ref;             // reference count per physical block
  struct Seq {
    std::vector<int32_t> blocks;        // logical block j -> physical block
    int64_t len = 0;                    // tokens
    uint64_t mark = 0;                  // last batch that named this sequence (repeat detection)
  };
  std::unordered_map<int64_t, Seq> seqs;
  uint64_t batch_epoch = 0;
  std::vector<pa_pool::Seq*> batch_seqs;                      // scratch of pa_pool_append_batch
  std::vector<std::pair<int32_t, int32_t>> batch_released;    // (block, references dropped by copies)

  int32_t take() {
    const int32_t b = free_list.pop_front();
    ref[b] = 1;
    return b;
  }
};

static inline int64_t blocks_for(int64_t n, int bs) { return (n + bs - 1) / bs; }

// Every call below does all of its allocation before it changes the pool, and no exception leaves the C
// ABI: an allocation failure is reported as PA_ERR_OOM (NULL from pa_pool_create) with the pool unchanged.

extern "C" pa_pool* pa_pool_create(int num_blocks, int block_size, const int32_t* free_order) {
  if (num_blocks < 0 || block_size <= 0) return nullptr;
  pa_pool* p = nullptr;
  try {
    p = new pa_pool;
    p->num_blocks = num_blocks;
    p->block_size = block_size;
    p->ref.assign(num_blocks, 0);
    p->free_list.slot.assign(num_blocks, 0);
    if (free_order) {
      std::vector<char> seen(num_blocks, 0);
      for (int i = 0; i < num_blocks; ++i) {
        const int32_t b = free_order[i];
        if (b < 0 || b >= num_blocks || seen[b]) {
          delete p;
          return nullptr;
        }
        seen[b] = 1;
        p->free_list.push_back(b);
      }
    } else {
      for (int i = 0; i < num_blocks; ++i) p->free_list.push_back(i);
    }
    return p;
  } catch (...) {
    delete p;
    return nullptr;
  }
}

extern "C" void pa_pool_destroy(pa_pool* pool) { delete pool; }

extern "C" int pa_seq_alloc(pa_pool* pool, int64_t seq_id, int num_tokens) {
  if (!pool || num_tokens < 0) return PA_ERR_INVALID;
  try {
    if (pool->seqs.count(seq_id)) return PA_ERR_NOT_FOUND;
    const int64_t need = blocks_for(num_tokens, pool->block_size);
    if (need > (int64_t)pool->free_list.size()) return PA_ERR_OOM;
    pa_pool::Seq s;
    s.blocks.reserve(need);
    s.len = num_tokens;
    pa_pool::Seq& in = pool->seqs.emplace(seq_id, std::move(s)).first->second;
    for (int64_t i = 0; i < need; ++i) in.blocks.push_back(pool->take());  // within capacity: no allocation
    return PA_OK;
  } catch (...) {
    return PA_ERR_OOM;
  }
}

extern "C" int pa_seq_fork(pa_pool* pool, int64_t parent_id, int64_t child_id, int n_prefix) {
  if (!pool || n_prefix < 0) return PA_ERR_INVALID;
  try {
    auto it = pool->seqs.find(parent_id);
    if (it == pool->seqs.end() || pool->seqs.count(child_id)) return PA_ERR_NOT_FOUND;
    if (n_prefix > it->second.len) return PA_ERR_INVALID;
    pa_pool::Seq c;
    const int64_t nb = blocks_for(n_prefix, pool->block_size);
    c.blocks.assign(it->second.blocks.begin(), it->second.blocks.begin() + nb);
    c.len = n_prefix;
    const pa_pool::Seq& in = pool->seqs.emplace(child_id, std::move(c)).first->second;
    for (int32_t b : in.blocks) pool->ref[b] += 1;
    return PA_OK;
  } catch (...) {
    return PA_ERR_OOM;
  }
}

// Does appending n tokens to s first copy its last block?  (A shared, partly filled last block.)
static bool needs_copy(const pa_pool* pool, const pa_pool::Seq& s, int64_t n) {
  return n > 0 && (s.len % pool->block_size) != 0 && pool->ref[s.blocks.back()] > 1;
}

// Blocks the pool must hand out to append n tokens to s (including the copy, if any).
static int64_t blocks_needed(const pa_pool* pool, const pa_pool::Seq& s, int64_t n, bool copy) {
  return blocks_for(s.len + n, pool->block_size) - (int64_t)s.blocks.size() + (copy ? 1 : 0);
}

// The state change of one append, once it is known to fit and s.blocks has the capacity: no allocation,
// cannot fail.  Writes the slots of the new tokens and returns whether the last block was copied.
static bool append_tokens(pa_pool* pool, pa_pool::Seq& s, int64_t n, int64_t* slots_out, int32_t* pair_out) {
  const int bs = pool->block_size;
  const int64_t n0 = s.len;
  const bool cow = needs_copy(pool, s, n);
  if (cow) {
    const int32_t old_b = s.blocks.back();
    const int32_t new_b = pool->take();
    pool->ref[old_b] -= 1;
    s.blocks.back() = new_b;
    if (pair_out) {
      pair_out[0] = old_b;
      pair_out[1] = new_b;
    }
  }
  for (int64_t p = n0; p < n0 + n; ++p) {
    if (p % bs == 0) s.blocks.push_back(pool->take());  // within capacity: no allocation
    if (slots_out) slots_out[p - n0] = (int64_t)s.blocks[p / bs] * bs + p % bs;
  }
  s.len = n0 + n;
  return cow;
}

extern "C" int pa_seq_append(pa_pool* pool, int64_t seq_id, int n, int64_t* slot_mapping_out,
                             int32_t* cow_pairs_out, int* num_cow_out) {
  if (!pool || n < 0) return PA_ERR_INVALID;
  try {
    auto it = pool->seqs.find(seq_id);
    if (it == pool->seqs.end()) return PA_ERR_NOT_FOUND;
    pa_pool::Seq& s = it->second;
    const int64_t need = blocks_needed(pool, s, n, needs_copy(pool, s, n));
    if (need > (int64_t)pool->free_list.size()) return PA_ERR_OOM;
    s.blocks.reserve(blocks_for(s.len + n, pool->block_size));
    const bool cow = append_tokens(pool, s, n, slot_mapping_out, cow_pairs_out);
    if (num_cow_out) *num_cow_out = cow ? 1 : 0;
    return PA_OK;
  } catch (...) {
    return PA_ERR_OOM;
  }
}

extern "C" int pa_pool_append_batch(pa_pool* pool, const int64_t* seq_ids, const int32_t* counts, int n,
                                    int64_t* slot_mapping_out, int32_t* cow_pairs_out, int* num_cow_out) {
  if (!pool || n < 0 || (n > 0 && (!seq_ids || !counts))) return PA_ERR_INVALID;
  try {
    // Dry run: find every sequence, reject repeats, and count the blocks the batch takes.  A copy made for
    // one sequence lowers the count of a block another sequence of the batch may share, exactly as
    // separate calls in this order would see it (`released`, short: copies are rare).
    std::vector<pa_pool::Seq*>& seq = pool->batch_seqs;
    auto& released = pool->batch_released;
    seq.resize(n);
    released.clear();
    const uint64_t epoch = ++pool->batch_epoch;
    int64_t need = 0;
    for (int i = 0; i < n; ++i) {
      if (counts[i] < 0) return PA_ERR_INVALID;
      auto it = pool->seqs.find(seq_ids[i]);
      if (it == pool->seqs.end()) return PA_ERR_NOT_FOUND;
      pa_pool::Seq& s = it->second;
      if (s.mark == epoch) return PA_ERR_INVALID;  // named twice in this batch
      s.mark = epoch;
      seq[i] = &s;
      bool copy = false;
      if (counts[i] > 0 && (s.len % pool->block_size) != 0) {
        const int32_t last = s.blocks.back();
        int32_t dropped = 0;
        size_t k = 0;
        for (; k < released.size() && released[k].first != last; ++k) {
        }
        if (k < released.size()) dropped = released[k].second;
        copy = pool->ref[last] - dropped > 1;
        if (copy) {
          if (k < released.size())
            released[k].second += 1;
          else
            released.emplace_back(last, 1);
        }
      }
      need += blocks_needed(pool, s, counts[i], copy);
    }
    if (need > (int64_t)pool->free_list.size()) return PA_ERR_OOM;
    for (int i = 0; i < n; ++i) seq[i]->blocks.reserve(blocks_for(seq[i]->len + counts[i], pool->block_size));
    // Apply: nothing below allocates or fails.
    int64_t off = 0;
    int ncow = 0;
    for (int i = 0; i < n; ++i) {
      int32_t* pair = cow_pairs_out ? cow_pairs_out + 2 * ncow : nullptr;
      if (append_tokens(pool, *seq[i], counts[i], slot_mapping_out ? slot_mapping_out + off : nullptr, pair)) ++ncow;
      off += counts[i];
    }
    if (num_cow_out) *num_cow_out = ncow;
    return PA_OK;
  } catch (...) {
    return PA_ERR_OOM;
  }
}

// Marks every id of a batch (a sequence named twice is an error); `must_exist` selects whether each id must
// name a live sequence or a free one.  Returns PA_OK or the error of the first offending id; sets nothing.
static int check_batch_ids(pa_pool* pool, const int64_t* ids, int n, bool must_exist, std::vector<int64_t>& seen) {
  seen.assign(ids, ids + n);
  std::sort(seen.begin(), seen.end());
  if (std::adjacent_find(seen.begin(), seen.end()) != seen.end()) return PA_ERR_INVALID;
  for (int i = 0; i < n; ++i) {
    const bool live = pool->seqs.count(ids[i]) != 0;
    if (live != must_exist) return PA_ERR_NOT_FOUND;
  }
  return PA_OK;
}

extern "C" int pa_pool_alloc_batch(pa_pool* pool, const int64_t* seq_ids, const int32_t* num_tokens, int n) {
  if (!pool || n < 0 || (n > 0 && (!seq_ids || !num_tokens))) return PA_ERR_INVALID;
  int inserted = 0;  // batch ids this call has put into the pool (ids 0..inserted-1, each absent on entry)
  try {
    std::vector<int64_t> scratch;
    const int st = check_batch_ids(pool, seq_ids, n, false, scratch);
    if (st != PA_OK) return st;
    int64_t need = 0;
    for (int i = 0; i < n; ++i) {
      if (num_tokens[i] < 0) return PA_ERR_INVALID;
      need += blocks_for(num_tokens[i], pool->block_size);
    }
    if (need > (int64_t)pool->free_list.size()) return PA_ERR_OOM;
    // every node and vector is allocated before the first block is taken
    std::vector<pa_pool::Seq*> made(n);
    for (int i = 0; i < n; ++i) {
      pa_pool::Seq s;
      s.blocks.reserve(blocks_for(num_tokens[i], pool->block_size));
      s.len = num_tokens[i];
      auto res = pool->seqs.emplace(seq_ids[i], std::move(s));
      made[i] = &res.first->second;
      inserted = i + 1;
    }
    for (int i = 0; i < n; ++i)
      for (int64_t j = 0, nb = blocks_for(num_tokens[i], pool->block_size); j < nb; ++j)
        made[i]->blocks.push_back(pool->take());
    return PA_OK;
  } catch (...) {
    // Only the id check or an insertion can throw, before any block is taken.  Remove exactly the sequences
    // inserted here (they hold no blocks yet); a sequence that was live on entry is never touched.
    for (int i = 0; i < inserted; ++i) pool->seqs.erase(seq_ids[i]);
    return PA_ERR_OOM;
  }
}

extern "C" int pa_pool_free_batch(pa_pool* pool, const int64_t* seq_ids, int n) {
  if (!pool || n < 0 || (n > 0 && !seq_ids)) return PA_ERR_INVALID;
  try {
    std::vector<int64_t> scratch;
    const int st = check_batch_ids(pool, seq_ids, n, true, scratch);
    if (st != PA_OK) return st;
  } catch (...) {
    return PA_ERR_OOM;
  }
  for (int i = 0; i < n; ++i) pa_seq_free(pool, seq_ids[i]);  // cannot fail now: every id is live and distinct
  return PA_OK;
}

extern "C" int pa_seq_free(pa_pool* pool, int64_t seq_id) {
  if (!pool) return PA_ERR_INVALID;
  auto it = pool->seqs.find(seq_id);
  if (it == pool->seqs.end()) return PA_ERR_NOT_FOUND;
  for (int32_t b : it->second.blocks) {
    pool->ref[b] -= 1;
    if (pool->ref[b] == 0) pool->free_list.push_back(b);  // the ring has room for every block
  }
  pool->seqs.erase(it);
  return PA_OK;
}

extern "C" int pa_seq_info(const pa_pool* pool, int64_t seq_id, int* len_out, int* blocks_out) {
  if (!pool) return PA_ERR_INVALID;
  auto it = pool->seqs.find(seq_id);
  if (it == pool->seqs.end()) return PA_ERR_NOT_FOUND;
  if (len_out) *len_out = (int)it->second.len;
  if (blocks_out) *blocks_out = (int)it->second.blocks.size();
  return PA_OK;
}

extern "C" int pa_pool_block_table(const pa_pool* pool, const int64_t* seq_ids, int n, int32_t* out,
                                   int max_blocks, int32_t* ctx_lens_out) {
  if (!pool || n < 0 || max_blocks < 0 || (n > 0 && (!seq_ids || !out))) return PA_ERR_INVALID;
  for (int i = 0; i < n; ++i) {  // check every row before writing any
    auto it = pool->seqs.find(seq_ids[i]);
    if (it == pool->seqs.end()) return PA_ERR_NOT_FOUND;
    if ((int64_t)it->second.blocks.size() > max_blocks) return PA_ERR_INVALID;
  }
  for (int i = 0; i < n; ++i) {
    const pa_pool::Seq& s = pool->seqs.find(seq_ids[i])->second;
    int32_t* row = out + (int64_t)i * max_blocks;
    size_t j = 0;
    for (; j < s.blocks.size(); ++j) row[j] = s.blocks[j];
    for (; j < (size_t)max_blocks; ++j) row[j] = -1;
    if (ctx_lens_out) ctx_lens_out[i] = (int32_t)s.len;
  }
  return PA_OK;
}

extern "C" int pa_pool_ref_count(const pa_pool* pool, int block_id) {
  if (!pool || block_id < 0 || block_id >= pool->num_blocks) return -1;
  return pool->ref[block_id];
}

extern "C" int pa_pool_stats(const pa_pool* pool, pa_pool_stats_t* out) {
  if (!pool || !out) return PA_ERR_INVALID;
  pa_pool_stats_t st{};
  st.num_blocks = pool->num_blocks;
  st.free_blocks = (int64_t)pool->free_list.size();
  for (int32_t r : pool->ref) {
    if (r > 0) st.used_blocks++;
    if (r > 1) st.shared_blocks++;
    st.ref_sum += r;
  }
  st.num_seqs = (int64_t)pool->seqs.size();
  for (const auto& kv : pool->seqs) {
    st.tokens += kv.second.len;
    st.table_refs += (int64_t)kv.second.blocks.size();
  }
  st.utilisation = st.table_refs ? (double)st.tokens / ((double)st.table_refs * pool->block_size) : 1.0;
  *out = st;
  return PA_OK;
}
