// pa_block_manager.cpp -- host manager of the paged KV pool (see include/pa_block_manager.h for the
// scheme and its sources). Plain C++: a vector stack of free blocks, a vector of reference counts and
// a hash map of sequences. Every entry point validates and checks capacity first, then performs every
// host allocation it needs (vector capacity, hash-map nodes), and only then mutates with operations
// that cannot throw, so a failed call -- an out-of-memory one included -- changes nothing. No
// exception crosses the C ABI: each entry point runs inside guarded(), which turns one into
// PA_ERR_HOST_MEMORY.
#include "pa_block_manager.h"

#include <algorithm>
#include <climits>
#include <exception>
#include <cstdint>
#include <mutex>
#include <new>
#include <unordered_map>
#include <unordered_set>
#include <vector>

namespace {

struct Sequence {
  std::vector<int32_t> blocks;  // device blocks when resident, host blocks when swapped
  int64_t tokens = 0;
  bool swapped = false;
};

}  // namespace

struct pa_block_manager {
  int num_blocks = 0;
  int block_size = 0;
  int num_host_blocks = 0;
  std::vector<int32_t> free_stack;  // back() is the top
  std::vector<int32_t> host_free;
  std::vector<int32_t> ref;
  std::unordered_map<int64_t, Sequence> seqs;
  std::mutex mu;

  int64_t blocks_for(int64_t tokens) const { return (tokens + block_size - 1) / block_size; }

  int32_t take() {
    const int32_t b = free_stack.back();
    free_stack.pop_back();
    ref[b] = 1;
    return b;
  }

  void release(int32_t b) {
    if (--ref[b] == 0) free_stack.push_back(b);
  }

  Sequence* resident(int64_t id) {
    auto it = seqs.find(id);
    return (it == seqs.end() || it->second.swapped) ? nullptr : &it->second;
  }

  // A sequence already known to exist (ids are validated before this is used); never inserts.
  Sequence& existing(int64_t id) { return seqs.find(id)->second; }

  // Does sequence s need a fresh block for its next token (a new block, or a copy of a shared one)?
  bool needs_block(const Sequence& s) const {
    if (s.tokens % block_size == 0) return true;
    return ref[s.blocks[s.tokens / block_size]] > 1;
  }

  bool distinct_resident(const int64_t* ids, int n) {
    std::unordered_set<int64_t> seen;
    seen.reserve(static_cast<size_t>(n) * 2);
    for (int i = 0; i < n; ++i)
      if (!resident(ids[i]) || !seen.insert(ids[i]).second) return false;
    return true;
  }

  // The append step itself; capacity already checked and reserved, so nothing here allocates.
  void append(const int64_t* ids, int n, int64_t* slots, int64_t* pairs, int* num_pairs) {
    int np = 0;
    for (int i = 0; i < n; ++i) {
      Sequence& s = existing(ids[i]);
      const int64_t logical = s.tokens / block_size;
      if (s.tokens % block_size == 0) {
        s.blocks.push_back(take());
      } else {
        const int32_t last = s.blocks[logical];
        if (ref[last] > 1) {
          const int32_t fresh = take();
          pairs[2 * np] = last;
          pairs[2 * np + 1] = fresh;
          ++np;
          release(last);
          s.blocks[logical] = fresh;
        }
      }
      slots[i] = static_cast<int64_t>(s.blocks[logical]) * block_size + s.tokens % block_size;
      ++s.tokens;
    }
    *num_pairs = np;
  }

  // Validates an append and reserves the block-list room it needs (a capacity change only, so the
  // manager's state is the same whether or not the append then happens).
  pa_status check_append(const int64_t* ids, int n) {
    if (!distinct_resident(ids, n)) return PA_ERR_INVALID_ARGUMENT;
    int64_t need = 0;
    for (int i = 0; i < n; ++i) need += needs_block(existing(ids[i])) ? 1 : 0;
    if (need > static_cast<int64_t>(free_stack.size())) return PA_ERR_OUT_OF_BLOCKS;
    for (int i = 0; i < n; ++i) {
      Sequence& s = existing(ids[i]);
      if (s.tokens % block_size == 0) s.blocks.reserve(s.blocks.size() + 1);
    }
    return PA_OK;
  }

  pa_status check_tables(const int64_t* ids, int n, int max_blocks) {
    for (int i = 0; i < n; ++i) {
      Sequence* s = resident(ids[i]);
      if (!s) return PA_ERR_INVALID_ARGUMENT;
      if (static_cast<int64_t>(s->blocks.size()) > max_blocks || s->tokens > INT32_MAX)
        return PA_ERR_INVALID_ARGUMENT;
    }
    return PA_OK;
  }

  void tables(const int64_t* ids, int n, int32_t* out, int max_blocks, int32_t pad, int32_t* lens) {
    for (int i = 0; i < n; ++i) {
      const Sequence& s = existing(ids[i]);
      int32_t* row = out + static_cast<int64_t>(i) * max_blocks;
      const int nb = static_cast<int>(s.blocks.size());
      for (int j = 0; j < nb; ++j) row[j] = s.blocks[j];
      for (int j = nb; j < max_blocks; ++j) row[j] = pad;
      lens[i] = static_cast<int32_t>(s.tokens);
    }
  }
};

namespace {

// Runs one entry point's body; an exception (in practice std::bad_alloc from a host allocation,
// which every body performs before mutating) becomes PA_ERR_HOST_MEMORY instead of crossing the ABI.
template <typename F>
pa_status guarded(F&& body) {
  try {
    return body();
  } catch (...) {
    return PA_ERR_HOST_MEMORY;
  }
}

}  // namespace

extern "C" {

pa_status pa_bm_create(int num_blocks, int block_size, int num_host_blocks, pa_block_manager** out) {
  if (!out || num_blocks <= 0 || block_size <= 0 || num_host_blocks < 0) return PA_ERR_INVALID_ARGUMENT;
  return guarded([&] {
    pa_block_manager* bm = new pa_block_manager();
    try {
      bm->num_blocks = num_blocks;
      bm->block_size = block_size;
      bm->num_host_blocks = num_host_blocks;
      bm->ref.assign(num_blocks, 0);
      // Full capacity up front: releasing a block or a host block later never reallocates.
      bm->free_stack.reserve(num_blocks);
      for (int b = num_blocks - 1; b >= 0; --b) bm->free_stack.push_back(b);
      bm->host_free.reserve(num_host_blocks);
      for (int b = num_host_blocks - 1; b >= 0; --b) bm->host_free.push_back(b);
    } catch (...) {
      delete bm;
      throw;
    }
    *out = bm;
    return PA_OK;
  });
}

void pa_bm_destroy(pa_block_manager* bm) { delete bm; }

pa_status pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, int64_t num_tokens, int64_t prefix_seq,
                             int64_t prefix_tokens, int64_t* slots_out, int64_t slots_capacity,
                             int64_t* num_slots_out) {
  if (!bm || !num_slots_out || seq_id < 0 || num_tokens < 0 || prefix_tokens < 0 || prefix_tokens > num_tokens)
    return PA_ERR_INVALID_ARGUMENT;
  if (slots_capacity < num_tokens || (num_tokens > 0 && !slots_out)) return PA_ERR_INVALID_ARGUMENT;
  return guarded([&] {
    std::lock_guard<std::mutex> lock(bm->mu);
    if (bm->seqs.count(seq_id)) return PA_ERR_INVALID_ARGUMENT;
    // A sequence never holds more tokens than the whole pool (shared blocks are pool blocks too);
    // checked first so that the block count below cannot overflow.
    if (num_tokens > static_cast<int64_t>(bm->num_blocks) * bm->block_size) return PA_ERR_OUT_OF_BLOCKS;
    const Sequence* parent = nullptr;
    int64_t shared = 0;
    if (prefix_seq != PA_BM_NO_SEQUENCE) {
      parent = bm->resident(prefix_seq);
      if (!parent) return PA_ERR_INVALID_ARGUMENT;
      shared = std::min(prefix_tokens, parent->tokens) / bm->block_size;
    }
    const int64_t need = bm->blocks_for(num_tokens) - shared;
    if (need > static_cast<int64_t>(bm->free_stack.size())) return PA_ERR_OUT_OF_BLOCKS;
    // Allocate first (the block list and the map node), then take blocks: nothing below throws.
    Sequence s;
    s.tokens = num_tokens;
    s.blocks.reserve(static_cast<size_t>(shared + need));
    Sequence& slot = bm->seqs.emplace(seq_id, Sequence{}).first->second;
    for (int64_t j = 0; j < shared; ++j) {
      const int32_t b = parent->blocks[j];
      ++bm->ref[b];
      s.blocks.push_back(b);
    }
    for (int64_t j = 0; j < need; ++j) s.blocks.push_back(bm->take());
    const int bs = bm->block_size;
    int64_t k = 0;
    for (int64_t t = shared * bs; t < num_tokens; ++t, ++k)
      slots_out[k] = static_cast<int64_t>(s.blocks[t / bs]) * bs + t % bs;
    *num_slots_out = k;
    slot = std::move(s);
    return PA_OK;
  });
}

pa_status pa_bm_fork(pa_block_manager* bm, int64_t parent, int64_t child) {
  if (!bm || child < 0) return PA_ERR_INVALID_ARGUMENT;
  return guarded([&] {
    std::lock_guard<std::mutex> lock(bm->mu);
    const Sequence* p = bm->resident(parent);
    if (!p || bm->seqs.count(child)) return PA_ERR_INVALID_ARGUMENT;
    Sequence c = *p;  // allocations first: the copy, then the map node
    Sequence& slot = bm->seqs.emplace(child, Sequence{}).first->second;
    for (int32_t b : c.blocks) ++bm->ref[b];
    slot = std::move(c);
    return PA_OK;
  });
}

pa_status pa_bm_append_slots(pa_block_manager* bm, const int64_t* seq_ids, int n, int64_t* slot_mapping_out,
                             int64_t* cow_pairs_out, int* num_cow_out) {
  if (!bm || n < 0 || !num_cow_out || (n > 0 && (!seq_ids || !slot_mapping_out || !cow_pairs_out)))
    return PA_ERR_INVALID_ARGUMENT;
  return guarded([&] {
    std::lock_guard<std::mutex> lock(bm->mu);
    const pa_status st = bm->check_append(seq_ids, n);
    if (st != PA_OK) return st;
    bm->append(seq_ids, n, slot_mapping_out, cow_pairs_out, num_cow_out);
    return PA_OK;
  });
}

pa_status pa_bm_block_tables(pa_block_manager* bm, const int64_t* seq_ids, int n, int32_t* tables_out,
                             int max_blocks, int32_t pad, int32_t* context_lens_out) {
  if (!bm || n < 0 || max_blocks < 0 || (n > 0 && (!seq_ids || !context_lens_out || (max_blocks > 0 && !tables_out))))
    return PA_ERR_INVALID_ARGUMENT;
  return guarded([&] {
    std::lock_guard<std::mutex> lock(bm->mu);
    const pa_status st = bm->check_tables(seq_ids, n, max_blocks);
    if (st != PA_OK) return st;
    bm->tables(seq_ids, n, tables_out, max_blocks, pad, context_lens_out);
    return PA_OK;
  });
}

pa_status pa_bm_plan_decode(pa_block_manager* bm, const int64_t* seq_ids, int n, int64_t* slot_mapping_out,
                            int64_t* cow_pairs_out, int* num_cow_out, int32_t* tables_out, int max_blocks,
                            int32_t pad, int32_t* context_lens_out) {
  if (!bm || n < 0 || max_blocks < 0 || !num_cow_out ||
      (n > 0 && (!seq_ids || !slot_mapping_out || !cow_pairs_out || !context_lens_out ||
                 (max_blocks > 0 && !tables_out))))
    return PA_ERR_INVALID_ARGUMENT;
  return guarded([&] {
    std::lock_guard<std::mutex> lock(bm->mu);
    pa_status st = bm->check_append(seq_ids, n);
    if (st != PA_OK) return st;
    // The tables after the append: a sequence gains a block exactly when its length is a multiple of
    // the block size; the length must still fit int32.
    for (int i = 0; i < n; ++i) {
      const Sequence& s = bm->existing(seq_ids[i]);
      const int64_t blocks_after =
          static_cast<int64_t>(s.blocks.size()) + (s.tokens % bm->block_size == 0 ? 1 : 0);
      if (blocks_after > max_blocks || s.tokens + 1 > INT32_MAX) return PA_ERR_INVALID_ARGUMENT;
    }
    bm->append(seq_ids, n, slot_mapping_out, cow_pairs_out, num_cow_out);
    bm->tables(seq_ids, n, tables_out, max_blocks, pad, context_lens_out);
    return PA_OK;
  });
}

pa_status pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id) {
  if (!bm) return PA_ERR_INVALID_ARGUMENT;
  return guarded([&] {
    std::lock_guard<std::mutex> lock(bm->mu);
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PA_ERR_INVALID_ARGUMENT;
    if (it->second.swapped) {
      for (int32_t h : it->second.blocks) bm->host_free.push_back(h);  // within the reserved capacity
    } else {
      for (int32_t b : it->second.blocks) bm->release(b);
    }
    bm->seqs.erase(it);
    return PA_OK;
  });
}

pa_status pa_bm_swap_out(pa_block_manager* bm, int64_t seq_id, int64_t* mapping_out, int capacity,
                         int* num_pairs_out) {
  if (!bm || !num_pairs_out || capacity < 0 || (capacity > 0 && !mapping_out)) return PA_ERR_INVALID_ARGUMENT;
  return guarded([&] {
    std::lock_guard<std::mutex> lock(bm->mu);
    Sequence* s = bm->resident(seq_id);
    if (!s || static_cast<int64_t>(s->blocks.size()) > capacity) return PA_ERR_INVALID_ARGUMENT;
    if (s->blocks.size() > bm->host_free.size()) return PA_ERR_OUT_OF_BLOCKS;
    std::vector<int32_t> host(s->blocks.size());  // the one allocation, before any change
    for (size_t j = 0; j < s->blocks.size(); ++j) {
      host[j] = bm->host_free.back();
      bm->host_free.pop_back();
      mapping_out[2 * j] = s->blocks[j];
      mapping_out[2 * j + 1] = host[j];
    }
    for (int32_t b : s->blocks) bm->release(b);
    s->blocks = std::move(host);
    s->swapped = true;
    *num_pairs_out = static_cast<int>(s->blocks.size());
    return PA_OK;
  });
}

pa_status pa_bm_swap_in(pa_block_manager* bm, int64_t seq_id, int64_t* mapping_out, int capacity,
                        int* num_pairs_out) {
  if (!bm || !num_pairs_out || capacity < 0 || (capacity > 0 && !mapping_out)) return PA_ERR_INVALID_ARGUMENT;
  return guarded([&] {
    std::lock_guard<std::mutex> lock(bm->mu);
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end() || !it->second.swapped) return PA_ERR_INVALID_ARGUMENT;
    Sequence& s = it->second;
    if (static_cast<int64_t>(s.blocks.size()) > capacity) return PA_ERR_INVALID_ARGUMENT;
    if (s.blocks.size() > bm->free_stack.size()) return PA_ERR_OUT_OF_BLOCKS;
    std::vector<int32_t> dev(s.blocks.size());  // the one allocation, before any change
    for (size_t j = 0; j < s.blocks.size(); ++j) {
      dev[j] = bm->take();
      mapping_out[2 * j] = s.blocks[j];
      mapping_out[2 * j + 1] = dev[j];
    }
    for (int32_t h : s.blocks) bm->host_free.push_back(h);  // within the reserved capacity
    s.blocks = std::move(dev);
    s.swapped = false;
    *num_pairs_out = static_cast<int>(s.blocks.size());
    return PA_OK;
  });
}

pa_status pa_bm_num_free_blocks(pa_block_manager* bm, int* device_out, int* host_out) {
  if (!bm) return PA_ERR_INVALID_ARGUMENT;
  return guarded([&] {
    std::lock_guard<std::mutex> lock(bm->mu);
    if (device_out) *device_out = static_cast<int>(bm->free_stack.size());
    if (host_out) *host_out = static_cast<int>(bm->host_free.size());
    return PA_OK;
  });
}

pa_status pa_bm_sequence_info(pa_block_manager* bm, int64_t seq_id, int64_t* num_tokens_out, int* num_blocks_out,
                              int* swapped_out) {
  if (!bm) return PA_ERR_INVALID_ARGUMENT;
  return guarded([&] {
    std::lock_guard<std::mutex> lock(bm->mu);
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PA_ERR_INVALID_ARGUMENT;
    if (num_tokens_out) *num_tokens_out = it->second.tokens;
    if (num_blocks_out) *num_blocks_out = static_cast<int>(it->second.blocks.size());
    if (swapped_out) *swapped_out = it->second.swapped ? 1 : 0;
    return PA_OK;
  });
}

pa_status pa_bm_ref_count(pa_block_manager* bm, int block, int* count_out) {
  if (!bm || !count_out) return PA_ERR_INVALID_ARGUMENT;
  return guarded([&] {
    std::lock_guard<std::mutex> lock(bm->mu);
    if (block < 0 || block >= bm->num_blocks) return PA_ERR_INVALID_ARGUMENT;
    *count_out = bm->ref[block];
    return PA_OK;
  });
}

}  // extern "C"
