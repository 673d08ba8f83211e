// Host-side block allocator: a stack of free physical block ids plus reference counts.
//
// Source: vLLM notes page, "PagedAttention / Block Manager": pages are handed out when a request
// needs them and marked reusable when it no longer does, with a free list (or a bitmap) so that
// both operations are O(1). "vLLM 前世今生" section 3.2: several sequences may point at one
// physical block (parallel sampling, beam search, shared prefixes), so a block carries a count of
// the sequences that reference it and returns to the free list when the last one lets go.
//
// alloc pops the top of the stack; freeing the last reference pushes the block back on top, so the
// block released most recently is reused first (warm in L2). Copy-on-write (前世今生 §3.2): a
// sequence about to write into a block other sequences share moves its reference to a fresh block,
// whose page the caller fills with pa_copy_blocks first. No GPU is involved.
#include <algorithm>
#include <cstdint>
#include <new>
#include <vector>

#include "../../include/pa.h"
#include "internal.h"

using pa::set_last_error;

struct pa_allocator {
  std::vector<int32_t> stack;  // free ids; top = back
  std::vector<int32_t> ref;    // 0 = free
};

namespace {

// Whether changing the count of every listed block by `delta` (+1 or -1) once per listing keeps all
// counts valid: every id allocated, no block freed more often than it is referenced, no count past
// INT32_MAX. Nothing is changed; a block listed k times is checked against k changes.
int check_batch(const pa_allocator* a, int32_t n, const int32_t* blocks, int delta) {
  std::vector<int32_t> ids;
  try {
    ids.assign(blocks, blocks + n);
  } catch (...) {
    return set_last_error(PA_ERR_INVALID_ARG, "out of host memory");
  }
  std::sort(ids.begin(), ids.end());
  const int32_t num_blocks = static_cast<int32_t>(a->ref.size());
  for (size_t i = 0; i < ids.size();) {
    const int32_t b = ids[i];
    size_t j = i;
    while (j < ids.size() && ids[j] == b) ++j;
    const int64_t times = static_cast<int64_t>(j - i);
    if (b < 0 || b >= num_blocks || a->ref[b] == 0)
      return set_last_error(PA_ERR_BAD_BLOCK, "block %d is not allocated (pool of %d)", b, num_blocks);
    if (delta < 0 && times > a->ref[b])
      return set_last_error(PA_ERR_BAD_BLOCK, "block %d listed %lld times but referenced %d times", b,
                            static_cast<long long>(times), a->ref[b]);
    if (delta > 0 && a->ref[b] + times > INT32_MAX)
      return set_last_error(PA_ERR_INVALID_ARG, "reference count of block %d would overflow", b);
    i = j;
  }
  return PA_OK;
}

}  // namespace

extern "C" {

pa_allocator* pa_allocator_create(int32_t num_blocks, const int32_t* initial_order) {
  if (num_blocks <= 0) {
    set_last_error(PA_ERR_INVALID_ARG, "num_blocks must be > 0 (got %d)", num_blocks);
    return nullptr;
  }
  pa_allocator* a = new (std::nothrow) pa_allocator;
  if (!a) {
    set_last_error(PA_ERR_INVALID_ARG, "out of host memory");
    return nullptr;
  }
  try {
    a->ref.assign(static_cast<size_t>(num_blocks), 0);
    a->stack.resize(static_cast<size_t>(num_blocks));
  } catch (...) {
    delete a;
    set_last_error(PA_ERR_INVALID_ARG, "out of host memory for %d blocks", num_blocks);
    return nullptr;
  }
  if (initial_order) {
    // Must be a permutation of [0, num_blocks); pops come out in this order.
    std::vector<char> seen(static_cast<size_t>(num_blocks), 0);
    for (int32_t i = 0; i < num_blocks; ++i) {
      const int32_t b = initial_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete a;
        set_last_error(PA_ERR_INVALID_ARG, "initial_order is not a permutation of [0, %d): entry %d is %d",
                       num_blocks, i, b);
        return nullptr;
      }
      seen[b] = 1;
      a->stack[num_blocks - 1 - i] = b;
    }
  } else {
    for (int32_t i = 0; i < num_blocks; ++i) a->stack[num_blocks - 1 - i] = i;
  }
  return a;
}

void pa_allocator_destroy(pa_allocator* a) { delete a; }

int32_t pa_block_alloc(pa_allocator* a) {
  if (!a) return set_last_error(PA_ERR_INVALID_ARG, "allocator is NULL");
  if (a->stack.empty()) return set_last_error(PA_ERR_EXHAUSTED, "all %zu blocks are in use", a->ref.size());
  const int32_t b = a->stack.back();
  a->stack.pop_back();
  a->ref[b] = 1;
  return b;
}

int pa_block_incref(pa_allocator* a, int32_t b) {
  if (!a) return set_last_error(PA_ERR_INVALID_ARG, "allocator is NULL");
  if (b < 0 || b >= static_cast<int32_t>(a->ref.size()) || a->ref[b] == 0)
    return set_last_error(PA_ERR_BAD_BLOCK, "block %d is not allocated", b);
  if (a->ref[b] == INT32_MAX) return set_last_error(PA_ERR_INVALID_ARG, "reference count of block %d would overflow", b);
  ++a->ref[b];
  return PA_OK;
}

int pa_block_free(pa_allocator* a, int32_t b) {
  if (!a) return set_last_error(PA_ERR_INVALID_ARG, "allocator is NULL");
  if (b < 0 || b >= static_cast<int32_t>(a->ref.size()) || a->ref[b] == 0)
    return set_last_error(PA_ERR_BAD_BLOCK, "block %d is not allocated", b);
  if (--a->ref[b] == 0) a->stack.push_back(b);
  return PA_OK;
}

int pa_block_cow(pa_allocator* a, int32_t b, int32_t* out_block) {
  if (!a || !out_block) return set_last_error(PA_ERR_INVALID_ARG, "allocator or out_block is NULL");
  if (b < 0 || b >= static_cast<int32_t>(a->ref.size()) || a->ref[b] == 0)
    return set_last_error(PA_ERR_BAD_BLOCK, "block %d is not allocated", b);
  if (a->ref[b] == 1) {  // sole owner: write in place
    *out_block = b;
    return 0;
  }
  if (a->stack.empty())
    return set_last_error(PA_ERR_EXHAUSTED, "block %d is shared and no block is free for its copy", b);
  const int32_t nb = pa_block_alloc(a);
  --a->ref[b];
  *out_block = nb;
  return 1;
}

int32_t pa_block_refcount(const pa_allocator* a, int32_t b) {
  if (!a) return set_last_error(PA_ERR_INVALID_ARG, "allocator is NULL");
  if (b < 0 || b >= static_cast<int32_t>(a->ref.size()))
    return set_last_error(PA_ERR_BAD_BLOCK, "block %d is outside the pool of %zu", b, a->ref.size());
  return a->ref[b];
}

int32_t pa_allocator_num_free(const pa_allocator* a) { return a ? static_cast<int32_t>(a->stack.size()) : PA_ERR_INVALID_ARG; }

int32_t pa_allocator_num_blocks(const pa_allocator* a) { return a ? static_cast<int32_t>(a->ref.size()) : PA_ERR_INVALID_ARG; }

int pa_blocks_alloc_n(pa_allocator* a, int32_t n, int32_t* out) {
  if (!a || n < 0 || (n > 0 && !out)) return set_last_error(PA_ERR_INVALID_ARG, "NULL allocator or output, or n < 0");
  if (static_cast<size_t>(n) > a->stack.size())
    return set_last_error(PA_ERR_EXHAUSTED, "%d blocks asked for, %zu free", n, a->stack.size());
  for (int32_t i = 0; i < n; ++i) out[i] = pa_block_alloc(a);
  return PA_OK;
}

// Both batch calls are all-or-nothing: the whole list is checked first, then applied in list order
// (so blocks whose last reference goes are pushed in that order, as n single frees would).
int pa_blocks_incref_n(pa_allocator* a, int32_t n, const int32_t* blocks) {
  if (!a || n < 0 || (n > 0 && !blocks)) return set_last_error(PA_ERR_INVALID_ARG, "NULL allocator or blocks, or n < 0");
  if (const int r = check_batch(a, n, blocks, +1)) return r;
  for (int32_t i = 0; i < n; ++i) ++a->ref[blocks[i]];
  return PA_OK;
}

int pa_blocks_free_n(pa_allocator* a, int32_t n, const int32_t* blocks) {
  if (!a || n < 0 || (n > 0 && !blocks)) return set_last_error(PA_ERR_INVALID_ARG, "NULL allocator or blocks, or n < 0");
  if (const int r = check_batch(a, n, blocks, -1)) return r;
  for (int32_t i = 0; i < n; ++i)
    if (--a->ref[blocks[i]] == 0) a->stack.push_back(blocks[i]);
  return PA_OK;
}

int pa_build_block_tables(pa_allocator* a, const int32_t* context_lens, int32_t num_seqs, int32_t max_blocks,
                          int32_t shared_prefix_tokens, int32_t* out) {
  if (!a || num_seqs < 0 || max_blocks < 0 || (num_seqs > 0 && (!context_lens || !out)))
    return set_last_error(PA_ERR_INVALID_ARG, "NULL allocator, lengths or output, or a negative count");
  if (shared_prefix_tokens < 0 || shared_prefix_tokens % PA_BLOCK_SIZE)
    return set_last_error(PA_ERR_INVALID_ARG, "shared_prefix_tokens must be a non-negative multiple of %d (got %d)",
                          PA_BLOCK_SIZE, shared_prefix_tokens);
  const int32_t npre = shared_prefix_tokens / PA_BLOCK_SIZE;
  // Count the allocations first (all-or-nothing): each sequence's own blocks past the prefix, plus
  // the prefix blocks, each allocated once by the first sequence that reaches it.
  int64_t fresh = 0;
  int32_t prefix_reach = 0;
  for (int32_t s = 0; s < num_seqs; ++s) {
    const int32_t n = context_lens[s];
    if (n < 0) return set_last_error(PA_ERR_INVALID_ARG, "context_lens[%d] is %d", s, n);
    const int32_t nb = n / PA_BLOCK_SIZE + (n % PA_BLOCK_SIZE != 0);
    if (nb > max_blocks)
      return set_last_error(PA_ERR_INVALID_ARG, "sequence %d needs %d blocks, the table has %d", s, nb, max_blocks);
    const int32_t in_prefix = std::min(npre, nb);
    fresh += nb - in_prefix;
    prefix_reach = std::max(prefix_reach, in_prefix);
  }
  fresh += prefix_reach;
  if (fresh > static_cast<int64_t>(a->stack.size()))
    return set_last_error(PA_ERR_EXHAUSTED, "the tables need %lld fresh blocks, %zu are free",
                          static_cast<long long>(fresh), a->stack.size());
  // Sequences in order, logical blocks in order: a prefix block already held is shared (one more
  // reference), anything else is popped from the free list. At most num_seqs references per
  // prefix block, so no count can overflow.
  std::vector<int32_t> prefix;
  try {
    prefix.reserve(static_cast<size_t>(prefix_reach));
  } catch (...) {
    return set_last_error(PA_ERR_INVALID_ARG, "out of host memory");
  }
  for (int32_t s = 0; s < num_seqs; ++s) {
    const int32_t n = context_lens[s];
    const int32_t nb = n / PA_BLOCK_SIZE + (n % PA_BLOCK_SIZE != 0);
    int32_t* row = out + static_cast<int64_t>(s) * max_blocks;
    for (int32_t j = 0; j < nb; ++j) {
      if (j < npre && j < static_cast<int32_t>(prefix.size())) {
        row[j] = prefix[j];
        ++a->ref[prefix[j]];
      } else {
        row[j] = pa_block_alloc(a);
        if (j < npre) prefix.push_back(row[j]);
      }
    }
    for (int32_t j = nb; j < max_blocks; ++j) row[j] = -1;
  }
  return PA_OK;
}

int pa_slots_for_positions(const int32_t* bt, int64_t row_stride, int32_t num_seqs, int32_t max_blocks,
                           const int32_t* token_seq, const int32_t* token_pos, int64_t num_tokens, int64_t* out) {
  if (num_tokens < 0 || (num_tokens > 0 && (!bt || !token_seq || !token_pos || !out)) || num_seqs < 0 ||
      max_blocks < 0 || row_stride < max_blocks)
    return set_last_error(PA_ERR_INVALID_ARG, "NULL pointer, negative count or row_stride < max_blocks");
  for (int64_t i = 0; i < num_tokens; ++i) {
    const int32_t s = token_seq[i], pos = token_pos[i];
    if (s < 0 || s >= num_seqs || pos < 0)
      return set_last_error(PA_ERR_INVALID_ARG, "token %lld: sequence %d / position %d out of range",
                            static_cast<long long>(i), s, pos);
    const int32_t j = pos / PA_BLOCK_SIZE;
    if (j >= max_blocks)
      return set_last_error(PA_ERR_INVALID_ARG, "token %lld: position %d is past the table's %d blocks",
                            static_cast<long long>(i), pos, max_blocks);
    const int32_t b = bt[static_cast<int64_t>(s) * row_stride + j];
    if (b < 0)
      return set_last_error(PA_ERR_INVALID_ARG, "token %lld: table entry %d of sequence %d is %d",
                            static_cast<long long>(i), j, s, b);
    out[i] = static_cast<int64_t>(b) * PA_BLOCK_SIZE + pos % PA_BLOCK_SIZE;
  }
  return PA_OK;
}

}  // extern "C"
