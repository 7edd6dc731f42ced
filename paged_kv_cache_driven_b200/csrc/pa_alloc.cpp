// Host block allocator of the paged KV cache.
//
// "vLLM KV Cache and PagedAttention Explained": 5단계 (fixed-size blocks of 16
// tokens; a request gets only the blocks it needs; the 17th token gets a new
// block), Step 6 "Prefill" (ceil(6 / 16) = 1 block at the start of prefill) and
// "Decode" (a new block when the length crosses a block boundary), Step 7 item 7
// (a finished request's blocks return to the pool, immediately reusable), Step 8
// (continuous batching refills freed slots). "PagedAttention" card,
// "무엇이 좋아지는가": on-demand allocation, waste bounded by each request's
// last block.
//
// Step 9 "Safe Sharing with Copy-on-Write": a block can be named by several
// tables (a shared prompt prefix, or the prompt of parallel samples forked from
// one request); each block keeps a reference count and goes back to the pool
// when it drops to zero. A sequence about to write into a partly filled block
// that other tables also name first gets a private copy: a new block is taken,
// the (old, new) pair is queued for pa_copy_blocks, and only this sequence's
// table entry changes.
//
// State: a LIFO free list (std::vector used as a stack; back() is handed out
// next), a reference count per block, a hash map from sequence id to {length,
// block table}, and the queue of pending copies. Every call is O(work it
// reports) and validates its arguments before changing anything.

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedattn.h"

struct pa_alloc {
  struct Seq {
    int len = 0;
    std::vector<int32_t> blocks;
  };
  int num_blocks = 0;
  int block_size = 0;
  std::vector<int32_t> free_list;
  std::vector<int32_t> refs;                       // tables naming each block
  std::vector<std::pair<int32_t, int32_t>> copies;  // pending copy-on-write (src, dst)
  std::unordered_map<int64_t, Seq> seqs;

  int64_t blocks_for(int64_t len) const { return (len + block_size - 1) / block_size; }

  // Growing seq s past its length writes into its last block when that block
  // is partly filled; a block other tables also name must be copied first.
  bool cow_needed(const Seq& s, int64_t new_len) const {
    return new_len > s.len && s.len % block_size != 0 && !s.blocks.empty() &&
           refs[static_cast<size_t>(s.blocks.back())] > 1;
  }

  int32_t pop_block() {
    const int32_t b = free_list.back();
    free_list.pop_back();
    refs[static_cast<size_t>(b)] = 1;
    return b;
  }

  // Gives s a private copy of its last block (free list known to be non-empty).
  void copy_on_write(Seq& s) {
    const int32_t src = s.blocks.back();
    const int32_t dst = pop_block();
    --refs[static_cast<size_t>(src)];
    s.blocks.back() = dst;
    copies.emplace_back(src, dst);
  }
};

namespace {

const pa_alloc::Seq* find_seq(const pa_alloc* a, int64_t id) {
  auto it = a->seqs.find(id);
  return it == a->seqs.end() ? nullptr : &it->second;
}

}  // namespace

extern "C" {

pa_status pa_alloc_create(int NB, int S, const int32_t* initial_order, pa_alloc** out) {
  if (!out || NB < 0 || S <= 0) return PA_ERR_INVALID;
  *out = nullptr;
  pa_alloc* a = new (std::nothrow) pa_alloc;
  if (!a) return PA_ERR_OOM;
  a->num_blocks = NB;
  a->block_size = S;
  try {
    a->refs.assign(static_cast<size_t>(NB), 0);
    a->copies.reserve(64);
    a->free_list.resize(static_cast<size_t>(NB));
    if (initial_order) {
      std::vector<uint8_t> seen(static_cast<size_t>(NB), 0);
      for (int k = 0; k < NB; ++k) {
        const int32_t id = initial_order[k];
        if (id < 0 || id >= NB || seen[id]) {
          delete a;
          return PA_ERR_INVALID;
        }
        seen[id] = 1;
        a->free_list[NB - 1 - k] = id;  // first in order = top of the stack
      }
    } else {
      for (int k = 0; k < NB; ++k) a->free_list[NB - 1 - k] = k;
    }
  } catch (...) {
    delete a;
    return PA_ERR_OOM;
  }
  *out = a;
  return PA_OK;
}

void pa_alloc_destroy(pa_alloc* a) { delete a; }

pa_status pa_seq_grow(pa_alloc* a, int64_t seq_id, int new_len) {
  if (!a || new_len < 0) return PA_ERR_INVALID;
  auto it = a->seqs.find(seq_id);
  const int cur_len = it == a->seqs.end() ? 0 : it->second.len;
  const size_t cur_blocks = it == a->seqs.end() ? 0 : it->second.blocks.size();
  if (new_len < cur_len) return PA_ERR_INVALID;
  const bool cow = it != a->seqs.end() && a->cow_needed(it->second, new_len);
  const int64_t grow = a->blocks_for(new_len) - static_cast<int64_t>(cur_blocks);
  if (grow + (cow ? 1 : 0) > static_cast<int64_t>(a->free_list.size())) return PA_ERR_OOM;
  try {
    pa_alloc::Seq& s = a->seqs[seq_id];  // may create
    s.blocks.reserve(s.blocks.size() + static_cast<size_t>(grow));
    a->copies.reserve(a->copies.size() + 1);
    if (cow) a->copy_on_write(s);
    for (int64_t k = 0; k < grow; ++k) s.blocks.push_back(a->pop_block());
    s.len = new_len;
  } catch (...) {
    return PA_ERR_OOM;  // only reachable on host allocation failure before any pop
  }
  return PA_OK;
}

pa_status pa_seq_free(pa_alloc* a, int64_t seq_id) {
  if (!a) return PA_ERR_INVALID;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_INVALID;
  // capacity was reserved for the whole pool at creation, so this cannot throw
  for (int32_t b : it->second.blocks)
    if (--a->refs[static_cast<size_t>(b)] == 0) a->free_list.push_back(b);
  a->seqs.erase(it);
  return PA_OK;
}

pa_status pa_seq_fork(pa_alloc* a, int64_t parent, int64_t child) {
  if (!a) return PA_ERR_INVALID;
  auto it = a->seqs.find(parent);
  if (it == a->seqs.end() || a->seqs.count(child)) return PA_ERR_INVALID;
  try {
    pa_alloc::Seq copy = it->second;
    for (int32_t b : copy.blocks) ++a->refs[static_cast<size_t>(b)];
    a->seqs.emplace(child, std::move(copy));
  } catch (...) {
    return PA_ERR_OOM;
  }
  return PA_OK;
}

pa_status pa_alloc_take_copies(pa_alloc* a, int32_t* src_dst, int cap, int* n) {
  if (!a || !n || cap < 0 || (cap > 0 && !src_dst)) return PA_ERR_INVALID;
  *n = static_cast<int>(a->copies.size());
  if (*n > cap) return PA_ERR_OUT_OF_RANGE;  // nothing taken
  for (int k = 0; k < *n; ++k) {
    src_dst[2 * k] = a->copies[static_cast<size_t>(k)].first;
    src_dst[2 * k + 1] = a->copies[static_cast<size_t>(k)].second;
  }
  a->copies.clear();
  return PA_OK;
}

pa_status pa_alloc_refcounts(const pa_alloc* a, int32_t* dst, int cap) {
  if (!a || !dst || cap < a->num_blocks) return PA_ERR_INVALID;
  if (a->num_blocks) std::memcpy(dst, a->refs.data(), sizeof(int32_t) * a->refs.size());
  return PA_OK;
}

pa_status pa_seq_len(const pa_alloc* a, int64_t seq_id, int* len) {
  if (!a || !len) return PA_ERR_INVALID;
  const pa_alloc::Seq* s = find_seq(a, seq_id);
  if (!s) return PA_ERR_INVALID;
  *len = s->len;
  return PA_OK;
}

pa_status pa_seq_block_table(const pa_alloc* a, int64_t seq_id, int32_t* dst, int cap, int* n) {
  if (!a || !n || cap < 0 || (cap > 0 && !dst)) return PA_ERR_INVALID;
  const pa_alloc::Seq* s = find_seq(a, seq_id);
  if (!s) return PA_ERR_INVALID;
  *n = static_cast<int>(s->blocks.size());
  if (static_cast<int>(s->blocks.size()) > cap) return PA_ERR_OUT_OF_RANGE;
  if (!s->blocks.empty()) std::memcpy(dst, s->blocks.data(), s->blocks.size() * sizeof(int32_t));
  return PA_OK;
}

pa_status pa_build_slot_mapping(const pa_alloc* a, const int64_t* seq_ids, const int* start_pos,
                                const int* n_tok, int n_seq, int64_t* dst) {
  if (!a || n_seq < 0 || (n_seq > 0 && (!seq_ids || !start_pos || !n_tok))) return PA_ERR_INVALID;
  // validate everything first so a failing call writes nothing
  int64_t total = 0;
  for (int k = 0; k < n_seq; ++k) {
    const pa_alloc::Seq* s = find_seq(a, seq_ids[k]);
    if (!s || n_tok[k] < 0) return PA_ERR_INVALID;
    if (start_pos[k] < 0 || static_cast<int64_t>(start_pos[k]) + n_tok[k] > s->len)
      return PA_ERR_OUT_OF_RANGE;
    total += n_tok[k];
  }
  if (total > 0 && !dst) return PA_ERR_INVALID;
  const int64_t S = a->block_size;
  int64_t w = 0;
  for (int k = 0; k < n_seq; ++k) {
    const pa_alloc::Seq* s = find_seq(a, seq_ids[k]);
    for (int64_t pos = start_pos[k]; pos < static_cast<int64_t>(start_pos[k]) + n_tok[k]; ++pos)
      dst[w++] = static_cast<int64_t>(s->blocks[pos / S]) * S + pos % S;
  }
  return PA_OK;
}

pa_status pa_check_slots(const int64_t* slots, int64_t T, int64_t n_slots, int64_t* first_bad) {
  if (T < 0 || n_slots < 0 || (T > 0 && !slots)) return PA_ERR_INVALID;
  std::vector<std::pair<int64_t, int64_t>> seen;  // (slot, index) of the non-padding entries
  seen.reserve(static_cast<size_t>(T));
  for (int64_t t = 0; t < T; ++t) {
    if (slots[t] < 0) continue;  // padding
    if (slots[t] >= n_slots) {
      if (first_bad) *first_bad = t;
      return PA_ERR_OUT_OF_RANGE;
    }
    seen.emplace_back(slots[t], t);
  }
  std::sort(seen.begin(), seen.end());
  for (size_t k = 1; k < seen.size(); ++k)
    if (seen[k].first == seen[k - 1].first) {
      if (first_bad) *first_bad = seen[k].second;  // the later of two entries naming one slot
      return PA_ERR_INVALID;
    }
  return PA_OK;
}

pa_status pa_build_block_tables(const pa_alloc* a, const int64_t* seq_ids, int n_seq, int MB,
                                int32_t* dst) {
  if (!a || n_seq < 0 || MB < 0 || (n_seq > 0 && (!seq_ids || !dst))) return PA_ERR_INVALID;
  for (int k = 0; k < n_seq; ++k) {
    const pa_alloc::Seq* s = find_seq(a, seq_ids[k]);
    if (!s) return PA_ERR_INVALID;
    if (static_cast<int64_t>(s->blocks.size()) > MB) return PA_ERR_OUT_OF_RANGE;
  }
  for (int k = 0; k < n_seq; ++k) {
    const pa_alloc::Seq* s = find_seq(a, seq_ids[k]);
    int32_t* row = dst + static_cast<int64_t>(k) * MB;
    const int n = static_cast<int>(s->blocks.size());
    if (n) std::memcpy(row, s->blocks.data(), static_cast<size_t>(n) * sizeof(int32_t));
    for (int j = n; j < MB; ++j) row[j] = -1;
  }
  return PA_OK;
}

pa_status pa_prepare_step(pa_alloc* a, const int64_t* seq_ids, int n_seq, int n_new, int MB,
                          int64_t* dst_slots, int32_t* dst_tables, int32_t* dst_lens) {
  if (!a || n_seq < 0 || n_new < 0 || MB < 0 || (n_seq > 0 && !seq_ids)) return PA_ERR_INVALID;
  {
    // each sequence at most once per step
    std::vector<int64_t> sorted(seq_ids, seq_ids + n_seq);
    std::sort(sorted.begin(), sorted.end());
    if (std::adjacent_find(sorted.begin(), sorted.end()) != sorted.end()) return PA_ERR_INVALID;
  }
  int64_t need = 0;
  for (int k = 0; k < n_seq; ++k) {
    const pa_alloc::Seq* s = find_seq(a, seq_ids[k]);
    if (!s) return PA_ERR_INVALID;
    const int64_t new_len = static_cast<int64_t>(s->len) + n_new;
    if (new_len > INT32_MAX) return PA_ERR_INVALID;
    const int64_t nb = a->blocks_for(new_len);
    if (dst_tables && nb > MB) return PA_ERR_OUT_OF_RANGE;
    need += nb - static_cast<int64_t>(s->blocks.size()) + (a->cow_needed(*s, new_len) ? 1 : 0);
  }
  if (need > static_cast<int64_t>(a->free_list.size())) return PA_ERR_OOM;
  try {
    a->copies.reserve(a->copies.size() + static_cast<size_t>(n_seq));
  } catch (...) {
    return PA_ERR_OOM;
  }
  for (int k = 0; k < n_seq; ++k) {
    pa_alloc::Seq& s = a->seqs.find(seq_ids[k])->second;
    const int old_len = s.len;
    const int new_len = old_len + n_new;
    if (a->cow_needed(s, new_len)) a->copy_on_write(s);
    const int64_t add = a->blocks_for(new_len) - static_cast<int64_t>(s.blocks.size());
    for (int64_t j = 0; j < add; ++j) s.blocks.push_back(a->pop_block());
    s.len = new_len;
    const int64_t S = a->block_size;
    if (dst_slots)
      for (int t = 0; t < n_new; ++t) {
        const int64_t pos = old_len + t;
        dst_slots[static_cast<int64_t>(k) * n_new + t] =
            static_cast<int64_t>(s.blocks[pos / S]) * S + pos % S;
      }
    if (dst_tables) {
      int32_t* row = dst_tables + static_cast<int64_t>(k) * MB;
      const int n = static_cast<int>(s.blocks.size());
      if (n) std::memcpy(row, s.blocks.data(), static_cast<size_t>(n) * sizeof(int32_t));
      for (int j = n; j < MB; ++j) row[j] = -1;
    }
    if (dst_lens) dst_lens[k] = new_len;
  }
  return PA_OK;
}

pa_status pa_alloc_stats(const pa_alloc* a, int* free_blocks, int64_t* used_slots,
                         int64_t* wasted_slots) {
  if (!a) return PA_ERR_INVALID;
  int64_t used = 0, held = 0;
  for (const auto& kv : a->seqs) {
    used += kv.second.len;
    held += static_cast<int64_t>(kv.second.blocks.size()) * a->block_size;
  }
  if (free_blocks) *free_blocks = static_cast<int>(a->free_list.size());
  if (used_slots) *used_slots = used;
  if (wasted_slots) *wasted_slots = held - used;
  return PA_OK;
}

pa_status pa_alloc_dump(const pa_alloc* a, int32_t* free_list, int cap, int* n) {
  if (!a || !n || cap < 0 || (cap > 0 && !free_list)) return PA_ERR_INVALID;
  *n = static_cast<int>(a->free_list.size());
  if (*n > cap) return PA_ERR_OUT_OF_RANGE;
  if (*n) std::memcpy(free_list, a->free_list.data(), static_cast<size_t>(*n) * sizeof(int32_t));
  return PA_OK;
}

}  // extern "C"
