// Host-side refcounted KV block allocator (include/pkv.h, "Host block allocator").
//
// Follows the vLLM and PagedAttention slides 10-14 (block table, a new frame
// only when the last block fills, one shared pool, copy on write for parallel
// samples, forked prefixes for beam search) and the dataarena note sections 2,
// 3.1, 3.2 and 4 step 2 (reference counts, sharing increments them, a branch
// that diverges inside a shared block gets a private copy, finished sequences
// free their frames).
//
// Readings where the pages are silent: the free list is a FIFO queue seeded
// with a caller-given frame order; allocation is all-or-nothing; a token goes
// in place into a last block with room and count 1, into a fresh frame plus a
// copy pair when that block is shared, and into a fresh frame (no copy) when
// the last block is full.
#include <cstdint>
#include <deque>
#include <new>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "pkv.h"

struct pkv_allocator {
  struct Seq {
    std::vector<int32_t> frames;  // logical block j -> frame
    int64_t len = 0;              // tokens
  };
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::deque<int32_t> free_frames;
  std::vector<int32_t> ref;
  std::unordered_map<int32_t, Seq> seqs;

  int32_t take() {
    const int32_t f = free_frames.front();
    free_frames.pop_front();
    ref[f] = 1;
    return f;
  }
  int64_t slot(const Seq& s, int64_t t) const {
    return static_cast<int64_t>(s.frames[t / block_size]) * block_size + t % block_size;
  }
  // Frames the next token of `s` needs given the counts in `counts`
  // (0 or 1); the counts are updated as the append would update them.
  int needs_frame(const Seq& s, std::unordered_map<int32_t, int32_t>& counts) const {
    if (s.len % block_size == 0) return 1;
    const int32_t last = s.frames.back();
    auto it = counts.find(last);
    int32_t c = it == counts.end() ? ref[last] : it->second;
    if (c > 1) {
      counts[last] = c - 1;
      return 1;
    }
    return 0;
  }
  // Append one token; the caller has checked that a frame is free when needed.
  int64_t append(Seq& s, int32_t* cow_src, int32_t* cow_dst) {
    const int64_t t = s.len;
    *cow_src = *cow_dst = -1;
    if (t % block_size == 0) {
      s.frames.push_back(take());
    } else {
      const int32_t last = s.frames.back();
      if (ref[last] > 1) {
        const int32_t fresh = take();
        ref[last] -= 1;
        s.frames.back() = fresh;
        *cow_src = last;
        *cow_dst = fresh;
      }
    }
    s.len = t + 1;
    return slot(s, t);
  }
};

extern "C" {

pkv_status pkv_alloc_create(int32_t num_blocks, int32_t block_size, const int32_t* frame_order,
                            pkv_allocator** out) {
  if (!out || num_blocks < 0 || block_size <= 0) return PKV_EINVAL;
  pkv_allocator* a = new (std::nothrow) pkv_allocator();
  if (!a) return PKV_ENOMEM;
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->ref.assign(num_blocks, 0);
  if (frame_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int32_t i = 0; i < num_blocks; ++i) {
      const int32_t f = frame_order[i];
      if (f < 0 || f >= num_blocks || seen[f]) {
        delete a;
        return PKV_EINVAL;
      }
      seen[f] = 1;
      a->free_frames.push_back(f);
    }
  } else {
    for (int32_t i = 0; i < num_blocks; ++i) a->free_frames.push_back(i);
  }
  *out = a;
  return PKV_OK;
}

void pkv_alloc_destroy(pkv_allocator* alloc) { delete alloc; }

pkv_status pkv_alloc_add_seq(pkv_allocator* a, int32_t seq_id, int32_t prompt_len,
                             int64_t* slots_out) {
  if (!a || prompt_len < 0 || a->seqs.count(seq_id)) return PKV_EINVAL;
  const int64_t need = (static_cast<int64_t>(prompt_len) + a->block_size - 1) / a->block_size;
  if (need > static_cast<int64_t>(a->free_frames.size())) return PKV_ENOMEM;
  pkv_allocator::Seq s;
  s.frames.reserve(need);
  for (int64_t j = 0; j < need; ++j) s.frames.push_back(a->take());
  s.len = prompt_len;
  if (slots_out)
    for (int64_t t = 0; t < prompt_len; ++t) slots_out[t] = a->slot(s, t);
  a->seqs.emplace(seq_id, std::move(s));
  return PKV_OK;
}

pkv_status pkv_alloc_fork(pkv_allocator* a, int32_t parent, int32_t child) {
  if (!a) return PKV_EINVAL;
  auto it = a->seqs.find(parent);
  if (it == a->seqs.end() || a->seqs.count(child)) return PKV_EINVAL;
  pkv_allocator::Seq c = it->second;
  for (int32_t f : c.frames) a->ref[f] += 1;
  a->seqs.emplace(child, std::move(c));
  return PKV_OK;
}

pkv_status pkv_alloc_append(pkv_allocator* a, int32_t seq_id, int64_t* slot_out, int32_t* cow_src,
                            int32_t* cow_dst) {
  if (!a || !slot_out || !cow_src || !cow_dst) return PKV_EINVAL;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_EINVAL;
  std::unordered_map<int32_t, int32_t> counts;
  if (a->needs_frame(it->second, counts) > static_cast<int>(a->free_frames.size()))
    return PKV_ENOMEM;
  *slot_out = a->append(it->second, cow_src, cow_dst);
  return PKV_OK;
}

pkv_status pkv_alloc_append_batch(pkv_allocator* a, const int32_t* seq_ids, int32_t n,
                                  int64_t* slots_out, int64_t* pairs_out, int32_t* num_pairs_out) {
  if (!a || n < 0 || (n > 0 && (!seq_ids || !slots_out || !pairs_out)) || !num_pairs_out)
    return PKV_EINVAL;
  // Check every id and count the frames the whole step needs before changing anything.
  std::unordered_set<int32_t> seen;
  std::unordered_map<int32_t, int32_t> counts;
  std::vector<pkv_allocator::Seq*> order;
  order.reserve(n);
  int64_t need = 0;
  for (int32_t i = 0; i < n; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end() || !seen.insert(seq_ids[i]).second) return PKV_EINVAL;
    need += a->needs_frame(it->second, counts);
    order.push_back(&it->second);
  }
  if (need > static_cast<int64_t>(a->free_frames.size())) return PKV_ENOMEM;
  int32_t np = 0;
  for (int32_t i = 0; i < n; ++i) {
    int32_t src, dst;
    slots_out[i] = a->append(*order[i], &src, &dst);
    if (src >= 0) {
      pairs_out[2 * np] = src;
      pairs_out[2 * np + 1] = dst;
      ++np;
    }
  }
  *num_pairs_out = np;
  return PKV_OK;
}

pkv_status pkv_alloc_beam_step(pkv_allocator* a, const int32_t* beams, int32_t k,
                               const int32_t* parents, int32_t k_new, int32_t* next_id,
                               int32_t* new_ids_out, int64_t* slots_out, int64_t* pairs_out,
                               int32_t* num_pairs_out) {
  if (!a || k < 0 || k_new < 0 || !next_id || !num_pairs_out ||
      (k > 0 && !beams) || (k_new > 0 && (!parents || !new_ids_out || !slots_out || !pairs_out)))
    return PKV_EINVAL;
  // Check everything and count the frames the step needs before changing anything.
  std::vector<pkv_allocator::Seq*> old(k);
  std::unordered_set<int32_t> seen;
  for (int32_t i = 0; i < k; ++i) {
    auto it = a->seqs.find(beams[i]);
    if (it == a->seqs.end() || !seen.insert(beams[i]).second) return PKV_EINVAL;
    old[i] = &it->second;
  }
  std::vector<int32_t> children(k, 0);
  for (int32_t j = 0; j < k_new; ++j) {
    if (parents[j] < 0 || parents[j] >= k) return PKV_EINVAL;
    children[parents[j]] += 1;
  }
  // ids of the new beams: a parent's first continuation keeps its id, the others
  // take fresh ids counting up from *next_id
  std::vector<int32_t> ids(k_new);
  std::vector<char> taken(k, 0);
  int32_t fresh = *next_id;
  for (int32_t j = 0; j < k_new; ++j) {
    const int32_t i = parents[j];
    if (!taken[i]) {
      taken[i] = 1;
      ids[j] = beams[i];
    } else {
      if (a->seqs.count(fresh)) return PKV_EINVAL;
      ids[j] = fresh++;
    }
  }
  // reference counts after the forks and frees, then the appends' needs
  std::unordered_map<int32_t, int32_t> counts;
  auto count_of = [&](int32_t f) {
    auto it = counts.find(f);
    return it == counts.end() ? a->ref[f] : it->second;
  };
  for (int32_t i = 0; i < k; ++i) {
    const int32_t delta = children[i] == 0 ? -1 : children[i] - 1;  // forks add, a free drops
    if (delta != 0)
      for (int32_t f : old[i]->frames) counts[f] = count_of(f) + delta;
  }
  int64_t freed = 0;
  for (const auto& kv : counts) freed += kv.second == 0 && a->ref[kv.first] > 0;
  int64_t need = 0;
  for (int32_t j = 0; j < k_new; ++j) {
    const pkv_allocator::Seq& sq = *old[parents[j]];
    if (sq.len % a->block_size == 0) {
      need += 1;
    } else {
      const int32_t last = sq.frames.back();
      const int32_t c = count_of(last);
      if (c > 1) {
        counts[last] = c - 1;
        need += 1;
      }
    }
  }
  if (need > static_cast<int64_t>(a->free_frames.size()) + freed) return PKV_ENOMEM;
  // forks, in new-beam order
  for (int32_t j = 0; j < k_new; ++j) {
    const int32_t i = parents[j];
    if (ids[j] != beams[i]) {
      pkv_allocator::Seq c = *old[i];
      for (int32_t f : c.frames) a->ref[f] += 1;
      a->seqs.emplace(ids[j], std::move(c));
    }
  }
  // beams without a continuation, in beam order
  for (int32_t i = 0; i < k; ++i)
    if (children[i] == 0) pkv_alloc_free_seq(a, beams[i]);
  // one token per new beam, in order
  int32_t np = 0;
  for (int32_t j = 0; j < k_new; ++j) {
    int32_t src, dst;
    slots_out[j] = a->append(a->seqs.at(ids[j]), &src, &dst);
    new_ids_out[j] = ids[j];
    if (src >= 0) {
      pairs_out[2 * np] = src;
      pairs_out[2 * np + 1] = dst;
      ++np;
    }
  }
  *num_pairs_out = np;
  *next_id = fresh;
  return PKV_OK;
}

pkv_status pkv_alloc_free_seq(pkv_allocator* a, int32_t seq_id) {
  if (!a) return PKV_EINVAL;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_EINVAL;
  for (int32_t f : it->second.frames) {
    if (--a->ref[f] == 0) a->free_frames.push_back(f);
  }
  a->seqs.erase(it);
  return PKV_OK;
}

pkv_status pkv_alloc_block_table(const pkv_allocator* a, const int32_t* seq_ids, int32_t n,
                                 int32_t max_blocks, int32_t* table_out, int32_t* lens_out) {
  if (!a || n < 0 || max_blocks < 0 || (n > 0 && (!seq_ids || !table_out))) return PKV_EINVAL;
  for (int32_t i = 0; i < n; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end()) return PKV_EINVAL;
    const auto& fr = it->second.frames;
    if (static_cast<int64_t>(fr.size()) > max_blocks) return PKV_ERANGE;
    int32_t* row = table_out + static_cast<int64_t>(i) * max_blocks;
    for (int32_t j = 0; j < max_blocks; ++j)
      row[j] = j < static_cast<int32_t>(fr.size()) ? fr[j] : -1;
    if (lens_out) lens_out[i] = static_cast<int32_t>(it->second.len);
  }
  return PKV_OK;
}

pkv_status pkv_alloc_refcount(const pkv_allocator* a, int32_t block, int32_t* count_out) {
  if (!a || !count_out || block < 0 || block >= a->num_blocks) return PKV_EINVAL;
  *count_out = a->ref[block];
  return PKV_OK;
}

pkv_status pkv_alloc_stats(const pkv_allocator* a, pkv_alloc_stats_t* out) {
  if (!a || !out) return PKV_EINVAL;
  int64_t used = 0, shared = 0, tokens = 0, logical = 0;
  for (int32_t r : a->ref) {
    used += r > 0;
    shared += r > 1;
  }
  for (const auto& kv : a->seqs) {
    tokens += kv.second.len;
    logical += static_cast<int64_t>(kv.second.frames.size());
  }
  out->used_blocks = used;
  out->free_blocks = static_cast<int64_t>(a->free_frames.size());
  out->tokens = tokens;
  out->shared_blocks = shared;
  out->logical_blocks = logical;
  return PKV_OK;
}

}  // extern "C"
