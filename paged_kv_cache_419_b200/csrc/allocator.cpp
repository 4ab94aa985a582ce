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
//
// Automatic prefix caching (dataarena note section 3.1): every full prompt
// block of a sequence added with pkv_alloc_add_seq_cached gets a key, the
// SHA-256 of the previous block's key and the block's token ids, so equal keys
// mean equal prefixes.  A request whose leading blocks have cached keys maps
// them to the existing frames (count + 1) and needs no KV written for them.  A
// cached frame whose count falls to 0 goes back to the free queue but keeps
// its key until it is taken for other content; a request that hits it before
// then takes it back out of the queue.
#include <cstdint>
#include <new>
#include <string>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "pkv.h"

namespace {

// SHA-256 (FIPS 180-4).  The round constants and initial hash value are the
// first 32 bits of the fractional parts of the cube roots of the first 64
// primes and of the square roots of the first 8 primes, computed here from
// that definition with exact integer roots.
struct Sha256Constants {
  uint32_t k[64], h0[8];
  static unsigned __int128 iroot(unsigned __int128 x, int degree) {  // floor(x^(1/degree))
    unsigned __int128 lo = 0, hi = static_cast<unsigned __int128>(1) << (degree == 2 ? 40 : 36);
    while (lo < hi) {
      const unsigned __int128 mid = (lo + hi + 1) / 2;
      unsigned __int128 p = mid * mid;
      if (degree == 3) p *= mid;
      if (p <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
  Sha256Constants() {
    int primes[64], n = 0;
    for (int c = 2; n < 64; ++c) {
      bool prime = true;
      for (int d = 2; d * d <= c; ++d) prime = prime && (c % d != 0);
      if (prime) primes[n++] = c;
    }
    for (int i = 0; i < 64; ++i)
      k[i] = static_cast<uint32_t>(iroot(static_cast<unsigned __int128>(primes[i]) << 96, 3));
    for (int i = 0; i < 8; ++i)
      h0[i] = static_cast<uint32_t>(iroot(static_cast<unsigned __int128>(primes[i]) << 64, 2));
  }
};

const Sha256Constants& sha_constants() {
  static const Sha256Constants c;
  return c;
}

uint32_t rotr(uint32_t x, int n) { return (x >> n) | (x << (32 - n)); }

void sha256(const uint8_t* msg, size_t len, uint8_t out[32]) {
  const Sha256Constants& c = sha_constants();
  uint32_t h[8];
  for (int i = 0; i < 8; ++i) h[i] = c.h0[i];
  // padded message: msg, 0x80, zeros, 64-bit big-endian bit length
  const size_t total = ((len + 8) / 64 + 1) * 64;
  std::vector<uint8_t> m(total, 0);
  for (size_t i = 0; i < len; ++i) m[i] = msg[i];
  m[len] = 0x80;
  const uint64_t bits = static_cast<uint64_t>(len) * 8;
  for (int i = 0; i < 8; ++i) m[total - 1 - i] = static_cast<uint8_t>(bits >> (8 * i));
  for (size_t off = 0; off < total; off += 64) {
    uint32_t w[64];
    for (int t = 0; t < 16; ++t)
      w[t] = (uint32_t(m[off + 4 * t]) << 24) | (uint32_t(m[off + 4 * t + 1]) << 16) |
             (uint32_t(m[off + 4 * t + 2]) << 8) | uint32_t(m[off + 4 * t + 3]);
    for (int t = 16; t < 64; ++t) {
      const uint32_t s0 = rotr(w[t - 15], 7) ^ rotr(w[t - 15], 18) ^ (w[t - 15] >> 3);
      const uint32_t s1 = rotr(w[t - 2], 17) ^ rotr(w[t - 2], 19) ^ (w[t - 2] >> 10);
      w[t] = w[t - 16] + s0 + w[t - 7] + s1;
    }
    uint32_t a = h[0], b = h[1], cc = h[2], d = h[3], e = h[4], f = h[5], g = h[6], hh = h[7];
    for (int t = 0; t < 64; ++t) {
      const uint32_t S1 = rotr(e, 6) ^ rotr(e, 11) ^ rotr(e, 25);
      const uint32_t ch = (e & f) ^ (~e & g);
      const uint32_t t1 = hh + S1 + ch + c.k[t] + w[t];
      const uint32_t S0 = rotr(a, 2) ^ rotr(a, 13) ^ rotr(a, 22);
      const uint32_t maj = (a & b) ^ (a & cc) ^ (b & cc);
      const uint32_t t2 = S0 + maj;
      hh = g; g = f; f = e; e = d + t1; d = cc; cc = b; b = a; a = t1 + t2;
    }
    h[0] += a; h[1] += b; h[2] += cc; h[3] += d; h[4] += e; h[5] += f; h[6] += g; h[7] += hh;
  }
  for (int i = 0; i < 8; ++i)
    for (int j = 0; j < 4; ++j) out[4 * i + j] = static_cast<uint8_t>(h[i] >> (24 - 8 * j));
}

// Key of a full block: SHA-256 of (the previous block's key, or 32 zero bytes
// for the first block) followed by the block's token ids as little-endian int32.
void block_key(const uint8_t parent[32], const int32_t* tokens, int32_t n, uint8_t out[32]) {
  std::vector<uint8_t> buf(32 + 4 * static_cast<size_t>(n));
  for (int i = 0; i < 32; ++i) buf[i] = parent ? parent[i] : 0;
  for (int32_t t = 0; t < n; ++t)
    for (int j = 0; j < 4; ++j)
      buf[32 + 4 * t + j] = static_cast<uint8_t>(static_cast<uint32_t>(tokens[t]) >> (8 * j));
  sha256(buf.data(), buf.size(), out);
}

}  // namespace

struct pkv_allocator {
  struct Seq {
    std::vector<int32_t> frames;  // logical block j -> frame
    int64_t len = 0;              // tokens
  };
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  // Free queue: exactly the frames with count 0, oldest first, as a doubly
  // linked list over frame ids (push at the tail, take from the head, and
  // remove a revived cached frame from anywhere, all O(1)).
  std::vector<int32_t> q_next, q_prev;
  int32_t q_head = -1, q_tail = -1;
  int64_t free_count = 0;
  std::vector<int32_t> ref;
  std::unordered_map<int32_t, Seq> seqs;
  // prefix cache: key of a cached full block -> frame, and frame -> key
  std::unordered_map<std::string, int32_t> cache;
  std::unordered_map<int32_t, std::string> frame_key;

  void q_push(int32_t f) {
    q_prev[f] = q_tail;
    q_next[f] = -1;
    if (q_tail >= 0) q_next[q_tail] = f; else q_head = f;
    q_tail = f;
    free_count += 1;
  }
  void q_remove(int32_t f) {
    if (q_prev[f] >= 0) q_next[q_prev[f]] = q_next[f]; else q_head = q_next[f];
    if (q_next[f] >= 0) q_prev[q_next[f]] = q_prev[f]; else q_tail = q_prev[f];
    free_count -= 1;
  }
  int32_t take() {
    const int32_t f = q_head;
    q_remove(f);
    ref[f] = 1;
    auto it = frame_key.find(f);  // new content: the frame leaves the prefix cache
    if (it != frame_key.end()) {
      cache.erase(it->second);
      frame_key.erase(it);
    }
    return f;
  }
  void release(int32_t f) {
    if (--ref[f] == 0) q_push(f);
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
  a->q_next.assign(num_blocks, -1);
  a->q_prev.assign(num_blocks, -1);
  if (frame_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int32_t i = 0; i < num_blocks; ++i) {
      const int32_t f = frame_order[i];
      if (f < 0 || f >= num_blocks || seen[f]) {
        delete a;
        return PKV_EINVAL;
      }
      seen[f] = 1;
      a->q_push(f);
    }
  } else {
    for (int32_t i = 0; i < num_blocks; ++i) a->q_push(i);
  }
  *out = a;
  return PKV_OK;
}

void pkv_alloc_destroy(pkv_allocator* alloc) { delete alloc; }

pkv_status pkv_alloc_add_seq(pkv_allocator* a, int32_t seq_id, int32_t prompt_len,
                             int64_t* slots_out) {
  if (!a || prompt_len < 0 || a->seqs.count(seq_id)) return PKV_EINVAL;
  const int64_t need = (static_cast<int64_t>(prompt_len) + a->block_size - 1) / a->block_size;
  if (need > a->free_count) return PKV_ENOMEM;
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
  if (a->needs_frame(it->second, counts) > a->free_count)
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
  if (need > a->free_count) return PKV_ENOMEM;
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
  if (need > a->free_count + freed) return PKV_ENOMEM;
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

pkv_status pkv_alloc_add_seq_cached(pkv_allocator* a, int32_t seq_id, const int32_t* token_ids,
                                    int32_t prompt_len, int64_t* slots_out, int32_t* cached_tokens_out) {
  if (!a || prompt_len < 0 || (prompt_len > 0 && !token_ids) || !cached_tokens_out ||
      a->seqs.count(seq_id))
    return PKV_EINVAL;
  const int32_t B = a->block_size;
  const int64_t nb = (static_cast<int64_t>(prompt_len) + B - 1) / B;
  const int64_t full = prompt_len / B;
  // keys of the full blocks, and the cached prefix (hits end at the first miss:
  // a key depends on every earlier token)
  std::vector<std::string> keys(full);
  std::vector<int32_t> hit;
  uint8_t parent[32], key[32];
  for (int64_t j = 0; j < full; ++j) {
    block_key(j ? parent : nullptr, token_ids + j * B, B, key);
    keys[j].assign(reinterpret_cast<const char*>(key), 32);
    for (int i = 0; i < 32; ++i) parent[i] = key[i];
    if (static_cast<int64_t>(hit.size()) == j) {
      auto it = a->cache.find(keys[j]);
      if (it != a->cache.end()) hit.push_back(it->second);
    }
  }
  // frames needed: the blocks past the cached prefix, from the free frames that
  // are not themselves part of that prefix
  int64_t revived = 0;
  for (int32_t f : hit) revived += a->ref[f] == 0;
  if (nb - static_cast<int64_t>(hit.size()) > a->free_count - revived) return PKV_ENOMEM;
  pkv_allocator::Seq sq;
  sq.frames.reserve(nb);
  for (int32_t f : hit) {
    if (a->ref[f] == 0) a->q_remove(f);  // a cached frame that was free: revived
    a->ref[f] += 1;
    sq.frames.push_back(f);
  }
  for (int64_t j = static_cast<int64_t>(hit.size()); j < nb; ++j) {
    const int32_t f = a->take();
    sq.frames.push_back(f);
    if (j < full) {  // a new full block enters the prefix cache
      a->cache[keys[j]] = f;
      a->frame_key[f] = keys[j];
    }
  }
  sq.len = prompt_len;
  if (slots_out)
    for (int64_t t = 0; t < prompt_len; ++t) slots_out[t] = a->slot(sq, t);
  *cached_tokens_out = static_cast<int32_t>(hit.size()) * B;
  a->seqs.emplace(seq_id, std::move(sq));
  return PKV_OK;
}

pkv_status pkv_block_hash(const uint8_t* parent_key, const int32_t* token_ids, int32_t n,
                          uint8_t* key_out) {
  if (n < 0 || (n > 0 && !token_ids) || !key_out) return PKV_EINVAL;
  block_key(parent_key, token_ids, n, key_out);
  return PKV_OK;
}

pkv_status pkv_alloc_free_seq(pkv_allocator* a, int32_t seq_id) {
  if (!a) return PKV_EINVAL;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_EINVAL;
  for (int32_t f : it->second.frames) a->release(f);
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
  out->free_blocks = a->free_count;
  out->cached_blocks = static_cast<int64_t>(a->cache.size());
  out->tokens = tokens;
  out->shared_blocks = shared;
  out->logical_blocks = logical;
  return PKV_OK;
}

}  // extern "C"
