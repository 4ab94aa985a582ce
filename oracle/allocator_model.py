"""Reference model of the refcounted KV block allocator, in plain Python.

TEST INFRASTRUCTURE (see the oracle package docstring for who may import it).

What it follows:

* vLLM and PagedAttention slides, slide 10: each request sees its blocks in
  logical order; the block table maps them to physical frames.  Slide 11: a new
  frame is taken only when the last block is full (prefill, the first decode
  step goes into the free slot, the second into a new frame).  Slide 12: one
  pool; any free frame serves any request.  Slide 13: parallel samples share
  the prompt's frames; only the last, partially filled block is ever copied.
* dataarena note, section 2: blocks of B tokens, worked example with reference
  counts; section 3.1: sharing a frame increments its reference count;
  section 3.2: a branch that writes a divergent token into a shared block gets a
  private frame holding a copy of the block's state; section 4 step 2: a
  finished sequence frees its frames.

Readings where the pages are silent:

* The free list is a FIFO queue, initially ``frame_order`` (default 0..N-1).
  A sequence takes frames from the head for its logical blocks in order; a
  frame whose count drops to 0 goes to the tail, in the order of the freeing
  sequence's logical blocks.
* Allocation is all-or-nothing: a request that needs more frames than are free
  fails with ENOMEM and changes nothing.
* A token is written in place into the last block when that block has room and
  its count is 1; when it has room and is shared (count > 1) the writer gets a
  new frame, the pair (shared frame, new frame) is emitted for the block copy,
  and the shared frame's count drops by one.  A full last block is never copied:
  the writer simply starts a new frame.
* slot = frame * B + offset (offset = token index mod B).

Automatic prefix caching (dataarena note, section 3.1: a cryptographic hash of
each prompt block; a request whose block hash already has a frame maps its
logical block to it and increments the count, so no KV is recomputed).  Readings:

* Only full prompt blocks are keyed; the key of block j is SHA-256 of the key of
  block j-1 (32 zero bytes for j = 0) and block j's token ids as little-endian
  int32, so equal keys mean equal prefixes and hits are always a leading run.
* A cached frame whose count falls to 0 returns to the free queue with its key;
  a later hit takes it back out of the queue, and taking it for other content
  drops the key.
"""
from __future__ import annotations

import hashlib
from collections import deque

ENOMEM = "ENOMEM"


class AllocatorError(RuntimeError):
    pass


class AllocatorModel:
    def __init__(self, num_blocks: int, block_size: int, frame_order=None):
        if num_blocks < 0 or block_size <= 0:
            raise AllocatorError("EINVAL")
        self.N = num_blocks
        self.B = block_size
        order = list(range(num_blocks)) if frame_order is None else [int(x) for x in frame_order]
        if sorted(order) != list(range(num_blocks)):
            raise AllocatorError("EINVAL")
        self.free = deque(order)
        self.ref = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}
        self.cache: dict[bytes, int] = {}      # prefix-cache key -> frame
        self.frame_key: dict[int, bytes] = {}  # frame -> its key

    # -- queries -----------------------------------------------------------
    def slot(self, seq: int, t: int) -> int:
        return self.tables[seq][t // self.B] * self.B + t % self.B

    def block_table(self, seqs, max_blocks: int):
        rows, lens = [], []
        for s in seqs:
            tab = self.tables[s]
            if len(tab) > max_blocks:
                raise AllocatorError("ERANGE")
            rows.append(tab + [-1] * (max_blocks - len(tab)))
            lens.append(self.lens[s])
        return rows, lens

    def stats(self):
        used = sum(1 for r in self.ref if r > 0)
        shared = sum(1 for r in self.ref if r > 1)
        tokens = sum(self.lens.values())
        logical = sum(len(t) for t in self.tables.values())
        return {"used_blocks": used, "free_blocks": len(self.free), "tokens": tokens,
                "shared_blocks": shared, "logical_blocks": logical, "cached_blocks": len(self.cache)}

    # -- operations --------------------------------------------------------
    def _take(self) -> int:
        b = self.free.popleft()
        self.ref[b] = 1
        key = self.frame_key.pop(b, None)  # new content: the frame leaves the prefix cache
        if key is not None:
            del self.cache[key]
        return b

    @staticmethod
    def block_key(parent, tokens) -> bytes:
        """Prefix-cache key of a full block (dataarena note section 3.1: a
        cryptographic hash of each prompt block): SHA-256 of the previous block's
        key (32 zero bytes for the first block) and the block's token ids as
        little-endian int32, so that equal keys mean equal prefixes."""
        data = (parent if parent is not None else bytes(32)) + b"".join(
            int(t).to_bytes(4, "little", signed=True) for t in tokens)
        return hashlib.sha256(data).digest()

    def add_seq_cached(self, seq: int, token_ids):
        """Like add_seq for a prompt given by its token ids, through the prefix
        cache: leading full blocks whose keys are cached map to those frames
        (count + 1; a free cached frame leaves the free queue), the rest take
        fresh frames and their full blocks enter the cache.  Returns (slots,
        cached_tokens)."""
        toks = [int(t) for t in token_ids]
        L = len(toks)
        if seq in self.tables:
            raise AllocatorError("EINVAL")
        nb, full = -(-L // self.B), L // self.B
        keys, hit, parent = [], [], None
        for j in range(full):
            parent = self.block_key(parent, toks[j * self.B:(j + 1) * self.B])
            keys.append(parent)
            if len(hit) == j and parent in self.cache:
                hit.append(self.cache[parent])
        revived = sum(1 for f in hit if self.ref[f] == 0)
        if nb - len(hit) > len(self.free) - revived:
            raise AllocatorError(ENOMEM)
        tab = []
        for f in hit:
            if self.ref[f] == 0:
                self.free.remove(f)
            self.ref[f] += 1
            tab.append(f)
        for j in range(len(hit), nb):
            f = self._take()
            tab.append(f)
            if j < full:
                self.cache[keys[j]] = f
                self.frame_key[f] = keys[j]
        self.tables[seq] = tab
        self.lens[seq] = L
        return [self.slot(seq, t) for t in range(L)], len(hit) * self.B

    def add_seq(self, seq: int, prompt_len: int):
        """Allocate frames for a prompt of ``prompt_len`` tokens; returns its slots."""
        if seq in self.tables or prompt_len < 0:
            raise AllocatorError("EINVAL")
        need = -(-prompt_len // self.B)
        if need > len(self.free):
            raise AllocatorError(ENOMEM)
        self.tables[seq] = [self._take() for _ in range(need)]
        self.lens[seq] = prompt_len
        return [self.slot(seq, t) for t in range(prompt_len)]

    def fork(self, parent: int, child: int):
        if parent not in self.tables or child in self.tables:
            raise AllocatorError("EINVAL")
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def append(self, seq: int):
        """Reserve the slot of the next token.  Returns (slot, cow_src, cow_dst),
        the last two -1 when no copy is needed."""
        if seq not in self.tables:
            raise AllocatorError("EINVAL")
        t = self.lens[seq]
        tab = self.tables[seq]
        src = dst = -1
        if t % self.B == 0:
            if not self.free:
                raise AllocatorError(ENOMEM)
            tab.append(self._take())
        else:
            last = tab[-1]
            if self.ref[last] > 1:
                if not self.free:
                    raise AllocatorError(ENOMEM)
                new = self._take()
                self.ref[last] -= 1
                tab[-1] = new
                src, dst = last, new
        self.lens[seq] = t + 1
        return self.slot(seq, t), src, dst

    def beam_step(self, beams, parents, next_id: int):
        """One beam-search step over the block tree (slide 14: candidates share
        their prefix like forked processes; kashii section 3: copy on write when
        tokens diverge).  New beam j continues beams[parents[j]]: the first
        continuation of a beam keeps its id, each further one is a fork with the
        next fresh id; beams with no continuation are freed; then every new beam
        appends one token.  Order: forks, frees, appends.  All-or-nothing:
        ENOMEM restores the state.  Returns (new_ids, slots, pairs, next_id)."""
        beams = [int(b) for b in beams]
        parents = [int(p) for p in parents]
        if len(set(beams)) != len(beams) or any(b not in self.tables for b in beams):
            raise AllocatorError("EINVAL")
        if any(p < 0 or p >= len(beams) for p in parents):
            raise AllocatorError("EINVAL")
        ids, first = [], set()
        for p in parents:
            if p not in first:
                first.add(p)
                ids.append(beams[p])
            else:
                if next_id in self.tables:
                    raise AllocatorError("EINVAL")
                ids.append(next_id)
                next_id += 1
        saved = ({k: list(v) for k, v in self.tables.items()}, dict(self.lens), list(self.ref),
                 deque(self.free), dict(self.cache), dict(self.frame_key))
        try:
            for j, p in enumerate(parents):
                if ids[j] != beams[p]:
                    self.fork(beams[p], ids[j])
            for i, b in enumerate(beams):
                if i not in first:
                    self.free_seq(b)
            slots, pairs = [], []
            for j in range(len(parents)):
                slot, src, dst = self.append(ids[j])
                slots.append(slot)
                if src >= 0:
                    pairs.append([src, dst])
        except AllocatorError:
            self.tables, self.lens, self.ref, self.free, self.cache, self.frame_key = saved
            raise
        return ids, slots, pairs, next_id

    def free_seq(self, seq: int):
        if seq not in self.tables:
            raise AllocatorError("EINVAL")
        for b in self.tables.pop(seq):
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        del self.lens[seq]
