"""Pins of the allocator reference model against the pages' traces and invariants."""
import json
import os

import numpy as np
import pytest

from oracle.allocator_model import AllocatorModel, AllocatorError, ENOMEM
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_new_frame_only_when_last_block_fills():
    g = golden("allocation_trace_slides_s11.json")
    assert len(g["steps"]) == 3
    B = 16
    a = AllocatorModel(8, B)
    slots = a.add_seq(0, 15)                       # prefill: one frame, one free slot
    assert a.tables[0] == [0] and slots == list(range(15))
    s1, src, dst = a.append(0)                     # first step: the free slot
    assert (s1, src, dst) == (15, -1, -1) and a.tables[0] == [0]
    s2, src, dst = a.append(0)                     # second step: a new frame
    assert a.tables[0] == [0, 1] and s2 == 1 * B + 0 and (src, dst) == (-1, -1)


def test_cow_four_samples_only_last_block_copied():
    g = golden("cow_dataarena_s3_2.json")
    n = g["samples"]
    B = 16
    a = AllocatorModel(128, B)
    a.add_seq(0, 1000)                             # 62 full blocks + 8 tokens in block 62
    for c in range(1, n):
        a.fork(0, c)
    shared = list(a.tables[0])
    assert all(a.ref[b] == n for b in shared)
    pairs = []
    for s in range(n):
        slot, src, dst = a.append(s)
        if src >= 0:
            pairs.append((src, dst))
    # samples 0..n-2 copy the partial last block; the last writer finds count 1
    assert len(pairs) == n - 1
    assert all(src == shared[-1] for src, _ in pairs)
    assert a.ref[shared[-1]] == 1 and a.tables[n - 1][-1] == shared[-1]
    # full shared blocks stay shared by all samples
    assert all(a.ref[b] == n for b in shared[:-1])
    for s in range(n):
        assert a.tables[s][:-1] == shared[:-1]


def test_full_shared_last_block_is_never_copied():
    a = AllocatorModel(16, 4)
    a.add_seq(0, 8)
    a.fork(0, 1)
    for s in (0, 1):
        _, src, dst = a.append(s)
        assert (src, dst) == (-1, -1)
    assert a.tables[0][:2] == a.tables[1][:2] and a.tables[0][2] != a.tables[1][2]


def test_free_returns_frames_in_fifo_order_and_refcounts():
    a = AllocatorModel(6, 4, frame_order=[5, 4, 3, 2, 1, 0])
    a.add_seq(0, 9)                                # frames 5, 4, 3
    a.fork(0, 1)
    a.free_seq(0)
    assert list(a.free) == [2, 1, 0]               # still held by seq 1
    a.free_seq(1)
    assert list(a.free) == [2, 1, 0, 5, 4, 3]
    assert all(r == 0 for r in a.ref)


def test_all_or_nothing_exhaustion():
    a = AllocatorModel(4, 16)
    a.add_seq(0, 40)                               # 3 frames
    before = (list(a.free), list(a.ref))
    with pytest.raises(AllocatorError, match=ENOMEM):
        a.add_seq(1, 17)                           # needs 2, one free
    assert (list(a.free), list(a.ref)) == before and 1 not in a.tables
    a.add_seq(1, 16)
    with pytest.raises(AllocatorError, match=ENOMEM):
        a.append(1)


@pytest.mark.parametrize("name", ["mha13b", "gqa8b", "long"])
def test_only_last_block_partial_and_waste_below_4_percent(name):
    g = golden("waste_bound_dataarena_s2.json")
    w = wl.WORKLOADS[name]
    rng = np.random.default_rng(w.seed)
    lens = wl.draw_lengths(w, rng)
    a = AllocatorModel(w.num_blocks, w.block_size)
    for s, L in enumerate(lens):
        a.add_seq(s, int(L))
    reserved = 0
    for s, L in enumerate(lens):
        nb = len(a.tables[s])
        reserved += nb * w.block_size
        # every block but the last holds B tokens; the last holds 1..B
        assert (nb - 1) * w.block_size < L <= nb * w.block_size
        assert nb * w.block_size - L <= w.block_size - 1
    waste = 1 - lens.sum() / reserved
    assert waste < g["waste_below"]


def test_shared_workload_memory_saving():
    """Sharing the 1000-token prompt among 4 samples needs far fewer frames than
    4 private copies (the slides report 6-66 % savings on real traces)."""
    w = wl.WORKLOADS["shared"]
    inp = wl.make_shared_inputs()
    a = AllocatorModel(w.num_blocks, w.block_size, inp.frame_order)
    n = w.samples_per_prompt
    for p in range(w.num_prompts):
        a.add_seq(p * n, inp.prompt_len)
        for c in range(1, n):
            a.fork(p * n, p * n + c)
    pairs = 0
    for step in range(int(inp.gen_lens.max())):
        for s in range(w.num_seqs):
            if inp.gen_lens[s] > step:
                _, src, _ = a.append(s)
                pairs += src >= 0
    st = a.stats()
    saving = 1 - st["used_blocks"] / st["logical_blocks"]
    assert 0.5 < saving < 0.75
    # per prompt: one copy per writer while the partial prompt block is shared
    writers = (inp.gen_lens.reshape(w.num_prompts, n) > 0).sum(axis=1)
    assert pairs == int(np.minimum(writers, n - 1).sum())


# ------------------------------------------------------------ beam search (slide 14)
def test_beam_step_candidates_share_the_prefix_like_forked_processes():
    """Slide 14: beam candidates share their prefix like forked processes.  Four
    candidates that all continue one beam hold every full block of it once (count
    4); the partial last block is copied once per writer while it is shared
    (slide 13's rule), so 3 copies, and the last writer appends in place."""
    a = AllocatorModel(64, 4)
    a.add_seq(0, 10)  # blocks 0, 1 full, block 2 holds 2 tokens
    ids, slots, pairs, nxt = a.beam_step([0], [0, 0, 0, 0], next_id=100)
    assert ids == [0, 100, 101, 102] and nxt == 103
    full = a.tables[0][:2]
    for s in ids:
        assert a.tables[s][:2] == full and a.lens[s] == 11
    assert all(a.ref[b] == 4 for b in full)
    assert len(pairs) == 3 and all(src == 2 for src, _ in pairs)
    # each pair's destination became that beam's private last block; the last writer kept the shared one
    assert [a.tables[s][2] for s in ids[:3]] == [dst for _, dst in pairs]
    assert a.tables[102][2] == 2 and a.ref[2] == 1
    # the appended token goes at offset 2 of each beam's last block
    assert slots == [a.tables[s][2] * 4 + 2 for s in ids]


def test_beam_step_frees_dropped_beams_and_copies_only_on_divergence():
    """Beams with no continuation release their frames (dataarena note section 4
    step 2); a beam that continues alone writes in place once its last block is
    private, so copies happen only where a shared partial block diverges."""
    a = AllocatorModel(64, 4)
    a.add_seq(0, 8)  # two full blocks
    ids, _, pairs, nxt = a.beam_step([0], [0, 0], next_id=10)
    assert ids == [0, 10] and pairs == []  # block boundary: new frames, nothing to copy
    ids, _, pairs, nxt = a.beam_step([0, 10], [1, 1], next_id=nxt)  # beam 0 dropped, 10 forks
    assert ids == [10, 11] and pairs and 0 not in a.tables
    ids, _, pairs, nxt = a.beam_step([10, 11], [0, 1], next_id=nxt)  # each continues itself
    assert pairs == []  # both last blocks are private now
    st = a.stats()
    assert st["used_blocks"] == 2 + 2 and st["logical_blocks"] == 2 * 3


def test_beam_tree_frames_closed_form():
    """k beams forked from a P-token prompt (P a multiple of B), each continuing
    itself for T steps, hold P/B + k * ceil(T/B) frames against k * (P/B +
    ceil(T/B)) unshared: the saving the pages quote 'up to 55 %' for beam search."""
    B, P, k, T = 16, 1024, 4, 100
    a = AllocatorModel(4096, B)
    a.add_seq(0, P)
    beams, nxt = [0], 1
    beams, _, _, nxt = a.beam_step(beams, [0] * k, nxt)
    for _ in range(T - 1):
        beams, _, pairs, nxt = a.beam_step(beams, list(range(k)), nxt)
        assert pairs == []
    st = a.stats()
    tb = -(-T // B)
    assert st["used_blocks"] == P // B + k * tb
    assert st["logical_blocks"] == k * (P // B + tb)


def test_beam_step_enomem_changes_nothing():
    a = AllocatorModel(4, 4)
    a.add_seq(0, 6)  # 2 frames, the second holding 2 tokens
    snap = lambda: ({k: list(v) for k, v in a.tables.items()}, dict(a.lens), list(a.ref), list(a.free))
    before = snap()
    with pytest.raises(AllocatorError):
        a.beam_step([0], [0, 0, 0, 0], next_id=5)  # 3 copies need 3 frames, 2 are free
    assert snap() == before
    with pytest.raises(AllocatorError):
        a.beam_step([0], [1], next_id=5)  # parent index out of range
    with pytest.raises(AllocatorError):
        a.beam_step([0, 0], [0], next_id=5)  # repeated beam


# ------------------------------------------------------------ prefix caching (dataarena note 3.1)
def _prompt(rng, n):
    return [int(x) for x in rng.integers(0, 32000, size=n)]


def test_prefix_cache_second_request_maps_to_the_same_frames():
    """A second request with the same system prompt maps its logical blocks to
    the frames of the first (count 2) and needs no KV written for them; only the
    full blocks are cached, so a private suffix and the partial last block get
    their own frames."""
    rng = np.random.default_rng(1)
    B = 16
    system = _prompt(rng, 5 * B)  # five full blocks
    a = AllocatorModel(64, B)
    s1, c1 = a.add_seq_cached(0, system + _prompt(rng, 20))
    assert c1 == 0 and len(a.cache) == 6  # 5 system blocks + 1 full user block
    s2, c2 = a.add_seq_cached(1, system + _prompt(rng, 7))
    assert c2 == 5 * B
    assert a.tables[1][:5] == a.tables[0][:5] and a.tables[1][5] != a.tables[0][5]
    assert all(a.ref[f] == 2 for f in a.tables[0][:5])
    assert s2[:5 * B] == s1[:5 * B]  # the cached tokens' slots are the first request's
    st = a.stats()
    assert st["used_blocks"] == 6 + 1 + 1 and st["logical_blocks"] == 7 + 6


def test_prefix_cache_keys_chain_the_whole_prefix():
    """A block's key covers every earlier token: a request that differs only in
    its first block reuses nothing, even where later blocks hold equal tokens."""
    rng = np.random.default_rng(2)
    B = 8
    blocks = [_prompt(rng, B) for _ in range(4)]
    a = AllocatorModel(64, B)
    a.add_seq_cached(0, sum(blocks, []))
    other = _prompt(rng, B)
    _, c = a.add_seq_cached(1, other + sum(blocks[1:], []))
    assert c == 0 and not set(a.tables[1]) & set(a.tables[0])
    k0 = AllocatorModel.block_key(None, blocks[0])
    assert a.cache[AllocatorModel.block_key(k0, blocks[1])] == a.tables[0][1]


def test_prefix_cache_survives_free_and_is_evicted_only_by_reuse():
    """Frames of a finished request stay cached while free (a later request
    revives them out of the free queue); once the pool hands them out for other
    content their keys are gone."""
    rng = np.random.default_rng(3)
    B = 4
    system = _prompt(rng, 3 * B)
    a = AllocatorModel(6, B)
    a.add_seq_cached(0, system)
    frames = list(a.tables[0])
    a.free_seq(0)
    assert a.stats()["cached_blocks"] == 3 and len(a.free) == 6
    _, c = a.add_seq_cached(1, system)
    assert c == 3 * B and a.tables[1] == frames and len(a.free) == 3
    a.free_seq(1)
    # the free queue now ends with the three cached frames; a 6-block request takes all of them
    a.add_seq(2, 6 * B)
    assert a.stats()["cached_blocks"] == 0
    a.free_seq(2)
    _, c = a.add_seq_cached(3, system)
    assert c == 0


def test_prefix_cache_enomem_changes_nothing():
    rng = np.random.default_rng(4)
    a = AllocatorModel(4, 4)
    a.add_seq_cached(0, _prompt(rng, 12))
    snap = ({k: list(v) for k, v in a.tables.items()}, list(a.ref), list(a.free), dict(a.cache))
    with pytest.raises(AllocatorError):
        a.add_seq_cached(1, _prompt(rng, 8))  # needs 2 frames, 1 is free
    assert ({k: list(v) for k, v in a.tables.items()}, list(a.ref), list(a.free), dict(a.cache)) == snap


def test_prefix_cache_block_after_a_different_prefix_is_not_reused():
    """A block's KV depends on every earlier token (dataarena note section 3.1
    hashes prompt blocks; the reading chains each key to its prefix).  With
    A = [X, Y] and C = [Z, W] cached, B = [X, W] reuses X's frame but not W's:
    W was cached after Z, not after X."""
    rng = np.random.default_rng(5)
    B = 4
    X, Y, Z, W = (_prompt(rng, B) for _ in range(4))
    a = AllocatorModel(32, B)
    a.add_seq_cached(0, X + Y)
    a.add_seq_cached(1, Z + W)
    _, c = a.add_seq_cached(2, X + W)
    assert c == B
    assert a.tables[2][0] == a.tables[0][0] and a.tables[2][1] not in (a.tables[0][1], a.tables[1][1])
