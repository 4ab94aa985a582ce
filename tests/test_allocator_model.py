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
