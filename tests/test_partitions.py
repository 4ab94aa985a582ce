"""How a decode call cuts each context into partitions, checked on the host.

The partition rules run in the planning, decode and merge kernels, and
pkv_test_partitions runs the same code on the CPU.  Which cut is used is a work
split (the pages leave it open, and any cut gives the same attention output
within the tolerance).  The properties that make a cut usable are checked here
for many random batches:
  * every token belongs to exactly one partition, and the last partition of a
    context is not empty;
  * sizes are whole 64-token stages;
  * a partition's blocks fit one 256-entry table buffer of the producer warp;
  * no context has more partitions than the workspace holds per context;
  * a fixed partition size is never exceeded;
  * under the two-size rule, the statically handed-out big partitions cover at
    most 7/8 of each context, and the tail partitions are at least 256 tokens;
  * the cut of a context depends on its length and the batch total only, not on
    the order of the sequences.
The GPU tests check the attention results under these cuts against the oracle.
"""
import numpy as np
import pytest

from paged_kv_cache_419_b200 import binding as B

STAGE = 64
TABLE_ENTRIES = 256
ROUND_ROBIN_SEQS = 64
MIN_SMALL = 256
BALANCED_MIN_PARTITION = 512  # workspace partitions per context under the default size


def draw_lengths(rng, S, max_ctx):
    kind = rng.integers(0, 4)
    if kind == 0:
        lens = rng.integers(0, max_ctx + 1, size=S)
    elif kind == 1:
        lens = np.clip(np.round(np.exp(rng.normal(np.log(512), 1.0, size=S))), 1, max_ctx)
    elif kind == 2:
        lens = rng.integers(max_ctx // 2, max_ctx + 1, size=S)
    else:
        lens = rng.integers(1, 200, size=S)
        lens[rng.integers(0, S)] = max_ctx
    lens = lens.astype(np.int64)
    lens[rng.random(S) < 0.05] = 0
    return lens.astype(np.int32)


def check_cut(lens, Hkv, max_ctx, bs, part, grid):
    n, nb, pb, ps = B.partitions(lens, Hkv, max_ctx, bs, part, grid)
    S = len(lens)
    L = np.clip(lens, 0, max_ctx).astype(np.int64)
    ws_part = part if part else BALANCED_MIN_PARTITION
    max_parts = max(1, -(-max_ctx // ws_part))
    balanced = part == 0 and S * Hkv < grid
    two_size = np.any((nb != n) | (pb != ps))
    assert not two_size or (balanced and S <= ROUND_ROBIN_SEQS)
    for s in range(S):
        assert 1 <= n[s] <= max_parts, (s, L[s], n[s], max_parts)
        assert 0 <= nb[s] <= n[s]
        if L[s] == 0:
            assert n[s] == 1
            continue
        for p in (pb[s], ps[s]):
            assert p > 0 and p % STAGE == 0, (s, p)
            assert -(-p // bs) <= TABLE_ENTRIES, (s, p, bs)
            if not balanced:
                assert p <= (part or 1024)
        covered = int(nb[s]) * int(pb[s]) + int(n[s] - nb[s]) * int(ps[s])
        last = int(ps[s]) if n[s] > nb[s] else int(pb[s])
        assert covered >= L[s] > covered - last, (s, L[s], n[s], nb[s], pb[s], ps[s])
        if two_size:
            assert 8 * int(nb[s]) * int(pb[s]) <= 7 * L[s]
            assert ps[s] >= MIN_SMALL and ps[s] <= pb[s]
    return n, nb, pb, ps


@pytest.mark.parametrize("seed", range(12))
def test_partition_invariants_random_batches(seed):
    rng = np.random.default_rng(1000 + seed)
    for _ in range(40):
        S = int(rng.choice([1, 2, 4, 8, 17, 63, 64, 65, 120, 256, 300]))
        Hkv = int(rng.choice([1, 2, 4, 8]))
        bs = int(rng.choice([8, 16, 32]))
        part = int(rng.choice([0, 0, 0, 64, 512, 1024, 2048]))
        grid = int(rng.choice([296, 444]))
        max_ctx = bs * int(rng.integers(1, 2049))
        check_cut(draw_lengths(rng, S, max_ctx), Hkv, max_ctx, bs, part, grid)


def test_cut_does_not_depend_on_sequence_order():
    rng = np.random.default_rng(7)
    for S, Hkv in ((4, 8), (40, 8), (64, 4), (120, 2), (300, 8)):
        lens = draw_lengths(rng, S, 32768)
        perm = rng.permutation(S)
        a = check_cut(lens, Hkv, 32768, 32, 0, 444)
        b = check_cut(lens[perm], Hkv, 32768, 32, 0, 444)
        for x, y in zip(a, b):
            assert np.array_equal(x[perm], y)


def test_two_sizes_reach_the_long_batch():
    """The long-context batch (4 contexts of 16-32K tokens, 8 kv heads, 32-token
    blocks, 444 CTAs) as measured: 424 static big partitions of 1856 tokens
    (the first wave, one per CTA but 20) and 288 claimed ones of 512."""
    lens = np.array([28286, 31835, 30825, 24762], np.int32)
    n, nb, pb, ps = check_cut(lens, 8, 32768, 32, 0, 444)
    assert list(pb) == [1856] * 4 and list(ps) == [512] * 4
    assert int(nb.sum()) * 8 == 424 and int((n - nb).sum()) * 8 == 288


def test_policy_switches_with_the_number_of_pairs():
    """The default size is balanced only while the batch has fewer (sequence,
    kv head) pairs than CTAs; from grid / Hkv sequences on it is 1024 tokens.
    With more than 64 sequences the balanced rule has one size: here each
    context's share of the grid is one partition."""
    lens = np.full(111, 3000, np.int32)
    n_few, nb_few, p_few, _ = check_cut(lens[:110], 4, 4096, 16, 0, 444)  # 440 pairs < 444
    n_many, _, p_many, _ = check_cut(lens, 4, 4096, 16, 0, 444)           # 444 pairs
    assert np.all(p_many == 1024) and np.all(n_many == 3)
    assert np.all(n_few == 1) and np.all(nb_few == 1) and np.all(p_few == 3008)


def test_bad_arguments_are_refused():
    with pytest.raises(B.PkvError):
        B.partitions(np.array([10], np.int32), 8, 1024, 12, 0, 444)   # block size
    with pytest.raises(B.PkvError):
        B.partitions(np.array([10], np.int32), 8, 1024, 16, 100, 444)  # not whole stages
    with pytest.raises(B.PkvError):
        B.partitions(np.array([10], np.int32), 0, 1024, 16, 0, 444)   # kv heads
