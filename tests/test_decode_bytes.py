"""The decode roofline's numerator on the host (no GPU): the bytes a decode step
must move (bench.algorithmic_bytes), checked against the arrays the oracle reads
and writes for the same batch, against the bench's gqa8b batch, and against
the pages' per-token K/V size of a 13B model."""
import numpy as np

import bench
import workloads as wl


def test_decode_bytes_equal_the_arrays_the_step_reads_and_writes():
    for name, n in (("tiny", None), ("mha13b", 4), ("gqa8b", 8), ("long", 1)):
        inp = wl.make_decode_inputs(name, num_seqs=n)
        nb = bench.algorithmic_bytes(inp.w, inp.context_lens)
        # K and V rows of every context token (the cached ones and the new one),
        # q read, out written (out has q's shape and type)
        assert nb["decode"] == inp.k_stream.nbytes + inp.v_stream.nbytes + 2 * inp.q.nbytes
        # the cache write: the new token's K and V rows, read and written, and its
        # int64 slot
        new_rows = inp.k_stream[inp.offsets[1:] - 1]
        assert nb["cache_write"] == 2 * 2 * new_rows.nbytes + 8 * inp.w.num_seqs
        assert nb["step"] == nb["decode"] + nb["cache_write"]
        # the block-table entries a decode reads (listed apart)
        blocks = sum(-(-int(L) // inp.w.block_size) for L in inp.context_lens)
        assert nb["tables"] == 4 * blocks + 4 * inp.w.num_seqs


def test_gqa8b_batch_bytes_as_reported():
    w = wl.WORKLOADS["gqa8b"]
    lens = wl.draw_lengths(w, np.random.default_rng(w.seed))
    assert int(lens.sum()) == 201_857
    nb = bench.algorithmic_bytes(w, lens)
    assert nb["decode"] == 831_000_576  # 201,857 x 8 kv heads x 512 B + 2 x 2 MB
    assert nb["cache_write"] == 2_099_200


def test_kv_bytes_per_token_of_the_13b_model():
    """P1 slide 5: a 13B model (hidden size 5120, 40 layers) keeps
    2 x 5120 x 40 x 2 B = 800 KB of K and V per token in fp16.  One decode
    layer of the mha13b shape (40 heads x 128 = 5120) reads 1/40 of it per
    context token."""
    w = wl.WORKLOADS["mha13b"]
    one = bench.algorithmic_bytes(w, np.array([1], np.int32))["decode"]
    two = bench.algorithmic_bytes(w, np.array([2], np.int32))["decode"]
    assert (two - one) * 40 == 2 * 5120 * 40 * 2 == 819_200
