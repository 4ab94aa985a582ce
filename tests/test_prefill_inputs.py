"""Host-side pieces of the prefill path (no GPU): the seeded batch layout and
the benchmark's flop count, checked by brute force."""
import numpy as np

import bench
import workloads as wl


def test_prefill_batch_layout():
    inp = wl.make_prefill_inputs("prefill")
    w = inp.w
    assert (inp.cached[:4] == 0).all() and (inp.cached <= 4096).all()
    assert ((inp.chunk >= 256) & (inp.chunk <= 2048)).all()
    assert inp.query_start[0] == 0 and np.array_equal(np.diff(inp.query_start), inp.chunk)
    assert inp.q.shape == (int(inp.chunk.sum()), w.num_heads, w.head_dim)
    assert np.array_equal(np.diff(inp.offsets), inp.context_lens)
    assert inp.k_stream.shape == (int(inp.context_lens.sum()), w.num_kv_heads, w.head_dim)
    # the pool holds every sequence's blocks and the table every row
    assert sum(-(-int(L) // w.block_size) for L in inp.context_lens) <= w.num_blocks
    assert int(inp.context_lens.max()) <= w.max_blocks_per_seq * w.block_size


def test_prefill_flops_count_every_causal_pair_once():
    w = wl.Workload("tiny-prefill", 3, 3, 4, 2, 64, 16, 64, wl.BF16, 16, 0.125,
                    lengths=("prefill", 0, 1, 1, 0))
    inp = wl.make_prefill_inputs(w, cached=[0, 7, 30], chunk=[5, 1, 12])
    pairs = 0
    for p0, T in zip(inp.cached, inp.chunk):
        for i in range(int(T)):
            pairs += len(range(0, int(p0) + i + 1))  # keys 0 .. p0 + i
    # q.K and P.V: one multiply-add (2 flops) per head dimension each, per query head
    assert bench.prefill_flops(inp) == pairs * 2 * 2 * w.head_dim * w.num_heads


def test_stored_tolerance_is_half_an_ulp_above_the_absolute_bound():
    from flow import stored_tolerance, TOL

    ref = np.array([0.0, 0.3, 2.5, 3.99, 4.0, 5.0, -6.0, 100.0])
    got = stored_tolerance(ref, wl.BF16)
    # bf16 spacing is 2^(e-7) in [2^e, 2^(e+1)); half of it from magnitude 4 up
    assert np.allclose(got, [TOL[wl.BF16]] * 4 + [2.0 ** -6, 2.0 ** -6, 2.0 ** -6, 2.0 ** -2])
    # fp16 spacing is 2^(e-10): half of it passes 2e-3 from magnitude 8 up
    assert np.allclose(stored_tolerance(np.array([1.0, 4.0, 8.0, 64.0]), wl.F16),
                       [TOL[wl.F16], TOL[wl.F16], 2.0 ** -8, 2.0 ** -5])
