"""Parity of the CUDA path with the CPU oracle (run on a B200).

Tolerances are the stated bar: max-abs error <= 2e-3 for fp16 and <= 1e-2 for
bf16 attention outputs against the fp64 oracle; cache writes and block copies
bit-exact.  The pool is filled with NaN before use, so a read of any byte that
no table entry / context length covers shows up as NaN in the output.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from oracle.allocator_model import AllocatorModel
import workloads as wl
from flow import (TOL, POISON, gpu_step_inputs, gpu_decode_step, oracle_step_inputs, oracle_decode,
                  max_abs_err, to_dev, from_dev, torch_dtype, rounded_oracle_stats)

pytestmark = pytest.mark.gpu


def _bin():
    from paged_kv_cache_419_b200 import binding
    return binding


def run_and_compare(inp, partition_size=0, seqs=None, check_cache=True, poison=True):
    B = _bin()
    b = gpu_step_inputs(inp, poison=poison)
    out = gpu_decode_step(inp, b, partition_size)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    ob = oracle_step_inputs(inp, poison=poison)
    assert np.array_equal(b.tables_host, ob.tables)
    ref = oracle_decode(inp, ob, seqs=seqs)
    rows = slice(None) if seqs is None else slice(*seqs)
    out_np = out.float().cpu().numpy()
    assert np.isfinite(out_np[rows]).all()
    err = max_abs_err(out, ref, rows)
    assert err <= TOL[inp.w.dtype], f"max-abs error {err}"
    if check_cache:
        used = np.unique(ob.tables[ob.tables >= 0])
        assert np.array_equal(from_dev(b.k_cache)[used], ob.k_cache[used])
        assert np.array_equal(from_dev(b.v_cache)[used], ob.v_cache[used])
    return out, ref, err, b, ob


# ------------------------------------------------------------ the workloads
def test_tiny_full():
    inp = wl.make_decode_inputs("tiny")
    run_and_compare(inp)


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_mha13b_block_sizes(bs):
    w = wl.WORKLOADS["mha13b"]
    w = w if bs == 16 else w.with_block_size(bs)
    inp = wl.make_decode_inputs(w)
    run_and_compare(inp)


def test_mha13b_contiguous_matches_oracle_and_paged():
    B = _bin()
    inp = wl.make_decode_inputs("mha13b")
    w = inp.w
    out_paged, ref, _, b, ob = run_and_compare(inp, check_cache=False)
    max_ctx = 2048
    k = torch.zeros(w.num_seqs, w.num_kv_heads, max_ctx, w.head_dim, dtype=torch_dtype(w.dtype), device="cuda")
    v = torch.zeros_like(k)
    ks, vs = to_dev(inp.k_stream, w.dtype), to_dev(inp.v_stream, w.dtype)
    for s in range(w.num_seqs):
        a, e = int(inp.offsets[s]), int(inp.offsets[s + 1])
        k[s, :, : e - a] = ks[a:e].transpose(0, 1)
        v[s, :, : e - a] = vs[a:e].transpose(0, 1)
    out = torch.empty_like(b.q)
    B.contiguous_attention_decode(out, b.q, k, v, b.lens, w.scale)
    torch.cuda.synchronize()
    assert max_abs_err(out, ref) <= TOL[w.dtype]
    # same partitions, same arithmetic order: the paged and contiguous kernels agree exactly
    assert torch.equal(out, out_paged)


@pytest.mark.parametrize("part", [512, 1024])
def test_gqa8b_full_size_all_sequences(part):
    """The benchmark's batch in the benchmark's launch configuration (partition
    1024, the default; and 512): every one of the 256 sequences, every head and
    every element against the oracle.  Also the error against the oracle rounded
    to bf16 (round to nearest even), in ulps: most elements are bit-identical to
    the rounded exact result."""
    inp = wl.make_decode_inputs("gqa8b")
    out, ref, err, b, ob = run_and_compare(inp, partition_size=part, check_cache=False)
    st = rounded_oracle_stats(out, ref, wl.BF16)
    print(f"gqa8b partition {part}: max-abs error {err:.3e}, vs rounded oracle {st}")
    assert st["within_1_ulp"] >= 0.99, st
    # sampled frames of the cache are bit-identical to the oracle's scatter
    used = np.unique(ob.tables[ob.tables >= 0])
    sample = np.random.default_rng(6).choice(used, 512, replace=False)
    got = b.k_cache[torch.from_numpy(sample).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, ob.k_cache[sample])
    got = b.v_cache[torch.from_numpy(sample).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, ob.v_cache[sample])


@pytest.mark.parametrize("part", [64, 512, 0, 2048])
def test_long_context_partitions(part):
    """4 x 16K-32K tokens; partition 0 is the default (1024), the benchmark's.
    At 64 tokens a context has up to 512 partitions, so the merge runs over
    several chunks of partition statistics.  Besides the max-abs bound, nearly
    every element must equal the oracle rounded to bf16: these outputs are small
    (|out| ~ 0.01), so a wrong merge weight can hide inside the absolute
    tolerance but not in this count."""
    inp = wl.make_decode_inputs("long")
    out, ref, err, _, _ = run_and_compare(inp, partition_size=part, check_cache=False)
    st = rounded_oracle_stats(out, ref, wl.BF16)
    print(f"long partition {part}: max-abs error {err:.3e}, vs rounded oracle {st}")
    assert st["within_1_ulp"] >= 0.99, st


def test_default_policy_balances_few_long_contexts():
    """A batch with fewer (sequence, kv head) pairs than decode CTAs, at the
    default partition size: partitions are sized per call from the batch's total
    (lengths from one token to 20K, so some contexts get one partition and some
    dozens).  Same bar as every other case, and bit-identical to the contiguous
    cache under the same policy."""
    B = _bin()
    lens = np.array([1, 63, 64, 65, 700, 5000, 20001, 12000], np.int32)
    bs = 32
    max_blocks = -(-int(lens.max()) // bs)
    w = wl.Workload("few", 12, len(lens), 8, 2, 128, bs, max_blocks * len(lens) + 3, wl.BF16,
                    max_blocks, 1.0 / np.sqrt(128), lengths=("uniform", 1, 2))
    inp = wl.make_decode_inputs(w, lengths=lens)
    out, ref, err, b, _ = run_and_compare(inp, check_cache=False)
    st = rounded_oracle_stats(out, ref, wl.BF16)
    print(f"few long contexts, default policy: max-abs {err:.3e}, vs rounded oracle {st}")
    assert st["within_1_ulp"] >= 0.99, st
    max_ctx = max_blocks * bs
    k = torch.zeros(w.num_seqs, w.num_kv_heads, max_ctx, w.head_dim, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    ks, vs = to_dev(inp.k_stream, w.dtype), to_dev(inp.v_stream, w.dtype)
    for s in range(w.num_seqs):
        a, e = int(inp.offsets[s]), int(inp.offsets[s + 1])
        k[s, :, : e - a] = ks[a:e].transpose(0, 1)
        v[s, :, : e - a] = vs[a:e].transpose(0, 1)
    out_c = torch.empty_like(b.q)
    B.contiguous_attention_decode(out_c, b.q, k, v, b.lens, w.scale)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    assert torch.equal(out_c, out)


def test_default_policy_two_size_partitions():
    """A few sequences with about a million (token, kv head) pairs in all: at
    the default size the long contexts are cut into large partitions of about
    7/8 of a CTA's share, which CTAs take in turn, and a tail of quarter-size
    partitions that CTAs claim as they finish.  The lengths give contexts made
    only of large items plus a tail (the 24K-32K ones), of both (7000), and of
    tail items alone, down to a single ragged one (1, 200, 1500): every element
    against the oracle, and bit-identical on a repeat (the claimed items land
    on different CTAs from call to call, but each partition's partial result
    does not depend on which CTA computed it)."""
    B = _bin()
    lens = np.array([32768, 30001, 1, 24000, 200, 1500, 7000, 29999], np.int32)
    bs = 32
    max_blocks = -(-int(lens.max()) // bs)
    w = wl.Workload("two-size", 12, len(lens), 32, 8, 128, bs, max_blocks * len(lens) + 3, wl.BF16,
                    max_blocks, 1.0 / np.sqrt(128), lengths=("uniform", 1, 2))
    inp = wl.make_decode_inputs(w, lengths=lens)
    out, ref, err, b, _ = run_and_compare(inp, check_cache=False)
    st = rounded_oracle_stats(out, ref, wl.BF16)
    print(f"two-size partitions, default policy: max-abs {err:.3e}, vs rounded oracle {st}")
    assert st["within_1_ulp"] >= 0.99, st
    out2 = torch.empty_like(out)
    for _ in range(3):
        B.paged_attention_decode(out2, b.q, b.k_cache, b.v_cache, b.tables, b.lens, w.scale)
        torch.cuda.synchronize()
        assert B.device_error() == 0
        assert torch.equal(out2, out)


@pytest.mark.parametrize("S,Hq,Hkv", [(64, 16, 4), (65, 16, 4), (120, 8, 2), (200, 8, 1)])
def test_default_policy_balanced_partitions_many_sequences(S, Hq, Hkv):
    """Fewer (sequence, kv head) pairs than decode CTAs, so the partitions are
    balanced per call at the default size, with many sequences.  64 is the
    most the round-robin schedule takes (every producer lane holds two
    sequences), and this batch is large enough for its two partition sizes;
    from 65 sequences on, the first partition of the first sequences runs
    statically and the rest comes from the plan's largest-first list.  Ragged
    lengths from 1 token to a few thousand, with some long contexts that span
    many partitions; every element against the oracle, and bit-identical on a
    repeat."""
    B = _bin()
    rng = np.random.default_rng(31 + S)
    lens = rng.integers(1, 3000, size=S).astype(np.int32)
    lens[rng.choice(S, size=4, replace=False)] = [6000, 7777, 9000, 8191]
    bs = 16
    max_blocks = -(-int(lens.max()) // bs)
    w = wl.Workload("balanced-list", 12, S, Hq, Hkv, 128, bs, int(np.sum(-(-lens // bs))) + S + 8,
                    wl.BF16, max_blocks, 1.0 / np.sqrt(128), lengths=("uniform", 1, 2))
    inp = wl.make_decode_inputs(w, lengths=lens)
    out, ref, err, b, _ = run_and_compare(inp, check_cache=False)
    st = rounded_oracle_stats(out, ref, wl.BF16)
    print(f"balanced partitions S={S} Hkv={Hkv}: max-abs {err:.3e}, vs rounded oracle {st}")
    assert st["within_1_ulp"] >= 0.99, st
    out2 = torch.empty_like(out)
    for _ in range(2):
        B.paged_attention_decode(out2, b.q, b.k_cache, b.v_cache, b.tables, b.lens, w.scale)
        torch.cuda.synchronize()
        assert B.device_error() == 0
        assert torch.equal(out2, out)


# ------------------------------------------------------------ normalisation pins
# Contexts that run as one stage, as a ragged stage, and across 2, 3 and 5
# partitions of the default 1024 tokens (so both normalisers run: the one at the
# end of a partition and the log-sum-exp merge across partitions).
PIN_LENGTHS = [1, 17, 64, 65, 1000, 1024, 1025, 2049, 5000]


def _pin_batch(dtype, G, lengths, seed):
    Hkv, D, bs = 2, 128, 16
    lens = np.array(lengths, np.int32)
    max_blocks = -(-int(lens.max()) // bs)
    w = wl.Workload("pin", seed, len(lens), G * Hkv, Hkv, D, bs, max_blocks * len(lens) + 3, dtype,
                    max_blocks, 1.0 / np.sqrt(D), lengths=("uniform", 1, 2))
    return wl.make_decode_inputs(w, lengths=lens)


@pytest.mark.parametrize("dtype", [wl.F16, wl.BF16])
@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("c", [1.0, -3.0])
def test_constant_values_give_the_constant(dtype, G, c):
    """V = c for every token gives out = c: the softmax weights, after both
    normalisers, sum to 1.  The weights enter the PV product rounded to the input
    type (relative error at most 2^-8 for bf16, 2^-11 plus the subnormal range
    for fp16) while the normaliser sums them unrounded, and out is rounded once
    more, so |out - c| <= |c| 2^-7 (bf16) / |c| 2^-9 (fp16); a normaliser off by
    1 % or more fails."""
    inp = _pin_batch(dtype, G, PIN_LENGTHS, seed=50 + G)
    cbits = wl.to_bits(np.array([c], np.float32), dtype)[0]
    inp = dataclasses.replace(inp, v_stream=np.full_like(inp.v_stream, cbits))
    out, ref, err, _, _ = run_and_compare(inp, check_cache=False)
    assert np.abs(ref - c).max() <= 1e-12        # the oracle: exactly c up to fp64 rounding
    dev = (out.double() - c).abs().max().item()
    bound = abs(c) * (2.0 ** -7 if dtype == wl.BF16 else 2.0 ** -9)
    assert dev <= bound, (dev, bound)


@pytest.mark.parametrize("dtype", [wl.F16, wl.BF16])
@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("D", [64, 128])
def test_single_token_context_returns_its_value_bit_exact(dtype, G, D):
    """A context of one token: its weight is exactly 1, so every query head of the
    group returns that token's V row bit for bit (mixed into a batch with longer
    contexts, which are checked against the oracle)."""
    Hkv, bs = 2, 16
    lens = np.array([1, 300, 1, 1, 2000, 1], np.int32)
    max_blocks = -(-int(lens.max()) // bs)
    w = wl.Workload("one", 60 + G, len(lens), G * Hkv, Hkv, D, bs, max_blocks * len(lens) + 3, dtype,
                    max_blocks, 1.0 / np.sqrt(D), lengths=("uniform", 1, 2))
    inp = wl.make_decode_inputs(w, lengths=lens)
    out, _, _, _, _ = run_and_compare(inp, check_cache=False)
    got = from_dev(out)
    for s in np.nonzero(lens == 1)[0]:
        v0 = inp.v_stream[inp.offsets[s]]                     # [Hkv, D]
        want = np.repeat(v0, G, axis=0)                       # query head h reads kv head h / G
        assert np.array_equal(got[s], want), s


# ------------------------------------------------------------ bounded waits
def test_merge_wait_timeout_sets_flag_and_returns():
    """The bounded-wait path, made to run out on purpose without a fault: the
    test hook makes the partition merge wait for one publication more than the
    decode grid makes, with a 20 ms bound.  The call returns, the timeout flag
    is set, and after the hook is cleared the same call is correct again."""
    import time

    B = _bin()
    inp = _pin_batch(wl.BF16, 4, [5000, 3000, 700, 2049], seed=70)
    b = gpu_step_inputs(inp)
    gpu_decode_step(inp, b)            # cache write of the new tokens; correct output
    torch.cuda.synchronize()
    assert B.device_error() == 0
    out = torch.zeros_like(b.q)
    try:
        B.set_merge_wait_hook(20_000_000, 1)
        t0 = time.perf_counter()
        B.paged_attention_decode(out, b.q, b.k_cache, b.v_cache, b.tables, b.lens, inp.w.scale)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        B.set_merge_wait_hook(0, 0)
    assert B.device_error() & B.DEVERR_WAIT_TIMEOUT
    assert elapsed < 5.0, elapsed
    B.paged_attention_decode(out, b.q, b.k_cache, b.v_cache, b.tables, b.lens, inp.w.scale)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    ob = oracle_step_inputs(inp)
    assert max_abs_err(out, oracle_decode(inp, ob)) <= TOL[wl.BF16]


# ------------------------------------------------------------ edge cases
EDGE_LENGTHS = [0, 1, 2, 7, 8, 9, 15, 16, 17, 31, 32, 33, 511, 512, 513, 1023, 1024, 1025, 2047]


@pytest.mark.parametrize("dtype", [wl.F16, wl.BF16])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_shapes_and_ragged_lengths(dtype, D, G, bs):
    Hkv = 2
    lens = np.array([1, 2, 7, 8, 9, 15, 16, 17, 31, 32, 33, 63, 64, 65, 511, 512, 513, 1030],
                    np.int32)
    max_blocks = -(-int(lens.max()) // bs) + 1
    w = wl.Workload("edge", 7, len(lens), G * Hkv, Hkv, D, bs, max_blocks * len(lens) + 5, dtype,
                    max_blocks, 1.0 / np.sqrt(D), lengths=("uniform", 1, 2))
    inp = wl.make_decode_inputs(w, lengths=lens)
    run_and_compare(inp, partition_size=512)


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_ragged_lengths_default_policy(bs):
    """The ragged lengths at the default partition policy: 36 (sequence, kv head)
    pairs, fewer than decode CTAs, so partitions are balanced per call under the
    round-robin schedule (their largest size depends on the block size)."""
    Hkv, G = 2, 4
    lens = np.array([1, 2, 7, 8, 9, 15, 16, 17, 31, 32, 33, 63, 64, 65, 511, 512, 513, 9030],
                    np.int32)
    max_blocks = -(-int(lens.max()) // bs) + 1
    w = wl.Workload("edge", 8, len(lens), G * Hkv, Hkv, 128, bs, max_blocks * len(lens) + 5, wl.BF16,
                    max_blocks, 1.0 / np.sqrt(128), lengths=("uniform", 1, 2))
    inp = wl.make_decode_inputs(w, lengths=lens)
    out, ref, err, b, _ = run_and_compare(inp, partition_size=0)
    st = rounded_oracle_stats(out, ref, wl.BF16)
    assert st["within_1_ulp"] >= 0.99, st


def test_zero_length_context_writes_zeros():
    lens = np.array([0, 5, 0, 40], np.int32)
    w = wl.Workload("zero", 8, 4, 8, 2, 128, 16, 64, wl.BF16, 4, 0.088, lengths=("uniform", 1, 2))
    inp_full = wl.make_decode_inputs(w, lengths=np.maximum(lens, 1))
    # build the batch with lengths >= 1, then set two lengths to 0 on both sides
    B = _bin()
    b = gpu_step_inputs(inp_full)
    out = gpu_decode_step(inp_full, b)
    lens_dev = torch.from_numpy(lens).cuda()
    out0 = torch.full_like(out, 3.0)
    B.paged_attention_decode(out0, b.q, b.k_cache, b.v_cache, b.tables, lens_dev, w.scale)
    torch.cuda.synchronize()
    assert torch.all(out0[0] == 0) and torch.all(out0[2] == 0)
    assert torch.equal(out0[1], out[1]) and torch.equal(out0[3], out[3])


def test_many_short_sequences():
    lens = np.random.default_rng(9).integers(1, 40, size=4096).astype(np.int32)
    w = wl.Workload("many", 9, 4096, 8, 2, 64, 16, 4096 * 3 + 8, wl.F16, 3, 0.125,
                    lengths=("uniform", 1, 2))
    inp = wl.make_decode_inputs(w, lengths=lens)
    run_and_compare(inp, check_cache=False)


def test_permutation_of_physical_frames_is_bit_identical():
    B = _bin()
    inp = wl.make_decode_inputs("mha13b")
    w = inp.w
    b = gpu_step_inputs(inp)
    out = gpu_decode_step(inp, b)
    pi = torch.from_numpy(np.random.default_rng(3).permutation(w.num_blocks)).cuda()
    k2 = torch.empty_like(b.k_cache)
    v2 = torch.empty_like(b.v_cache)
    k2[pi] = b.k_cache
    v2[pi] = b.v_cache
    t2 = torch.where(b.tables >= 0, pi[b.tables.clamp(min=0).long()].int(), b.tables)
    out2 = torch.empty_like(out)
    B.paged_attention_decode(out2, b.q, k2, v2, t2, b.lens, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_partition_size_changes_stay_within_tolerance():
    inp = wl.make_decode_inputs("mha13b")
    outs = [run_and_compare(inp, partition_size=p, check_cache=False)[0] for p in (64, 512, 2048)]
    assert (outs[0].float() - outs[2].float()).abs().max().item() <= 2 * TOL[inp.w.dtype]


# ------------------------------------------------------------ cache write / copy
@pytest.mark.parametrize("dtype", [wl.F16, wl.BF16])
@pytest.mark.parametrize("D", [64, 128])
def test_reshape_and_cache_bit_exact(dtype, D):
    B = _bin()
    N, Hkv, bs, T = 96, 4, 16, 300
    kc, vc = wl.random_pool(30 + D, N, Hkv, bs, D, dtype)
    key, value = wl.make_token_rows(31 + D, T, Hkv, D, dtype)
    slots = wl.random_slots(32 + D, T, N * bs, num_skipped=17)
    gk, gv = to_dev(kc, dtype), to_dev(vc, dtype)
    B.reshape_and_cache(to_dev(key, dtype), to_dev(value, dtype), gk, gv, torch.from_numpy(slots).cuda())
    torch.cuda.synchronize()
    assert B.device_error() == 0
    oracle.reshape_and_cache(kc, vc, key, value, slots, bs)
    assert np.array_equal(from_dev(gk), kc) and np.array_equal(from_dev(gv), vc)


def test_copy_blocks_bit_exact():
    B = _bin()
    N, Hkv, bs, D = 64, 8, 16, 128
    kc, vc = wl.random_pool(40, N, Hkv, bs, D, wl.BF16)
    rng = np.random.default_rng(41)
    frames = rng.permutation(N)
    pairs = np.stack([frames[:20], frames[20:40]], axis=1).astype(np.int64)
    pairs = np.concatenate([pairs, [[frames[50], frames[50]]]])   # src == dst is a no-op
    gk, gv = to_dev(kc, wl.BF16), to_dev(vc, wl.BF16)
    B.copy_blocks(gk, gv, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    assert B.device_error() == 0
    oracle.copy_blocks(kc, vc, pairs)
    assert np.array_equal(from_dev(gk), kc) and np.array_equal(from_dev(gv), vc)


# ------------------------------------------------------------ shared prefix + CoW
def test_shared_prefix_parallel_sampling_with_copy_on_write():
    """16 prompts x 4 samples: the prompt is written once, forked 3 times; every
    generated token goes through allocator append -> copy_blocks (CoW pairs) ->
    cache write, step by step; then decode over the mixed shared/private tables.
    The oracle replays the same script with the allocator model."""
    Bn = _bin()
    inp = wl.make_shared_inputs()
    w = inp.w
    n = w.samples_per_prompt
    S = w.num_seqs
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    td = torch_dtype(w.dtype)
    gk = torch.full(shape, POISON[w.dtype], dtype=torch.int16, device="cuda").view(td)
    gv = torch.full(shape, POISON[w.dtype], dtype=torch.int16, device="cuda").view(td)
    ok = np.full(shape, POISON[w.dtype], np.uint16)
    ov = np.full(shape, POISON[w.dtype], np.uint16)
    na = Bn.BlockAllocator(w.num_blocks, w.block_size, inp.frame_order)
    ma = AllocatorModel(w.num_blocks, w.block_size, inp.frame_order)
    for p in range(w.num_prompts):
        slots = na.add_seq(p * n, inp.prompt_len)
        assert slots.tolist() == ma.add_seq(p * n, inp.prompt_len)
        Bn.reshape_and_cache(to_dev(inp.prompt_k[p], w.dtype), to_dev(inp.prompt_v[p], w.dtype), gk, gv,
                             torch.from_numpy(slots).cuda())
        oracle.reshape_and_cache(ok, ov, inp.prompt_k[p], inp.prompt_v[p], slots, w.block_size)
        for c in range(1, n):
            na.fork(p * n, p * n + c)
            ma.fork(p * n, p * n + c)
    total_pairs = 0
    for step in range(int(inp.gen_lens.max())):
        ids = [s for s in range(S) if inp.gen_lens[s] > step]
        slots, pairs = na.append_batch(ids)
        exp = [ma.append(s) for s in ids]
        assert slots.tolist() == [e[0] for e in exp]
        assert pairs.tolist() == [[e[1], e[2]] for e in exp if e[1] >= 0]
        rows = np.array([inp.gen_offsets[s] + step for s in ids])
        if len(pairs):
            Bn.copy_blocks(gk, gv, torch.from_numpy(pairs).cuda())
            oracle.copy_blocks(ok, ov, pairs)
            total_pairs += len(pairs)
        Bn.reshape_and_cache(to_dev(inp.gen_k[rows], w.dtype), to_dev(inp.gen_v[rows], w.dtype), gk, gv,
                             torch.from_numpy(slots).cuda())
        oracle.reshape_and_cache(ok, ov, inp.gen_k[rows], inp.gen_v[rows], slots, w.block_size)
    writers = (inp.gen_lens.reshape(w.num_prompts, n) > 0).sum(axis=1)
    assert total_pairs == int(np.minimum(writers, n - 1).sum())
    table, lens = na.block_table(np.arange(S, dtype=np.int32), w.max_blocks_per_seq)
    mt, ml = ma.block_table(range(S), w.max_blocks_per_seq)
    assert table.tolist() == mt and lens.tolist() == ml
    q = to_dev(inp.q, w.dtype)
    out = torch.empty_like(q)
    Bn.paged_attention_decode(out, q, gk, gv, torch.from_numpy(table).cuda(),
                              torch.from_numpy(lens).cuda(), w.scale)
    torch.cuda.synchronize()
    assert Bn.device_error() == 0
    used = np.unique(table[table >= 0])
    assert np.array_equal(from_dev(gk)[used], ok[used]) and np.array_equal(from_dev(gv)[used], ov[used])
    ref = oracle.paged_decode(inp.q, ok, ov, np.array(mt, np.int32), np.array(ml, np.int32), w.scale,
                              w.num_kv_heads, w.block_size, w.dtype)
    assert max_abs_err(out, ref) <= TOL[w.dtype]


def test_beam_search_block_tree_decode():
    """Beam search over a block tree (slide 14): 4 beams from one 1000-token
    prompt, 200 steps.  Each step goes allocator beam_step (forks, frees,
    appends) -> copy_blocks (CoW pairs) -> cache write of the new tokens; the
    native allocator and the model must agree on every step.  Then decode the
    final beams with the same kernel against the oracle's replay, and check that
    the tree holds far fewer frames than unshared beams would."""
    Bn = _bin()
    inp = wl.make_beam_inputs()
    w = inp.w
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    td = torch_dtype(w.dtype)
    gk = torch.full(shape, POISON[w.dtype], dtype=torch.int16, device="cuda").view(td)
    gv = torch.full(shape, POISON[w.dtype], dtype=torch.int16, device="cuda").view(td)
    ok = np.full(shape, POISON[w.dtype], np.uint16)
    ov = np.full(shape, POISON[w.dtype], np.uint16)
    na = Bn.BlockAllocator(w.num_blocks, w.block_size, inp.frame_order)
    ma = AllocatorModel(w.num_blocks, w.block_size, inp.frame_order)
    slots = na.add_seq(0, inp.prompt_len)
    assert slots.tolist() == ma.add_seq(0, inp.prompt_len)
    Bn.reshape_and_cache(to_dev(inp.prompt_k, w.dtype), to_dev(inp.prompt_v, w.dtype), gk, gv,
                         torch.from_numpy(slots).cuda())
    oracle.reshape_and_cache(ok, ov, inp.prompt_k, inp.prompt_v, slots, w.block_size)
    beams, nid_n, nid_m = np.zeros(1, np.int32), 1, 1
    for step in range(inp.steps):
        ids, slots, pairs, nid_n = na.beam_step(beams, inp.parents[step], nid_n)
        e_ids, e_slots, e_pairs, nid_m = ma.beam_step(beams.tolist(), inp.parents[step], nid_m)
        assert ids.tolist() == e_ids and slots.tolist() == e_slots and pairs.tolist() == e_pairs
        if len(pairs):
            Bn.copy_blocks(gk, gv, torch.from_numpy(pairs).cuda())
            oracle.copy_blocks(ok, ov, pairs)
        Bn.reshape_and_cache(to_dev(inp.step_k[step], w.dtype), to_dev(inp.step_v[step], w.dtype), gk, gv,
                             torch.from_numpy(slots).cuda())
        oracle.reshape_and_cache(ok, ov, inp.step_k[step], inp.step_v[step], slots, w.block_size)
        beams = ids
    table, lens = na.block_table(beams, w.max_blocks_per_seq)
    mt, ml = ma.block_table(beams.tolist(), w.max_blocks_per_seq)
    assert table.tolist() == mt and lens.tolist() == ml
    assert (lens == inp.prompt_len + inp.steps).all()
    st = na.stats()
    assert st["used_blocks"] < 0.5 * st["logical_blocks"]  # the tree, not copies
    q = to_dev(inp.q, w.dtype)
    out = torch.empty_like(q)
    Bn.paged_attention_decode(out, q, gk, gv, torch.from_numpy(table).cuda(), torch.from_numpy(lens).cuda(),
                              w.scale, partition_size=512)
    torch.cuda.synchronize()
    assert Bn.device_error() == 0
    used = np.unique(table[table >= 0])
    assert np.array_equal(from_dev(gk)[used], ok[used]) and np.array_equal(from_dev(gv)[used], ov[used])
    ref = oracle.paged_decode(inp.q, ok, ov, np.array(mt, np.int32), np.array(ml, np.int32), w.scale,
                              w.num_kv_heads, w.block_size, w.dtype)
    assert max_abs_err(out, ref) <= TOL[w.dtype]


def test_prefix_cache_reuses_frames_and_writes_no_kv():
    """Automatic prefix caching (dataarena note section 3.1): 16 requests on 4
    shared 1024-token system prompts.  Each request goes through the cached
    add_seq of the native allocator (checked against the model) and writes K/V
    only for its tokens past the cached ones, so a system prompt is written once.
    Decoding every request over the shared frames matches the oracle, and the
    cached frames' contents equal the oracle's."""
    Bn = _bin()
    inp = wl.make_prefix_inputs(num_seqs=16)
    w = inp.w
    S = w.num_seqs
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    td = torch_dtype(w.dtype)
    gk = torch.full(shape, POISON[w.dtype], dtype=torch.int16, device="cuda").view(td)
    gv = torch.full(shape, POISON[w.dtype], dtype=torch.int16, device="cuda").view(td)
    ok = np.full(shape, POISON[w.dtype], np.uint16)
    ov = np.full(shape, POISON[w.dtype], np.uint16)
    na = Bn.BlockAllocator(w.num_blocks, w.block_size, inp.frame_order)
    ma = AllocatorModel(w.num_blocks, w.block_size, inp.frame_order)
    written = 0
    for i in range(S):
        slots, cached = na.add_seq_cached(i, inp.token_ids[i])
        e_slots, e_cached = ma.add_seq_cached(i, inp.token_ids[i])
        assert slots.tolist() == e_slots and cached == e_cached
        rows_k = np.concatenate([inp.system_k[inp.system[i]], inp.own_k[inp.own_offsets[i]:inp.own_offsets[i + 1]]])
        rows_v = np.concatenate([inp.system_v[inp.system[i]], inp.own_v[inp.own_offsets[i]:inp.own_offsets[i + 1]]])
        new = slice(cached, len(slots))  # only the tokens past the cached prefix
        Bn.reshape_and_cache(to_dev(rows_k[new], w.dtype), to_dev(rows_v[new], w.dtype), gk, gv,
                             torch.from_numpy(slots[new].copy()).cuda())
        oracle.reshape_and_cache(ok, ov, rows_k[new], rows_v[new], slots[new], w.block_size)
        written += len(slots) - cached
    total = sum(len(t) for t in inp.token_ids)
    firsts = len(set(inp.system.tolist()))
    # each system prompt's full blocks are written once
    full = (inp.prompt_len // w.block_size) * w.block_size
    assert written == total - (S - firsts) * full
    table, lens = na.block_table(np.arange(S, dtype=np.int32), w.max_blocks_per_seq)
    mt, ml = ma.block_table(range(S), w.max_blocks_per_seq)
    assert table.tolist() == mt and lens.tolist() == ml
    q = to_dev(inp.q, w.dtype)
    out = torch.empty_like(q)
    Bn.paged_attention_decode(out, q, gk, gv, torch.from_numpy(table).cuda(), torch.from_numpy(lens).cuda(),
                              w.scale)
    torch.cuda.synchronize()
    assert Bn.device_error() == 0
    used = np.unique(table[table >= 0])
    assert np.array_equal(from_dev(gk)[used], ok[used]) and np.array_equal(from_dev(gv)[used], ov[used])
    ref = oracle.paged_decode(inp.q, ok, ov, np.array(mt, np.int32), np.array(ml, np.int32), w.scale,
                              w.num_kv_heads, w.block_size, w.dtype)
    assert max_abs_err(out, ref) <= TOL[w.dtype]


# ------------------------------------------------------------ bad device data
def test_bad_indices_set_device_flags_without_faulting():
    B = _bin()
    inp = wl.make_decode_inputs("tiny")
    w = inp.w
    b = gpu_step_inputs(inp)
    gpu_decode_step(inp, b)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    out = torch.empty_like(b.q)
    bad = b.tables.clone()
    bad[0, 0] = w.num_blocks + 5
    B.paged_attention_decode(out, b.q, b.k_cache, b.v_cache, bad, b.lens, w.scale)
    assert B.device_error() & B.DEVERR_TABLE_ENTRY
    lens = b.lens.clone()
    lens[1] = w.max_blocks_per_seq * w.block_size + 3
    B.paged_attention_decode(out, b.q, b.k_cache, b.v_cache, b.tables, lens, w.scale)
    assert B.device_error() & B.DEVERR_CONTEXT_LEN
    slots = torch.tensor([w.num_blocks * w.block_size + 1, -1, 3, 4], dtype=torch.int64, device="cuda")
    B.reshape_and_cache(b.new_k, b.new_v, b.k_cache, b.v_cache, slots)
    assert B.device_error() == B.DEVERR_SLOT
    B.copy_blocks(b.k_cache, b.v_cache, torch.tensor([[0, w.num_blocks]], dtype=torch.int64, device="cuda"))
    assert B.device_error() == B.DEVERR_COPY_PAIR
    assert B.device_error() == 0


def test_validate_env_rejects_order_dependent_copy_lists(monkeypatch):
    B = _bin()
    N, Hkv, bs, D = 32, 2, 16, 64
    kc, vc = wl.random_pool(44, N, Hkv, bs, D, wl.F16)
    gk, gv = to_dev(kc, wl.F16), to_dev(vc, wl.F16)
    monkeypatch.setenv("PKV_VALIDATE", "1")
    for bad in ([[1, 2], [2, 3]],          # frame 2 is written and read
                [[1, 5], [4, 5]]):         # two pairs write frame 5
        with pytest.raises(B.PkvError) as e:
            B.copy_blocks(gk, gv, torch.tensor(bad, dtype=torch.int64, device="cuda"))
        assert e.value.status == B.PKV_EINVAL
    with pytest.raises(B.PkvError) as e:
        B.copy_blocks(gk, gv, torch.tensor([[1, N]], dtype=torch.int64, device="cuda"))
    assert e.value.status == B.PKV_ERANGE
    B.copy_blocks(gk, gv, torch.tensor([[1, 2], [3, 4], [6, 6]], dtype=torch.int64, device="cuda"))
    torch.cuda.synchronize()
    assert B.device_error() == 0
    oracle.copy_blocks(kc, vc, np.array([[1, 2], [3, 4], [6, 6]], np.int64))
    assert np.array_equal(from_dev(gk), kc) and np.array_equal(from_dev(gv), vc)


def test_validate_env_rejects_bad_tables_before_launch(monkeypatch):
    B = _bin()
    inp = wl.make_decode_inputs("tiny")
    w = inp.w
    b = gpu_step_inputs(inp)
    monkeypatch.setenv("PKV_VALIDATE", "1")
    bad = b.tables.clone()
    bad[2, 0] = -1
    out = torch.zeros_like(b.q)
    with pytest.raises(B.PkvError) as e:
        B.paged_attention_decode(out, b.q, b.k_cache, b.v_cache, bad, b.lens, w.scale)
    assert e.value.status == B.PKV_ERANGE
    B.paged_attention_decode(out, b.q, b.k_cache, b.v_cache, b.tables, b.lens, w.scale)
    torch.cuda.synchronize()
    assert B.device_error() == 0
