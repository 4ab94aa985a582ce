"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test states what fixes the expected value: a worked example printed on the
pages (fixtures under tests/golden/), a closed form, a special case that reduces
to a library routine, an exact rational computation, or an invariant of the
definition.  The attention pins are chosen so that a dropped term, a wrong sign,
a wrong scale, a swapped head or token index or a transposed operand in the
oracle fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle.allocator_model import AllocatorModel
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def f16(x):
    return np.asarray(x, dtype=np.float16).view(np.uint16)


def bf16(x):
    return torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f16_val(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def one_seq_pool(K, V, B=4, frames=None, dtype=wl.F16):
    """Lay out one sequence's K, V [Hkv, L, D] (already bit patterns) in a pool,
    logical block j in frame frames[j], by plain array indexing."""
    Hkv, L, D = K.shape
    nb = -(-L // B)
    frames = list(range(nb)) if frames is None else list(frames)
    N = max(frames) + 2 if frames else 1
    kc = np.zeros((N, Hkv, B, D), dtype=np.uint16)
    vc = np.zeros_like(kc)
    for t in range(L):
        kc[frames[t // B], :, t % B, :] = K[:, t, :]
        vc[frames[t // B], :, t % B, :] = V[:, t, :]
    table = np.full((1, max(nb, 1)), -1, dtype=np.int32)
    table[0, :nb] = frames
    return kc, vc, table


# --------------------------------------------------------------------------
# element decoding: the oracle's own fp16/bf16 decoders vs numpy / torch
# --------------------------------------------------------------------------

def test_f16_decode_all_bit_patterns():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = oracle.to_double(bits, wl.F16)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_bf16_decode_all_bit_patterns():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = oracle.to_double(bits, wl.BF16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


# --------------------------------------------------------------------------
# attention: special cases and closed forms
# --------------------------------------------------------------------------

def _decode_one(K, V, q, scale, B=4, frames=None, dtype=wl.F16):
    kc, vc, table = one_seq_pool(K, V, B, frames)
    Hkv, L, D = K.shape
    return oracle.paged_decode(q[None], kc, vc, table, np.array([L], np.int32), scale, Hkv, B,
                               dtype)[0]


def test_single_token_returns_its_value_exactly():
    rng = np.random.default_rng(10)
    K = f16(rng.standard_normal((2, 1, 8)))
    V = f16(rng.standard_normal((2, 1, 8)))
    q = f16(rng.standard_normal((4, 8)))
    out = _decode_one(K, V, q, 0.37)
    for h in range(4):
        assert np.array_equal(out[h], f16_val(V[h // 2, 0]))


def test_zero_query_gives_mean_of_values():
    rng = np.random.default_rng(11)
    K = f16(rng.standard_normal((1, 37, 16)))
    V = f16(rng.standard_normal((1, 37, 16)))
    q = f16(np.zeros((1, 16)))
    out = _decode_one(K, V, q, 0.25, B=8, frames=[4, 0, 2, 1, 3])
    np.testing.assert_allclose(out[0], f16_val(V[0]).mean(axis=0), rtol=0, atol=1e-15)


def test_constant_values_give_the_constant():
    rng = np.random.default_rng(12)
    K = f16(rng.standard_normal((1, 29, 16)))
    V = f16(np.full((1, 29, 16), -1.75))
    q = f16(rng.standard_normal((1, 16)))
    out = _decode_one(K, V, q, 0.9)
    np.testing.assert_allclose(out[0], -1.75, rtol=0, atol=1e-14)


def test_two_tokens_closed_form_sigmoid():
    # out = v0 + sigmoid(s1 - s0) (v1 - v0), s_i = scale * (q . k_i) with integer dot products
    q = np.array([1, 2, -1, 0.5])
    k0 = np.array([1, 0, 1, 2])      # q.k0 = 1 - 1 + 1 = 1
    k1 = np.array([2, 1, -1, 0])     # q.k1 = 2 + 2 + 1 = 5
    v0 = np.array([1.0, -2.0, 0.5, 3.0])
    v1 = np.array([-1.0, 4.0, 0.25, 0.0])
    scale = 0.3
    K = f16(np.stack([k0, k1])[None])
    V = f16(np.stack([v0, v1])[None])
    out = _decode_one(K, V, f16(q[None]), scale)
    w1 = scipy.special.expit(scale * (5 - 1))
    np.testing.assert_allclose(out[0], v0 + w1 * (v1 - v0), rtol=0, atol=1e-14)


@pytest.mark.parametrize("dtype", [wl.F16, wl.BF16])
def test_exact_rational_with_scale_ln2(dtype):
    # With scale = ln 2 and integer dot products n_t, the weights are 2^n_t / sum 2^n,
    # so the output is an exact rational computed here with Fractions.
    rng = np.random.default_rng(13)
    L, D = 11, 4
    qi = rng.integers(-2, 3, size=D)
    Ki = rng.integers(-2, 3, size=(L, D))
    Vi = rng.integers(-8, 9, size=(L, D)) / 4.0
    enc = f16 if dtype == wl.F16 else bf16
    out = _decode_one(enc(Ki[None]), enc(Vi[None]), enc(qi[None]), math.log(2), B=4,
                      frames=[2, 0, 1], dtype=dtype)
    n = [int(np.dot(qi, Ki[t])) for t in range(L)]
    Z = sum(Fraction(2) ** e for e in n)
    exact = [sum(Fraction(2) ** n[t] * Fraction(Vi[t, d]) for t in range(L)) / Z for d in range(D)]
    np.testing.assert_allclose(out[0], [float(x) for x in exact], rtol=1e-13, atol=1e-13)


def test_one_hot_key_selects_its_value_and_head_mapping():
    # Hq = 8, Hkv = 2: query heads 0-3 read kv head 0, heads 4-7 read kv head 1.
    # kv head g has one key aligned with q at token t_g; the output of every query
    # head is that token's value row of its own kv head (leakage below 1e-5).
    L, D = 23, 8
    t_of = {0: 5, 1: 17}
    q = np.zeros((8, D)); q[:, 0] = 4.0
    K = np.zeros((2, L, D))
    for g, t in t_of.items():
        K[g, t, 0] = 4.0
    V = np.arange(2 * L * D, dtype=np.float64).reshape(2, L, D) / 64.0
    out = _decode_one(f16(K), f16(V), f16(q), 1.0, B=8, frames=[1, 2, 0])
    for h in range(8):
        g = h // 4
        np.testing.assert_allclose(out[h], V[g, t_of[g]], atol=2e-4)
        assert np.abs(out[h] - V[1 - g, t_of[1 - g]]).max() > 1.0


def test_value_head_mapping_is_contiguous_groups():
    rng = np.random.default_rng(14)
    Hq, Hkv, L, D = 12, 3, 19, 8
    K = f16(rng.standard_normal((Hkv, L, D)))
    V = f16(np.broadcast_to(np.arange(Hkv, dtype=np.float64)[:, None, None] + 1, (Hkv, L, D)))
    q = f16(rng.standard_normal((Hq, D)))
    out = _decode_one(K, V, q, 0.5)
    for h in range(Hq):
        np.testing.assert_allclose(out[h], h // (Hq // Hkv) + 1, rtol=0, atol=1e-14)


def test_large_scores_do_not_overflow():
    # scores of order 1e5: the max subtraction keeps every exponent <= 0
    L, D = 6, 64
    q = np.full((1, D), 100.0)
    K = np.zeros((1, L, D)); K[0, 3] = 100.0; K[0, 4] = 99.0
    V = np.arange(L * D, dtype=np.float64).reshape(1, L, D) / 8.0
    out = _decode_one(f16(K), f16(V), f16(q), 1.0 / 8.0)
    assert np.isfinite(out).all()
    np.testing.assert_allclose(out[0], V[0, 3], atol=1e-12)


def test_weights_sum_to_one_and_follow_library_softmax():
    rng = np.random.default_rng(15)
    L, D = 50, 16
    qi = rng.integers(-3, 4, size=D)
    Ki = rng.integers(-3, 4, size=(L, D))
    kc, vc, table = one_seq_pool(f16(Ki[None]), f16(rng.standard_normal((1, L, D))), 8,
                                 frames=[6, 1, 3, 0, 2, 5, 4])
    scale = 0.125
    w = oracle.attention_weights(f16(qi[None, None]), kc, vc, table, np.array([L], np.int32), 0, 0,
                                 scale, 1, 8, wl.F16)
    assert w.shape == (L,) and (w > 0).all()
    assert abs(w.sum() - 1.0) < 1e-14
    ref = scipy.special.softmax(scale * (Ki @ qi).astype(np.float64))
    np.testing.assert_allclose(w, ref, rtol=1e-13, atol=0)


def test_score_shift_and_scale_invariance():
    rng = np.random.default_rng(16)
    L, D = 40, 8
    q = np.zeros((1, D)); q[0, 0] = 2.0
    K = rng.integers(-4, 5, size=(1, L, D)).astype(np.float64)
    V = f16(rng.standard_normal((1, L, D)))
    base = _decode_one(f16(K), V, f16(q), 0.25)
    # adding the same vector to every key shifts all scores equally
    K2 = K.copy(); K2[..., 0] += 3.0
    np.testing.assert_allclose(_decode_one(f16(K2), V, f16(q), 0.25), base, atol=1e-13)
    # doubling q and halving scale leaves the scores unchanged
    np.testing.assert_allclose(_decode_one(f16(K), V, f16(2 * q), 0.125), base, atol=1e-14)


def test_empty_context_gives_zero_output():
    q = f16(np.ones((1, 1, 8)))
    kc = np.zeros((2, 1, 4, 8), np.uint16)
    out = oracle.paged_decode(q, kc, kc, np.full((1, 2), -1, np.int32), np.array([0], np.int32),
                              1.0, 1, 4, wl.F16)
    assert np.array_equal(out, np.zeros_like(out))


# --------------------------------------------------------------------------
# paging: worked examples, paged = dense, permutation invariance
# --------------------------------------------------------------------------

def test_dataarena_worked_example_tokens_land_in_frames_7_2_11():
    g = golden("block_table_dataarena_s2.json")
    B = g["block_size"]
    n_tokens = g["logical_blocks_tokens"][-1][1] + 1
    # 12 frames; hand them out in the order the example shows
    order = g["logical_to_physical"] + [f for f in range(12) if f not in g["logical_to_physical"]]
    alloc = AllocatorModel(12, B, frame_order=order)
    slots = alloc.add_seq(0, n_tokens)
    assert alloc.tables[0] == g["logical_to_physical"]
    for b, c in g["ref_counts"].items():
        assert alloc.ref[int(b)] == c
    # write token t's row = t into the pool with the oracle scatter, then read the frames
    D = 8
    key = f16(np.repeat(np.arange(n_tokens, dtype=np.float64)[:, None, None], D, axis=2))
    kc = np.zeros((12, 1, B, D), np.uint16)
    vc = np.zeros_like(kc)
    oracle.reshape_and_cache(kc, vc, key, key, np.array(slots), B)
    for (lo, hi), frame in zip(g["logical_blocks_tokens"], g["logical_to_physical"]):
        got = f16_val(kc[frame, 0, : hi - lo + 1, 0])
        assert list(got) == list(range(lo, hi + 1))
    # only the last logical block is partial: 10 of its 16 slots hold tokens
    assert n_tokens - B * (len(g["logical_to_physical"]) - 1) == 10


def test_kashii_example_all_three_blocks_full():
    g = golden("block_table_kashii_s1.json")
    B = g["block_size"]
    n = g["logical_blocks_tokens"][-1][1] + 1
    order = g["logical_to_physical"] + [f for f in range(128) if f not in g["logical_to_physical"]]
    alloc = AllocatorModel(128, B, frame_order=order)
    alloc.add_seq(0, n)
    assert alloc.tables[0] == g["logical_to_physical"]
    assert n % B == 0  # no partial block


def test_slides_block_table_with_unallocated_entry():
    g = golden("block_table_slides_s10.json")
    frames = [p for p in g["physical"] if p is not None]
    table = np.array([[p if p is not None else -1 for p in g["physical"]]], np.int32)
    B, D = 4, 8
    rng = np.random.default_rng(17)
    kc = f16(rng.standard_normal((8, 1, B, D)))
    vc = f16(rng.standard_normal((8, 1, B, D)))
    q = f16(rng.standard_normal((1, 1, D)))
    L = len(frames) * B
    # a context covered by the three mapped blocks never touches the 'nothing' entry
    out = oracle.paged_decode(q, kc, vc, table, np.array([L], np.int32), 0.5, 1, B, wl.F16)
    assert np.isfinite(out).all()
    # one more token would need the unmapped fourth block: the oracle refuses
    with pytest.raises(oracle.OracleError):
        oracle.paged_decode(q, kc, vc, table, np.array([L + 1], np.int32), 0.5, 1, B, wl.F16)


def _oracle_pool_from_stream(inp, model: AllocatorModel):
    """Write every token of a DecodeInputs batch into a fresh pool through the
    allocator model's slots and the oracle's scatter."""
    w = inp.w
    kc = np.zeros((w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim), np.uint16)
    vc = np.zeros_like(kc)
    slots = []
    for s in range(w.num_seqs):
        slots += model.add_seq(s, int(inp.context_lens[s]))
    oracle.reshape_and_cache(kc, vc, inp.k_stream, inp.v_stream, np.array(slots, np.int64),
                             w.block_size)
    tables, lens = model.block_table(range(w.num_seqs), w.max_blocks_per_seq)
    return kc, vc, np.array(tables, np.int32), np.array(lens, np.int32)


def _dense_from_stream(inp, max_ctx):
    w = inp.w
    shape = (w.num_seqs, w.num_kv_heads, max_ctx, w.head_dim)
    k = np.zeros(shape, np.uint16)
    v = np.zeros(shape, np.uint16)
    for s in range(w.num_seqs):
        a, b = inp.offsets[s], inp.offsets[s + 1]
        k[s, :, : b - a] = inp.k_stream[a:b].transpose(1, 0, 2)
        v[s, :, : b - a] = inp.v_stream[a:b].transpose(1, 0, 2)
    return k, v


@pytest.mark.parametrize("name,bs", [("tiny", 16), ("tiny", 8), ("tiny", 32)])
def test_paged_equals_dense_over_logically_gathered_kv(name, bs):
    w = wl.WORKLOADS[name].with_block_size(bs) if bs != 16 else wl.WORKLOADS[name]
    inp = wl.make_decode_inputs(w)
    kc, vc, tables, lens = _oracle_pool_from_stream(inp, AllocatorModel(w.num_blocks, bs, inp.frame_order))
    paged = oracle.paged_decode(inp.q, kc, vc, tables, lens, w.scale, w.num_kv_heads, bs, w.dtype)
    k, v = _dense_from_stream(inp, int(lens.max()))
    dense = oracle.dense_decode(inp.q, k, v, lens, w.scale, w.dtype)
    assert np.array_equal(paged, dense)


def test_permutation_of_physical_frames_is_bit_exact():
    w = wl.WORKLOADS["tiny"]
    inp = wl.make_decode_inputs(w)
    kc, vc, tables, lens = _oracle_pool_from_stream(inp, AllocatorModel(w.num_blocks, 16, inp.frame_order))
    base = oracle.paged_decode(inp.q, kc, vc, tables, lens, w.scale, w.num_kv_heads, 16, w.dtype)
    pi = np.random.default_rng(18).permutation(w.num_blocks)
    kc2 = np.empty_like(kc); kc2[pi] = kc
    vc2 = np.empty_like(vc); vc2[pi] = vc
    tables2 = np.where(tables >= 0, pi[np.maximum(tables, 0)], -1).astype(np.int32)
    out = oracle.paged_decode(inp.q, kc2, vc2, tables2, lens, w.scale, w.num_kv_heads, 16, w.dtype)
    assert np.array_equal(out, base)


def test_out_of_range_table_entry_is_refused():
    q = f16(np.ones((1, 1, 8)))
    kc = np.zeros((4, 1, 4, 8), np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.paged_decode(q, kc, kc, np.array([[1, 4]], np.int32), np.array([6], np.int32), 1.0,
                            1, 4, wl.F16)


# --------------------------------------------------------------------------
# cache write and block copy
# --------------------------------------------------------------------------

def test_reshape_and_cache_scatter_and_skip():
    N, Hkv, B, D = 6, 2, 4, 8
    kc, vc = wl.random_pool(20, N, Hkv, B, D, wl.F16)
    k0, v0 = kc.copy(), vc.copy()
    key, value = wl.make_token_rows(21, 5, Hkv, D, wl.F16)
    slots = np.array([0, 23, -1, 9, 14], np.int64)
    oracle.reshape_and_cache(kc, vc, key, value, slots, B)
    expect_k, expect_v = k0.copy(), v0.copy()
    for i, s in enumerate(slots):
        if s >= 0:
            expect_k[s // B, :, s % B] = key[i]
            expect_v[s // B, :, s % B] = value[i]
    assert np.array_equal(kc, expect_k) and np.array_equal(vc, expect_v)
    # token 1 went to the last slot of the last frame
    assert np.array_equal(kc[5, :, 3], key[1])


def test_reshape_and_cache_rejects_slot_past_pool():
    kc = np.zeros((2, 1, 4, 8), np.uint16)
    key = np.ones((1, 1, 8), np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.reshape_and_cache(kc, kc.copy(), key, key, np.array([8], np.int64), 4)


def test_copy_blocks_copies_whole_frames_only():
    N, Hkv, B, D = 8, 2, 16, 8
    kc, vc = wl.random_pool(22, N, Hkv, B, D, wl.BF16)
    k0, v0 = kc.copy(), vc.copy()
    pairs = np.array([[1, 5], [3, 0], [6, 6]], np.int64)
    oracle.copy_blocks(kc, vc, pairs)
    for f in range(N):
        src = {5: 1, 0: 3}.get(f, f)
        assert np.array_equal(kc[f], k0[src]) and np.array_equal(vc[f], v0[src])


def test_copy_blocks_rejects_bad_frame():
    kc = np.zeros((2, 1, 4, 8), np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.copy_blocks(kc, kc.copy(), np.array([[0, 2]], np.int64))


# --------------------------------------------------------------------------
# closed forms printed on the pages
# --------------------------------------------------------------------------

def test_kv_bytes_per_token_13b_closed_form():
    g = golden("kv_size_slides_s5.json")
    two, hidden, layers, elt = g["factors"]
    per_token = oracle.kv_bytes_per_token(hidden, layers, elt)
    assert two == 2
    assert per_token == 819200 == g["kilobytes_per_token"] * 1024
    request = per_token * g["request_tokens"]
    assert abs(request / 1e9 - g["request_gigabytes"]) < 0.1  # 1.678e9 B, printed as 1.6 GB
    # the kernel's per-layer view of the same shape: 40 heads x 128 = 5120
    assert 2 * 40 * 128 * elt * layers == per_token


# --------------------------------------------------------------------------
# rounding of results to the storage type (round to nearest, ties to even)
# --------------------------------------------------------------------------

def _format_values(dtype):
    """All finite values of fp16 / bf16 in increasing order, with their bit patterns
    (numpy / torch decoders, independent of the oracle)."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    if dtype == wl.F16:
        vals = bits.view(np.float16).astype(np.float64)
    else:
        vals = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    keep = np.isfinite(vals) & ~((vals == 0) & (bits >= 0x8000))  # one zero (+0)
    order = np.argsort(vals[keep], kind="stable")
    return vals[keep][order], bits[keep][order]


def _nearest_even_reference(x, vals, bits):
    """Nearest representable value to x by exact rational comparison with its two
    bracketing neighbours; a tie goes to the pattern whose last bit is 0; beyond
    the largest finite value the halfway point to the next power step decides
    between the maximum and infinity."""
    top, top_bits = vals[-1], int(bits[-1])
    inf_bits = 0x7C00 if top < 1e6 else 0x7F80
    ax = abs(x)
    sign = 0x8000 if x < 0 or (x == 0 and math.copysign(1.0, x) < 0) else 0
    if ax > top:
        ulp = top - vals[-2]
        return sign | (inf_bits if Fraction(ax) >= Fraction(top) + Fraction(ulp) / 2 else top_bits)
    i = int(np.searchsorted(vals, ax, side="left"))
    if vals[i] == ax:
        return sign | int(bits[i])
    lo, hi = i - 1, i
    dlo = Fraction(ax) - Fraction(vals[lo])
    dhi = Fraction(vals[hi]) - Fraction(ax)
    if dlo < dhi:
        pick = lo
    elif dhi < dlo:
        pick = hi
    else:
        pick = lo if int(bits[lo]) % 2 == 0 else hi
    return sign | int(bits[pick])


@pytest.mark.parametrize("dtype", [wl.F16, wl.BF16])
def test_round_to_dtype_is_identity_on_every_representable_value(dtype):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = oracle.to_double(bits, dtype)
    finite = np.isfinite(vals)
    assert np.array_equal(oracle.round_to_dtype(vals[finite], dtype), bits[finite])
    inf = np.isinf(vals)
    assert np.array_equal(oracle.round_to_dtype(vals[inf], dtype), bits[inf])


@pytest.mark.parametrize("dtype", [wl.F16, wl.BF16])
def test_round_to_dtype_midpoints_go_to_even_and_neighbours_to_the_nearer(dtype):
    vals, bits = _format_values(dtype)
    pos = vals > 0
    v, b = vals[pos], bits[pos]
    mid = (v[:-1] + v[1:]) / 2           # exact in fp64 (a few more bits than the format)
    got = oracle.round_to_dtype(mid, dtype)
    even = np.where(b[:-1] % 2 == 0, b[:-1], b[1:])
    assert np.array_equal(got, even)
    assert np.array_equal(oracle.round_to_dtype(np.nextafter(mid, np.inf), dtype), b[1:])
    assert np.array_equal(oracle.round_to_dtype(np.nextafter(mid, -np.inf), dtype), b[:-1])
    # the same on the negative side, with the sign bit set
    assert np.array_equal(oracle.round_to_dtype(-mid, dtype), even | 0x8000)


@pytest.mark.parametrize("dtype", [wl.F16, wl.BF16])
def test_round_to_dtype_matches_exact_nearest_search(dtype):
    vals, bits = _format_values(dtype)
    rng = np.random.default_rng(11 + dtype)
    top = vals[-1]
    tiny = vals[vals > 0][0]
    x = np.concatenate([
        rng.standard_normal(1500),
        np.exp(rng.uniform(np.log(tiny / 4), np.log(top * 1.01), 1500)) * rng.choice([-1, 1], 1500),
        rng.uniform(0, 4 * tiny, 300),                       # subnormal range
        np.array([top, top * (1 + 2.0 ** -12), top * 1.5, -top * 1.5, 0.0, -0.0]),
    ])
    got = oracle.round_to_dtype(x, dtype)
    want = np.array([_nearest_even_reference(float(t), vals, bits) for t in x], dtype=np.uint16)
    assert np.array_equal(got, want)


def test_round_to_f16_matches_numpy_conversion():
    # numpy converts float64 -> float16 with one round-to-nearest-even step
    rng = np.random.default_rng(12)
    x = np.concatenate([rng.standard_normal(200000) * 10.0 ** rng.integers(-9, 5, 200000),
                        rng.uniform(-70000, 70000, 20000)])
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.round_to_dtype(x, wl.F16), want)
