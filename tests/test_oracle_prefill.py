"""Pins of the paged prefill oracle (oracle_paged_prefill): causal attention of
T new prompt tokens of one sequence over the paged cache (the prefill phase of
the vLLM and PagedAttention slides, slide 3, over the block table of slides
9-10).  Checked against closed forms, invariants and the pinned decode oracle;
nothing here touches a GPU."""
import numpy as np
import pytest
import scipy.special

import oracle
import workloads as wl

B, HKV, G, D = 8, 2, 2, 16
HQ = HKV * G
N = 32


def _case(seed, p0, T, dtype=wl.F16):
    rng = np.random.default_rng(seed)
    kc, vc = wl.random_pool(seed, N, HKV, B, D, dtype)
    nb = -(-(p0 + T) // B)
    row = np.full(nb + 2, -1, np.int32)
    row[:nb] = rng.permutation(N)[:nb]
    q = wl.to_bits(rng.standard_normal((T, HQ, D)).astype(np.float32), dtype)
    return q, kc, vc, row


def test_each_query_is_a_decode_over_its_causal_prefix():
    """Query i of a prefill at positions p0.. is the decode of a context of
    p0 + i + 1 tokens through the same block-table row (the decode oracle is
    pinned on its own); bit-identical, since both gather and attend alike."""
    p0, T = 13, 11
    q, kc, vc, row = _case(1, p0, T)
    out = oracle.paged_prefill(q, kc, vc, row, p0, 0.25, HKV, B, wl.F16)
    for i in range(T):
        ref = oracle.paged_decode(q[i][None], kc, vc, row[None], np.array([p0 + i + 1], np.int32), 0.25,
                                  HKV, B, wl.F16)
        assert np.array_equal(out[i], ref[0])


def test_first_prompt_token_returns_its_own_value():
    """At position 0 the softmax has one term: every head returns V of token 0 of
    its kv head exactly."""
    q, kc, vc, row = _case(2, 0, 3)
    out = oracle.paged_prefill(q, kc, vc, row, 0, 0.7, HKV, B, wl.F16)
    for h in range(HQ):
        expect = oracle.to_double(vc[row[0], h // G, 0], wl.F16)
        assert np.array_equal(out[0, h], expect)


def test_causal_later_tokens_do_not_leak():
    """Changing the cache row of position p0 + j changes the outputs of queries
    j, j+1, ... and leaves every earlier query bit-identical."""
    p0, T, j = 5, 9, 4
    q, kc, vc, row = _case(3, p0, T)
    out = oracle.paged_prefill(q, kc, vc, row, p0, 0.5, HKV, B, wl.F16)
    t = p0 + j
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[row[t // B], :, t % B] ^= np.uint16(0x0400)  # flip an exponent bit of every element
    vc2[row[t // B], :, t % B] ^= np.uint16(0x0400)
    out2 = oracle.paged_prefill(q, kc2, vc2, row, p0, 0.5, HKV, B, wl.F16)
    assert np.array_equal(out[:j], out2[:j])
    assert not np.array_equal(out[j], out2[j])


def test_frame_relabelling_is_bit_identical():
    p0, T = 21, 6
    q, kc, vc, row = _case(4, p0, T, wl.BF16)
    out = oracle.paged_prefill(q, kc, vc, row, p0, 0.3, HKV, B, wl.BF16)
    pi = np.random.default_rng(5).permutation(N)
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[pi], vc2[pi] = kc, vc
    row2 = np.where(row >= 0, pi[np.maximum(row, 0)], -1).astype(np.int32)
    assert np.array_equal(out, oracle.paged_prefill(q, kc2, vc2, row2, p0, 0.3, HKV, B, wl.BF16))


def test_second_prompt_token_two_term_closed_form():
    """Query 1 of a prompt sees two tokens: out = v0 + sigmoid(s1 - s0)(v1 - v0)
    with s_t = scale q . k_t (integer dot products, exact in fp16)."""
    qv = np.array([1, 2, -1, 0.5] * (D // 4))
    k0 = np.array([1, 0, 1, 2] * (D // 4))    # q.k0 = 1 per group of 4
    k1 = np.array([2, 1, -1, 0] * (D // 4))   # q.k1 = 5 per group of 4
    v0 = np.linspace(-1, 1, D)
    v1 = np.linspace(2, -3, D)
    kc = np.zeros((N, HKV, B, D), np.uint16)
    vc = np.zeros((N, HKV, B, D), np.uint16)
    row = np.array([7, -1], np.int32)
    for g in range(HKV):
        kc[7, g, 0], kc[7, g, 1] = wl.to_bits(k0, wl.F16), wl.to_bits(k1, wl.F16)
        vc[7, g, 0], vc[7, g, 1] = wl.to_bits(v0, wl.F16), wl.to_bits(v1, wl.F16)
    q = np.stack([wl.to_bits(np.tile(qv, (HQ, 1)), wl.F16)] * 2)
    scale = 0.05
    out = oracle.paged_prefill(q, kc, vc, row, 0, scale, HKV, B, wl.F16)
    f = lambda x: oracle.to_double(wl.to_bits(x, wl.F16), wl.F16)  # the values as stored
    w1 = scipy.special.expit(scale * (5 - 1) * (D // 4))
    for h in range(HQ):
        np.testing.assert_allclose(out[1, h], f(v0) + w1 * (f(v1) - f(v0)), rtol=0, atol=1e-12)
        np.testing.assert_array_equal(out[0, h], f(v0))


def test_range_errors():
    q, kc, vc, row = _case(6, 3, 4)
    with pytest.raises(oracle.OracleError):
        oracle.paged_prefill(q, kc, vc, row[:0], 3, 0.5, HKV, B, wl.F16)  # table too short
    bad = row.copy()
    bad[0] = N
    with pytest.raises(oracle.OracleError):
        oracle.paged_prefill(q, kc, vc, bad, 3, 0.5, HKV, B, wl.F16)      # frame outside the pool
