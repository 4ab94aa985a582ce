"""Parity of the paged prefill kernel with the CPU oracle (run on a B200).

Each batch goes through the library on the GPU (C++ allocator -> cache write of
every token, cached and new -> prefill attention) and through the oracle on the
CPU (allocator model -> oracle scatter -> oracle_paged_prefill), from the same
seeded inputs.  The pool is filled with NaN first, so a read of any slot that no
table entry or context length covers shows up as NaN.  Tolerances: max-abs error
2e-3 (fp16) / 1e-2 (bf16) against the fp64 oracle.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from oracle.allocator_model import AllocatorModel
import workloads as wl
from flow import TOL, POISON, to_dev, from_dev, torch_dtype, rounded_oracle_stats, stored_tolerance

pytestmark = pytest.mark.gpu


def _bin():
    from paged_kv_cache_419_b200 import binding
    return binding


def _workload(dtype, D, G, bs, frames, max_blocks, seed=80, Hkv=2):
    return wl.Workload("prefill-test", seed, 1, G * Hkv, Hkv, D, bs, frames, dtype, max_blocks,
                       1.0 / np.sqrt(D), lengths=("prefill", 0, 1, 1, 0))


def gpu_prefill_batch(inp: wl.PrefillInputs, poison=True):
    """Pool, allocator and cache write of every token through the library."""
    B = _bin()
    w = inp.w
    S = w.num_seqs
    alloc = B.BlockAllocator(w.num_blocks, w.block_size, inp.frame_order)
    slots = [alloc.add_seq(s, int(inp.context_lens[s])) for s in range(S)]
    table, lens = alloc.block_table(np.arange(S, dtype=np.int32), w.max_blocks_per_seq)
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    td = torch_dtype(w.dtype)
    fill = POISON[w.dtype] if poison else 0
    kc = torch.full(shape, fill, dtype=torch.int16, device="cuda").view(td)
    vc = torch.full(shape, fill, dtype=torch.int16, device="cuda").view(td)
    B.reshape_and_cache(to_dev(inp.k_stream, w.dtype), to_dev(inp.v_stream, w.dtype), kc, vc,
                        torch.from_numpy(np.concatenate(slots)).cuda())
    return kc, vc, table, lens


def run_prefill(inp, kc, vc, table, lens, qs=None):
    B = _bin()
    w = inp.w
    q = to_dev(inp.q, w.dtype)
    out = torch.full_like(q, float("nan"))
    qs = inp.query_start if qs is None else qs
    B.paged_prefill(out, q, kc, vc, torch.from_numpy(table).cuda(), torch.from_numpy(qs).cuda(),
                    torch.from_numpy(lens).cuda(), w.scale, int(inp.chunk.max()))
    torch.cuda.synchronize()
    return out


def oracle_prefill_batch(inp, poison=True, rows=None):
    """The oracle over its own pool; rows (optional): {seq: [row indices in the
    chunk]} to compute only those query rows (each as a one-token chunk at its
    position, which is the same definition)."""
    w = inp.w
    S = w.num_seqs
    m = AllocatorModel(w.num_blocks, w.block_size, inp.frame_order)
    slots = []
    for s in range(S):
        slots += m.add_seq(s, int(inp.context_lens[s]))
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    fill = POISON[w.dtype] if poison else 0
    kc = np.full(shape, fill, np.uint16)
    vc = np.full(shape, fill, np.uint16)
    oracle.reshape_and_cache(kc, vc, inp.k_stream, inp.v_stream, np.array(slots, np.int64), w.block_size)
    tables, _ = m.block_table(range(S), w.max_blocks_per_seq)
    tables = np.array(tables, np.int32)
    out = np.zeros(inp.q.shape, np.float64)
    for s in range(S):
        a = int(inp.query_start[s])
        p0 = int(inp.cached[s])
        if int(inp.chunk[s]) == 0:
            continue  # no new tokens: no rows
        if rows is None:
            out[a:a + int(inp.chunk[s])] = oracle.paged_prefill(
                inp.q[a:a + int(inp.chunk[s])], kc, vc, tables[s], p0, w.scale, w.num_kv_heads,
                w.block_size, w.dtype)
        else:
            for i in rows.get(s, []):
                out[a + i:a + i + 1] = oracle.paged_prefill(inp.q[a + i:a + i + 1], kc, vc, tables[s],
                                                            p0 + i, w.scale, w.num_kv_heads,
                                                            w.block_size, w.dtype)
    return out, tables


def max_err(out, ref, rows=None):
    g = out.double().cpu().numpy()
    if rows is not None:
        g, ref = g[rows], ref[rows]
    return float(np.abs(g - ref).max())


def assert_within_tolerance(out, ref, dtype, rows=None):
    """Every element within the tolerance, or within half an ulp of the exact
    value in the output type where that is larger (stored_tolerance)."""
    g = out.double().cpu().numpy()
    if rows is not None:
        g, ref = g[rows], ref[rows]
    bound = stored_tolerance(ref, dtype)
    worst = float((np.abs(g - ref) - bound).max())
    assert worst <= 0.0, (worst, float(np.abs(g - ref).max()))


# Cached prefixes of 0 (a whole prompt), a few tokens and several tiles; chunks
# of 1 token, across tile and block boundaries, and several query tiles.
CACHED = [0, 5, 40, 300, 129]
CHUNK = [130, 1, 77, 200, 256]


@pytest.mark.parametrize("dtype", [wl.F16, wl.BF16])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_prefill_matches_oracle(dtype, D, G, bs):
    mb = -(-(max(c + t for c, t in zip(CACHED, CHUNK))) // bs) + 1
    w = _workload(dtype, D, G, bs, frames=len(CACHED) * mb + 7, max_blocks=mb, seed=81 + G)
    inp = wl.make_prefill_inputs(w, cached=CACHED, chunk=CHUNK)
    kc, vc, table, lens = gpu_prefill_batch(inp)
    out = run_prefill(inp, kc, vc, table, lens)
    assert _bin().device_error() == 0
    ref, tables = oracle_prefill_batch(inp)
    assert np.array_equal(tables, table)
    assert torch.isfinite(out).all()
    err = max_err(out, ref)
    assert_within_tolerance(out, ref, dtype)
    if dtype == wl.BF16 and D == 128 and G == 4 and bs == 16:
        print(f"prefill vs rounded oracle: {rounded_oracle_stats(out, ref, dtype)}, max-abs {err:.3e}")


def test_prefill_first_prompt_token_returns_its_value_bit_exact():
    """Token 0 of a whole prompt (nothing cached) sees only itself: weight 1, so
    every head of a group returns its V row bit for bit."""
    w = _workload(wl.BF16, 128, 4, 16, frames=64, max_blocks=20, seed=90)
    inp = wl.make_prefill_inputs(w, cached=[0, 0, 17], chunk=[300, 1, 40])
    kc, vc, table, lens = gpu_prefill_batch(inp)
    out = run_prefill(inp, kc, vc, table, lens)
    got = from_dev(out)
    for s in (0, 1):
        row = inp.query_start[s]
        v0 = inp.v_stream[inp.offsets[s]]                       # [Hkv, D]
        assert np.array_equal(got[row], np.repeat(v0, w.group, axis=0)), s


@pytest.mark.parametrize("dtype", [wl.F16, wl.BF16])
@pytest.mark.parametrize("c", [1.0, -3.0])
def test_prefill_constant_values_give_the_constant_exactly(dtype, c):
    """V = c everywhere: the output is a convex combination of equal rows whose
    weights are normalised by their own (rounded) sum, so out = c exactly after
    the final rounding."""
    w = _workload(dtype, 128, 4, 16, frames=200, max_blocks=40, seed=91)
    inp = wl.make_prefill_inputs(w, cached=CACHED, chunk=CHUNK)
    cbits = wl.to_bits(np.array([c], np.float32), dtype)[0]
    inp = dataclasses.replace(inp, v_stream=np.full_like(inp.v_stream, cbits))
    kc, vc, table, lens = gpu_prefill_batch(inp)
    out = run_prefill(inp, kc, vc, table, lens)
    assert torch.all(out.double() == c)


def test_prefill_in_chunks_equals_whole_prompt_bit_exact():
    """A prompt prefilled as one chunk or as three consecutive chunks (each
    attending over the cache the earlier ones filled) gives bit-identical rows:
    a row's arithmetic depends only on its keys, in the same tile order."""
    w = _workload(wl.BF16, 128, 4, 16, frames=64, max_blocks=40, seed=92)
    whole = wl.make_prefill_inputs(w, cached=[0], chunk=[600])
    kc, vc, table, lens = gpu_prefill_batch(whole)
    out_whole = run_prefill(whole, kc, vc, table, lens)
    pieces = []
    for a, b in ((0, 150), (150, 420), (420, 600)):
        part = dataclasses.replace(whole, q=whole.q[a:b], cached=np.array([a], np.int32),
                                   chunk=np.array([b - a], np.int32),
                                   query_start=np.array([0, b - a], np.int32))
        lens_b = np.array([b], np.int32)
        pieces.append(run_prefill(part, kc, vc, table, lens_b))
    assert torch.equal(torch.cat(pieces), out_whole)


def test_prefill_permutation_of_physical_frames_is_bit_identical():
    B = _bin()
    w = _workload(wl.BF16, 128, 4, 16, frames=200, max_blocks=40, seed=93)
    inp = wl.make_prefill_inputs(w, cached=CACHED, chunk=CHUNK)
    kc, vc, table, lens = gpu_prefill_batch(inp)
    out = run_prefill(inp, kc, vc, table, lens)
    pi = np.random.default_rng(3).permutation(w.num_blocks)
    pit = torch.from_numpy(pi).cuda()
    k2, v2 = torch.empty_like(kc), torch.empty_like(vc)
    k2[pit] = kc
    v2[pit] = vc
    t2 = np.where(table >= 0, pi[np.maximum(table, 0)], table).astype(np.int32)
    out2 = run_prefill(inp, k2, v2, t2, lens)
    assert B.device_error() == 0
    assert torch.equal(out, out2)


def test_prefill_last_token_agrees_with_decode():
    """The last new token of a chunk sees exactly the context the decode of that
    token sees: prefill and decode (different kernels and arithmetic) agree
    within the tolerance."""
    B = _bin()
    w = _workload(wl.BF16, 128, 4, 16, frames=200, max_blocks=40, seed=94)
    inp = wl.make_prefill_inputs(w, cached=CACHED, chunk=CHUNK)
    kc, vc, table, lens = gpu_prefill_batch(inp)
    out = run_prefill(inp, kc, vc, table, lens)
    last = torch.from_numpy(inp.query_start[1:] - 1).long().cuda()
    q_last = to_dev(inp.q, w.dtype)[last].contiguous()
    dec = torch.empty_like(q_last)
    B.paged_attention_decode(dec, q_last, kc, vc, torch.from_numpy(table).cuda(),
                             torch.from_numpy(lens).cuda(), w.scale)
    torch.cuda.synchronize()
    # both within the tolerance of the exact value: within twice it of each other
    assert (dec.double() - out[last].double()).abs().max().item() <= 2 * TOL[wl.BF16]


def test_prefill_bad_lengths_set_flags_without_faulting():
    B = _bin()
    w = _workload(wl.F16, 64, 2, 16, frames=64, max_blocks=20, seed=95)
    inp = wl.make_prefill_inputs(w, cached=[10, 0], chunk=[30, 50])
    kc, vc, table, lens = gpu_prefill_batch(inp)
    run_prefill(inp, kc, vc, table, lens)
    assert B.device_error() == 0
    bad = lens.copy()
    bad[0] = 20  # shorter than its 30-token chunk: clamped to 30
    run_prefill(inp, kc, vc, table, bad)
    assert B.device_error() & B.DEVERR_CONTEXT_LEN
    qs = inp.query_start.copy()
    qs[2] = qs[2] + 5  # past the query rows: the chunk is skipped
    q = to_dev(inp.q, w.dtype)
    out = torch.zeros_like(q)
    B.paged_prefill(out, q, kc, vc, torch.from_numpy(table).cuda(), torch.from_numpy(qs).cuda(),
                    torch.from_numpy(lens).cuda(), w.scale, 60)
    torch.cuda.synchronize()
    assert B.device_error() & B.DEVERR_CONTEXT_LEN


def test_prefill_odd_group_empty_chunk_and_spare_row_tiles():
    """Three query heads per kv head (an odd group: each CTA takes two
    consecutive 128-row tiles of one head), a sequence with no new tokens in the
    batch, and max_query_len above the longest chunk, so the grid has row tiles
    with no rows.  Every row of every chunk against the oracle; the q rows past
    the last chunk belong to no sequence and their output rows stay untouched."""
    B = _bin()
    cached, chunk = [5, 0, 64, 17, 200], [0, 1, 129, 300, 45]
    mb = -(-max(c + t for c, t in zip(cached, chunk)) // 16) + 1
    w = _workload(wl.BF16, 128, 3, 16, frames=len(cached) * mb + 7, max_blocks=mb, seed=97)
    inp = wl.make_prefill_inputs(w, cached=cached, chunk=chunk)
    kc, vc, table, lens = gpu_prefill_batch(inp)
    spare = 9
    q = to_dev(inp.q, w.dtype)
    q = torch.cat([q, torch.zeros((spare,) + tuple(q.shape[1:]), dtype=q.dtype, device=q.device)])
    out = torch.full_like(q, float("nan"))
    B.paged_prefill(out, q, kc, vc, torch.from_numpy(table).cuda(),
                    torch.from_numpy(inp.query_start).cuda(), torch.from_numpy(lens).cuda(), w.scale, 512)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    rows = int(inp.query_start[-1])
    assert torch.isnan(out[rows:]).all()
    ref, tables = oracle_prefill_batch(inp)
    assert np.array_equal(tables, table)
    assert torch.isfinite(out[:rows]).all()
    assert_within_tolerance(out[:rows], ref, wl.BF16)


def test_prefill_full_size_batch_sampled_rows():
    """The benchmark's chunked-prefill batch (16 sequences, 32/8 heads, bf16,
    chunks of 256-2048 tokens after 0-4096 cached ones) in the benchmark's launch;
    the oracle checks 24 rows of every sequence (first, last and random ones,
    every head), each computed on its own as a one-token chunk at its position."""
    inp = wl.make_prefill_inputs("prefill")
    kc, vc, table, lens = gpu_prefill_batch(inp)
    out = run_prefill(inp, kc, vc, table, lens)
    assert _bin().device_error() == 0
    assert torch.isfinite(out).all()
    rng = np.random.default_rng(96)
    rows = {}
    for s in range(inp.w.num_seqs):
        T = int(inp.chunk[s])
        rows[s] = sorted({0, T - 1, min(127, T - 1), min(128, T - 1)} |
                         set(rng.choice(T, size=20, replace=False).tolist()))
    ref, _ = oracle_prefill_batch(inp, rows=rows)
    idx = np.concatenate([inp.query_start[s] + np.array(r) for s, r in rows.items()])
    assert_within_tolerance(out, ref, wl.BF16, idx)
