"""One decode step, run twice from the same seeded inputs:

* on the GPU through the library (C++ allocator -> cache write kernel -> decode
  kernels), and
* on the CPU through the oracle (allocator model -> oracle scatter -> oracle
  decode).

The two sides share only the inputs from ``workloads``.  Each sequence's first
L-1 tokens are the cached context (written as a prefill); the decode step then
appends token L-1 (allocator append -> cache write) and attends over all L.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import oracle
from oracle.allocator_model import AllocatorModel
import workloads as wl

TOL = {wl.F16: 2e-3, wl.BF16: 1e-2}   # max-abs error against the fp64 oracle
POISON = {wl.F16: 0x7E00, wl.BF16: 0x7FC0}   # quiet NaN bit patterns


def torch_dtype(dtype):
    return torch.float16 if dtype == wl.F16 else torch.bfloat16


def to_dev(bits: np.ndarray, dtype, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch_dtype(dtype)).to(device)


def from_dev(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def split_stream(inp: wl.DecodeInputs):
    """Rows of the cached context (all but each sequence's last token) and the
    appended token's rows."""
    last = inp.offsets[1:] - 1
    keep = np.ones(inp.total_tokens, dtype=bool)
    keep[last] = False
    return (inp.k_stream[keep], inp.v_stream[keep], inp.k_stream[last], inp.v_stream[last])


@dataclasses.dataclass
class GpuBatch:
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    tables: torch.Tensor
    lens: torch.Tensor
    new_k: torch.Tensor
    new_v: torch.Tensor
    new_slots: torch.Tensor
    tables_host: np.ndarray


def gpu_step_inputs(inp: wl.DecodeInputs, poison: bool = True, device="cuda") -> GpuBatch:
    """Allocate the pool, write the cached context with the cache-write kernel and
    reserve the decode step's slots with the C++ allocator.  The appended token is
    not written yet (``gpu_decode_step`` does that)."""
    from paged_kv_cache_419_b200.binding import BlockAllocator, reshape_and_cache

    w = inp.w
    S = w.num_seqs
    alloc = BlockAllocator(w.num_blocks, w.block_size, inp.frame_order)
    pre = [alloc.add_seq(s, int(inp.context_lens[s]) - 1) for s in range(S)]
    new_slots, pairs = alloc.append_batch(np.arange(S, dtype=np.int32))
    assert pairs.shape[0] == 0
    table, lens = alloc.block_table(np.arange(S, dtype=np.int32), w.max_blocks_per_seq)
    assert np.array_equal(lens, inp.context_lens)
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    fill = POISON[w.dtype] if poison else 0
    td = torch_dtype(w.dtype)
    k_cache = torch.full(shape, fill, dtype=torch.int16, device=device).view(td) if poison else torch.zeros(shape, dtype=td, device=device)
    v_cache = torch.full(shape, fill, dtype=torch.int16, device=device).view(td) if poison else torch.zeros(shape, dtype=td, device=device)
    pk, pv, nk, nv = split_stream(inp)
    if pk.shape[0]:
        reshape_and_cache(to_dev(pk, w.dtype, device), to_dev(pv, w.dtype, device), k_cache, v_cache,
                          torch.from_numpy(np.concatenate(pre)).to(device))
    tab = np.where(table >= 0, table, -1).astype(np.int32)
    return GpuBatch(
        q=to_dev(inp.q, w.dtype, device), k_cache=k_cache, v_cache=v_cache,
        tables=torch.from_numpy(tab).to(device), lens=torch.from_numpy(lens.astype(np.int32)).to(device),
        new_k=to_dev(nk, w.dtype, device), new_v=to_dev(nv, w.dtype, device),
        new_slots=torch.from_numpy(new_slots.astype(np.int64)).to(device), tables_host=tab)


def gpu_decode_step(inp: wl.DecodeInputs, b: GpuBatch, partition_size: int = 0, out=None,
                    workspace=None):
    from paged_kv_cache_419_b200.binding import paged_attention_decode, reshape_and_cache

    w = inp.w
    reshape_and_cache(b.new_k, b.new_v, b.k_cache, b.v_cache, b.new_slots)
    if out is None:
        out = torch.empty_like(b.q)
    paged_attention_decode(out, b.q, b.k_cache, b.v_cache, b.tables, b.lens, w.scale,
                           partition_size=partition_size, workspace=workspace)
    return out


@dataclasses.dataclass
class OracleBatch:
    k_cache: np.ndarray
    v_cache: np.ndarray
    tables: np.ndarray
    lens: np.ndarray


def oracle_step_inputs(inp: wl.DecodeInputs, poison: bool = True) -> OracleBatch:
    """The same step on the CPU: allocator model, oracle scatter of the context and
    of the appended token.  The pool starts with the same fill as the GPU pool
    (NaN bit patterns, or zeros), so whole frames can be compared byte for byte."""
    w = inp.w
    S = w.num_seqs
    m = AllocatorModel(w.num_blocks, w.block_size, inp.frame_order)
    pre = []
    for s in range(S):
        pre += m.add_seq(s, int(inp.context_lens[s]) - 1)
    new = [m.append(s)[0] for s in range(S)]
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    fill = POISON[w.dtype] if poison else 0
    kc = np.full(shape, fill, np.uint16)
    vc = np.full(shape, fill, np.uint16)
    pk, pv, nk, nv = split_stream(inp)
    oracle.reshape_and_cache(kc, vc, pk, pv, np.array(pre, np.int64), w.block_size)
    oracle.reshape_and_cache(kc, vc, nk, nv, np.array(new, np.int64), w.block_size)
    tables, lens = m.block_table(range(S), w.max_blocks_per_seq)
    return OracleBatch(kc, vc, np.array(tables, np.int32), np.array(lens, np.int32))


def oracle_decode(inp: wl.DecodeInputs, ob: OracleBatch, seqs=None) -> np.ndarray:
    w = inp.w
    return oracle.paged_decode(inp.q, ob.k_cache, ob.v_cache, ob.tables, ob.lens, w.scale,
                               w.num_kv_heads, w.block_size, w.dtype, seqs=seqs)


def max_abs_err(gpu_out: torch.Tensor, ref: np.ndarray, rows=None) -> float:
    g = gpu_out.detach().float().cpu().numpy().astype(np.float64)
    if rows is not None:
        g, ref = g[rows], ref[rows]
    return float(np.abs(g - ref).max()) if g.size else 0.0


def ulp_distance(out_bits: np.ndarray, ref_bits: np.ndarray) -> np.ndarray:
    """Number of representable 16-bit values between two fp16 / bf16 bit patterns
    (sign-magnitude mapped onto one ordered integer line; +0 and -0 coincide)."""
    def line(b):
        b = b.astype(np.int64)
        mag = b & 0x7FFF
        return np.where(b & 0x8000, -mag, mag)
    return np.abs(line(out_bits) - line(ref_bits))


def rounded_oracle_stats(gpu_out: torch.Tensor, ref: np.ndarray, dtype) -> dict:
    """Error of the GPU output against the oracle rounded to the output type (round
    to nearest even, one rounding from fp64): share of bit-identical elements,
    share within one ulp, and the largest distance in ulps."""
    got = from_dev(gpu_out).reshape(-1)
    want = oracle.round_to_dtype(ref, dtype).reshape(-1)
    d = ulp_distance(got, want)
    return {"elements": int(d.size), "identical": float(np.mean(d == 0)),
            "within_1_ulp": float(np.mean(d <= 1)), "max_ulp": int(d.max()) if d.size else 0}


def stored_tolerance(ref: np.ndarray, dtype) -> np.ndarray:
    """Per-element bound for an output stored in fp16 / bf16: the absolute
    tolerance, or half an ulp of the exact value in the output type when that is
    larger (bf16 values of magnitude 4 and up are 2^-5 apart, so even the exact
    result rounded once can miss 1e-2; the decode's outputs are averages of many
    rows and stay far below that, a prefill row over a handful of keys need not)."""
    mant = 8 if dtype == wl.BF16 else 11      # significant bits of the format
    a = np.abs(ref)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    half_ulp = np.where(a > 0, np.exp2(e - mant), 0.0)
    return np.maximum(TOL[dtype], half_ulp)
