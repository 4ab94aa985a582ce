"""The allocation-free decode entry point (pkv_paged_attention_decode_static).

It serves callers that cannot allocate device memory at decode time (a fixed
up-front memory plan, a plugin hook that must not allocate, an allocator owned
by someone else): its scratch lives in one array inside the library.  These
tests call it through the C ABI and check its output against the workspace-
taking entry point on two calls in a row with different batches, queued back to
back on one stream (the shared scratch keeps the previous call's contents, which
must not leak into the next result).  The two entry points run the same kernels
with the same partitions, so the outputs must be bit-identical, well inside the
tolerance the other parity tests use.

The file name sorts last so that a run stopping at the first failure has run
every other test first; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl
from flow import gpu_step_inputs, gpu_decode_step

pytestmark = pytest.mark.gpu


def _static_decode(b, w, out, partition_size):
    from paged_kv_cache_419_b200 import binding as B

    S, Hq, D = b.q.shape
    N, Hkv, Bs, _ = b.k_cache.shape
    return B.lib().pkv_paged_attention_decode_static(
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(b.q.data_ptr()),
        ctypes.c_void_p(b.k_cache.data_ptr()), ctypes.c_void_p(b.v_cache.data_ptr()),
        ctypes.c_void_p(b.tables.data_ptr()), ctypes.c_void_p(b.lens.data_ptr()),
        S, b.tables.shape[1], N, float(w.scale), Hq, Hkv, D, Bs,
        B.PKV_F16 if b.q.dtype == torch.float16 else B.PKV_BF16, partition_size,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _batch(seed, lengths):
    w = wl.WORKLOADS["long"]
    inp = wl.make_decode_inputs(w, seed=seed, lengths=np.array(lengths, np.int32))
    b = gpu_step_inputs(inp)
    ref = gpu_decode_step(inp, b, partition_size=512)   # workspace-taking entry point
    return inp.w, b, ref


def test_static_scratch_matches_workspace_entry_on_two_calls_in_a_row():
    from paged_kv_cache_419_b200 import binding as B

    # two different long-context batches: 4 x (16K..32K) tokens need 4 MiB of scratch
    batches = [_batch(40, [32768, 16384, 20001, 25000]), _batch(41, [17000, 31999, 16384, 29000])]
    torch.cuda.synchronize()
    assert B.device_error() == 0
    # Both calls queued back to back on one stream with no host synchronisation in
    # between, each into its own output: the second call's planning kernel resets
    # the shared array's counters while nothing of the first call is still running.
    outs = [torch.full_like(ref, float("nan")) for _, _, ref in batches]
    for (w, b, _), out in zip(batches, outs):
        assert _static_decode(b, w, out, 512) == B.PKV_OK
    torch.cuda.synchronize()
    assert B.device_error() == 0
    for (_, _, ref), out in zip(batches, outs):
        # same partitions, same arithmetic order: bit-identical to the workspace entry
        assert torch.equal(out, ref)
    # and once more, one call at a time, reusing the array's leftover contents
    for (w, b, ref), out in zip(batches, outs):
        out.fill_(float("nan"))
        assert _static_decode(b, w, out, 512) == B.PKV_OK
        torch.cuda.synchronize()
        assert B.device_error() == 0
        assert torch.equal(out, ref)


def test_static_scratch_rejects_shapes_beyond_its_size():
    from paged_kv_cache_419_b200 import binding as B

    w = wl.WORKLOADS["gqa8b"]
    need = B.decode_workspace_bytes(w.num_seqs, w.num_heads, w.head_dim,
                                    w.max_blocks_per_seq * w.block_size, 512)
    assert need > 16 << 20
    inp = wl.make_decode_inputs(w, num_seqs=w.num_seqs, lengths=np.full(w.num_seqs, 16, np.int32))
    b = gpu_step_inputs(inp, poison=False)
    out = torch.zeros_like(b.q)
    assert _static_decode(b, w, out, 512) == B.PKV_EUNSUPPORTED
    torch.cuda.synchronize()
    assert torch.all(out == 0)
