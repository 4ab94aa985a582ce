"""ctypes binding of libpkv.so (include/pkv.h).

Argument marshalling only: tensors become device pointers and sizes, the
current torch CUDA stream becomes the cudaStream_t, and a non-zero status
becomes a ``PkvError``.  Every step of the computation runs in the library's
CUDA kernels; there is no fallback of any kind.  PyTorch supplies device memory
and streams.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpkv.so")

PKV_OK, PKV_EINVAL, PKV_EUNSUPPORTED, PKV_ECUDA, PKV_ENOMEM, PKV_ERANGE = 0, -1, -2, -3, -4, -5
PKV_F16, PKV_BF16 = 0, 1
DEVERR_TABLE_ENTRY, DEVERR_CONTEXT_LEN, DEVERR_SLOT, DEVERR_COPY_PAIR, DEVERR_WAIT_TIMEOUT = (
    1, 2, 4, 8, 16)

# Every function include/pkv.h declares.
EXPORTS = (
    "pkv_status_string", "pkv_last_cuda_error", "pkv_cuda_error_name", "pkv_device_error",
    "pkv_decode_workspace_bytes",
    "pkv_paged_attention_decode", "pkv_paged_attention_decode_static",
    "pkv_contiguous_attention_decode", "pkv_reshape_and_cache",
    "pkv_copy_blocks", "pkv_alloc_create", "pkv_alloc_destroy", "pkv_alloc_add_seq",
    "pkv_alloc_fork", "pkv_alloc_append", "pkv_alloc_append_batch", "pkv_alloc_free_seq",
    "pkv_alloc_beam_step", "pkv_alloc_block_table", "pkv_alloc_refcount", "pkv_alloc_stats",
    "pkv_alloc_add_seq_cached", "pkv_block_hash", "pkv_test_set_merge_wait", "pkv_paged_prefill",
    "pkv_test_partitions",
)


class PkvError(RuntimeError):
    """A pkv_* call returned an error status; for PKV_ECUDA the message names the
    CUDA error behind it (``cuda_error``, the cudaError_t value)."""

    def __init__(self, status: int, what: str):
        self.status = status
        self.cuda_error = last_cuda_error() if status == PKV_ECUDA else 0
        msg = f"{what}: {status_string(status)}"
        if status == PKV_ECUDA:
            msg += f" ({cuda_error_name(self.cuda_error)})"
        super().__init__(msg)


class AllocStats(ctypes.Structure):
    _fields_ = [("used_blocks", ctypes.c_int64), ("free_blocks", ctypes.c_int64),
                ("tokens", ctypes.c_int64), ("shared_blocks", ctypes.c_int64),
                ("logical_blocks", ctypes.c_int64), ("cached_blocks", ctypes.c_int64)]


def block_hash(parent_key, token_ids) -> bytes:
    """Prefix-cache key of one block (pkv_block_hash): SHA-256 of the parent key
    (32 zero bytes when None) and the token ids as little-endian int32."""
    import numpy as np

    toks = np.ascontiguousarray(token_ids, dtype=np.int32)
    out = (ctypes.c_uint8 * 32)()
    par = None if parent_key is None else (ctypes.c_uint8 * 32).from_buffer_copy(bytes(parent_key))
    _check(lib().pkv_block_hash(par, toks.ctypes.data_as(ctypes.c_void_p), toks.shape[0], out),
           "pkv_block_hash")
    return bytes(out)


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library.  Raises if libpkv.so has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_419_b200.build` "
                "(there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, i64, sz, f32 = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                                ctypes.c_float)
        sig = {
            "pkv_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "pkv_device_error": ([P, ctypes.c_int, P], ctypes.c_int),
            "pkv_decode_workspace_bytes": ([i32, i32, i32, i32, i32], sz),
            "pkv_paged_attention_decode": (
                [P, P, P, P, P, P, i32, i32, i32, f32, i32, i32, i32, i32, ctypes.c_int, i32, P, sz,
                 P], ctypes.c_int),
            "pkv_paged_attention_decode_static": (
                [P, P, P, P, P, P, i32, i32, i32, f32, i32, i32, i32, i32, ctypes.c_int, i32, P],
                ctypes.c_int),
            "pkv_contiguous_attention_decode": (
                [P, P, P, P, P, i32, i32, f32, i32, i32, i32, ctypes.c_int, i32, P, sz, P],
                ctypes.c_int),
            "pkv_reshape_and_cache": ([P, P, P, P, P, i32, i32, i32, i32, i32, ctypes.c_int, P],
                                      ctypes.c_int),
            "pkv_copy_blocks": ([P, P, P, i32, i64, i32, P], ctypes.c_int),
            "pkv_alloc_create": ([i32, i32, P, P], ctypes.c_int),
            "pkv_alloc_destroy": ([P], None),
            "pkv_alloc_add_seq": ([P, i32, i32, P], ctypes.c_int),
            "pkv_alloc_fork": ([P, i32, i32], ctypes.c_int),
            "pkv_alloc_append": ([P, i32, P, P, P], ctypes.c_int),
            "pkv_alloc_append_batch": ([P, P, i32, P, P, P], ctypes.c_int),
            "pkv_alloc_free_seq": ([P, i32], ctypes.c_int),
            "pkv_alloc_beam_step": ([P, P, i32, P, i32, P, P, P, P, P], ctypes.c_int),
            "pkv_alloc_add_seq_cached": ([P, i32, P, i32, P, P], ctypes.c_int),
            "pkv_block_hash": ([P, P, i32, P], ctypes.c_int),
            "pkv_alloc_block_table": ([P, P, i32, i32, P, P], ctypes.c_int),
            "pkv_alloc_refcount": ([P, i32, P], ctypes.c_int),
            "pkv_alloc_stats": ([P, ctypes.POINTER(AllocStats)], ctypes.c_int),
            "pkv_test_set_merge_wait": ([ctypes.c_uint64, ctypes.c_uint32], ctypes.c_int),
            "pkv_test_partitions": ([P, i32, i32, i32, i32, i32, i32, P, P, P, P], ctypes.c_int),
            "pkv_last_cuda_error": ([], ctypes.c_int),
            "pkv_cuda_error_name": ([ctypes.c_int], ctypes.c_char_p),
            "pkv_paged_prefill": ([P, P, P, P, P, P, P, i32, i32, i32, i32, i32, f32, i32, i32, i32, i32,
                                   ctypes.c_int, P], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().pkv_status_string(status).decode()


def last_cuda_error() -> int:
    """cudaError_t behind the last PKV_ECUDA of this thread (0 if none)."""
    return int(lib().pkv_last_cuda_error())


def cuda_error_name(error: int) -> str:
    return lib().pkv_cuda_error_name(error).decode()


def _check(status: int, what: str):
    if status != PKV_OK:
        raise PkvError(status, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return PKV_F16
    if t.dtype == torch.bfloat16:
        return PKV_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; fp16 or bf16")


def _dev(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


# ---------------------------------------------------------------- decode
def decode_workspace_bytes(num_seqs: int, num_heads: int, head_dim: int, max_context_len: int,
                           partition_size: int = 0) -> int:
    return int(lib().pkv_decode_workspace_bytes(num_seqs, num_heads, head_dim, max_context_len,
                                                 partition_size))


def _workspace(workspace, need: int, device):
    if need == 0:
        raise ValueError("invalid decode arguments (no workspace size)")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace too small: {need} bytes needed")
    return workspace, workspace.numel() * workspace.element_size()


def paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                           partition_size: int = 0, workspace=None, stream=None):
    """out[s,h] = softmax(scale q[s,h] K_s^T) V_s over the paged cache.

    q, out: [S, Hq, D]; k_cache, v_cache: [N, Hkv, B, D] (fp16/bf16);
    block_tables int32 [S, MB]; context_lens int32 [S]."""
    S, Hq, D = q.shape
    N, Hkv, B, D2 = k_cache.shape
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != (S, Hq, D):
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables must be [S, MB] and context_lens [S]")
    MB = block_tables.shape[1]
    need = decode_workspace_bytes(S, Hq, D, MB * B, partition_size)
    ws, ws_bytes = _workspace(workspace, need, q.device)
    dt = _dtype_code(q)
    for t, n in ((out, "out"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        if t.dtype != q.dtype:
            raise TypeError(f"{n} must have q's dtype")
    _check(lib().pkv_paged_attention_decode(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), _dev(context_lens, "context_lens", torch.int32),
        S, MB, N, float(scale), Hq, Hkv, D, B, dt, partition_size,
        None if ws is None else ctypes.c_void_p(ws.data_ptr()), ws_bytes, _stream(stream)),
        "pkv_paged_attention_decode")
    return out


def contiguous_attention_decode(out, q, k, v, context_lens, scale: float, partition_size: int = 0,
                                workspace=None, stream=None):
    """Same attention over a contiguous cache k, v: [S, Hkv, max_ctx, D]."""
    S, Hq, D = q.shape
    S2, Hkv, max_ctx, D2 = k.shape
    if S2 != S or D2 != D or tuple(v.shape) != tuple(k.shape) or tuple(out.shape) != (S, Hq, D):
        raise ValueError("shape mismatch")
    need = decode_workspace_bytes(S, Hq, D, max_ctx, partition_size)
    ws, ws_bytes = _workspace(workspace, need, q.device)
    _check(lib().pkv_contiguous_attention_decode(
        _dev(out, "out"), _dev(q, "q"), _dev(k, "k"), _dev(v, "v"),
        _dev(context_lens, "context_lens", torch.int32), S, max_ctx, float(scale), Hq, Hkv, D,
        _dtype_code(q), partition_size, None if ws is None else ctypes.c_void_p(ws.data_ptr()),
        ws_bytes, _stream(stream)), "pkv_contiguous_attention_decode")
    return out


# ---------------------------------------------------------- cache write / copy
def paged_prefill(out, q, k_cache, v_cache, block_tables, query_start, context_lens, scale: float,
                  max_query_len: int, stream=None):
    """Causal attention of each sequence's new tokens (q rows query_start[s] ..
    query_start[s+1]) over its paged context of context_lens[s] tokens
    (pkv_paged_prefill).  q, out: [total_tokens, Hq, D]; caches [N, Hkv, B, D]."""
    total, Hq, D = q.shape
    N, Hkv, Bs, D2 = k_cache.shape
    if D2 != D or tuple(out.shape) != tuple(q.shape):
        raise ValueError("shape mismatch between q, out and the caches")
    S = context_lens.shape[0]
    if query_start.shape[0] != S + 1:
        raise ValueError("query_start must hold num_seqs + 1 offsets")
    _check(lib().pkv_paged_prefill(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), _dev(query_start, "query_start", torch.int32),
        _dev(context_lens, "context_lens", torch.int32), S, int(max_query_len), total,
        block_tables.shape[1], N, float(scale), Hq, Hkv, D, Bs, _dtype_code(q), _stream(stream)),
        "pkv_paged_prefill")


def reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, stream=None):
    """Scatter key/value [T, Hkv, D] into the caches [N, Hkv, B, D] at slot_mapping (int64 [T])."""
    T, Hkv, D = key.shape
    N, Hkv2, B, D2 = k_cache.shape
    if Hkv2 != Hkv or D2 != D or tuple(value.shape) != tuple(key.shape) or slot_mapping.shape != (T,):
        raise ValueError("shape mismatch")
    _check(lib().pkv_reshape_and_cache(
        _dev(key, "key"), _dev(value, "value"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(slot_mapping, "slot_mapping", torch.int64), T, Hkv, D, B, N, _dtype_code(k_cache),
        _stream(stream)), "pkv_reshape_and_cache")


def copy_blocks(k_cache, v_cache, src_dst_pairs, stream=None):
    """Copy whole frames src -> dst in both caches; src_dst_pairs int64 [n, 2] on the device."""
    n = src_dst_pairs.shape[0] if src_dst_pairs.numel() else 0
    N = k_cache.shape[0]
    block_bytes = k_cache[0].numel() * k_cache.element_size()
    _check(lib().pkv_copy_blocks(
        _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(src_dst_pairs, "src_dst_pairs", torch.int64) if n else None, n, block_bytes, N,
        _stream(stream)), "pkv_copy_blocks")


def device_error(clear: bool = True, stream=None) -> int:
    flags = ctypes.c_uint(0)
    _check(lib().pkv_device_error(ctypes.byref(flags), int(clear), _stream(stream)),
           "pkv_device_error")
    return flags.value


def set_merge_wait_hook(limit_ns: int = 0, extra: int = 0):
    """Bounded-wait test hook (pkv_test_set_merge_wait): later decode calls make
    the partition merge wait for ``extra`` more publications than the decode grid
    makes and give up after ``limit_ns`` (0, 0 restores normal operation)."""
    _check(lib().pkv_test_set_merge_wait(int(limit_ns), int(extra)), "pkv_test_set_merge_wait")


def partitions(context_lens, num_kv_heads: int, max_context_len: int, block_size: int,
               partition_size: int, grid_ctas: int):
    """Partition rule test hook (pkv_test_partitions, host only): per context,
    (n_parts, n_big, p_big, p_small) as int32 arrays; the first n_big partitions
    hold p_big tokens, the others p_small, the last one shorter."""
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    S = int(lens.shape[0])
    outs = [np.zeros(S, np.int32) for _ in range(4)]
    _check(lib().pkv_test_partitions(lens.ctypes.data, S, int(num_kv_heads), int(max_context_len),
                                     int(block_size), int(partition_size), int(grid_ctas),
                                     *[o.ctypes.data for o in outs]), "pkv_test_partitions")
    return tuple(outs)


# ---------------------------------------------------------------- allocator
class BlockAllocator:
    """Host refcounted block allocator (libpkv's C++ implementation)."""

    def __init__(self, num_blocks: int, block_size: int, frame_order=None):
        import numpy as np

        self._np = np
        self.num_blocks = num_blocks
        self.block_size = block_size
        h = ctypes.c_void_p()
        order = None
        if frame_order is not None:
            order = np.ascontiguousarray(frame_order, dtype=np.int32)
            if order.shape != (num_blocks,):
                raise ValueError("frame_order must have num_blocks entries")
        _check(lib().pkv_alloc_create(num_blocks, block_size,
                                      None if order is None else order.ctypes.data_as(ctypes.c_void_p),
                                      ctypes.byref(h)), "pkv_alloc_create")
        self._h = h

    def close(self):
        if self._h:
            lib().pkv_alloc_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_seq(self, seq_id: int, prompt_len: int):
        slots = self._np.empty(max(prompt_len, 1), dtype=self._np.int64)
        _check(lib().pkv_alloc_add_seq(self._h, seq_id, prompt_len,
                                       slots.ctypes.data_as(ctypes.c_void_p)), "pkv_alloc_add_seq")
        return slots[:prompt_len]

    def add_seq_cached(self, seq_id: int, token_ids):
        """New sequence through the prefix cache: returns (slots, cached_tokens)."""
        np = self._np
        toks = np.ascontiguousarray(token_ids, dtype=np.int32)
        n = toks.shape[0]
        slots = np.empty(max(n, 1), dtype=np.int64)
        cached = ctypes.c_int32()
        _check(lib().pkv_alloc_add_seq_cached(self._h, seq_id, toks.ctypes.data_as(ctypes.c_void_p), n,
                                              slots.ctypes.data_as(ctypes.c_void_p), ctypes.byref(cached)),
               "pkv_alloc_add_seq_cached")
        return slots[:n], cached.value

    def fork(self, parent: int, child: int):
        _check(lib().pkv_alloc_fork(self._h, parent, child), "pkv_alloc_fork")

    def append(self, seq_id: int):
        slot, src, dst = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib().pkv_alloc_append(self._h, seq_id, ctypes.byref(slot), ctypes.byref(src),
                                      ctypes.byref(dst)), "pkv_alloc_append")
        return slot.value, src.value, dst.value

    def append_batch(self, seq_ids):
        np = self._np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
        n = ids.shape[0]
        slots = np.empty(max(n, 1), dtype=np.int64)
        pairs = np.empty((max(n, 1), 2), dtype=np.int64)
        npairs = ctypes.c_int32()
        _check(lib().pkv_alloc_append_batch(self._h, ids.ctypes.data_as(ctypes.c_void_p), n,
                                            slots.ctypes.data_as(ctypes.c_void_p),
                                            pairs.ctypes.data_as(ctypes.c_void_p),
                                            ctypes.byref(npairs)), "pkv_alloc_append_batch")
        return slots[:n], pairs[: npairs.value]

    def free_seq(self, seq_id: int):
        _check(lib().pkv_alloc_free_seq(self._h, seq_id), "pkv_alloc_free_seq")

    def beam_step(self, beams, parents, next_id: int):
        """One beam-search step (pkv_alloc_beam_step): returns (new_ids, slots,
        copy pairs, next_id)."""
        np = self._np
        b = np.ascontiguousarray(beams, dtype=np.int32)
        p = np.ascontiguousarray(parents, dtype=np.int32)
        k, kn = b.shape[0], p.shape[0]
        ids = np.empty(max(kn, 1), dtype=np.int32)
        slots = np.empty(max(kn, 1), dtype=np.int64)
        pairs = np.empty((max(kn, 1), 2), dtype=np.int64)
        nid, npairs = ctypes.c_int32(next_id), ctypes.c_int32()
        _check(lib().pkv_alloc_beam_step(self._h, b.ctypes.data_as(ctypes.c_void_p), k,
                                         p.ctypes.data_as(ctypes.c_void_p), kn, ctypes.byref(nid),
                                         ids.ctypes.data_as(ctypes.c_void_p),
                                         slots.ctypes.data_as(ctypes.c_void_p),
                                         pairs.ctypes.data_as(ctypes.c_void_p), ctypes.byref(npairs)),
               "pkv_alloc_beam_step")
        return ids[:kn], slots[:kn], pairs[: npairs.value], nid.value

    def block_table(self, seq_ids, max_blocks: int):
        np = self._np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
        n = ids.shape[0]
        table = np.empty((max(n, 1), max(max_blocks, 1)), dtype=np.int32)
        lens = np.empty(max(n, 1), dtype=np.int32)
        _check(lib().pkv_alloc_block_table(self._h, ids.ctypes.data_as(ctypes.c_void_p), n,
                                           max_blocks, table.ctypes.data_as(ctypes.c_void_p),
                                           lens.ctypes.data_as(ctypes.c_void_p)),
               "pkv_alloc_block_table")
        return table[:n, :max_blocks], lens[:n]

    def refcount(self, block: int) -> int:
        c = ctypes.c_int32()
        _check(lib().pkv_alloc_refcount(self._h, block, ctypes.byref(c)), "pkv_alloc_refcount")
        return c.value

    def stats(self) -> dict:
        st = AllocStats()
        _check(lib().pkv_alloc_stats(self._h, ctypes.byref(st)), "pkv_alloc_stats")
        return {f: getattr(st, f) for f, _ in AllocStats._fields_}
