"""CPU oracle for paged decode attention (fp64), the cache write and the block copy.

TEST INFRASTRUCTURE.  Only the tests, the package smoke check and the CPU
baseline leg of the benchmark may import this package; the CUDA library and its
Python binding never do, and the two share no code.

``oracle.c`` holds the arithmetic (plain C, fp64, written from the definitions
cited in its header); this module compiles it with gcc on first use and wraps it
with numpy.  ``allocator_model`` is a pure-Python reference model of the block
allocator.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

OR_OK, OR_EINVAL, OR_ERANGE, OR_ENOMEM = 0, -1, -2, -4


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, strict IEEE: no fast-math,
    no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                               "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        # PKV_ORACLE_LIB names another build of oracle.c; the mutation tests use it
        # to run the pins against a copy with a planted mistake.
        path = os.environ.get("PKV_ORACLE_LIB") or build()
        L = ctypes.CDLL(path)
        P, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        L.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_f16_to_double.restype = dbl
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_double.restype = dbl
        L.oracle_double_to_f16.argtypes = [dbl]
        L.oracle_double_to_f16.restype = ctypes.c_uint16
        L.oracle_double_to_bf16.argtypes = [dbl]
        L.oracle_double_to_bf16.restype = ctypes.c_uint16
        L.oracle_round_array.argtypes = [P, P, i64, i32]
        L.oracle_round_array.restype = ctypes.c_int
        L.oracle_paged_decode.argtypes = [P, P, P, P, P, i32, P, i32, i32, dbl, i32, i32, i32, i32,
                                          i32, i32]
        L.oracle_attention_weights.argtypes = [P, P, P, P, P, i32, P, i32, i32, dbl, i32, i32, i32,
                                               i32, i32, i32]
        L.oracle_dense_decode.argtypes = [P, P, P, P, P, i32, i32, i32, dbl, i32, i32, i32, i32]
        L.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32]
        L.oracle_copy_blocks.argtypes = [P, P, P, i32, i64, i32]
        L.oracle_paged_prefill.argtypes = [P, P, P, P, P, i32, i32, i32, dbl, i32, i32, i32, i32, i32,
                                           i32]
        for f in ("oracle_paged_decode", "oracle_attention_weights", "oracle_dense_decode",
                  "oracle_reshape_and_cache", "oracle_copy_blocks", "oracle_paged_prefill"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


class OracleError(RuntimeError):
    def __init__(self, rc, what):
        super().__init__(f"{what}: oracle status {rc}")
        self.rc = rc


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def to_double(bits: np.ndarray, dtype: int) -> np.ndarray:
    """fp16 (dtype 0) / bf16 (dtype 1) bit patterns -> float64, element by element."""
    f = lib().oracle_f16_to_double if dtype == 0 else lib().oracle_bf16_to_double
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([f(int(b)) for b in flat], dtype=np.float64).reshape(np.shape(bits))


def round_to_dtype(x, dtype: int) -> np.ndarray:
    """float64 values -> fp16 (dtype 0) / bf16 (dtype 1) bit patterns, each rounded
    to nearest with ties to even, straight from fp64 (one rounding)."""
    src = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(src.shape, dtype=np.uint16)
    rc = lib().oracle_round_array(_ptr(out), _ptr(src), src.size, int(dtype))
    if rc != OR_OK:
        raise OracleError(rc, "round_to_dtype")
    return out


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, block_size,
                 dtype, seqs=None) -> np.ndarray:
    """softmax(scale q K^T) V per (sequence, query head), K/V gathered through the
    block table in logical order.  q: uint16 [S, Hq, D]; caches uint16
    [N, Hkv, B, D]; returns float64 [S, Hq, D].  ``seqs``: optional (begin, end)
    range; rows outside it are zero."""
    q = _c(q, np.uint16)
    kc, vc = _c(k_cache, np.uint16), _c(v_cache, np.uint16)
    tables = _c(block_tables, np.int32)
    lens = _c(context_lens, np.int32)
    S, Hq, D = q.shape
    N = kc.shape[0]
    out = np.zeros((S, Hq, D), dtype=np.float64)
    b, e = (0, S) if seqs is None else seqs
    rc = lib().oracle_paged_decode(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(tables),
                                   tables.shape[1], _ptr(lens), b, e, float(scale), Hq,
                                   num_kv_heads, D, block_size, N, dtype)
    if rc != OR_OK:
        raise OracleError(rc, "paged_decode")
    return out


def paged_prefill(q, k_cache, v_cache, table_row, p0, scale, num_kv_heads, block_size, dtype) -> np.ndarray:
    """Causal attention of T new tokens of one sequence at positions p0 .. p0 + T - 1
    (their K/V already in the cache): query i sees positions 0 .. p0 + i through the
    block-table row.  q: uint16 [T, Hq, D]; returns float64 [T, Hq, D]."""
    q = _c(q, np.uint16)
    kc, vc = _c(k_cache, np.uint16), _c(v_cache, np.uint16)
    row = _c(table_row, np.int32)
    T, Hq, D = q.shape
    out = np.zeros((T, Hq, D), dtype=np.float64)
    rc = lib().oracle_paged_prefill(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(row), row.shape[0],
                                    int(p0), T, float(scale), Hq, num_kv_heads, D, block_size,
                                    kc.shape[0], dtype)
    if rc != OR_OK:
        raise OracleError(rc, "paged_prefill")
    return out


def attention_weights(q, k_cache, v_cache, block_tables, context_lens, s, h, scale, num_kv_heads,
                      block_size, dtype) -> np.ndarray:
    q = _c(q, np.uint16)
    kc, vc = _c(k_cache, np.uint16), _c(v_cache, np.uint16)
    tables = _c(block_tables, np.int32)
    lens = _c(context_lens, np.int32)
    S, Hq, D = q.shape
    w = np.zeros(max(int(lens[s]), 1), dtype=np.float64)
    rc = lib().oracle_attention_weights(_ptr(w), _ptr(q), _ptr(kc), _ptr(vc), _ptr(tables),
                                        tables.shape[1], _ptr(lens), s, h, float(scale), Hq,
                                        num_kv_heads, D, block_size, kc.shape[0], dtype)
    if rc != OR_OK:
        raise OracleError(rc, "attention_weights")
    return w[: int(lens[s])]


def dense_decode(q, k, v, context_lens, scale, dtype, seqs=None) -> np.ndarray:
    """Decode over a contiguous cache k, v: uint16 [S, Hkv, max_ctx, D]."""
    q = _c(q, np.uint16)
    k, v = _c(k, np.uint16), _c(v, np.uint16)
    lens = _c(context_lens, np.int32)
    S, Hq, D = q.shape
    Hkv, max_ctx = k.shape[1], k.shape[2]
    out = np.zeros((S, Hq, D), dtype=np.float64)
    b, e = (0, S) if seqs is None else seqs
    rc = lib().oracle_dense_decode(_ptr(out), _ptr(q), _ptr(k), _ptr(v), _ptr(lens), b, e,
                                   max_ctx, float(scale), Hq, Hkv, D, dtype)
    if rc != OR_OK:
        raise OracleError(rc, "dense_decode")
    return out


def reshape_and_cache(k_cache, v_cache, key, value, slot_mapping, block_size):
    """In-place scatter of key/value rows [T, Hkv, D] into the caches [N, Hkv, B, D]."""
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    key, value = _c(key, k_cache.dtype), _c(value, k_cache.dtype)
    slots = _c(slot_mapping, np.int64)
    N, Hkv, B, D = k_cache.shape
    assert B == block_size
    rc = lib().oracle_reshape_and_cache(_ptr(k_cache), _ptr(v_cache), _ptr(key), _ptr(value),
                                        _ptr(slots), slots.shape[0], Hkv, D, B,
                                        k_cache.dtype.itemsize, N)
    if rc != OR_OK:
        raise OracleError(rc, "reshape_and_cache")


def copy_blocks(k_cache, v_cache, pairs):
    """In-place copy of whole frames, pairs int64 [n, 2] of (src, dst), in order."""
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    pairs = _c(pairs, np.int64).reshape(-1, 2)
    N = k_cache.shape[0]
    block_bytes = k_cache[0].nbytes
    rc = lib().oracle_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(pairs), pairs.shape[0],
                                  block_bytes, N)
    if rc != OR_OK:
        raise OracleError(rc, "copy_blocks")


def kv_bytes_per_token(hidden: int, layers: int, elt_bytes: int) -> int:
    """K and V of one token across all layers: 2 x hidden x layers x bytes per element
    (vLLM and PagedAttention slides, slide 5)."""
    return 2 * hidden * layers * elt_bytes
