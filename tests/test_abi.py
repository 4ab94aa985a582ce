"""The C-ABI library loads on a machine without a GPU, exports every function
include/pkv.h declares, and rejects bad arguments on the host before any CUDA
call.  No test here launches or allocates anything on a device."""
import ctypes
import os
import re

import pytest
import torch

from paged_kv_cache_419_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pkv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"^[A-Za-z_][\w \*]*?\b(pkv_\w+)\s*\(", text, flags=re.M))


def test_header_declares_the_binding_export_list():
    assert declared_functions() == set(B.EXPORTS)


def test_library_exports_every_declared_function():
    lib = B.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings():
    for code in (B.PKV_OK, B.PKV_EINVAL, B.PKV_EUNSUPPORTED, B.PKV_ECUDA, B.PKV_ENOMEM, B.PKV_ERANGE):
        assert B.status_string(code).startswith("PKV_")


def test_cuda_error_names():
    assert B.cuda_error_name(0) == "cudaSuccess"
    assert B.cuda_error_name(2) == "cudaErrorMemoryAllocation"


@pytest.mark.skipif(torch.cuda.is_available(), reason="needs a machine without a GPU")
def test_cuda_failure_is_reported_with_its_cuda_error():
    """Without a GPU the first CUDA call of pkv_device_error fails; the status is
    PKV_ECUDA and the binding's error names the CUDA error behind it."""
    flags = ctypes.c_uint(0)
    status = B.lib().pkv_device_error(ctypes.byref(flags), 1, None)  # default stream
    with pytest.raises(B.PkvError) as e:
        B._check(status, "pkv_device_error")
    assert e.value.status == B.PKV_ECUDA
    assert e.value.cuda_error != 0 and B.last_cuda_error() == e.value.cuda_error
    assert B.cuda_error_name(e.value.cuda_error) in str(e.value)
    assert B.cuda_error_name(e.value.cuda_error).startswith("cudaError")


def _layout_bytes(S, Hq, D, ctx, part=512):
    # partition_size 0 (the default policy) bounds the workspace as 512-token partitions
    r = lambda x: (x + 255) // 256 * 256
    P = max(1, -(-ctx // part))
    rec = 32
    return 256 + r(4 * S) + r(4 * S * Hq) + r(S * P * rec) + (r(S * Hq * P * (D + 2) * 4) if P > 1 else 0)


def test_workspace_bytes_formula():
    # one partition per context: counters and the work list only
    assert B.decode_workspace_bytes(256, 32, 128, 512) == _layout_bytes(256, 32, 128, 512)
    assert B.decode_workspace_bytes(256, 32, 128, 512) < 1 << 20
    assert B.decode_workspace_bytes(256, 32, 128, 1024, 1024) < 1 << 20
    # 4096 tokens under the default policy: P = 8 cells of (D + 2) floats
    assert B.decode_workspace_bytes(256, 32, 128, 4096) == _layout_bytes(256, 32, 128, 4096)
    assert B.decode_workspace_bytes(256, 32, 128, 4096) > 256 * 32 * 8 * 130 * 4
    # an explicit 512: P = 8
    assert B.decode_workspace_bytes(256, 32, 128, 4096, 512) == _layout_bytes(256, 32, 128, 4096, 512)
    assert B.decode_workspace_bytes(4, 32, 128, 32768, 1024) == _layout_bytes(4, 32, 128, 32768, 1024)
    # invalid partition sizes give 0
    assert B.decode_workspace_bytes(4, 32, 128, 32768, 48) == 0
    assert B.decode_workspace_bytes(4, 32, 128, 32768, 4096) == 0


FAKE = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: every call below fails first


def _paged(**kw):
    args = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, tables=FAKE, lens=FAKE, S=4, MB=8, N=64,
                scale=0.1, Hq=8, Hkv=8, D=64, Bs=16, dt=B.PKV_F16, part=0, ws=None, wsb=0)
    args.update(kw)
    a = args
    return B.lib().pkv_paged_attention_decode(a["out"], a["q"], a["k"], a["v"], a["tables"],
                                              a["lens"], a["S"], a["MB"], a["N"], a["scale"],
                                              a["Hq"], a["Hkv"], a["D"], a["Bs"], a["dt"],
                                              a["part"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(D=96), B.PKV_EUNSUPPORTED),
    (dict(D=256), B.PKV_EUNSUPPORTED),
    (dict(Bs=12), B.PKV_EUNSUPPORTED),
    (dict(Bs=64), B.PKV_EUNSUPPORTED),
    (dict(Hq=12, Hkv=8), B.PKV_EUNSUPPORTED),     # Hq % Hkv != 0
    (dict(Hq=48, Hkv=3), B.PKV_EUNSUPPORTED),     # group of 16
    (dict(dt=7), B.PKV_EUNSUPPORTED),
    (dict(S=-1), B.PKV_EINVAL),
    (dict(MB=0), B.PKV_EINVAL),
    (dict(N=0), B.PKV_EINVAL),
    (dict(Hkv=0), B.PKV_EINVAL),
    (dict(q=None), B.PKV_EINVAL),
    (dict(out=None), B.PKV_EINVAL),
    (dict(tables=None), B.PKV_EINVAL),
    (dict(k=ctypes.c_void_p((1 << 20) + 8)), B.PKV_EINVAL),   # misaligned
    (dict(part=48), B.PKV_EINVAL),                # not a multiple of 64
    (dict(part=96), B.PKV_EINVAL),
    (dict(part=4096), B.PKV_EINVAL),              # above 2048
    (dict(MB=64), B.PKV_EINVAL),                  # no workspace given
])
def test_paged_decode_rejects_bad_arguments_before_launch(kw, status):
    assert _paged(**kw) == status


def test_zero_sequences_is_a_no_op():
    assert _paged(S=0, q=None, out=None) == B.PKV_OK


def test_cache_ops_reject_bad_arguments_before_launch():
    L = B.lib()
    # head_dim 4 (8 bytes per row) cannot be moved in 16-byte vectors
    assert L.pkv_reshape_and_cache(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 4, 16, 8, 0, None) == B.PKV_EUNSUPPORTED
    # head_dim 96: 12 vectors per row, not a power of two
    assert L.pkv_reshape_and_cache(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 96, 16, 8, 0, None) == B.PKV_EUNSUPPORTED
    assert L.pkv_reshape_and_cache(None, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 8, 0, None) == B.PKV_EINVAL
    assert L.pkv_reshape_and_cache(FAKE, FAKE, FAKE, FAKE, FAKE, -1, 2, 64, 16, 8, 0, None) == B.PKV_EINVAL
    assert L.pkv_reshape_and_cache(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, 64, 16, 8, 0, None) == B.PKV_OK
    assert L.pkv_copy_blocks(FAKE, FAKE, FAKE, 3, 24, 8, None) == B.PKV_EINVAL      # not 16-byte multiple
    assert L.pkv_copy_blocks(FAKE, FAKE, None, 3, 4096, 8, None) == B.PKV_EINVAL
    assert L.pkv_copy_blocks(FAKE, FAKE, FAKE, 70000, 4096, 8, None) == B.PKV_EUNSUPPORTED
    assert L.pkv_copy_blocks(FAKE, FAKE, FAKE, 0, 4096, 8, None) == B.PKV_OK


def test_contiguous_decode_rejects_bad_arguments_before_launch():
    L = B.lib()
    f = L.pkv_contiguous_attention_decode
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 512, 0.1, 8, 8, 80, 0, 0, None, 0, None) == B.PKV_EUNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, None, 4, 512, 0.1, 8, 8, 64, 0, 0, None, 0, None) == B.PKV_EINVAL
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2048, 0.1, 8, 8, 64, 0, 0, None, 0, None) == B.PKV_EINVAL
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 256, 0.1, 8, 8, 64, 0, 0, None, 0, None) == B.PKV_EINVAL
