"""B200-native paged KV-cache attention, decode and prefill (vLLM / PagedAttention method).

The compute lives in ``libpkv.so`` (CUDA for sm_100a, C ABI in include/pkv.h);
``binding`` is its ctypes binding.  Names are re-exported lazily so that
importing the package does not load the library until a call needs it.
"""

_EXPORTS = (
    "paged_attention_decode", "contiguous_attention_decode", "paged_prefill", "reshape_and_cache",
    "copy_blocks",
    "decode_workspace_bytes", "device_error", "BlockAllocator", "PkvError", "block_hash",
)

__all__ = list(_EXPORTS)


def __getattr__(name):
    if name in _EXPORTS:
        from . import binding

        return getattr(binding, name)
    raise AttributeError(name)
