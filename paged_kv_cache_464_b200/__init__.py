"""paged_kv_cache_464_b200: paged-KV decode attention for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libpa_b200.so`` (hand-written CUDA
kernels); ``capi`` is its thin ctypes binding.  Importing this package does not
load the library; the first call through ``capi`` does, and it raises if the
library is missing -- there is no CPU fallback.
"""
__all__ = ["capi", "inputs"]


def __getattr__(name):
    if name in ("reshape_and_cache", "decode", "copy_blocks", "decode_workspace_bytes",
                "get_device_error", "PaError"):
        from . import capi
        return getattr(capi, name)
    raise AttributeError(name)
