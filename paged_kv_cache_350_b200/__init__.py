"""paged_kv_cache_350_b200 — paged KV-cache decode attention for B200 (sm_100a).

The product is the C-ABI library ``libpagedattn.so`` (``include/pa.h``): batched
single-token decode attention that reads K/V from a block pool through
per-sequence block tables, the two kernels that keep the pool consistent
(``reshape_and_cache``, ``copy_blocks``; ``pa_decode_append`` fuses the first into
the decode), and a host block allocator with
reference counts.  This package is its Python face: ``binding`` marshals torch
tensors into the C calls (same names), ``cache.PagedKVCache`` chains one decode
step end to end, and ``build`` compiles the library in-tree.

The library is loaded on first use of any of these names; if it is missing that
raises ImportError (there is no fallback).  ``paged_kv_cache_350_b200.build``
imports without it.
"""

_BINDING_NAMES = {
    "PA_BF16", "PA_F32", "PA_PATH_AUTO", "PA_PATH_GENERIC", "PA_PATH_TENSOR", "PAError",
    "Allocator", "pa_copy_blocks", "pa_decode", "pa_decode_workspace_size", "pa_decode_plan", "pa_decode_no_alloc",
    "pa_decode_append",
    "pa_decode_shared_prefix", "pa_decode_shared_prefix_workspace_size",
    "pa_reshape_and_cache", "pa_status_from_device_flag", "lib",
}

__all__ = sorted(_BINDING_NAMES | {"PagedKVCache"})


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    if name == "PagedKVCache":
        from .cache import PagedKVCache
        return PagedKVCache
    if name == "__version__":
        from . import binding
        return binding.lib.pa_version().decode()
    raise AttributeError(name)
