"""paged_kv_cache_447_b200 -- a paged KV-cache data plane for NVIDIA B200 (sm_100a).

The compute lives in ``libpagedkv.so`` (hand-written CUDA behind the C ABI declared in
``include/pkv.h``).  This package is its thin Python binding: ``kv_store``, ``rope_apply``,
``paged_decode_attention``, ``paged_decode_step``, ``paged_prefill_attention``,
``slot_mapping``, ``copy_blocks``
and helpers take torch tensors,
pass their device pointers and sizes across the C ABI and raise on a non-zero status.
PyTorch only provides device memory and streams.

The binding is loaded on first use of any of those names; if the shared library has not
been built (``python -c "import __graft_entry__ as g; g.build()"``) that first use raises.
``workloads`` (seeded input generators) does not need the library.
"""
from __future__ import annotations

import importlib

_BINDING_NAMES = {
    "kv_store", "rope_apply", "paged_decode_attention", "paged_prefill_attention",
    "paged_decode_attention_noalloc", "NOALLOC_SCRATCH_BYTES", "slot_mapping", "copy_blocks",
    "paged_decode_step", "decode_step_workspace_bytes", "decode_step_workspace",
    "block_pool", "block_pool_alloc", "block_pool_free",
    "set_decode_step_mode", "STEP_AUTO", "STEP_FUSED", "STEP_SPLIT",
    "rope_build_table", "decode_workspace_bytes", "cache_bytes", "get_error", "strerror",
    "debug_wait_timeout", "version", "library_path", "load_library", "PagedKVError",
    "BF16", "FP8_E4M3",
}

__all__ = sorted(_BINDING_NAMES) + ["workloads"]


def __getattr__(name):
    if name in _BINDING_NAMES:
        binding = importlib.import_module(".binding", __name__)
        return getattr(binding, name)
    if name == "workloads":
        return importlib.import_module(".workloads", __name__)
    raise AttributeError(name)
