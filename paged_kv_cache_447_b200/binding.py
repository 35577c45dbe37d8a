"""ctypes binding of libpagedkv.so -- argument marshalling only.

Every function takes torch tensors that already live on the GPU (the caller owns them),
checks dtype/shape/contiguity on the host, and passes their device pointers and sizes to
the C entry point of the same name (see include/pkv.h).  Work is enqueued on the current
torch CUDA stream unless ``stream`` is given.  A non-zero status raises PagedKVError.
There is no fallback: if the shared library is missing, loading it raises."""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_LIB_NAME = "libpagedkv.so"
_HERE = os.path.dirname(os.path.abspath(__file__))

BF16 = 0
FP8_E4M3 = 1
NOALLOC_SCRATCH_BYTES = 8 << 20  # PKV_NOALLOC_SCRATCH_BYTES in include/pkv.h

_STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported shape or dtype",
           -3: "workspace missing or too small", -4: "CUDA runtime error",
           -5: "a bounded wait inside a kernel ran out",
           -6: "slot, block id or position out of range", -7: "pointer not 16-byte aligned",
           -8: "call needs more than the built-in decode scratch array",
           -9: "block pool cannot cover the allocation"}


class PagedKVError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {code} ({_STATUS.get(code, 'unknown')})")
        self.code = code


def library_path() -> str:
    return os.environ.get("PKV_LIBRARY", os.path.join(_HERE, _LIB_NAME))


_lib = None


def load_library():
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m paged_kv_cache_447_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    P, I, LL, F, D, SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float,
                          ctypes.c_double, ctypes.c_size_t)
    sig = {
        "pkv_version": ([], I),
        "pkv_strerror": ([I], ctypes.c_char_p),
        "pkv_rope_build_table": ([P, I, I, D], I),
        "pkv_cache_bytes": ([I, LL, I, I, I, I], SZ),
        "pkv_kv_store": ([P, P, P, P, P, I, I, I, I, LL, I, P, P, P, I, P, P, I, P], I),
        "pkv_rope_apply": ([P, P, P, I, P, P, I, I, I, I, I, P], I),
        "pkv_decode_workspace_bytes": ([I, I, I, I], SZ),
        "pkv_paged_decode_attention": ([P, P, P, P, P, I, P, I, I, I, I, I, LL, F, I, P, P, P,
                                        I, P, SZ, P], I),
        "pkv_paged_prefill_attention": ([P, P, P, P, P, P, I, P, I, I, I, I, I, I, LL, F, I,
                                         P, P, P, I, I, P], I),
        "pkv_paged_decode_attention_noalloc": ([P, P, P, P, P, I, P, I, I, I, I, I, LL, F, I,
                                                P, P, P, I, P], I),
        "pkv_decode_step_workspace_bytes": ([I, I, I, I], SZ),
        "pkv_paged_decode_step": ([P, P, P, P, P, P, P, I, P, I, I, I, I, I, LL, F, I, P, P, P, I,
                                   P, SZ, P], I),
        "pkv_slot_mapping": ([P, P, I, P, P, I, I, I, LL, P], I),
        "pkv_block_pool_bytes": ([LL], SZ),
        "pkv_block_pool_init": ([P, LL, P], I),
        "pkv_block_pool_alloc": ([P, LL, P, I, P, P, I, I, P], I),
        "pkv_block_pool_free": ([P, LL, P, I, P], I),
        "pkv_copy_blocks": ([P, P, P, I, I, I, I, LL, I, P], I),
        "pkv_get_error": ([P], I),
        "pkv_debug_wait_timeout": ([LL, P], I),
        "pkv_set_decode_step_mode": ([I], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _check(fn: str, code: int):
    if code != 0:
        raise PagedKVError(fn, code)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _cache_dtype(k_cache: torch.Tensor) -> int:
    if k_cache.dtype == torch.bfloat16:
        return BF16
    if k_cache.dtype in (torch.uint8, torch.float8_e4m3fn):
        return FP8_E4M3
    raise TypeError(f"cache dtype {k_cache.dtype} (bf16 or uint8/float8_e4m3fn codes)")


def _i32(t, name):
    if t is None:
        return None
    if t.dtype != torch.int32:
        raise TypeError(f"{name} must be int32")
    return t


def _bf16(t, name):
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bf16")
    return t


# ------------------------------------------------------------------------------ API

def version() -> int:
    return load_library().pkv_version()


def strerror(code: int) -> str:
    return load_library().pkv_strerror(code).decode()


def rope_build_table(max_pos: int, head_dim: int, base: float = 10000.0) -> torch.Tensor:
    """Host (CPU) fp32 table [max_pos, head_dim]: cos(p*theta_i) then sin(p*theta_i)."""
    out = torch.empty((max_pos, head_dim), dtype=torch.float32)
    _check("pkv_rope_build_table",
           load_library().pkv_rope_build_table(ctypes.c_void_p(out.data_ptr()), max_pos,
                                               head_dim, float(base)))
    return out


def cache_bytes(num_layers: int, num_blocks: int, block_size: int, n_kv_heads: int,
                head_dim: int, cache_dtype: int = BF16) -> int:
    return int(load_library().pkv_cache_bytes(num_layers, num_blocks, block_size, n_kv_heads,
                                              head_dim, cache_dtype))


def kv_store(k, v, k_cache, v_cache, slot_mapping, *, k_scale=None, v_scale=None,
             rope_cos_sin=None, cu_seqlens=None, context_lens=None, stream=None) -> None:
    """Scatter k/v [T, Hkv, D] into k_cache/v_cache [NB, bs, Hkv, D] at slot_mapping[T]."""
    T, H, D = k.shape
    NB, bs = k_cache.shape[0], k_cache.shape[1]
    _bf16(k, "k"); _bf16(v, "v"); _i32(slot_mapping, "slot_mapping")
    max_pos = rope_cos_sin.shape[0] if rope_cos_sin is not None else 0
    B = context_lens.shape[0] if context_lens is not None else 0
    _check("pkv_kv_store", load_library().pkv_kv_store(
        _p(k), _p(v), _p(k_cache), _p(v_cache), _p(slot_mapping), T, H, D, bs, NB,
        _cache_dtype(k_cache), _p(k_scale), _p(v_scale), _p(rope_cos_sin), max_pos,
        _p(_i32(cu_seqlens, "cu_seqlens")), _p(_i32(context_lens, "context_lens")), B,
        _stream(stream)))


def slot_mapping(block_tables, cu_seqlens, context_lens, num_tokens: int, num_blocks: int, *,
                 block_size: int = 16, out=None, stream=None) -> torch.Tensor:
    """int32 [num_tokens] cache slot of every new token (num_tokens = cu_seqlens[-1])."""
    _i32(block_tables, "block_tables"); _i32(cu_seqlens, "cu_seqlens")
    _i32(context_lens, "context_lens")
    if out is None:
        out = torch.empty(num_tokens, dtype=torch.int32, device=block_tables.device)
    _i32(out, "out")
    _check("pkv_slot_mapping", load_library().pkv_slot_mapping(
        _p(out), _p(block_tables), block_tables.shape[1], _p(cu_seqlens), _p(context_lens),
        context_lens.shape[0], num_tokens, block_size, num_blocks, _stream(stream)))
    return out


def block_pool(num_blocks: int, device=None, stream=None) -> torch.Tensor:
    """A device block pool of num_blocks blocks, all free (int32 tensor; element 0 is the
    number of free blocks)."""
    n = int(load_library().pkv_block_pool_bytes(num_blocks))
    if n == 0:
        raise PagedKVError("pkv_block_pool_bytes", -1)
    pool = torch.empty(n // 4, dtype=torch.int32, device=device or "cuda")
    _check("pkv_block_pool_init", load_library().pkv_block_pool_init(_p(pool), num_blocks,
                                                                      _stream(stream)))
    return pool


def _pool_blocks(pool: torch.Tensor) -> int:
    return (pool.numel() - 4) // 2


def block_pool_alloc(pool, block_tables, cu_seqlens, context_lens, *, block_size: int = 16,
                     stream=None) -> None:
    """Write into block_tables the blocks each sequence's new tokens need (in place)."""
    _i32(pool, "pool"); _i32(block_tables, "block_tables"); _i32(cu_seqlens, "cu_seqlens")
    _i32(context_lens, "context_lens")
    _check("pkv_block_pool_alloc", load_library().pkv_block_pool_alloc(
        _p(pool), _pool_blocks(pool), _p(block_tables), block_tables.shape[1], _p(cu_seqlens),
        _p(context_lens), context_lens.shape[0], block_size, _stream(stream)))


def block_pool_free(pool, block_ids, *, stream=None) -> None:
    """Return the int32 block ids to the pool, in order."""
    _i32(pool, "pool"); _i32(block_ids, "block_ids")
    n = block_ids.numel()
    _check("pkv_block_pool_free", load_library().pkv_block_pool_free(
        _p(pool), _pool_blocks(pool), _p(block_ids) if n else None, n, _stream(stream)))


STEP_AUTO, STEP_FUSED, STEP_SPLIT = 0, 1, 2


def set_decode_step_mode(mode: int) -> int:
    """How paged_decode_step runs (STEP_AUTO / STEP_FUSED / STEP_SPLIT); returns the previous
    mode."""
    r = load_library().pkv_set_decode_step_mode(int(mode))
    if r < 0:
        raise PagedKVError("pkv_set_decode_step_mode", r)
    return r


def copy_blocks(k_cache, v_cache, block_pairs, *, stream=None) -> None:
    """Copy physical blocks src -> dst of both caches for every (src, dst) row of the int32
    [n, 2] block_pairs (copy on write)."""
    _i32(block_pairs, "block_pairs")
    NB, bs, H, D = k_cache.shape
    n = block_pairs.shape[0] if block_pairs.numel() else 0
    _check("pkv_copy_blocks", load_library().pkv_copy_blocks(
        _p(k_cache), _p(v_cache), _p(block_pairs) if n else None, n, H, D, bs, NB,
        _cache_dtype(k_cache), _stream(stream)))


def rope_apply(q, k, rope_cos_sin, cu_seqlens, context_lens, *, stream=None) -> None:
    """Rotate q [T, Hq, D] and/or k [T, Hkv, D] in place (either may be None)."""
    ref = q if q is not None else k
    T, _, D = ref.shape
    Hq = q.shape[1] if q is not None else 0
    Hkv = k.shape[1] if k is not None else 0
    _check("pkv_rope_apply", load_library().pkv_rope_apply(
        _p(q), _p(k), _p(rope_cos_sin), rope_cos_sin.shape[0], _p(_i32(cu_seqlens, "cu")),
        _p(_i32(context_lens, "context_lens")), context_lens.shape[0], T, Hq, Hkv, D,
        _stream(stream)))


def decode_workspace_bytes(num_seqs: int, n_q_heads: int, n_kv_heads: int, head_dim: int) -> int:
    return int(load_library().pkv_decode_workspace_bytes(num_seqs, n_q_heads, n_kv_heads,
                                                         head_dim))


def paged_decode_attention(q, k_cache, v_cache, block_tables, context_lens, *, scale=None,
                           k_scale=None, v_scale=None, rope_cos_sin=None, workspace=None,
                           out=None, stream=None) -> torch.Tensor:
    """q [B, Hq, D] bf16 -> out [B, Hq, D] bf16 over the paged cache."""
    B, Hq, D = q.shape
    NB, bs, Hkv, _ = k_cache.shape
    _bf16(q, "q")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    need = decode_workspace_bytes(B, Hq, Hkv, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    max_pos = rope_cos_sin.shape[0] if rope_cos_sin is not None else 0
    _check("pkv_paged_decode_attention", load_library().pkv_paged_decode_attention(
        _p(out), _p(q), _p(k_cache), _p(v_cache), _p(_i32(block_tables, "block_tables")),
        block_tables.shape[1], _p(_i32(context_lens, "context_lens")), B, Hq, Hkv, D, bs, NB,
        float(scale), _cache_dtype(k_cache), _p(k_scale), _p(v_scale), _p(rope_cos_sin),
        max_pos, _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def decode_step_workspace_bytes(num_seqs: int, n_q_heads: int, n_kv_heads: int,
                                head_dim: int) -> int:
    return int(load_library().pkv_decode_step_workspace_bytes(num_seqs, n_q_heads, n_kv_heads,
                                                              head_dim))


def decode_step_workspace(num_seqs: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                          device=None) -> torch.Tensor:
    """A zero-filled workspace for paged_decode_step (reusable: every call leaves it zero)."""
    return torch.zeros(decode_step_workspace_bytes(num_seqs, n_q_heads, n_kv_heads, head_dim),
                       dtype=torch.uint8, device=device or "cuda")


def paged_decode_step(q, k, v, k_cache, v_cache, block_tables, context_lens, workspace, *,
                      scale=None, k_scale=None, v_scale=None, rope_cos_sin=None, out=None,
                      stream=None) -> torch.Tensor:
    """One decode step in one launch: store k/v [B, Hkv, D] (each sequence's new token, at
    position context_lens[b] - 1) into the paged cache and attend with q [B, Hq, D].
    ``workspace`` comes from decode_step_workspace (zero-filled)."""
    B, Hq, D = q.shape
    NB, bs, Hkv, _ = k_cache.shape
    _bf16(q, "q"); _bf16(k, "k"); _bf16(v, "v")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    max_pos = rope_cos_sin.shape[0] if rope_cos_sin is not None else 0
    _check("pkv_paged_decode_step", load_library().pkv_paged_decode_step(
        _p(out), _p(q), _p(k), _p(v), _p(k_cache), _p(v_cache),
        _p(_i32(block_tables, "block_tables")), block_tables.shape[1],
        _p(_i32(context_lens, "context_lens")), B, Hq, Hkv, D, bs, NB, float(scale),
        _cache_dtype(k_cache), _p(k_scale), _p(v_scale), _p(rope_cos_sin), max_pos,
        _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def paged_prefill_attention(q, k_cache, v_cache, cu_seqlens, block_tables, context_lens,
                            max_new_tokens: int, *, scale=None, k_scale=None, v_scale=None,
                            rope_cos_sin=None, out=None, stream=None) -> torch.Tensor:
    """q [T, Hq, D] bf16 (rows grouped by cu_seqlens) -> out [T, Hq, D] bf16."""
    T, Hq, D = q.shape
    NB, bs, Hkv, _ = k_cache.shape
    _bf16(q, "q")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    max_pos = rope_cos_sin.shape[0] if rope_cos_sin is not None else 0
    _check("pkv_paged_prefill_attention", load_library().pkv_paged_prefill_attention(
        _p(out), _p(q), _p(k_cache), _p(v_cache), _p(_i32(cu_seqlens, "cu_seqlens")),
        _p(_i32(block_tables, "block_tables")), block_tables.shape[1],
        _p(_i32(context_lens, "context_lens")), context_lens.shape[0], T, Hq, Hkv, D, bs, NB,
        float(scale), _cache_dtype(k_cache), _p(k_scale), _p(v_scale), _p(rope_cos_sin),
        max_pos, int(max_new_tokens), _stream(stream)))
    return out


def paged_decode_attention_noalloc(q, k_cache, v_cache, block_tables, context_lens, *,
                                   scale=None, k_scale=None, v_scale=None, rope_cos_sin=None,
                                   out=None, stream=None) -> torch.Tensor:
    """Decode attention without a workspace argument, for callers that cannot allocate
    device memory at decode time (for example an engine that gave nearly all HBM to its
    KV-block pool).  The library uses its own fixed 8 MiB device array instead, shared by
    every call on the device: calls must not overlap on the GPU.  Pass ``out`` to keep
    the call itself free of allocations."""
    B, Hq, D = q.shape
    NB, bs, Hkv, _ = k_cache.shape
    _bf16(q, "q")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    max_pos = rope_cos_sin.shape[0] if rope_cos_sin is not None else 0
    _check("pkv_paged_decode_attention_noalloc",
           load_library().pkv_paged_decode_attention_noalloc(
               _p(out), _p(q), _p(k_cache), _p(v_cache), _p(_i32(block_tables, "block_tables")),
               block_tables.shape[1], _p(_i32(context_lens, "context_lens")), B, Hq, Hkv, D, bs,
               NB, float(scale), _cache_dtype(k_cache), _p(k_scale), _p(v_scale),
               _p(rope_cos_sin), max_pos, _stream(stream)))
    return out


def get_error(stream=None) -> int:
    """Synchronise the stream; return and clear the device error word (0 = none)."""
    return int(load_library().pkv_get_error(_stream(stream)))


def debug_wait_timeout(timeout_ns: int, stream=None) -> None:
    _check("pkv_debug_wait_timeout",
           load_library().pkv_debug_wait_timeout(int(timeout_ns), _stream(stream)))


load_library()
