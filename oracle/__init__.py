"""CPU oracle for the paged KV-cache data plane -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference
leg may import this package.  The product (``paged_kv_cache_447_b200``) never imports,
links or runs it, and the two share no code: the arithmetic lives in ``pkv_oracle.c``
(plain fp64 C, compiled here with gcc) and this module only marshals numpy arrays.

What each function follows, and what pins it (tests/test_oracle_pins.py):

=====================  ====================================================  ===========================
function               passage                                               pinned by
=====================  ====================================================  ===========================
``bf16_from_f64``      bf16 = binary32 with 8 significant bits (format)      exact rational rounding of
                                                                             random doubles (fractions)
``e4m3_encode/decode`` FP8 KV cache, 1 byte/element ("LLM primer", §17.6);  all 256 codes vs
                       OCP E4M3-FN is the workload's format                  torch.float8_e4m3fn,
                                                                             monotonicity, saturation
``rope_table/rope``    RoPE rotates Q/K inside attention ("LLM primer",      pos 0 = identity, pairwise
                       §21.2; "Inside the Nano-vLLM engine", §3.2)           norm kept, relative-position
                                                                             property, quarter turn, direct
                                                                             fp64 rotation at position p
``positions``          new token r of sequence b at L_b - n_b + r (the new   hand-worked positions
                       tokens are the newest; "Inside the Nano-vLLM          (tests/golden); attention on q
                       engine", §2.1, §3.1)                                  rotated at hand-written
                                                                             positions; prefix + chunk
                                                                             shift invariance
``kv_store``           K/V cached per token, written by a cache kernel       round trip through the block
                       ("Nano-vLLM Part 2", §5.1-5.3); fixed 16-token        table equals the source rows;
                       blocks + block table ("Inside the Nano-vLLM engine",  slot -1 writes nothing
                       §2.2)
``attention``          softmax(QK^T/sqrt(d))V with causal mask and max       worked example "I eat fish"
                       subtraction ("Inside the Nano-vLLM engine", §3,       weights 0.60/0.40/0.00
                       §3.2; "LLM primer", §22 steps 6-8)                    ("LLM primer", §22 step 7-8);
                                                                             torch SDPA on the gathered
                                                                             K/V; L=1 returns V; rows sum
                                                                             to 1; x1e4 logits finite;
                                                                             block-permutation and shared-
                                                                             prefix invariance; E4M3 caches:
                                                                             SDPA on torch-dequantised
                                                                             codes x scales
``kv_cache_bytes``     2 x layers x kv_heads x head_dim x tokens x bytes     printed sizes ("LLM primer",
                       ("LLM primer", §17.3, §17.6)                          §17.3, §17.6, §23.2 exp. 2)
``slot_mapping``       block table lists a sequence's physical blocks, 16    hand-worked example
                       tokens each ("Inside the Nano-vLLM engine", §2.2)     (tests/golden); brute-force
                                                                             enumeration of each table's
                                                                             slots; -1 past the table
``copy_blocks``        shared prefix blocks, copy on write ("Inside the      numpy block slicing: dst
                       Nano-vLLM engine", §2.2; "LLM primer", §17.7)         equals old src, rest unchanged
``pool_*``             blocks come from a pool on demand and go back when   hand-worked sequence
                       a request finishes ("Inside the Nano-vLLM engine",    (tests/golden); invariants
                       §2.2; "LLM primer", §17.7)                            (no id held twice, ids
                                                                             conserved, tables cover every
                                                                             token); random alloc/free runs
                                                                             against a set-based model
=====================  ====================================================  ===========================
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile pkv_oracle.c with gcc (fp64, no FMA contraction, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        lib.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.orc_bf16_to_f64.restype = D
        lib.orc_f64_to_bf16.argtypes = [D]
        lib.orc_f64_to_bf16.restype = ctypes.c_uint16
        lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.orc_e4m3_decode.restype = D
        lib.orc_e4m3_encode.argtypes = [D]
        lib.orc_e4m3_encode.restype = ctypes.c_uint8
        lib.orc_rope_table.argtypes = [P, I, I, D]
        lib.orc_rope_table.restype = None
        lib.orc_positions.argtypes = [P, P, I, P]
        lib.orc_positions.restype = None
        lib.orc_rope.argtypes = [P, I, I, I, P, P]
        lib.orc_rope.restype = None
        lib.orc_kv_store.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P, P, P]
        lib.orc_kv_store.restype = None
        lib.orc_attention.argtypes = [P, P, P, P, P, I, P, I, I, I, I, I, I, D, I, P, P, P,
                                      P, I, P]
        lib.orc_attention.restype = None
        lib.orc_attention_weights.argtypes = [P, P, P, P, I, P, I, I, I, I, I, I, D, P, I, I, P]
        lib.orc_attention_weights.restype = None
        lib.orc_kv_cache_bytes.argtypes = [ctypes.c_int64] * 5
        lib.orc_slot_mapping.argtypes = [P, P, I, P, P, I, I, ctypes.c_int64]
        lib.orc_slot_mapping.restype = None
        lib.orc_copy_blocks.argtypes = [P, P, P, I, ctypes.c_int64, ctypes.c_int64]
        lib.orc_copy_blocks.restype = None
        lib.orc_kv_cache_bytes.restype = ctypes.c_int64
        lib.orc_pool_init.argtypes = [P, ctypes.c_int32]
        lib.orc_pool_init.restype = None
        lib.orc_pool_alloc.argtypes = [P, ctypes.c_int32, P, I, P, P, I, I]
        lib.orc_pool_alloc.restype = I
        lib.orc_pool_free.argtypes = [P, ctypes.c_int32, P, I]
        lib.orc_pool_free.restype = I
        lib.orc_num_threads.argtypes = []
        lib.orc_num_threads.restype = ctypes.c_int
        _lib = lib
        return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------- formats

def bf16_to_f64(bits):
    """bf16 bit patterns (uint16) -> float64, exact."""
    b = _c(bits, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_from_f64(x):
    """float64 -> bf16 bit patterns, round-to-nearest-even on the real value."""
    lib = _load()
    x = np.asarray(x, dtype=np.float64)
    flat = [lib.orc_f64_to_bf16(float(v)) for v in x.ravel()]
    return np.array(flat, dtype=np.uint16).reshape(x.shape)


def e4m3_decode(codes):
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.orc_e4m3_decode(int(v)) for v in c.ravel()],
                    dtype=np.float64).reshape(c.shape)


def e4m3_encode(x):
    lib = _load()
    x = np.asarray(x, dtype=np.float64)
    return np.array([lib.orc_e4m3_encode(float(v)) for v in x.ravel()],
                    dtype=np.uint8).reshape(x.shape)


# --------------------------------------------------------------------------- RoPE

def rope_table(max_pos: int, head_dim: int, base: float = 10000.0) -> np.ndarray:
    """[max_pos, head_dim] float32: row p = cos(p*theta_i) for i < D/2, then sin."""
    lib = _load()
    out = np.empty((max_pos, head_dim), dtype=np.float32)
    lib.orc_rope_table(_ptr(out), max_pos, head_dim, float(base))
    return out


def positions(cu_seqlens, context_lens) -> np.ndarray:
    lib = _load()
    cu = _c(cu_seqlens, np.int32)
    cl = _c(context_lens, np.int32)
    out = np.zeros(int(cu[-1]), dtype=np.int64)
    lib.orc_positions(_ptr(cu), _ptr(cl), len(cl), _ptr(out))
    return out


def rope(x_bits, pos, table) -> np.ndarray:
    """Rotate x [T, H, D] (bf16 bits) at pos[T]; returns new bf16 bits."""
    lib = _load()
    x = _c(x_bits, np.uint16).copy()
    T, H, D = x.shape
    p = _c(pos, np.int64)
    tab = _c(table, np.float32)
    assert p.shape == (T,) and (T == 0 or int(p.max()) < tab.shape[0])
    lib.orc_rope(_ptr(x), T, H, D, _ptr(p), _ptr(tab))
    return x


# --------------------------------------------------------------------------- store

def kv_store(k_bits, v_bits, k_cache, v_cache, slot_mapping, block_size: int, fp8: bool = False,
             k_scale=None, v_scale=None, table=None, pos=None) -> None:
    """Scatter k/v [T, Hkv, D] into k_cache/v_cache [NB, bs, Hkv, D] (modified in place).

    Caches are uint16 (bf16 bits) or uint8 (E4M3 codes) numpy arrays."""
    lib = _load()
    k = _c(k_bits, np.uint16)
    v = _c(v_bits, np.uint16)
    T, H, D = k.shape
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    assert k_cache.dtype == (np.uint8 if fp8 else np.uint16)
    sm = _c(slot_mapping, np.int32)
    ks = _c(k_scale, np.float32) if fp8 else None
    vs = _c(v_scale, np.float32) if fp8 else None
    tab = _c(table, np.float32) if table is not None else None
    p = _c(pos, np.int64) if table is not None else None
    lib.orc_kv_store(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(sm), T, H, D,
                     block_size, int(fp8), _ptr(ks), _ptr(vs), _ptr(tab), _ptr(p))


# --------------------------------------------------------------------------- attention

def attention(q_bits, k_cache, v_cache, cu_seqlens, block_tables, context_lens, scale: float,
              block_size: int, n_kv_heads: int, fp8: bool = False, k_scale=None, v_scale=None,
              table=None, rows=None) -> np.ndarray:
    """Paged causal attention, fp64.  q [T, Hq, D] bf16 bits.

    rows=None -> [T, Hq, D]; rows = int array [R, 2] of (token, q head) -> [R, D]."""
    lib = _load()
    q = _c(q_bits, np.uint16)
    T, Hq, D = q.shape
    cu = _c(cu_seqlens, np.int32)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    ks = _c(k_scale, np.float32) if fp8 else None
    vs = _c(v_scale, np.float32) if fp8 else None
    tab = _c(table, np.float32) if table is not None else None
    kc = np.ascontiguousarray(k_cache)
    vc = np.ascontiguousarray(v_cache)
    if rows is None:
        r = None
        out = np.zeros((T, Hq, D), dtype=np.float64)
        nr = 0
    else:
        r = _c(rows, np.int32).reshape(-1, 2)
        nr = r.shape[0]
        out = np.zeros((nr, D), dtype=np.float64)
    lib.orc_attention(_ptr(q), _ptr(kc), _ptr(vc), _ptr(cu), _ptr(bt), bt.shape[1], _ptr(cl),
                      len(cl), T, Hq, n_kv_heads, D, block_size, float(scale), int(fp8),
                      _ptr(ks), _ptr(vs), _ptr(tab), _ptr(r), nr, _ptr(out))
    return out


def attention_weights(q_bits, k_cache, cu_seqlens, block_tables, context_lens, scale: float,
                      block_size: int, n_kv_heads: int, rows, lmax: int) -> np.ndarray:
    """Softmax rows p_j (bf16 cache only) for the requested (token, head) rows."""
    lib = _load()
    q = _c(q_bits, np.uint16)
    T, Hq, D = q.shape
    cu = _c(cu_seqlens, np.int32)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    r = _c(rows, np.int32).reshape(-1, 2)
    out = np.zeros((r.shape[0], lmax), dtype=np.float64)
    kc = np.ascontiguousarray(k_cache)
    lib.orc_attention_weights(_ptr(q), _ptr(kc), _ptr(cu), _ptr(bt), bt.shape[1], _ptr(cl),
                              len(cl), T, Hq, n_kv_heads, D, block_size, float(scale), _ptr(r),
                              r.shape[0], lmax, _ptr(out))
    return out


# --------------------------------------------------------------------------- sizing

def kv_cache_bytes(num_layers: int, n_kv_heads: int, head_dim: int, cached_tokens: int,
                   bytes_per_element: int) -> int:
    return int(_load().orc_kv_cache_bytes(num_layers, n_kv_heads, head_dim, cached_tokens,
                                          bytes_per_element))


def slot_mapping(block_tables, cu_seqlens, context_lens, block_size: int,
                 num_blocks: int) -> np.ndarray:
    """int32 slot of every new token of the batch (-1 past the table / bad block id)."""
    bt = _c(block_tables, np.int32)
    cu = _c(cu_seqlens, np.int32)
    cl = _c(context_lens, np.int32)
    out = np.full(int(cu[-1]), -1, dtype=np.int32)
    _load().orc_slot_mapping(_ptr(out), _ptr(bt), bt.shape[1], _ptr(cu), _ptr(cl), len(cl),
                             block_size, num_blocks)
    return out


def copy_blocks(k_cache, v_cache, pairs) -> None:
    """In place: block dst of both caches (numpy, [NB, ...]) becomes a copy of block src."""
    pr = _c(np.asarray(pairs).reshape(-1, 2), np.int32)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    nb = k_cache.shape[0]
    block_bytes = k_cache.nbytes // nb
    _load().orc_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(pr), pr.shape[0], block_bytes, nb)


def pool_init(num_blocks: int) -> np.ndarray:
    """Block pool state (int32): [free count, stack of free ids bottom first, free flags]."""
    pool = np.zeros(1 + 2 * num_blocks, dtype=np.int32)
    _load().orc_pool_init(_ptr(pool), num_blocks)
    return pool


def pool_alloc(pool, block_tables, cu_seqlens, context_lens, block_size: int = 16) -> int:
    """Give every sequence the blocks its new tokens need (written into block_tables in
    place); 0, or -1 (nothing taken) when the pool or a table is too small."""
    nb = (pool.shape[0] - 1) // 2
    assert block_tables.flags.c_contiguous and block_tables.dtype == np.int32
    cu = _c(cu_seqlens, np.int32)
    cl = _c(context_lens, np.int32)
    return int(_load().orc_pool_alloc(_ptr(pool), nb, _ptr(block_tables), block_tables.shape[1],
                                      _ptr(cu), _ptr(cl), len(cl), block_size))


def pool_free(pool, ids) -> int:
    """Return ids to the pool; the number of ids rejected (outside the pool or already free)."""
    nb = (pool.shape[0] - 1) // 2
    ids = _c(np.asarray(ids).reshape(-1), np.int32)
    return int(_load().orc_pool_free(_ptr(pool), nb, _ptr(ids), len(ids)))


def num_threads() -> int:
    """OpenMP threads the oracle's parallel loops use."""
    return int(_load().orc_num_threads())
