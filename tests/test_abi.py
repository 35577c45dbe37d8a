"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol
the header declares, rejects bad arguments before touching the device, and its host
helpers (RoPE table, cache sizing) agree with the oracle and the pages."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_447_b200 as pkv
from paged_kv_cache_447_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "pkv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(binding.library_path())
    syms = _declared_symbols()
    assert len(syms) >= 10
    for s in syms:
        assert hasattr(lib, s), f"missing export {s}"


def test_version_and_strerror():
    assert pkv.version() >> 16 == 1
    assert pkv.strerror(-2) == "unsupported shape or dtype"


def test_rope_table_bitwise_equals_oracle_table():
    for D, P in ((64, 200), (128, 4096)):
        lib_tab = pkv.rope_build_table(P, D, 10000.0).numpy()
        orc_tab = oracle.rope_table(P, D, 10000.0)
        assert np.array_equal(lib_tab.view(np.uint32), orc_tab.view(np.uint32))


def test_cache_bytes_formula_and_pages_examples():
    # library allocation size == the pages' formula with cached_tokens = blocks x 16
    for layers, nb, h, d, dt, eb in ((32, 256, 8, 128, pkv.BF16, 2), (1, 4224, 8, 128, pkv.BF16, 2),
                                     (32, 1, 32, 128, pkv.FP8_E4M3, 1), (3, 7, 2, 64, pkv.BF16, 2)):
        assert pkv.cache_bytes(layers, nb, 16, h, d, dt) == oracle.kv_cache_bytes(layers, h, d, nb * 16, eb)
    # 4096 tokens of a 32-layer, 8-kv-head, head_dim-128 model = 536,870,912 B (0.5 GiB)
    assert pkv.cache_bytes(32, 4096 // 16, 16, 8, 128, pkv.BF16) == 536870912
    # torch allocation of the cache tensors for the same shape
    k = torch.empty((4096 // 16, 16, 8, 128), dtype=torch.bfloat16)
    assert 32 * 2 * k.numel() * k.element_size() == 536870912
    assert pkv.cache_bytes(0, 1, 16, 1, 64, 5) == 0


def test_host_argument_checks_need_no_device():
    lib = binding.load_library()
    n = None
    # head_dim 96 is not compiled
    assert lib.pkv_kv_store(n, n, n, n, n, 4, 2, 96, 16, 32, 0, n, n, n, 0, n, n, 0, n) == -2
    # block size 8 is not compiled
    assert lib.pkv_kv_store(n, n, n, n, n, 4, 2, 64, 8, 32, 0, n, n, n, 0, n, n, 0, n) == -2
    # null pointers
    assert lib.pkv_kv_store(n, n, n, n, n, 4, 2, 64, 16, 32, 0, n, n, n, 0, n, n, 0, n) == -1
    # Hq not a multiple of Hkv
    assert lib.pkv_paged_decode_attention(n, n, n, n, n, 4, n, 2, 6, 4, 64, 16, 32, 1.0, 0, n, n,
                                          n, 0, n, 0, n) == -1
    # group 3 not compiled
    assert lib.pkv_paged_decode_attention(n, n, n, n, n, 4, n, 2, 6, 2, 64, 16, 32, 1.0, 0, n, n,
                                          n, 0, n, 0, n) == -2
    # fp8 without scales (misaligned check comes first with fake pointers, so use aligned ones)
    buf = ctypes.create_string_buffer(64)
    addr = (ctypes.addressof(buf) + 15) & ~15
    p = ctypes.c_void_p(addr)
    assert lib.pkv_kv_store(p, p, p, p, p, 4, 2, 64, 16, 32, 1, n, n, n, 0, n, n, 0, n) == -1
    assert lib.pkv_kv_store(ctypes.c_void_p(addr + 2), p, p, p, p, 4, 2, 64, 16, 32, 0, n, n, n,
                            0, n, n, 0, n) == -7
    # zero tokens is a no-op
    assert lib.pkv_kv_store(n, n, n, n, n, 0, 2, 64, 16, 32, 0, n, n, n, 0, n, n, 0, n) == 0
    assert lib.pkv_rope_build_table(n, 4, 64, 1e4) == -1
    assert lib.pkv_rope_build_table(p, 4, 63, 1e4) == -1


def test_block_helpers_host_checks_need_no_device():
    lib = binding.load_library()
    n = None
    buf = ctypes.create_string_buffer(64)
    p = ctypes.c_void_p((ctypes.addressof(buf) + 15) & ~15)
    # slot mapping: block size 8 not compiled; negative sizes; null pointers; empty is a no-op
    assert lib.pkv_slot_mapping(p, p, 4, p, p, 2, 5, 8, 32, n) == -2
    assert lib.pkv_slot_mapping(p, p, 4, p, p, -1, 5, 16, 32, n) == -1
    assert lib.pkv_slot_mapping(n, p, 4, p, p, 2, 5, 16, 32, n) == -1
    assert lib.pkv_slot_mapping(p, p, 0, p, p, 2, 5, 16, 32, n) == -1
    assert lib.pkv_slot_mapping(n, n, 4, n, n, 2, 0, 16, 32, n) == 0
    # slots are int32: num_blocks * block_size must stay below 2^31
    assert lib.pkv_slot_mapping(p, p, 4, p, p, 2, 5, 16, 1 << 27, n) == -2
    # block copies: shape checks, null pairs, misaligned cache, empty is a no-op
    assert lib.pkv_copy_blocks(p, p, p, 1, 2, 96, 16, 32, 0, n) == -2
    assert lib.pkv_copy_blocks(p, p, n, 1, 2, 64, 16, 32, 0, n) == -1
    assert lib.pkv_copy_blocks(p, p, p, -1, 2, 64, 16, 32, 0, n) == -1
    assert lib.pkv_copy_blocks(ctypes.c_void_p(p.value + 4), p, p, 1, 2, 64, 16, 32, 0, n) == -7
    assert lib.pkv_copy_blocks(n, n, n, 0, 2, 64, 16, 32, 0, n) == 0


def test_workspace_size_is_positive_and_monotone():
    a = pkv.decode_workspace_bytes(64, 32, 32, 128)
    b = pkv.decode_workspace_bytes(128, 32, 32, 128)
    assert 0 < a < b
    assert pkv.decode_workspace_bytes(64, 32, 5, 128) == 0


def test_missing_library_fails_loudly():
    """No CPU fallback: without the CUDA library every entry point raises at first use."""
    import subprocess
    import sys
    code = ("import paged_kv_cache_447_b200 as pkv\n"
            "try:\n    pkv.version()\nexcept ImportError as e:\n    print('raised', e)\n")
    env = dict(os.environ, PKV_LIBRARY=os.path.join(ROOT, "no_such_libpagedkv.so"))
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.startswith("raised") and "missing" in r.stdout
