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
    # block sizes other than 8, 16, 32 are not compiled
    assert lib.pkv_kv_store(n, n, n, n, n, 4, 2, 64, 12, 32, 0, n, n, n, 0, n, n, 0, n) == -2
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
    # slot mapping: block size 12 not compiled; negative sizes; null pointers; empty is a no-op
    assert lib.pkv_slot_mapping(p, p, 4, p, p, 2, 5, 12, 32, n) == -2
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


def test_decode_step_mode_control():
    """The decode-step mode: unknown modes are refused and change nothing; a set returns the
    previous mode."""
    lib = binding.load_library()
    assert lib.pkv_set_decode_step_mode(7) == -1
    assert lib.pkv_set_decode_step_mode(-1) == -1
    prev = pkv.set_decode_step_mode(pkv.STEP_SPLIT)
    assert prev == pkv.STEP_AUTO
    assert pkv.set_decode_step_mode(pkv.STEP_FUSED) == pkv.STEP_SPLIT
    assert pkv.set_decode_step_mode(pkv.STEP_AUTO) == pkv.STEP_FUSED
    with pytest.raises(pkv.PagedKVError):
        pkv.set_decode_step_mode(3)


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


# ---- the header's prototypes, the binding's ctypes signatures and a C caller agree

_CTYPE = {"int": ctypes.c_int, "long long": ctypes.c_longlong, "size_t": ctypes.c_size_t,
          "float": ctypes.c_float, "double": ctypes.c_double, "void": None}


def _prototypes():
    """name -> (return type, [parameter types]) for every function pkv.h declares."""
    src = open(os.path.join(ROOT, "include", "pkv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"#[^\n]*", "", src)
    protos = {}
    for ret, name, params in re.findall(
            r"((?:const\s+)?[A-Za-z_][A-Za-z0-9_ ]*?\s*\**)\s*\b(pkv_[a-z0-9_]+)\s*\(([^)]*)\)\s*;",
            src, flags=re.S):
        ps = [p.strip() for p in params.split(",")]
        types = []
        for p in ps:
            if p in ("void", ""):
                continue
            p = re.sub(r"\s+", " ", p)
            t = re.sub(r"\s*\b[A-Za-z_][A-Za-z0-9_]*$", "", p)  # drop the parameter name
            types.append(t.strip())
        protos[name] = (re.sub(r"\s+", " ", ret.strip()), types)
    return protos


def _as_ctype(t: str):
    t = t.replace("const ", "").strip()
    if t.endswith("*") or t == "pkv_stream_t":
        return "char*" if t == "char *" else ctypes.c_void_p
    return _CTYPE[t]


def test_binding_signatures_match_the_header():
    """Every argtypes / restype the ctypes binding sets equals what pkv.h declares, in
    order -- an int passed where the header has long long (or a swapped pair) fails."""
    protos = _prototypes()
    lib = binding.load_library()
    assert set(protos) == set(_declared_symbols())
    for name, (ret, params) in protos.items():
        fn = getattr(lib, name)
        want = [_as_ctype(p) for p in params]
        got = list(fn.argtypes or [])
        assert len(got) == len(want), (name, params)
        for i, (g, w) in enumerate(zip(got, want)):
            if w == "char*":
                w = ctypes.c_char_p
            assert g is w, f"{name} argument {i}: binding {g}, header {params[i]}"
        wr = _as_ctype(ret)
        if ret.replace(" ", "") == "constchar*":
            wr = ctypes.c_char_p
        assert fn.restype is wr, f"{name} returns {ret}, binding {fn.restype}"


def _build_c_driver(tmp_path):
    """Compile tests/abi_check.c against include/pkv.h only (-Wall -Werror) and link it to
    the library."""
    import subprocess
    src = os.path.join(ROOT, "tests", "abi_check.c")
    exe = str(tmp_path / "abi_check")
    libdir = os.path.dirname(binding.library_path())
    cuda = "/usr/local/cuda"
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-O1", "-I", os.path.join(ROOT, "include"),
           "-I", f"{cuda}/include", src, "-o", exe, "-L", libdir, "-lpagedkv",
           f"-Wl,-rpath,{libdir}", "-L", f"{cuda}/lib64", "-lcudart", f"-Wl,-rpath,{cuda}/lib64", "-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_c_caller_host_entry_points(tmp_path):
    """A C program that includes pkv.h calls every host-side entry point and the argument
    checks that return before touching a device."""
    import subprocess
    exe = _build_c_driver(tmp_path)
    r = subprocess.run([exe, "host"], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "host checks passed" in r.stdout


@pytest.mark.gpu
def test_c_caller_runs_the_hot_path(tmp_path):
    """The same C program stores a tiny batch (K rotated), runs prefill and decode through
    the header's prototypes with device buffers it allocates itself, and writes the outputs;
    they must match the oracle."""
    import subprocess
    from paged_kv_cache_447_b200 import workloads as W
    from helpers import oracle_attention, oracle_caches, oracle_store
    exe = _build_c_driver(tmp_path)
    wl = W.tiny(seed=1)
    pre, dec = wl.steps
    kc, vc = oracle_caches(wl)
    files = {}

    def put(name, arr):
        path = str(tmp_path / name)
        np.ascontiguousarray(arr).tofile(path)
        files[name] = path

    put("k_cache", kc)
    put("v_cache", vc)
    for tag, st in (("pre", pre), ("dec", dec)):
        for f in ("q", "k", "v"):
            put(f"{tag}_{f}", W.bits(getattr(st, f)))
        for f in ("slot_mapping", "cu_seqlens", "context_lens", "block_tables"):
            put(f"{tag}_{f}", getattr(st, f).numpy().astype(np.int32))
    dims = [wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.num_blocks, wl.max_pos,
            pre.num_seqs, pre.num_tokens, pre.block_tables.shape[1], pre.max_new_tokens,
            dec.num_seqs, dec.num_tokens, dec.block_tables.shape[1]]
    r = subprocess.run([exe, "device", str(tmp_path)] + [str(x) for x in dims],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    # oracle side: the same two steps
    outs = {}
    for tag, st in (("pre", pre), ("dec", dec)):
        oracle_store(wl, st, kc, vc)
        outs[tag] = oracle_attention(wl, st, kc, vc)
    for tag, st in (("pre", pre), ("dec", dec)):
        got = np.fromfile(str(tmp_path / f"out_{tag}"), dtype=np.uint16)
        got = oracle.bf16_to_f64(got).reshape(outs[tag].shape)
        err = np.abs(got - outs[tag])
        assert err.max() <= 1e-2 and err.mean() <= 1e-3, (tag, err.max())
    assert np.array_equal(np.fromfile(str(tmp_path / "k_cache_out"), dtype=np.uint16).reshape(kc.shape), kc)
