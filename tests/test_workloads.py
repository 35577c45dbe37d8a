"""The seeded synthetic inputs (CPU): deterministic per seed, shaped like the five
configurations, and internally consistent -- every stored token's slot is where its
sequence's block table puts its position, tables never share a physical block except the
aliased prefix, and the lognormal mix stays inside its clip range."""
import numpy as np
import pytest
import torch

from paged_kv_cache_447_b200 import workloads as W


def _positions(st):
    pos = []
    for b in range(st.num_seqs):
        n = int(st.cu_seqlens[b + 1] - st.cu_seqlens[b])
        L = int(st.context_lens[b])
        pos += list(range(L - n, L))
    return np.array(pos)


def _check_step(wl, st, shared=()):
    T = st.num_tokens
    assert st.q.shape == (T, wl.n_q_heads, wl.head_dim) and st.q.dtype == torch.bfloat16
    assert st.k.shape == st.v.shape == (T, wl.n_kv_heads, wl.head_dim)
    assert int(st.cu_seqlens[0]) == 0 and int(st.cu_seqlens[-1]) == T
    assert torch.all(st.cu_seqlens[1:] >= st.cu_seqlens[:-1])
    n = (st.cu_seqlens[1:] - st.cu_seqlens[:-1])
    assert torch.all(st.context_lens >= n)
    assert torch.all(n[:st.decode_seqs] == 1)
    # every token's slot is at its position in its table
    pos = _positions(st)
    for t in range(T):
        b = int(np.searchsorted(st.cu_seqlens.numpy(), t, side="right") - 1)
        s = int(st.slot_mapping[t])
        assert s == int(st.block_tables[b, pos[t] // 16]) * 16 + pos[t] % 16
    # tables cover their contexts with valid ids; blocks are private except the shared ones
    owner = {}
    for b in range(st.num_seqs):
        need = (int(st.context_lens[b]) + 15) // 16
        row = st.block_tables[b].tolist()
        assert all(0 <= x < wl.num_blocks for x in row[:need])
        for x in row[:need]:
            if x in shared:
                continue
            assert owner.setdefault(x, b) == b, f"block {x} in two tables"


def test_deterministic_per_seed():
    a, b = W.qwen_decode(seed=2), W.qwen_decode(seed=2)
    assert torch.equal(a.steps[0].q, b.steps[0].q) and torch.equal(a.k_cache, b.k_cache)
    assert torch.equal(a.steps[0].block_tables, b.steps[0].block_tables)
    c = W.qwen_decode(seed=3)
    assert not torch.equal(a.steps[0].q, c.steps[0].q)


def test_tiny_flow():
    wl = W.tiny(seed=1)
    pre, dec = wl.steps
    assert pre.context_lens.tolist() == [5, 17, 33, 60] and dec.context_lens.tolist() == [6, 18, 34, 61]
    assert wl.num_blocks == 32 and (wl.n_q_heads, wl.n_kv_heads, wl.head_dim) == (4, 2, 64)
    for st in wl.steps:
        _check_step(wl, st)


def test_qwen_decode_shape():
    wl = W.qwen_decode(seed=2)
    st = wl.steps[0]
    assert st.num_seqs == 64 and st.decode_seqs == 64
    assert (wl.n_q_heads, wl.n_kv_heads, wl.head_dim) == (32, 32, 128)
    assert int(st.context_lens.min()) >= 128 and int(st.context_lens.max()) <= 2048
    _check_step(wl, st)


def test_gqa_decode_shape():
    wl = W.gqa_decode(seed=3)
    st = wl.steps[0]
    assert st.num_seqs == 32 and torch.all(st.context_lens == 4096)
    assert (wl.n_q_heads, wl.n_kv_heads, wl.head_dim) == (32, 8, 128)
    _check_step(wl, st)


def test_shared_prefix_aliases_one_prefix():
    wl = W.shared_prefix(seed=4, requests=6, prefix=64, new=100)
    st = wl.steps[0]
    shared = wl.notes["shared_prefix_blocks"]
    assert len(shared) == 4
    for b in range(st.num_seqs):
        assert st.block_tables[b, :4].tolist() == shared
    assert torch.all(st.context_lens == 164)
    _check_step(wl, st, shared=set(shared))


@pytest.mark.parametrize("fp8", [False, True])
def test_mix_lengths_and_scales(fp8):
    wl = W.mix(seed=5, fp8=fp8)
    st = wl.steps[0]
    assert st.decode_seqs == 256 and st.num_seqs == 260
    L = st.context_lens
    assert int(L[:256].min()) >= 1 and int(L.max()) <= 32768
    n = (st.cu_seqlens[1:] - st.cu_seqlens[:-1])
    assert n[256:].tolist() == [512] * 4
    # median of the lognormal decode lengths near 1024 (sigma 1, 256 draws)
    assert 600 < float(L[:256].float().median()) < 1700
    if fp8:
        assert wl.k_cache.dtype == torch.uint8 and wl.k_scale.shape == (8,)
        amax = st.k.float().abs().permute(1, 0, 2).reshape(8, -1).amax(1)
        assert torch.allclose(wl.k_scale, amax / 448.0)
    _check_step(wl, st)
