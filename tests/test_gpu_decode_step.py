"""GPU parity of the decode step (pkv_paged_decode_step): storing each sequence's new token and
attending over the cache -- in one kernel, or as store + attention + merge, or as the batch
size picks -- gives the same cache bytes and the same output bits as pkv_kv_store followed
by pkv_paged_decode_attention, matches the oracle, and leaves the workspace's counters at
zero for the next call."""
import numpy as np
import pytest
import torch

import paged_kv_cache_447_b200 as pkv
from paged_kv_cache_447_b200 import workloads as W

from helpers import DeviceWorkload, compare, oracle_attention, oracle_caches, oracle_store

pytestmark = pytest.mark.gpu


def _decode_rows(full: W.Workload) -> W.Workload:
    st = full.steps[-1]
    sub = W.sub_step(st, range(st.decode_seqs))
    return W.Workload(full.name, full.seed, full.n_q_heads, full.n_kv_heads, full.head_dim,
                      full.num_blocks, full.cache_dtype, full.k_cache, full.v_cache, [sub],
                      full.max_pos, full.k_scale, full.v_scale)


def _small_batch(seed=11, batch=4, context=4096, fp8=False):
    full = W.gqa_decode(seed=seed, batch=batch, context=context)
    if not fp8:
        return full
    st = full.steps[0]
    ks, vs = W._fp8_scales(st.k, st.v)
    g = torch.Generator().manual_seed(seed)
    kc, vc = W._fill_cache(g, full.num_blocks, full.n_kv_heads, full.head_dim, True, ks, vs)
    return W.Workload(full.name, seed, full.n_q_heads, full.n_kv_heads, full.head_dim,
                      full.num_blocks, "fp8", kc, vc, [st], full.max_pos, ks, vs)


def _slots_from_tables(st: W.Step) -> torch.Tensor:
    L = st.context_lens.long()
    p = L - 1
    blk = st.block_tables.long().gather(1, (p // 16).clamp(min=0).unsqueeze(1)).squeeze(1)
    return torch.where(L > 0, blk * 16 + p % 16, torch.full_like(p, -1)).to(torch.int32)


def _check(wl: W.Workload, oracle_rows=None):
    st = wl.steps[-1]
    fp8 = wl.cache_dtype == "fp8"
    # the step's slots are the ones its block tables give for position L_b - 1
    assert torch.equal(_slots_from_tables(st), st.slot_mapping)
    a = DeviceWorkload(wl)
    a.store(st)
    ref = a.decode(st)
    # every mode: one launch, store + attention + merge, and whichever the batch size picks
    for mode in (pkv.STEP_FUSED, pkv.STEP_SPLIT, pkv.STEP_AUTO):
        pkv.set_decode_step_mode(mode)
        try:
            b = DeviceWorkload(wl)
            ws = pkv.decode_step_workspace(st.num_seqs, wl.n_q_heads, wl.n_kv_heads, wl.head_dim)
            for _ in range(2):  # twice in a row: the first call must leave its counters at zero
                out = pkv.paged_decode_step(st.q.cuda(), st.k.cuda(), st.v.cuda(), b.k_cache,
                                            b.v_cache, st.block_tables.cuda(), st.context_lens.cuda(),
                                            ws, scale=wl.scale, k_scale=b.k_scale,
                                            v_scale=b.v_scale, rope_cos_sin=b.table)
                torch.cuda.synchronize()
                assert pkv.get_error() == 0
                assert torch.equal(b.k_cache, a.k_cache) and torch.equal(b.v_cache, a.v_cache), mode
                assert torch.equal(out, ref), (mode, float((out.float() - ref.float()).abs().max()))
            nctr = st.num_seqs * wl.n_kv_heads * 4
            assert int(ws[-((nctr + 15) // 16 * 16):].count_nonzero()) == 0
        finally:
            pkv.set_decode_step_mode(pkv.STEP_AUTO)
    if oracle_rows is not False:
        kc, vc = oracle_caches(wl)
        oracle_store(wl, st, kc, vc)
        want = oracle_attention(wl, st, kc, vc)
        compare(out, want, fp8=fp8, what=f"{wl.name} decode step")


def test_decode_step_tiny():
    wl = W.tiny(seed=1)
    # the tiny workload's decode step follows its prefill: store the prompts first
    pre, dec = wl.steps
    kc, vc = wl.k_cache.clone(), wl.v_cache.clone()
    d = DeviceWorkload(wl)
    d.store(pre)
    wl2 = W.Workload(wl.name, wl.seed, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.num_blocks,
                     "bf16", d.k_cache.cpu(), d.v_cache.cpu(), [dec], wl.max_pos)
    _check(wl2)
    del kc, vc


def test_decode_step_qwen_full_size():
    _check(W.qwen_decode(seed=2))


def test_decode_step_gqa_layer():
    _check(W.gqa_decode(seed=3))


@pytest.mark.parametrize("fp8", [False, True])
def test_decode_step_lognormal_mix(fp8):
    _check(_decode_rows(W.mix(seed=5, fp8=fp8)))


@pytest.mark.parametrize("fp8", [False, True])
def test_decode_step_small_batch(fp8):
    """The latency-bound case the fused step is for: 4 sequences of 4096 tokens, so every
    sequence is split across many CTAs and merged in-kernel."""
    _check(_small_batch(fp8=fp8))


def _lognormal_batch(seed, hq, hkv, d, fp8, batch=24, hi=3000):
    g = torch.Generator().manual_seed(seed)
    lens = W.lognormal_lengths(g, batch, hi=hi)
    counts = [W.blocks_needed(L) for L in lens]
    nb = sum(counts) + 4
    perm = torch.randperm(nb, generator=g)
    bt = W._assign_blocks(perm, counts, max_blocks=max(counts) + 1)
    st = W._step("step", g, hq, hkv, d, [1] * batch, lens, bt, decode_seqs=batch)
    ks = vs = None
    if fp8:
        ks, vs = W._fp8_scales(st.k, st.v)
    kc, vc = W._fill_cache(g, nb, hkv, d, fp8, ks, vs)
    return W.Workload("step", seed, hq, hkv, d, nb, "fp8" if fp8 else "bf16", kc, vc, [st],
                      max_pos=max(lens) + 1, k_scale=ks, v_scale=vs)


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("hq,hkv,d", [(8, 8, 64), (8, 4, 64), (16, 2, 128), (8, 1, 128)])
def test_decode_step_groups_and_head_dims(hq, hkv, d, fp8):
    _check(_lognormal_batch(30 + hq + d, hq, hkv, d, fp8))


@pytest.fixture(params=["fused", "split"])
def step_mode(request):
    pkv.set_decode_step_mode(pkv.STEP_FUSED if request.param == "fused" else pkv.STEP_SPLIT)
    yield request.param
    pkv.set_decode_step_mode(pkv.STEP_AUTO)


def test_decode_step_empty_and_out_of_table(step_mode):
    """A sequence with no context stores nothing and gets a zero row; a block-table entry
    outside the pool stores nothing and raises the bounds flag (in both step modes)."""
    wl = W.qwen_decode(seed=2, batch=6)
    st = wl.steps[0]
    ctx = st.context_lens.clone()
    ctx[2] = 0
    d = DeviceWorkload(wl)
    before_k = d.k_cache.clone()
    ws = pkv.decode_step_workspace(st.num_seqs, wl.n_q_heads, wl.n_kv_heads, wl.head_dim)
    out = pkv.paged_decode_step(st.q.cuda(), st.k.cuda(), st.v.cuda(), d.k_cache, d.v_cache,
                                st.block_tables.cuda(), ctx.cuda(), ws, rope_cos_sin=d.table)
    torch.cuda.synchronize()
    assert pkv.get_error() == 0
    assert torch.count_nonzero(out[2].float()) == 0
    slot2 = int(_slots_from_tables(st)[2])
    flat = lambda c: c.view(-1, wl.n_kv_heads, wl.head_dim)
    assert torch.equal(flat(d.k_cache)[slot2], flat(before_k)[slot2])
    bt = st.block_tables.clone()
    last = (int(st.context_lens[4]) - 1) // 16
    bt[4, last] = wl.num_blocks + 7
    pkv.paged_decode_step(st.q.cuda(), st.k.cuda(), st.v.cuda(), d.k_cache, d.v_cache, bt.cuda(),
                          st.context_lens.cuda(), ws, rope_cos_sin=d.table)
    assert pkv.get_error() == -6


def test_decode_step_rejects_a_short_workspace():
    wl = W.tiny(seed=1)
    st = wl.steps[1]
    d = DeviceWorkload(wl)
    n = pkv.decode_step_workspace_bytes(st.num_seqs, wl.n_q_heads, wl.n_kv_heads, wl.head_dim)
    ws = torch.zeros(n - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_decode_step(st.q.cuda(), st.k.cuda(), st.v.cuda(), d.k_cache, d.v_cache,
                              st.block_tables.cuda(), st.context_lens.cuda(), ws)
    assert e.value.code == -3
