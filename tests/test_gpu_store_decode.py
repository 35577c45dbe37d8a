"""GPU parity of kv_store, rope_apply and paged decode attention against the oracle.

Every test drives the library through its C ABI (ctypes binding) on seeded workloads from
paged_kv_cache_447_b200.workloads; the oracle gets the same inputs on the CPU."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_447_b200 as pkv
from paged_kv_cache_447_b200 import workloads as W

from helpers import (DeviceWorkload, cache_bits, compare, oracle_attention, oracle_caches,
                     oracle_store)

pytestmark = pytest.mark.gpu


def _assert_no_device_error():
    assert pkv.get_error() == 0


# ----------------------------------------------------------------------------- kv_store

@pytest.mark.parametrize("rope", [False, True])
@pytest.mark.parametrize("which", ["tiny", "shared_prefix_small", "mix_fp8_small"])
def test_kv_store_bit_exact(which, rope):
    wl = {"tiny": lambda: W.tiny(seed=1),
          "shared_prefix_small": lambda: W.shared_prefix(seed=4, requests=3, prefix=64, new=200),
          "mix_fp8_small": lambda: W.mix(seed=5, decodes=40, chunks=2, chunk_len=100, fp8=True,
                                         max_context=2048)}[which]()
    d = DeviceWorkload(wl)
    kc, vc = oracle_caches(wl)
    for st in wl.steps:
        sm = st.slot_mapping.clone()
        sm[::7] = -1                                  # padding tokens write nothing
        st2 = W.Step(st.name, st.q, st.k, st.v, sm, st.cu_seqlens, st.context_lens,
                     st.block_tables, st.decode_seqs)
        d.store(st2, rope=rope)
        oracle_store(wl, st2, kc, vc, rope=rope)
    torch.cuda.synchronize()
    _assert_no_device_error()
    assert np.array_equal(cache_bits(d.k_cache), kc)
    assert np.array_equal(cache_bits(d.v_cache), vc)


def test_kv_store_full_shared_prefix_size_bit_exact():
    wl = W.shared_prefix(seed=4)                      # 65,536 new tokens x 8 kv heads x 128
    d = DeviceWorkload(wl)
    kc, vc = oracle_caches(wl)
    st = wl.steps[0]
    d.store(st)
    oracle_store(wl, st, kc, vc)
    _assert_no_device_error()
    assert np.array_equal(cache_bits(d.k_cache), kc)
    assert np.array_equal(cache_bits(d.v_cache), vc)


def test_kv_store_out_of_range_slot_is_flagged_not_written():
    wl = W.tiny(seed=1)
    d = DeviceWorkload(wl)
    st = wl.steps[1]
    sm = st.slot_mapping.clone()
    sm[0] = wl.num_blocks * 16 + 5                    # past the cache
    before = cache_bits(d.k_cache).copy()
    pkv.kv_store(st.k.cuda(), st.v.cuda(), d.k_cache, d.v_cache, sm.cuda())
    assert pkv.get_error() == -6
    after = cache_bits(d.k_cache)
    flat_b = before.reshape(-1, 2, 64); flat_a = after.reshape(-1, 2, 64)
    for t in range(1, 4):
        s = int(sm[t])
        assert np.array_equal(flat_a[s], W.bits(st.k)[t])
    changed = np.any(flat_a != flat_b, axis=(1, 2))
    assert changed.sum() == 3


# ----------------------------------------------------------------------------- rope

def test_rope_apply_bit_exact():
    wl = W.shared_prefix(seed=4, requests=4, prefix=32, new=300)
    st = wl.steps[0]
    q = st.q.cuda(); k = st.k.cuda()
    tab = pkv.rope_build_table(wl.max_pos, wl.head_dim).cuda()
    pkv.rope_apply(q, k, tab, st.cu_seqlens.cuda(), st.context_lens.cuda())
    torch.cuda.synchronize()
    _assert_no_device_error()
    otab = oracle.rope_table(wl.max_pos, wl.head_dim)
    pos = oracle.positions(st.cu_seqlens.numpy(), st.context_lens.numpy())
    assert np.array_equal(cache_bits(q), oracle.rope(W.bits(st.q), pos, otab))
    assert np.array_equal(cache_bits(k), oracle.rope(W.bits(st.k), pos, otab))


def test_rope_position_past_table_is_flagged():
    wl = W.tiny(seed=1)
    st = wl.steps[0]
    q = st.q.cuda()
    tab = pkv.rope_build_table(10, wl.head_dim).cuda()   # too short for positions up to 59
    pkv.rope_apply(q, None, tab, st.cu_seqlens.cuda(), st.context_lens.cuda())
    assert pkv.get_error() == -6


# ----------------------------------------------------------------------------- decode

def _decode_case(wl, rope=True, rows=None):
    d = DeviceWorkload(wl)
    kc, vc = oracle_caches(wl)
    st = wl.steps[-1]
    for prev in wl.steps[:-1]:
        d.store(prev, rope=rope)
        oracle_store(wl, prev, kc, vc, rope=rope)
    d.store(st, rope=rope)
    oracle_store(wl, st, kc, vc, rope=rope)
    out = d.decode(st, rope=rope)
    torch.cuda.synchronize()
    _assert_no_device_error()
    ref = oracle_attention(wl, st, kc, vc, rope=rope, rows=rows)
    return out, ref, d


@pytest.mark.parametrize("rope", [False, True])
def test_decode_tiny(rope):
    wl = W.tiny(seed=1)
    out, ref, _ = _decode_case(wl, rope)
    compare(out, ref, what="tiny decode")


def test_decode_qwen_mha_full_size():
    """Qwen-7B-style MHA decode at full size: 64 sequences, L ~ U[128, 2048], every row."""
    wl = W.qwen_decode(seed=2)
    out, ref, _ = _decode_case(wl)
    compare(out, ref, what="qwen decode")


def test_decode_gqa_one_layer_full_size():
    """Mistral-7B-style GQA decode, one layer at full size (32 x 4096 tokens)."""
    wl = W.gqa_decode(seed=3)
    out, ref, _ = _decode_case(wl)
    compare(out, ref, what="gqa decode")


@pytest.mark.parametrize("fp8", [False, True])
def test_decode_lognormal_mix(fp8):
    """The decode rows of the continuous-batching mix (lognormal lengths up to 32k)."""
    full = W.mix(seed=5, fp8=fp8)
    st = full.steps[0]
    dec = W.sub_step(st, range(st.decode_seqs))
    wl = W.Workload(full.name, full.seed, 32, 8, 128, full.num_blocks, full.cache_dtype,
                    full.k_cache, full.v_cache, [dec], full.max_pos, full.k_scale, full.v_scale)
    out, ref, _ = _decode_case(wl)
    compare(out, ref, fp8=fp8, what="mix decode")


@pytest.mark.parametrize("lens", [[1, 16, 17, 0, 33], [0, 0, 0], [5000, 1, 2, 3],
                                  [16 * 7] * 9])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_decode_edge_lengths_and_groups(lens, group):
    """Empty contexts (zero rows), single tokens, exact block multiples, ragged tails and
    one long sequence among short ones, for every compiled GQA group size."""
    g = torch.Generator().manual_seed(100 + group)
    hkv, d = 2, 128
    hq = hkv * group
    counts = [W.blocks_needed(L) for L in lens]
    nb = sum(counts) + 3
    perm = torch.randperm(nb, generator=g)
    bt = W._assign_blocks(perm, counts, max_blocks=max(max(counts), 1) + 1)
    kc, vc = W._fill_cache(g, nb, hkv, d, False)
    B = len(lens)
    st = W.Step("edge", W._randn_bf16(g, B, hq, d), W._randn_bf16(g, B, hkv, d),
                W._randn_bf16(g, B, hkv, d), torch.full((B,), -1, dtype=torch.int32),
                torch.arange(B + 1, dtype=torch.int32), torch.tensor(lens, dtype=torch.int32),
                bt, B)
    wl = W.Workload("edge", 0, hq, hkv, d, nb, "bf16", kc, vc, [st], max_pos=max(lens) + 1)
    dw = DeviceWorkload(wl)
    out = dw.decode(st, rope=False)
    torch.cuda.synchronize()
    _assert_no_device_error()
    ref = oracle_attention(wl, st, W.bits(kc), W.bits(vc), rope=False)
    compare(out, ref, what=f"edge {lens} G={group}")
    for b, L in enumerate(lens):
        if L == 0:
            assert torch.all(out[b] == 0)


def test_decode_unused_slots_hold_nan():
    """NaN sentinels in every slot no sequence owns (including the tails of last blocks)
    never reach the output."""
    wl = W.qwen_decode(seed=2, batch=8, lo=1, hi=300, nan_fill=True)
    st = wl.steps[0]
    # give every owned slot a finite value first (positions < L_b - 1) via the oracle-free
    # generator: write random rows at the owned slots on both sides
    g = torch.Generator().manual_seed(77)
    kc = wl.k_cache.clone(); vc = wl.v_cache.clone()
    for b in range(st.num_seqs):
        L = int(st.context_lens[b])
        for j in range(L):
            s = int(st.block_tables[b, j // 16]) * 16 + j % 16
            kc[s // 16, s % 16] = W._randn_bf16(g, 32, 128)
            vc[s // 16, s % 16] = W._randn_bf16(g, 32, 128)
    wl.k_cache, wl.v_cache = kc, vc
    out, ref, _ = _decode_case(wl)
    compare(out, ref, what="nan sentinels")


def _grouped_case(seed, lens, group, d, fp8, hkv=2, nan_unowned=False):
    """A decode step over a random cache with ragged lengths; optionally every K and V slot
    no sequence owns (the tails of last blocks included) holds NaN (E4M3: code 0x7F)."""
    g = torch.Generator().manual_seed(seed)
    hq = hkv * group
    counts = [W.blocks_needed(L) for L in lens]
    nb = sum(counts) + 4
    perm = torch.randperm(nb, generator=g)
    bt = W._assign_blocks(perm, counts, max_blocks=max(max(counts), 1) + 1)
    ks = vs = None
    if fp8:
        ks = (0.5 + torch.rand(hkv, generator=g)) / 100.0
        vs = (0.5 + torch.rand(hkv, generator=g)) / 100.0
    kc, vc = W._fill_cache(g, nb, hkv, d, fp8, ks, vs)
    if nan_unowned:
        owned = torch.zeros(nb * 16, dtype=torch.bool)
        for b, L in enumerate(lens):
            for j in range(L):
                owned[int(bt[b, j // 16]) * 16 + j % 16] = True
        fill = 0x7F if fp8 else float("nan")
        kc.view(nb * 16, hkv, d)[~owned] = fill
        vc.view(nb * 16, hkv, d)[~owned] = fill
    B = len(lens)
    st = W.Step("grouped", W._randn_bf16(g, B, hq, d), W._randn_bf16(g, B, hkv, d),
                W._randn_bf16(g, B, hkv, d), torch.full((B,), -1, dtype=torch.int32),
                torch.arange(B + 1, dtype=torch.int32), torch.tensor(lens, dtype=torch.int32),
                bt, B)
    wl = W.Workload("grouped", seed, hq, hkv, d, nb, "fp8" if fp8 else "bf16", kc, vc, [st],
                    max_pos=max(lens) + 1, k_scale=ks, v_scale=vs)
    dw = DeviceWorkload(wl)
    out = dw.decode(st, rope=False)
    torch.cuda.synchronize()
    _assert_no_device_error()
    ref = oracle_attention(wl, st, W.bits(kc), W.bits(vc), rope=False)
    return out, ref


@pytest.mark.parametrize("d,fp8", [(64, False), (128, False), (64, True), (128, True)])
@pytest.mark.parametrize("group", [2, 4, 8])
def test_decode_grouped_nan_sentinels(group, d, fp8):
    """Grouped heads: NaN in every K and V slot no sequence owns (the tails of last blocks
    included) never reaches the output, whatever the group size, head dim and cache type."""
    out, ref = _grouped_case(300 + group + d, [1, 15, 17, 250, 16 * 5, 1000], group, d, fp8,
                             nan_unowned=True)
    assert torch.isfinite(out.float()).all()
    compare(out, ref, fp8=fp8, what=f"nan sentinels G={group} D={d} fp8={fp8}")


@pytest.mark.parametrize("lens", [[1, 16, 17, 0, 33], [5000, 1, 2, 3], [16 * 7] * 9])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_decode_fp8_edge_lengths_and_groups(lens, group):
    """E4M3 caches with per-head scales: empty, single-token, block-multiple and ragged
    contexts for every compiled group size (head dim 128)."""
    out, ref = _grouped_case(500 + group, lens, group, 128, True)
    compare(out, ref, fp8=True, what=f"fp8 edge {lens} G={group}")
    for b, L in enumerate(lens):
        if L == 0:
            assert torch.all(out[b] == 0)


@pytest.mark.parametrize("group", [2, 4])
def test_decode_fp8_odd_kv_heads(group):
    """E4M3 with an odd kv-head count: units hold one kv head (two-head units need pairs)."""
    out, ref = _grouped_case(700 + group, [5000, 1, 17, 250], group, 128, True, hkv=3)
    compare(out, ref, fp8=True, what=f"fp8 odd kv heads G={group}")


def test_decode_block_id_out_of_range_is_flagged():
    wl = W.tiny(seed=1)
    st = wl.steps[1]
    bt = st.block_tables.clone()
    bt[2, 1] = wl.num_blocks + 3
    d = DeviceWorkload(wl)
    pkv.paged_decode_attention(st.q.cuda(), d.k_cache, d.v_cache, bt.cuda(),
                               st.context_lens.cuda())
    assert pkv.get_error() == -6


def test_decode_workspace_too_small_is_rejected():
    wl = W.tiny(seed=1)
    st = wl.steps[1]
    d = DeviceWorkload(wl)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_decode_attention(st.q.cuda(), d.k_cache, d.v_cache, st.block_tables.cuda(),
                                   st.context_lens.cuda(), workspace=ws)
    assert e.value.code == -3


def test_decode_is_deterministic_and_batch_independent():
    wl = W.qwen_decode(seed=2, batch=16, lo=10, hi=900)
    d = DeviceWorkload(wl)
    st = wl.steps[0]
    o1 = d.decode(st, rope=False)
    o2 = d.decode(st, rope=False)
    assert torch.equal(o1, o2)
    for b in (0, 7, 15):
        sub = W.sub_step(st, [b])
        ob = d.decode(sub, rope=False)
        torch.testing.assert_close(ob[0].float(), o1[b].float(), atol=2e-3, rtol=0)


def test_bounded_wait_times_out_and_context_survives():
    """Failure detection: a kernel whose mbarrier never completes gives up after the limit,
    reports PKV_E_TIMEOUT, and the context keeps working."""
    pkv.debug_wait_timeout(5_000_000)                 # 5 ms
    assert pkv.get_error() == -5
    assert pkv.get_error() == 0                       # cleared
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0


@pytest.mark.parametrize("scales", [(1.0, 0.0625), (0.3, 3.0), (1e-3, 7.0), (448.0, 2.0 ** -9)])
def test_kv_store_e4m3_every_bf16_value(scales):
    """The E4M3 quantiser of kv_store on every bf16 bit pattern (NaN included), for two heads
    with their own scales: code for code as the oracle's (fp64 quotient, round to nearest
    even, saturate).  Scales that are powers of two put many quotients exactly on rounding
    midpoints, where the product's fp32 shortcut has to take the exact decision."""
    H, D = 2, 128
    vals = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    T = 65536 // (H * D) * 2                   # every pattern once per head
    k = np.concatenate([vals, vals]).reshape(T, H, D)
    v = k[::-1].copy()
    bs = 16
    NB = T // bs
    slots = np.arange(T, dtype=np.int32)
    ks = np.array(scales, dtype=np.float32)
    vs = ks[::-1].copy()
    kc = np.zeros((NB, bs, H, D), dtype=np.uint8)
    vc = np.zeros_like(kc)
    oracle.kv_store(k, v, kc, vc, slots, bs, fp8=True, k_scale=ks, v_scale=vs)
    dk = torch.from_numpy(k.view(np.int16)).view(torch.bfloat16).cuda()
    dv = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).cuda()
    gk = torch.zeros((NB, bs, H, D), dtype=torch.uint8, device="cuda")
    gv = torch.zeros_like(gk)
    pkv.kv_store(dk, dv, gk, gv, torch.from_numpy(slots).cuda(), k_scale=torch.from_numpy(ks).cuda(),
                 v_scale=torch.from_numpy(vs).cuda())
    torch.cuda.synchronize()
    _assert_no_device_error()
    assert np.array_equal(gk.cpu().numpy(), kc)
    assert np.array_equal(gv.cpu().numpy(), vc)
