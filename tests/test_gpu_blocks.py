"""GPU parity of the block bookkeeping helpers against the oracle: slot mapping from block
tables (bit-exact), copy-on-write block copies (bit-exact, bf16 and E4M3), and a shared
prefix that diverges: copy, slot, store and decode through the library equal private caches
attended by the oracle."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_447_b200 as pkv
from paged_kv_cache_447_b200 import workloads as W

from helpers import DeviceWorkload, cache_bits, compare, oracle_attention

pytestmark = pytest.mark.gpu


def _cu(new):
    return torch.tensor(np.concatenate([[0], np.cumsum(new)]), dtype=torch.int32)


@pytest.mark.parametrize("which", ["mix", "shared_prefix", "tiny"])
def test_slot_mapping_bit_exact(which):
    wl = {"mix": lambda: W.mix(seed=5),
          "shared_prefix": lambda: W.shared_prefix(seed=4, requests=5, prefix=48, new=300),
          "tiny": lambda: W.tiny(seed=1)}[which]()
    for st in wl.steps:
        T = int(st.cu_seqlens[-1])
        got = pkv.slot_mapping(st.block_tables.cuda(), st.cu_seqlens.cuda(), st.context_lens.cuda(),
                               T, wl.num_blocks)
        torch.cuda.synchronize()
        assert pkv.get_error() == 0
        ref = oracle.slot_mapping(st.block_tables.numpy(), st.cu_seqlens.numpy(),
                                  st.context_lens.numpy(), 16, wl.num_blocks)
        assert np.array_equal(got.cpu().numpy(), ref)
        # the workloads' own slot mappings (the store inputs) agree for every stored token
        sm = st.slot_mapping.numpy()
        assert np.array_equal(ref[sm >= 0], sm[sm >= 0])


def test_slot_mapping_out_of_table_is_flagged_and_minus_one():
    bt = torch.tensor([[3, -1], [9, 1]], dtype=torch.int32).cuda()
    cu = _cu([2, 1]).cuda()
    ctx = torch.tensor([18, 1], dtype=torch.int32).cuda()   # positions 16, 17 -> entry -1
    got = pkv.slot_mapping(bt, cu, ctx, 3, 8)                # block 9 >= num_blocks
    torch.cuda.synchronize()
    assert pkv.get_error() == -6
    assert got.cpu().tolist() == [-1, -1, -1]


@pytest.mark.parametrize("fp8", [False, True])
def test_copy_blocks_bit_exact(fp8):
    g = torch.Generator().manual_seed(21)
    nb, hkv, d = 40, 8, 128
    if fp8:
        kc = torch.randint(0, 256, (nb, 16, hkv, d), generator=g, dtype=torch.uint8)
        vc = torch.randint(0, 256, (nb, 16, hkv, d), generator=g, dtype=torch.uint8)
    else:
        kc = W._randn_bf16(g, nb, 16, hkv, d)
        vc = W._randn_bf16(g, nb, 16, hkv, d)
    pairs = [(3, 7), (0, 11), (5, 5), (20, 39), (38, 1)]
    dk, dv = kc.cuda(), vc.cuda()
    pkv.copy_blocks(dk, dv, torch.tensor(pairs, dtype=torch.int32).cuda())
    torch.cuda.synchronize()
    assert pkv.get_error() == 0
    ok, ov = W.bits(kc).copy(), W.bits(vc).copy()
    oracle.copy_blocks(ok, ov, pairs)
    assert np.array_equal(cache_bits(dk), ok) and np.array_equal(cache_bits(dv), ov)


def test_copy_blocks_bad_id_is_flagged_and_skipped():
    g = torch.Generator().manual_seed(22)
    kc = W._randn_bf16(g, 6, 16, 2, 64)
    vc = W._randn_bf16(g, 6, 16, 2, 64)
    dk, dv = kc.cuda(), vc.cuda()
    pkv.copy_blocks(dk, dv, torch.tensor([(2, 9), (1, 4)], dtype=torch.int32).cuda())
    torch.cuda.synchronize()
    assert pkv.get_error() == -6
    ok, ov = W.bits(kc).copy(), W.bits(vc).copy()
    oracle.copy_blocks(ok, ov, [(1, 4)])
    assert np.array_equal(cache_bits(dk), ok) and np.array_equal(cache_bits(dv), ov)


@pytest.mark.parametrize("fp8", [False, True])
def test_copy_on_write_divergence_decode(fp8):
    """Sixteen requests share a 40-token prefix (its third block is partial).  Each request
    takes a private copy of the partial block, then a prefill of its own 9 tokens and one
    decode step run through slot_mapping + kv_store + attention.  Outputs equal the oracle
    on the same final cache; the two full shared blocks are never written."""
    g = torch.Generator().manual_seed(23)
    R, hq, hkv, d, prefix, own = 16, 32, 8, 128, 40, 9
    nb = 3 + R * 2 + 4
    ks = vs = None
    if fp8:
        ks = (0.5 + torch.rand(hkv, generator=g)) / 100.0
        vs = (0.5 + torch.rand(hkv, generator=g)) / 100.0
    kc, vc = W._fill_cache(g, nb, hkv, d, fp8, ks, vs)
    shared = [0, 1, 2]                       # prefix tokens 0..39 live here (block 2 partial)
    copies = [(2, 3 + 2 * r) for r in range(R)]
    tables = torch.full((R, 4), -1, dtype=torch.int32)
    for r in range(R):
        tables[r, :4] = torch.tensor([0, 1, 3 + 2 * r, 4 + 2 * r], dtype=torch.int32)
    wl = W.Workload("cow", 0, hq, hkv, d, nb, "fp8" if fp8 else "bf16", kc, vc, [],
                    max_pos=prefix + own + 2, k_scale=ks, v_scale=vs)
    dw = DeviceWorkload(wl)
    before = cache_bits(dw.k_cache)[:2].copy()
    pkv.copy_blocks(dw.k_cache, dw.v_cache, torch.tensor(copies, dtype=torch.int32).cuda())
    okc, ovc = W.bits(kc).copy(), W.bits(vc).copy()
    oracle.copy_blocks(okc, ovc, copies)
    # prefill of each request's own tokens, then one decode token each
    for n_new, L in ((own, prefix + own), (1, prefix + own + 1)):
        B = R
        cu = _cu([n_new] * B)
        ctx = torch.full((B,), L, dtype=torch.int32)
        T = n_new * B
        sm = pkv.slot_mapping(tables.cuda(), cu.cuda(), ctx.cuda(), T, nb)
        st = W.Step("cow", W._randn_bf16(g, T, hq, d), W._randn_bf16(g, T, hkv, d),
                    W._randn_bf16(g, T, hkv, d), sm.cpu(), cu, ctx, tables,
                    B if n_new == 1 else 0)
        dw.store(st, rope=True)
        oracle.kv_store(W.bits(st.k), W.bits(st.v), okc, ovc, oracle.slot_mapping(
            tables.numpy(), cu.numpy(), ctx.numpy(), 16, nb), 16, fp8=fp8,
            k_scale=None if not fp8 else ks.numpy(), v_scale=None if not fp8 else vs.numpy(),
            table=oracle.rope_table(wl.max_pos, d), pos=oracle.positions(cu.numpy(), ctx.numpy()))
    out = dw.decode(st, rope=True)
    torch.cuda.synchronize()
    assert pkv.get_error() == 0
    assert np.array_equal(cache_bits(dw.k_cache), okc) and np.array_equal(cache_bits(dw.v_cache), ovc)
    assert np.array_equal(cache_bits(dw.k_cache)[:2], before)
    ref = oracle_attention(wl, st, okc, ovc, rope=True)
    compare(out, ref, fp8=fp8, what=f"copy-on-write decode fp8={fp8}")
