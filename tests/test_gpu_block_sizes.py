"""Block sizes 8, 16 and 32 ("Inside the Nano-vLLM engine: KV cache, attention and tensor
parallelism", §2.2 uses 16 tokens per block as an example, not a constant): slot mapping,
store, prefill, decode attention, the one-launch decode step and the block pool, each against
the oracle run with the same block size.  Lengths are chosen around the block and 16-token
tile boundaries (1, bs - 1, bs, bs + 1, 17, 33, ...)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_447_b200 as pkv
from paged_kv_cache_447_b200 import workloads as W

from helpers import DeviceWorkload, compare, oracle_attention, oracle_caches, oracle_store

pytestmark = pytest.mark.gpu

SHAPES = [(64, 8, 8, False), (128, 16, 4, False), (128, 8, 2, True), (64, 8, 4, True),
          (128, 32, 8, False), (128, 32, 8, True)]


def _lengths(bs):
    return [1, bs - 1, bs, bs + 1, 17, 33, 47, 250, 1001]


@pytest.mark.parametrize("bs", [8, 32])
@pytest.mark.parametrize("d,hq,hkv,fp8", SHAPES)
def test_slots_store_and_prefill(bs, d, hq, hkv, fp8):
    ctxs = _lengths(bs)
    news = [min(L, n) for L, n in zip(ctxs, [1, 5, bs, bs + 1, 17, 20, 47, 130, 300])]
    wl = W.paged_batch(100 + bs + d + hq, hq, hkv, d, news, ctxs, block_size=bs, fp8=fp8)
    st = wl.steps[0]
    # slot mapping on the device = the generator's slots = the oracle's
    slots = pkv.slot_mapping(st.block_tables.cuda(), st.cu_seqlens.cuda(), st.context_lens.cuda(),
                             st.num_tokens, wl.num_blocks, block_size=bs)
    orc = oracle.slot_mapping(st.block_tables.numpy(), st.cu_seqlens.numpy(),
                              st.context_lens.numpy(), bs, wl.num_blocks)
    assert np.array_equal(slots.cpu().numpy(), orc)
    assert np.array_equal(orc, st.slot_mapping.numpy())
    dwl = DeviceWorkload(wl)
    kc, vc = oracle_caches(wl)
    dwl.store(st)
    oracle_store(wl, st, kc, vc)
    out = dwl.prefill(st)
    torch.cuda.synchronize()
    assert pkv.get_error() == 0
    assert np.array_equal(W.bits(dwl.k_cache.cpu()), kc) and np.array_equal(W.bits(dwl.v_cache.cpu()), vc)
    compare(out, oracle_attention(wl, st, kc, vc), fp8=fp8, what=f"prefill bs={bs}")


@pytest.mark.parametrize("mode", ["fused", "split"])
@pytest.mark.parametrize("bs", [8, 32])
@pytest.mark.parametrize("d,hq,hkv,fp8", SHAPES)
def test_decode_and_decode_step(bs, d, hq, hkv, fp8, mode):
    ctxs = _lengths(bs) + [4096, 2 * bs + 3]
    wl = W.paged_batch(200 + bs + d + hq, hq, hkv, d, [1] * len(ctxs), ctxs, block_size=bs,
                       fp8=fp8, decode_seqs=len(ctxs))
    st = wl.steps[0]
    a = DeviceWorkload(wl)
    a.store(st)
    ref = a.decode(st)
    b = DeviceWorkload(wl)
    ws = pkv.decode_step_workspace(st.num_seqs, hq, hkv, d)
    pkv.set_decode_step_mode(pkv.STEP_FUSED if mode == "fused" else pkv.STEP_SPLIT)
    try:
        out = pkv.paged_decode_step(st.q.cuda(), st.k.cuda(), st.v.cuda(), b.k_cache, b.v_cache,
                                    st.block_tables.cuda(), st.context_lens.cuda(), ws, scale=wl.scale,
                                    k_scale=b.k_scale, v_scale=b.v_scale, rope_cos_sin=b.table)
        torch.cuda.synchronize()
    finally:
        pkv.set_decode_step_mode(pkv.STEP_AUTO)
    assert pkv.get_error() == 0
    assert torch.equal(b.k_cache, a.k_cache) and torch.equal(b.v_cache, a.v_cache)
    assert torch.equal(out, ref)
    if mode == "fused":
        kc, vc = oracle_caches(wl)
        oracle_store(wl, st, kc, vc)
        compare(ref, oracle_attention(wl, st, kc, vc), fp8=fp8, what=f"decode bs={bs}")


@pytest.mark.parametrize("bs", [8, 32])
def test_pool_and_block_copies(bs):
    """Pool allocation counts blocks of bs tokens; block copies move whole blocks of bs rows."""
    nb = 40
    pool = pkv.block_pool(nb)
    orc = oracle.pool_init(nb)
    ctx = np.array([1, bs, bs + 1, 3 * bs + 5], np.int32)
    cu = np.concatenate([[0], np.cumsum(ctx)]).astype(np.int32)
    bt = np.full((4, 8), -1, np.int32)
    bt_dev = torch.from_numpy(bt.copy()).cuda()
    pkv.block_pool_alloc(pool, bt_dev, torch.from_numpy(cu).cuda(), torch.from_numpy(ctx).cuda(),
                         block_size=bs)
    assert oracle.pool_alloc(orc, bt, cu, ctx, block_size=bs) == 0
    assert pkv.get_error() == 0
    assert np.array_equal(bt_dev.cpu().numpy(), bt)
    assert int(pool[0].item()) == int(orc[0]) == nb - sum(-(-int(L) // bs) for L in ctx)
    g = torch.Generator().manual_seed(bs)
    kc = torch.randn(nb, bs, 2, 64, generator=g).to(torch.bfloat16)
    vc = torch.randn(nb, bs, 2, 64, generator=g).to(torch.bfloat16)
    okc, ovc = W.bits(kc).copy(), W.bits(vc).copy()
    dk, dv = kc.cuda(), vc.cuda()
    pairs = np.array([[3, 7], [0, 12], [39, 1]], np.int32)
    pkv.copy_blocks(dk, dv, torch.from_numpy(pairs).cuda())
    oracle.copy_blocks(okc, ovc, pairs)
    torch.cuda.synchronize()
    assert np.array_equal(W.bits(dk.cpu()), okc) and np.array_equal(W.bits(dv.cpu()), ovc)


@pytest.mark.parametrize("bs", [8, 16])
@pytest.mark.parametrize("hq,hkv,fp8", [(4, 4, False), (16, 4, False), (16, 2, True), (8, 8, True)])
def test_head_dim_256_store_rope_and_decode(bs, hq, hkv, fp8):
    """Head dim 256: the store (K rotated) is bit-exact, standalone RoPE matches the oracle
    bit for bit, decode attention and the decode step match the oracle (and each other bit
    for bit); prefill refuses the shape."""
    d = 256
    ctxs = [1, 15, 16, 17, 300, 2000]
    wl = W.paged_batch(300 + bs + hq, hq, hkv, d, [1] * len(ctxs), ctxs, block_size=bs, fp8=fp8,
                       decode_seqs=len(ctxs))
    st = wl.steps[0]
    a = DeviceWorkload(wl)
    kc, vc = oracle_caches(wl)
    a.store(st)
    oracle_store(wl, st, kc, vc)
    torch.cuda.synchronize()
    assert np.array_equal(W.bits(a.k_cache.cpu()), kc) and np.array_equal(W.bits(a.v_cache.cpu()), vc)
    ref = a.decode(st)
    compare(ref, oracle_attention(wl, st, kc, vc), fp8=fp8, what=f"decode d=256 bs={bs}")
    b = DeviceWorkload(wl)
    ws = pkv.decode_step_workspace(st.num_seqs, hq, hkv, d)
    out = pkv.paged_decode_step(st.q.cuda(), st.k.cuda(), st.v.cuda(), b.k_cache, b.v_cache,
                                st.block_tables.cuda(), st.context_lens.cuda(), ws, scale=wl.scale,
                                k_scale=b.k_scale, v_scale=b.v_scale, rope_cos_sin=b.table)
    torch.cuda.synchronize()
    assert pkv.get_error() == 0
    assert torch.equal(out, ref) and torch.equal(b.k_cache, a.k_cache)
    q = st.q.cuda().clone()
    pkv.rope_apply(q, None, a.table, st.cu_seqlens.cuda(), st.context_lens.cuda())
    pos = oracle.positions(st.cu_seqlens.numpy(), st.context_lens.numpy())
    assert np.array_equal(W.bits(q.cpu()), oracle.rope(W.bits(st.q), pos, oracle.rope_table(wl.max_pos, d)))
    with pytest.raises(pkv.PagedKVError) as e:
        a.prefill(st)
    assert e.value.code == -2
