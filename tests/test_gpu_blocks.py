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


# ---------------------------------------------------------------- block pool on the device

def _pool_state(pool: torch.Tensor):
    p = pool.cpu().numpy()
    nb = (p.shape[0] - 4) // 2
    return int(p[0]), p[4:4 + nb], p[4 + nb:]


def _same_pool(gpu_pool, orc_pool):
    n, stack, flags = _pool_state(gpu_pool)
    nb = stack.shape[0]
    assert n == int(orc_pool[0])
    assert np.array_equal(stack[:n], orc_pool[1:1 + n])
    assert np.array_equal(flags, orc_pool[1 + nb:])


def test_block_pool_random_traffic_bit_exact():
    """Batches of admissions and growth (some larger than the pool can cover) and frees of
    finished sequences, on the device and in the oracle: after every call the free count,
    the stack of free ids, the free flags and every table written are identical."""
    rng = np.random.default_rng(3)
    nb, mb = 96, 24
    pool = pkv.block_pool(nb)
    orc = oracle.pool_init(nb)
    _same_pool(pool, orc)
    live = {}
    next_id = 0
    refused = 0
    for _ in range(120):
        if live and rng.random() < 0.35:
            ids = []
            for s in rng.choice(list(live), size=min(len(live), int(rng.integers(1, 3))), replace=False):
                ids += live.pop(int(s))[1]
            pkv.block_pool_free(pool, torch.tensor(ids, dtype=torch.int32, device="cuda"))
            assert oracle.pool_free(orc, ids) == 0
            assert pkv.get_error() == 0
        else:
            batch = [(s, int(rng.integers(1, 30))) for s in list(live)[:4]]
            for _ in range(int(rng.integers(0, 3))):
                batch.append((next_id, int(rng.integers(1, 200))))
                next_id += 1
            if not batch:
                continue
            bt = np.full((len(batch), mb), -1, np.int32)
            ctx, new = [], []
            for i, (s, n) in enumerate(batch):
                L0, table = live.get(s, (0, []))
                bt[i, :len(table)] = table
                ctx.append(L0 + n)
                new.append(n)
            cu = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
            ctx = np.array(ctx, np.int32)
            bt_dev = torch.from_numpy(bt.copy()).cuda()
            pkv.block_pool_alloc(pool, bt_dev, torch.from_numpy(cu).cuda(), torch.from_numpy(ctx).cuda())
            rc = oracle.pool_alloc(orc, bt, cu, ctx)
            code = pkv.get_error()
            if rc != 0:
                refused += 1
                assert code in (-9, -6)
            else:
                assert code == 0
                for i, (s, n) in enumerate(batch):
                    live[s] = (int(ctx[i]), [int(x) for x in bt[i] if x >= 0])
            assert np.array_equal(bt_dev.cpu().numpy(), bt)
        _same_pool(pool, orc)
    assert refused > 0  # the run did exercise the all-or-nothing refusal


def test_block_pool_rejects_double_and_foreign_frees():
    nb = 8
    pool = pkv.block_pool(nb)
    orc = oracle.pool_init(nb)
    bt = torch.full((1, 4), -1, dtype=torch.int32, device="cuda")
    cu = torch.tensor([0, 40], dtype=torch.int32, device="cuda")
    ctx = torch.tensor([40], dtype=torch.int32, device="cuda")
    pkv.block_pool_alloc(pool, bt, cu, ctx)
    btn = np.full((1, 4), -1, np.int32)
    oracle.pool_alloc(orc, btn, cu.cpu().numpy(), ctx.cpu().numpy())
    assert pkv.get_error() == 0
    ids = [2, 0, 2, 9, -1, 5, 1]   # 2 twice, 9 and -1 outside, 5 not allocated
    pkv.block_pool_free(pool, torch.tensor(ids, dtype=torch.int32, device="cuda"))
    assert pkv.get_error() == -6
    assert oracle.pool_free(orc, ids) == 4
    _same_pool(pool, orc)
    assert _pool_state(pool)[0] == 8


def test_block_pool_end_to_end_alloc_store_decode_free():
    """Blocks from the pool, slots from the tables, the store and decode attention over
    them, then the blocks back: the cache is what the oracle stores at the same slots and
    the output matches the oracle."""
    g = torch.Generator().manual_seed(12)
    hq, hkv, d, nb, mb = 8, 2, 128, 64, 16
    pool = pkv.block_pool(nb)
    kc = torch.zeros((nb, 16, hkv, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    okc = np.zeros((nb, 16, hkv, d), np.uint16)
    ovc = np.zeros_like(okc)
    table = pkv.rope_build_table(512, d).cuda()
    otab = oracle.rope_table(512, d)
    bt = torch.full((3, mb), -1, dtype=torch.int32, device="cuda")
    lens = [0, 0, 0]
    for step, new in enumerate(([37, 5, 140], [1, 1, 1], [1, 20, 1])):
        ctx = [L + n for L, n in zip(lens, new)]
        cu = torch.tensor(np.concatenate([[0], np.cumsum(new)]), dtype=torch.int32, device="cuda")
        ctx_t = torch.tensor(ctx, dtype=torch.int32, device="cuda")
        pkv.block_pool_alloc(pool, bt, cu, ctx_t)
        T = sum(new)
        slots = pkv.slot_mapping(bt, cu, ctx_t, T, nb)
        k = W._randn_bf16(g, T, hkv, d).cuda()
        v = W._randn_bf16(g, T, hkv, d).cuda()
        q = W._randn_bf16(g, T, hq, d).cuda()
        pkv.kv_store(k, v, kc, vc, slots, rope_cos_sin=table, cu_seqlens=cu, context_lens=ctx_t)
        pos = oracle.positions(cu.cpu().numpy(), np.array(ctx, np.int32))
        oracle.kv_store(W.bits(k.cpu()), W.bits(v.cpu()), okc, ovc, slots.cpu().numpy(), 16,
                        table=otab, pos=pos)
        out = pkv.paged_prefill_attention(q, kc, vc, cu, bt, ctx_t, max(new), rope_cos_sin=table)
        torch.cuda.synchronize()
        assert pkv.get_error() == 0
        assert np.array_equal(W.bits(kc.cpu()), okc) and np.array_equal(W.bits(vc.cpu()), ovc)
        ref = oracle.attention(W.bits(q.cpu()), okc, ovc, cu.cpu().numpy(), bt.cpu().numpy(),
                               np.array(ctx, np.int32), 1.0 / np.sqrt(d), 16, hkv, table=otab)
        err = np.abs(out.float().cpu().numpy() - ref)
        assert err.max() <= 1e-2 and err.mean() <= 1e-3
        lens = ctx
    used = int(sum(-(-L // 16) for L in lens))
    assert _pool_state(pool)[0] == nb - used
    held = bt.cpu().numpy()
    ids = torch.from_numpy(held[held >= 0].astype(np.int32)).cuda()
    assert ids.numel() == used and len(set(ids.tolist())) == used
    pkv.block_pool_free(pool, ids)
    assert pkv.get_error() == 0 and _pool_state(pool)[0] == nb
