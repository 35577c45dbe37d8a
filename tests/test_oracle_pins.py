"""Pins of the CPU oracle to facts the pages and the mathematics fix (no GPU needed).

Each test ties one oracle function to something other than itself: values printed on the
pages (tests/golden/), closed forms, invariants, exact rational arithmetic, brute force on
tiny inputs, or an independent library routine (torch's SDPA / float8 conversion)."""
import math
import os
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_447_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- sizes

def _golden_rows(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name), encoding="utf-8"):
        line = line.split("#", 1)[0].strip()
        if line:
            rows.append(line.split())
    return rows


def test_kv_sizes_match_printed_values():
    rows = _golden_rows("kv_sizes.txt")
    assert len(rows) >= 6
    for r in rows:
        layers, heads, dim, tokens, nbytes, expect = (int(x) for x in r)
        assert oracle.kv_cache_bytes(layers, heads, dim, tokens, nbytes) == expect


def test_kv_sizes_printed_approximations():
    # "LLM primer" §17.3: ~0.5 GB per 4096-token sequence, 16 GB for 32, 0.25 GB with 4 heads
    gib = 1 << 30
    assert oracle.kv_cache_bytes(32, 8, 128, 4096, 2) / gib == 0.5
    assert oracle.kv_cache_bytes(32, 8, 128, 32 * 4096, 2) / gib == 16.0
    assert oracle.kv_cache_bytes(32, 4, 128, 4096, 2) / gib == 0.25
    # "Inside the Nano-vLLM engine" §2.1: 262,144 B ~ 256 KB per token; ~25.6 MB per 100
    # tokens; ~256 MB for 10 such requests (FP8 reading of the formula, see kv_sizes.txt)
    per_tok = oracle.kv_cache_bytes(32, 32, 128, 1, 1)
    assert per_tok / 1024 == 256
    assert abs(100 * per_tok / 1e6 - 25.6) / 25.6 < 0.03
    assert abs(1000 * per_tok / 1e6 - 256) / 256 < 0.03
    # linear in every factor (a dropped or doubled term breaks one of these)
    base = oracle.kv_cache_bytes(3, 5, 7, 11, 2)
    assert oracle.kv_cache_bytes(6, 5, 7, 11, 2) == 2 * base
    assert oracle.kv_cache_bytes(3, 10, 7, 11, 2) == 2 * base
    assert oracle.kv_cache_bytes(3, 5, 14, 11, 2) == 2 * base
    assert oracle.kv_cache_bytes(3, 5, 7, 22, 2) == 2 * base
    assert oracle.kv_cache_bytes(3, 5, 7, 11, 1) * 2 == base


# ----------------------------------------------------------------------------- bf16

def _exact_bf16_rne(x: float) -> float:
    """Round the real value x to bf16 with exact rationals (ties to even)."""
    if x == 0:
        return x
    s = -1.0 if x < 0 else 1.0
    a = Fraction(abs(x))
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    # |x| = a * 2^e, a in [1, 2)
    q = max(e - 7, -133)
    n = Fraction(abs(x)) / Fraction(2) ** q
    fl = math.floor(n)
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    r = Fraction(fl) * Fraction(2) ** q
    if r >= Fraction(2) ** 128:
        return s * math.inf
    return s * float(r)


def test_bf16_rounding_exact_rationals():
    rng = random.Random(7)
    vals = []
    for _ in range(3000):
        vals.append(rng.uniform(-8, 8) * 2.0 ** rng.randint(-140, 120))
    # values within one binary32 ulp of a bf16 midpoint (the double-rounding trap)
    for _ in range(500):
        m = rng.randint(128, 255) + 0.5
        e = rng.randint(-120, 120)
        mid = m * 2.0 ** (e - 7)
        for eps in (2.0 ** -30, -2.0 ** -30, 0.0):
            vals.append(mid * (1 + eps))
    got = oracle.bf16_to_f64(oracle.bf16_from_f64(np.array(vals)))
    for v, gv in zip(vals, got):
        ev = _exact_bf16_rne(v)
        assert gv == ev or (math.isinf(ev) and math.isinf(gv)), (v, gv, ev)


def test_bf16_matches_torch_on_float32_inputs():
    # for inputs that are exactly binary32, torch's float32->bf16 cast is RNE
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(20000, generator=g) * torch.exp(torch.randn(20000, generator=g) * 8))
    ref = W.bits(x.to(torch.bfloat16))
    got = oracle.bf16_from_f64(x.double().numpy())
    assert np.array_equal(got, ref)


# ----------------------------------------------------------------------------- fp8

def test_e4m3_decode_all_codes_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2                            # S.1111.111 only
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.nanmax(ours) == 448.0 and np.nanmin(ours) == -448.0


def test_e4m3_encode_is_nearest_even_and_saturating():
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    finite = [(int(c), v) for c, v in zip(codes, vals) if not np.isnan(v)]
    # round trip on every finite code (the two zeros keep their sign)
    enc = oracle.e4m3_encode(np.array([v for _, v in finite]))
    for (c, v), e in zip(finite, enc):
        assert e == c or (v == 0 and (e & 0x7F) == 0)
    # brute force nearest over all codes, ties to the even code, on random inputs
    pos = sorted({v for _, v in finite if v >= 0})
    rng = np.random.default_rng(11)
    xs = np.concatenate([rng.uniform(-500, 500, 4000), rng.normal(0, 0.02, 2000),
                         [(a + b) / 2 for a, b in zip(pos[:-1], pos[1:])]])
    got = oracle.e4m3_decode(oracle.e4m3_encode(xs))
    for x, gv in zip(xs, got):
        a = min(abs(x), 448.0)
        best = min(pos, key=lambda p: (abs(p - a), 0))
        ties = [p for p in pos if abs(p - a) == abs(best - a)]
        if len(ties) > 1:  # exact midpoint: the code with an even mantissa wins
            best = [p for p in ties
                    if int(oracle.e4m3_encode(np.array([p]))[0]) % 2 == 0][0]
        assert abs(gv) == best and (gv == 0 or np.sign(gv) == np.sign(x)), (x, gv, best)
    # monotone
    sweep = np.linspace(-460, 460, 20001)
    dec = oracle.e4m3_decode(oracle.e4m3_encode(sweep))
    assert np.all(np.diff(dec) >= 0)
    # in-range agreement with torch's conversion
    inr = rng.uniform(-448, 448, 5000).astype(np.float32)
    ref = torch.from_numpy(inr).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(inr.astype(np.float64)), ref)


# ----------------------------------------------------------------------------- RoPE

def test_rope_table_closed_form():
    D, P = 64, 300
    tab = oracle.rope_table(P, D, 10000.0)
    p = np.arange(P, dtype=np.float64)[:, None]
    theta = 10000.0 ** (-(2.0 * np.arange(D // 2)) / D)
    cos_ref = np.cos(p * theta).astype(np.float32)
    sin_ref = np.sin(p * theta).astype(np.float32)
    ulp = np.spacing(np.abs(cos_ref)).astype(np.float64)
    assert np.all(np.abs(tab[:, :D // 2] - cos_ref) <= ulp)
    assert np.all(np.abs(tab[:, D // 2:] - sin_ref) <= np.spacing(np.abs(sin_ref)))
    assert np.all(tab[0, :D // 2] == 1.0) and np.all(tab[0, D // 2:] == 0.0)
    # pair 0 has theta = 1: angle = position in radians
    assert tab[5, 0] == np.float32(math.cos(5.0)) and tab[5, D // 2] == np.float32(math.sin(5.0))


def _rand_bits(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return W.bits(torch.randn(*shape, generator=g).to(torch.bfloat16))


def test_rope_position_zero_is_identity_and_norm_is_kept():
    D = 128
    tab = oracle.rope_table(4096, D)
    x = _rand_bits((50, 4, D), 1)
    assert np.array_equal(oracle.rope(x, np.zeros(50, np.int64), tab), x)
    pos = np.random.default_rng(2).integers(0, 4096, 50)
    y = oracle.bf16_to_f64(oracle.rope(x, pos, tab))
    xf = oracle.bf16_to_f64(x)
    n_in = xf[..., :D // 2] ** 2 + xf[..., D // 2:] ** 2
    n_out = y[..., :D // 2] ** 2 + y[..., D // 2:] ** 2
    # a rotation keeps each (i, i+D/2) pair's norm; bf16 output rounding bounds the change
    assert np.all(np.abs(np.sqrt(n_out) - np.sqrt(n_in)) <= 2 * 2.0 ** -8 * np.sqrt(n_in) + 1e-30)


def test_rope_quarter_turn_and_pairing():
    # pair 0 (theta=1) at position p rotates (x_0, x_{D/2}) by p radians; build x with a
    # single nonzero in slot 0 and check the closed form -- a swapped pairing (i, i+1) or
    # a sign flip lands the value in the wrong slot or with the wrong sign.
    D = 64
    tab = oracle.rope_table(64, D)
    x = np.zeros((1, 1, D), np.uint16)
    x[0, 0, 0] = W.bits(torch.tensor([1.0], dtype=torch.bfloat16))[0]
    for p in (1, 2, 7, 33):
        y = oracle.bf16_to_f64(oracle.rope(x, np.array([p]), tab))[0, 0]
        assert abs(y[0] - math.cos(p)) <= 2 ** -8 and abs(y[D // 2] - math.sin(p)) <= 2 ** -8
        assert np.count_nonzero(y) <= 2
    x[0, 0, 0] = 0
    x[0, 0, D // 2] = W.bits(torch.tensor([1.0], dtype=torch.bfloat16))[0]
    y = oracle.bf16_to_f64(oracle.rope(x, np.array([1]), tab))[0, 0]
    assert abs(y[0] + math.sin(1)) <= 2 ** -8 and abs(y[D // 2] - math.cos(1)) <= 2 ** -8


def test_rope_relative_position_property():
    # <R(p) q, R(p') k> depends only on p - p' (up to bf16 output rounding)
    D = 128
    tab = oracle.rope_table(2048, D)
    q = _rand_bits((1, 1, D), 3)
    k = _rand_bits((1, 1, D), 4)
    def dot(pq, pk):
        a = oracle.bf16_to_f64(oracle.rope(q, np.array([pq]), tab))
        b = oracle.bf16_to_f64(oracle.rope(k, np.array([pk]), tab))
        return float((a * b).sum())
    ref = dot(10, 3)
    for shift in (1, 100, 1500):
        assert abs(dot(10 + shift, 3 + shift) - ref) < 0.15


# ---- where new tokens sit when part of the sequence is cached

POS_EXAMPLE = dict(ctx=[20, 1, 32, 17, 41], new=[3, 1, 2, 17, 1])


def test_positions_hand_worked_example():
    """Positions of new tokens after a cached prefix (chunked prefill and decode rows),
    worked by hand in tests/golden/positions.txt."""
    rows = _golden_rows("positions.txt")
    cu = np.concatenate([[0], np.cumsum(POS_EXAMPLE["new"])]).astype(np.int32)
    got = oracle.positions(cu, np.array(POS_EXAMPLE["ctx"], np.int32))
    assert [int(x) for x in got] == [int(r[1]) for r in rows]


def test_rope_at_position_is_direct_rotation():
    """One vector rotated by the oracle at position p equals a direct fp64 cos/sin rotation
    by p * theta_i (within the bf16 output rounding), for p where p - 1 and p + 1 differ:
    a position off by one, or read from another row, fails."""
    D = 64
    tab = oracle.rope_table(512, D)
    x = _rand_bits((1, 1, D), 11)
    xf = oracle.bf16_to_f64(x)[0, 0]
    theta = 10000.0 ** (-(2.0 * np.arange(D // 2)) / D)
    for p in (1, 17, 36, 40, 300):
        y = oracle.bf16_to_f64(oracle.rope(x, np.array([p]), tab))[0, 0]
        c, s = np.cos(p * theta), np.sin(p * theta)
        ref = np.concatenate([xf[:D // 2] * c - xf[D // 2:] * s, xf[D // 2:] * c + xf[:D // 2] * s])
        tol = 2.0 ** -8 * np.abs(ref) + 1e-6
        assert np.all(np.abs(y - ref) <= tol), p
        for wrong in (p - 1, p + 1):
            yw = oracle.bf16_to_f64(oracle.rope(x, np.array([wrong]), tab))[0, 0]
            assert np.any(np.abs(yw - ref) > tol)


def _mixed_batch(seed, lens_new, lens_ctx, hq=4, hkv=2, d=64, nb=16):
    """Random bf16 caches, a permuted block table per sequence and q for the new tokens."""
    g = torch.Generator().manual_seed(seed)
    kc = W.bits(torch.randn(nb, 16, hkv, d, generator=g).to(torch.bfloat16)).copy()
    vc = W.bits(torch.randn(nb, 16, hkv, d, generator=g).to(torch.bfloat16)).copy()
    perm = torch.randperm(nb, generator=g).numpy()
    bt = np.full((len(lens_ctx), nb), -1, np.int32)
    used = 0
    for b, L in enumerate(lens_ctx):
        k = W.blocks_needed(L)
        bt[b, :k] = perm[used:used + k]
        used += k
    cu = np.concatenate([[0], np.cumsum(lens_new)]).astype(np.int32)
    q = W.bits(torch.randn(int(cu[-1]), hq, d, generator=g).to(torch.bfloat16))
    return kc, vc, bt, cu, np.array(lens_ctx, np.int32), q


def test_attention_rotates_q_at_cached_offset():
    """attention(table=...) on a decode row (L = 37) and on a 5-token chunk after 35 cached
    tokens equals attention on q rotated beforehand at positions written out by hand
    (36; then 35 .. 39).  The slips a position rule can make (the row's index inside the
    chunk, or one off either way) give outputs far outside rounding."""
    kc, vc, bt, cu, cl, q = _mixed_batch(21, [1, 5], [37, 40])
    tab = oracle.rope_table(64, 64)
    scale = 0.125
    args = (kc, vc, cu, bt, cl, scale, 16, 2)
    got = oracle.attention(q, *args, table=tab)
    by_hand = np.array([36, 35, 36, 37, 38, 39])
    ref = oracle.attention(oracle.rope(q, by_hand, tab), *args)
    assert np.array_equal(got, ref)
    for wrong in (np.array([0, 0, 1, 2, 3, 4]), by_hand - 1, by_hand + 1):
        alt = oracle.attention(oracle.rope(q, wrong, tab), *args)
        assert np.max(np.abs(alt - ref)) > 1e-2


def _prefix_then_chunk(q, k, v, P, n, nb, tab, pos_rule):
    """Store a P-token prefix, then an n-token chunk, into empty caches (K rotated on the
    way in), then attend with the chunk's queries.  pos_rule None: the oracle's own
    positions/slot rules drive both calls and q is rotated by attention(table=...);
    otherwise pos_rule is the explicit position array of all P + n tokens, slots are
    enumerated from the table and q is rotated beforehand at pos_rule[P:]."""
    hkv, d = k.shape[1], k.shape[2]
    kc = np.zeros((nb, 16, hkv, d), np.uint16)
    vc = np.zeros_like(kc)
    bt = np.arange(nb, dtype=np.int32)[::-1].copy()[None, :]   # blocks in reverse order
    L = P + n
    if pos_rule is None:
        for lo, hi in ((0, P), (P, L)):
            cu = np.array([0, hi - lo], np.int32)
            cl = np.array([hi], np.int32)
            slots = oracle.slot_mapping(bt, cu, cl, 16, nb)
            oracle.kv_store(k[lo:hi], v[lo:hi], kc, vc, slots, 16, table=tab,
                            pos=oracle.positions(cu, cl))
        return oracle.attention(q, kc, vc, np.array([0, n], np.int32), bt,
                                np.array([L], np.int32), 0.125, 16, hkv, table=tab)
    slots = np.array([bt[0, j // 16] * 16 + j % 16 for j in range(L)], np.int32)
    oracle.kv_store(k, v, kc, vc, slots, 16, table=tab, pos=pos_rule)
    return oracle.attention(oracle.rope(q, pos_rule[P:], tab), kc, vc,
                            np.array([0, n], np.int32), bt, np.array([L], np.int32), 0.125, 16,
                            hkv)


def test_prefix_and_chunk_positions_are_relative():
    """RoPE makes attention depend on q and k positions only through their difference.
    A 21-token prefix stored by one call and a 7-token chunk by the next, attended through
    the oracle's own position rule, equals the same tokens placed explicitly at 0..27 (bit
    for bit) and at s..s+27 for shifts s (within bf16 rounding of the rotated values).  A
    rule that placed the chunk at its local indices 0..6 is far off."""
    g = torch.Generator().manual_seed(23)
    P, n, hq, hkv, d = 21, 7, 4, 2, 64
    k = W.bits(torch.randn(P + n, hkv, d, generator=g).to(torch.bfloat16))
    v = W.bits(torch.randn(P + n, hkv, d, generator=g).to(torch.bfloat16))
    q = W.bits(torch.randn(n, hq, d, generator=g).to(torch.bfloat16))
    tab = oracle.rope_table(4096, d)
    got = _prefix_then_chunk(q, k, v, P, n, 4, tab, None)
    explicit = np.arange(P + n)
    assert np.array_equal(got, _prefix_then_chunk(q, k, v, P, n, 4, tab, explicit))
    for s in (1, 100, 3000):
        shifted = _prefix_then_chunk(q, k, v, P, n, 4, tab, explicit + s)
        assert np.max(np.abs(shifted - got)) < 2e-2, s
    local = np.concatenate([np.arange(P), np.arange(n)])
    assert np.max(np.abs(_prefix_then_chunk(q, k, v, P, n, 4, tab, local) - got)) > 5e-2
    one_short = explicit.copy()
    one_short[P:] -= 1
    assert np.max(np.abs(_prefix_then_chunk(q, k, v, P, n, 4, tab, one_short) - got)) > 5e-2


# ----------------------------------------------------------------------------- store

def test_kv_store_round_trip_and_padding():
    wl = W.tiny(seed=1)
    st = wl.steps[0]
    kc = W.bits(wl.k_cache).copy()
    vc = W.bits(wl.v_cache).copy()
    before_k, before_v = kc.copy(), vc.copy()
    sm = st.slot_mapping.numpy().copy()
    sm[3] = -1                                           # a padding token writes nothing
    oracle.kv_store(W.bits(st.k), W.bits(st.v), kc, vc, sm, 16)
    flat_k = kc.reshape(-1, wl.n_kv_heads, wl.head_dim)
    flat_v = vc.reshape(-1, wl.n_kv_heads, wl.head_dim)
    for t, s in enumerate(sm):
        if s >= 0:
            assert np.array_equal(flat_k[s], W.bits(st.k)[t])
            assert np.array_equal(flat_v[s], W.bits(st.v)[t])
    touched = np.zeros(flat_k.shape[0], bool)
    touched[sm[sm >= 0]] = True
    assert np.array_equal(flat_k[~touched], before_k.reshape(flat_k.shape)[~touched])
    assert np.array_equal(flat_v[~touched], before_v.reshape(flat_v.shape)[~touched])
    # the slot of token 3 was left alone
    s3 = int(st.slot_mapping[3])
    assert np.array_equal(flat_k[s3], before_k.reshape(flat_k.shape)[s3])


def test_kv_store_rope_equals_rotate_then_store():
    wl = W.tiny(seed=1)
    st = wl.steps[0]
    tab = oracle.rope_table(wl.max_pos, wl.head_dim)
    pos = oracle.positions(st.cu_seqlens.numpy(), st.context_lens.numpy())
    assert np.array_equal(pos, np.concatenate([np.arange(n) for n in (5, 17, 33, 60)]))
    kc1 = W.bits(wl.k_cache).copy(); vc1 = W.bits(wl.v_cache).copy()
    oracle.kv_store(W.bits(st.k), W.bits(st.v), kc1, vc1, st.slot_mapping.numpy(), 16,
                    table=tab, pos=pos)
    kc2 = W.bits(wl.k_cache).copy(); vc2 = W.bits(wl.v_cache).copy()
    krot = oracle.rope(W.bits(st.k), pos, tab)
    oracle.kv_store(krot, W.bits(st.v), kc2, vc2, st.slot_mapping.numpy(), 16)
    assert np.array_equal(kc1, kc2) and np.array_equal(vc1, vc2)


def test_kv_store_fp8_codes_are_nearest():
    wl = W.mix(seed=5, decodes=8, chunks=1, chunk_len=16, fp8=True, max_context=256)
    st = wl.steps[0]
    kc = W.bits(wl.k_cache).copy(); vc = W.bits(wl.v_cache).copy()
    oracle.kv_store(W.bits(st.k), W.bits(st.v), kc, vc, st.slot_mapping.numpy(), 16, fp8=True,
                    k_scale=wl.k_scale.numpy(), v_scale=wl.v_scale.numpy())
    flat = kc.reshape(-1, wl.n_kv_heads, wl.head_dim)
    allv = oracle.e4m3_decode(np.arange(127, dtype=np.uint8))
    kf = oracle.bf16_to_f64(W.bits(st.k))
    for t, s in enumerate(st.slot_mapping.numpy()[:6]):
        for h in range(wl.n_kv_heads):
            target = kf[t, h] / float(wl.k_scale[h])
            got = oracle.e4m3_decode(flat[s, h])
            err = np.abs(np.abs(got) - np.minimum(np.abs(target), 448))
            best = np.min(np.abs(allv[None, :] - np.minimum(np.abs(target), 448)[:, None]), axis=1)
            assert np.all(err <= best + 1e-12)


# ----------------------------------------------------------------------------- attention

def _single_seq_cache(k_rows, v_rows, hkv, d, nb=4, perm=None):
    """Cache + block table holding k_rows/v_rows [L, hkv, d] (bf16 bits) for one sequence."""
    L = k_rows.shape[0]
    nblk = W.blocks_needed(L)
    perm = list(range(nb)) if perm is None else perm
    kc = np.zeros((nb, 16, hkv, d), np.uint16)
    vc = np.zeros((nb, 16, hkv, d), np.uint16)
    bt = np.full((1, nb), -1, np.int32)
    bt[0, :nblk] = perm[:nblk]
    slots = np.array([bt[0, j // 16] * 16 + j % 16 for j in range(L)], np.int32)
    oracle.kv_store(k_rows, v_rows, kc, vc, slots, 16)
    return kc, vc, bt


def test_worked_example_i_eat_fish():
    rows = _golden_rows("worked_example.txt")
    d = 64
    bf = lambda a: W.bits(torch.tensor(a, dtype=torch.float32).to(torch.bfloat16))
    # logits s(I) - s(eat) = ln(0.60/0.40) = ln 1.5, made with bf16 inputs:
    # q = [1, 0, ...], k(I) = [c, ...], k(eat) = 0, scale 1 -> s = (c, 0)
    q = np.zeros((3, 1, d), np.float32); q[:, 0, 0] = 1.0
    k = np.zeros((3, 1, d), np.float32); k[0, 0, 0] = math.log(1.5); k[2, 0, 0] = 3.0
    v = np.random.default_rng(0).normal(size=(3, 1, d)).astype(np.float32)
    kc, vc, bt = _single_seq_cache(bf(k), bf(v), 1, d)
    cu = np.array([0, 3], np.int32); cl = np.array([3], np.int32)
    w = oracle.attention_weights(bf(q), kc, cu, bt, cl, 1.0, 16, 1,
                                 rows=np.array([[1, 0]]), lmax=3)[0]
    for _, j, pw in rows:
        assert abs(w[int(j)] - float(pw)) < 5e-3
    assert w[2] == 0.0                                   # masked exactly
    o = oracle.attention(bf(q), kc, vc, cu, bt, cl, 1.0, 16, 1)[1, 0]
    vv = oracle.bf16_to_f64(bf(v))[:, 0]
    assert np.allclose(o, 0.6 * vv[0] + 0.4 * vv[1], atol=5e-3 * np.abs(vv).max())
    assert np.allclose(o, w[0] * vv[0] + w[1] * vv[1], atol=1e-12)


def _sdpa_reference(wl, st, table=None, kv=None):
    """torch's CPU SDPA (fp64) on K/V gathered with numpy fancy indexing and an explicit
    boolean bottom-right causal mask -- an independent statement of the definition.
    kv: optional fp64 caches [NB, 16, Hkv, D] (default: the workload's bf16 caches)."""
    q = oracle.bf16_to_f64(W.bits(st.q))
    if table is not None:
        pos = oracle.positions(st.cu_seqlens.numpy(), st.context_lens.numpy())
        q = oracle.bf16_to_f64(oracle.rope(W.bits(st.q), pos, table))
    if kv is None:
        kv = (oracle.bf16_to_f64(W.bits(wl.k_cache)), oracle.bf16_to_f64(W.bits(wl.v_cache)))
    kc = kv[0].reshape(-1, wl.n_kv_heads, wl.head_dim)
    vc = kv[1].reshape(-1, wl.n_kv_heads, wl.head_dim)
    G = wl.n_q_heads // wl.n_kv_heads
    out = np.zeros_like(q)
    for b in range(st.num_seqs):
        a, e = int(st.cu_seqlens[b]), int(st.cu_seqlens[b + 1])
        L = int(st.context_lens[b]); n = e - a
        j = np.arange(L)
        slots = st.block_tables[b].numpy()[j // 16] * 16 + j % 16
        K = torch.from_numpy(kc[slots]).permute(1, 0, 2).repeat_interleave(G, 0)
        V = torch.from_numpy(vc[slots]).permute(1, 0, 2).repeat_interleave(G, 0)
        Q = torch.from_numpy(q[a:e]).permute(1, 0, 2)
        mask = torch.from_numpy((j[None, :] <= (L - n + np.arange(n))[:, None]))
        o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask,
                                                             scale=wl.scale)
        out[a:e] = o.permute(1, 0, 2).numpy()
    return out


@pytest.mark.parametrize("which", ["prefill", "decode"])
def test_attention_matches_torch_sdpa(which):
    wl = W.tiny(seed=1)
    kc = W.bits(wl.k_cache).copy(); vc = W.bits(wl.v_cache).copy()
    pre, dec = wl.steps
    oracle.kv_store(W.bits(pre.k), W.bits(pre.v), kc, vc, pre.slot_mapping.numpy(), 16)
    st = pre
    if which == "decode":
        oracle.kv_store(W.bits(dec.k), W.bits(dec.v), kc, vc, dec.slot_mapping.numpy(), 16)
        st = dec
    wl2 = W.Workload(wl.name, wl.seed, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.num_blocks,
                     "bf16", torch.from_numpy(kc.view(np.int16)).view(torch.bfloat16),
                     torch.from_numpy(vc.view(np.int16)).view(torch.bfloat16), [st],
                     max_pos=wl.max_pos)
    tab = oracle.rope_table(wl.max_pos, wl.head_dim)
    for table in (None, tab):
        got = oracle.attention(W.bits(st.q), kc, vc, st.cu_seqlens.numpy(),
                               st.block_tables.numpy(), st.context_lens.numpy(), wl.scale, 16,
                               wl.n_kv_heads, table=table)
        ref = _sdpa_reference(wl2, st, table)
        assert np.max(np.abs(got - ref)) < 1e-12


def test_fp8_attention_matches_sdpa_on_torch_dequantised_cache():
    """E4M3 caches: the oracle's attention (its own code decoder, times the head's scale)
    equals SDPA on the cache dequantised by torch's float8_e4m3fn with the same scales."""
    wl = W.mix(seed=5, decodes=6, chunks=1, chunk_len=24, fp8=True, max_context=300)
    st = wl.steps[0]
    kc = W.bits(wl.k_cache).copy()
    vc = W.bits(wl.v_cache).copy()
    ks, vs = wl.k_scale.double(), wl.v_scale.double()

    def deq(codes, scale):
        x = torch.from_numpy(codes).view(torch.float8_e4m3fn).double()
        return (x * scale.view(1, 1, -1, 1)).numpy()

    kv = (deq(kc, ks), deq(vc, vs))
    got = oracle.attention(W.bits(st.q), kc, vc, st.cu_seqlens.numpy(), st.block_tables.numpy(),
                           st.context_lens.numpy(), wl.scale, 16, wl.n_kv_heads, fp8=True,
                           k_scale=wl.k_scale.numpy(), v_scale=wl.v_scale.numpy())
    ref = _sdpa_reference(wl, st, None, kv)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_context_len_one_returns_v_and_rows_sum_to_one():
    d, hkv = 64, 2
    g = torch.Generator().manual_seed(9)
    k = W.bits(torch.randn(40, hkv, d, generator=g).to(torch.bfloat16))
    v = W.bits(torch.randn(40, hkv, d, generator=g).to(torch.bfloat16))
    q = W.bits(torch.randn(1, 4, d, generator=g).to(torch.bfloat16))
    kc, vc, bt = _single_seq_cache(k, v, hkv, d, nb=4, perm=[2, 0, 3, 1])
    o = oracle.attention(q, kc, vc, np.array([0, 1]), bt, np.array([1]), 0.125, 16, hkv)
    for h in range(4):
        assert np.array_equal(o[0, h], oracle.bf16_to_f64(v[0, h // 2]))
    w = oracle.attention_weights(q, kc, np.array([0, 1]), bt, np.array([40]), 0.125, 16, hkv,
                                 rows=np.array([[0, h] for h in range(4)]), lmax=40)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-14) and np.all(w >= 0)


def test_max_subtraction_keeps_huge_logits_finite():
    d, hkv = 64, 1
    g = torch.Generator().manual_seed(4)
    k = W.bits((torch.randn(20, hkv, d, generator=g) * 100).to(torch.bfloat16))
    v = W.bits(torch.randn(20, hkv, d, generator=g).to(torch.bfloat16))
    q = W.bits((torch.randn(1, 1, d, generator=g) * 1e4).to(torch.bfloat16))
    kc, vc, bt = _single_seq_cache(k, v, hkv, d)
    o = oracle.attention(q, kc, vc, np.array([0, 1]), bt, np.array([20]), 1.0, 16, hkv)
    assert np.all(np.isfinite(o))
    # with logits this far apart the softmax is one-hot on the largest score
    s = oracle.bf16_to_f64(k)[:, 0] @ oracle.bf16_to_f64(q)[0, 0]
    assert np.array_equal(o[0, 0], oracle.bf16_to_f64(v)[int(np.argmax(s)), 0])


def test_block_permutation_invariance():
    wl = W.tiny(seed=1)
    pre = wl.steps[0]
    kc = W.bits(wl.k_cache).copy(); vc = W.bits(wl.v_cache).copy()
    oracle.kv_store(W.bits(pre.k), W.bits(pre.v), kc, vc, pre.slot_mapping.numpy(), 16)
    args = (pre.cu_seqlens.numpy(), pre.block_tables.numpy(), pre.context_lens.numpy(),
            wl.scale, 16, wl.n_kv_heads)
    ref = oracle.attention(W.bits(pre.q), kc, vc, *args)
    perm = np.random.default_rng(5).permutation(wl.num_blocks)   # new id of block i
    kc2 = np.empty_like(kc); vc2 = np.empty_like(vc)
    kc2[perm] = kc; vc2[perm] = vc
    bt2 = pre.block_tables.numpy().copy()
    bt2[bt2 >= 0] = perm[bt2[bt2 >= 0]]
    got = oracle.attention(W.bits(pre.q), kc2, vc2, args[0], bt2, *args[2:])
    assert np.array_equal(got, ref)


def test_shared_prefix_aliasing_equals_copies():
    wl = W.shared_prefix(seed=4, requests=3, prefix=32, new=20, hq=4, hkv=2, d=64)
    st = wl.steps[0]
    kc = W.bits(wl.k_cache).copy(); vc = W.bits(wl.v_cache).copy()
    oracle.kv_store(W.bits(st.k), W.bits(st.v), kc, vc, st.slot_mapping.numpy(), 16)
    bt = st.block_tables.numpy()
    assert np.all(bt[:, :2] == bt[0, :2])                    # the prefix is aliased
    args = (st.cu_seqlens.numpy(), st.context_lens.numpy())
    ref = oracle.attention(W.bits(st.q), kc, vc, args[0], bt, args[1], wl.scale, 16, 2)
    # un-share: give every request its own copy of the prefix blocks
    nb = wl.num_blocks
    kc2 = np.concatenate([kc, np.zeros((2 * 3,) + kc.shape[1:], kc.dtype)])
    vc2 = np.concatenate([vc, np.zeros((2 * 3,) + vc.shape[1:], vc.dtype)])
    bt2 = bt.copy()
    for r in range(3):
        for i in range(2):
            new_id = nb + 2 * r + i
            kc2[new_id] = kc[bt[r, i]]; vc2[new_id] = vc[bt[r, i]]
            bt2[r, i] = new_id
    got = oracle.attention(W.bits(st.q), kc2, vc2, args[0], bt2, args[1], wl.scale, 16, 2)
    assert np.array_equal(got, ref)


def test_padding_and_unused_slots_never_reach_output():
    wl = W.tiny(seed=1, nan_fill=True)
    pre = wl.steps[0]
    kc = W.bits(wl.k_cache).copy(); vc = W.bits(wl.v_cache).copy()
    oracle.kv_store(W.bits(pre.k), W.bits(pre.v), kc, vc, pre.slot_mapping.numpy(), 16)
    o = oracle.attention(W.bits(pre.q), kc, vc, pre.cu_seqlens.numpy(),
                         pre.block_tables.numpy(), pre.context_lens.numpy(), wl.scale, 16, 2)
    assert np.all(np.isfinite(o))
    # an empty context gives a zero row
    o0 = oracle.attention(W.bits(pre.q[:1]), kc, vc, np.array([0, 1]), pre.block_tables.numpy()[:1],
                          np.array([0]), wl.scale, 16, 2)
    assert np.all(o0 == 0)


def test_batch_independence():
    """A continuous-batching mix gives, row for row, what each sequence gives alone."""
    wl = W.mix(seed=5, decodes=6, chunks=2, chunk_len=24, max_context=300)
    st = wl.steps[0]
    kc = W.bits(wl.k_cache).copy(); vc = W.bits(wl.v_cache).copy()
    oracle.kv_store(W.bits(st.k), W.bits(st.v), kc, vc, st.slot_mapping.numpy(), 16)
    full = oracle.attention(W.bits(st.q), kc, vc, st.cu_seqlens.numpy(),
                            st.block_tables.numpy(), st.context_lens.numpy(), wl.scale, 16, 8)
    for b in (0, 5, 6, 7):
        sub = W.sub_step(st, [b])
        alone = oracle.attention(W.bits(sub.q), kc, vc, sub.cu_seqlens.numpy(),
                                 sub.block_tables.numpy(), sub.context_lens.numpy(), wl.scale,
                                 16, 8)
        a, e = int(st.cu_seqlens[b]), int(st.cu_seqlens[b + 1])
        assert np.array_equal(alone, full[a:e])


def test_planted_mistakes_are_caught():
    """Sanity of the pins themselves: perturb the oracle's output the way plausible bugs
    would and check the SDPA pin notices."""
    wl = W.tiny(seed=1)
    pre = wl.steps[0]
    kc = W.bits(wl.k_cache).copy(); vc = W.bits(wl.v_cache).copy()
    oracle.kv_store(W.bits(pre.k), W.bits(pre.v), kc, vc, pre.slot_mapping.numpy(), 16)
    wl2 = W.Workload(wl.name, wl.seed, 4, 2, 64, wl.num_blocks, "bf16",
                     torch.from_numpy(kc.view(np.int16)).view(torch.bfloat16),
                     torch.from_numpy(vc.view(np.int16)).view(torch.bfloat16), [pre], max_pos=61)
    ref = _sdpa_reference(wl2, pre)
    good = oracle.attention(W.bits(pre.q), kc, vc, pre.cu_seqlens.numpy(),
                            pre.block_tables.numpy(), pre.context_lens.numpy(), wl.scale, 16, 2)
    assert np.max(np.abs(good - ref)) < 1e-12
    # wrong GQA mapping (h % Hkv instead of h / G)
    bt = pre.block_tables.numpy()
    swapped = oracle.attention(W.bits(pre.q)[:, [0, 2, 1, 3]], kc, vc, pre.cu_seqlens.numpy(),
                               bt, pre.context_lens.numpy(), wl.scale, 16, 2)[:, [0, 2, 1, 3]]
    assert np.max(np.abs(swapped - ref)) > 1e-3
    # off-by-one causal alignment (context one short)
    short = oracle.attention(W.bits(pre.q), kc, vc, pre.cu_seqlens.numpy(), bt,
                             pre.context_lens.numpy() - 1, wl.scale, 16, 2)
    assert np.max(np.abs(short - ref)) > 1e-3


# ----------------------------------------------------------------------------- block bookkeeping

SLOT_EXAMPLE = dict(tables=[[7, 2, 9], [5, -1, -1], [4, 0, -1], [6, 3, -1]],
                    ctx=[20, 1, 32, 17], new=[3, 1, 2, 17])


def _cu(new):
    return np.concatenate([[0], np.cumsum(new)]).astype(np.int32)


def test_slot_mapping_hand_worked_example():
    rows = _golden_rows("slot_mapping.txt")
    got = oracle.slot_mapping(np.array(SLOT_EXAMPLE["tables"], np.int32), _cu(SLOT_EXAMPLE["new"]),
                              np.array(SLOT_EXAMPLE["ctx"], np.int32), 16, 10)
    assert [int(x) for x in got] == [int(r[1]) for r in rows]


def test_slot_mapping_brute_force_enumeration():
    """Enumerate each sequence's slots block by block in table order (the p-th entry is
    the slot of position p) and take the last n_b: no division or modulo involved."""
    g = np.random.default_rng(5)
    bs, nb = 16, 64
    for _ in range(30):
        B = int(g.integers(1, 6))
        lens = g.integers(1, 120, B)
        new = [int(g.integers(1, L + 1)) for L in lens]
        maxb = int((lens.max() + bs - 1) // bs) + 1
        perm = g.permutation(nb)
        tables = np.full((B, maxb), -1, np.int32)
        cur = 0
        for b in range(B):
            k = int((lens[b] + bs - 1) // bs)
            tables[b, :k] = perm[cur:cur + k]
            cur += k
        got = oracle.slot_mapping(tables, _cu(new), lens.astype(np.int32), bs, nb)
        exp = []
        for b in range(B):
            enum = [int(blk) * bs + o for blk in tables[b] if blk >= 0 for o in range(bs)]
            exp += enum[int(lens[b]) - new[b]:int(lens[b])]
        assert got.tolist() == exp


def test_slot_mapping_out_of_table_is_minus_one():
    bt = np.array([[3, -1]], np.int32)
    assert oracle.slot_mapping(bt, [0, 1], [17], 16, 8).tolist() == [-1]   # entry -1
    assert oracle.slot_mapping(bt, [0, 1], [33], 16, 8).tolist() == [-1]   # past the table
    assert oracle.slot_mapping(np.array([[9]], np.int32), [0, 1], [1], 16, 8).tolist() == [-1]
    assert oracle.slot_mapping(bt, [0, 2], [1], 16, 8).tolist() == [-1, 48]  # position -1, 0


def test_copy_blocks_copies_whole_blocks_only():
    g = np.random.default_rng(7)
    for dtype, hi in ((np.uint16, 2 ** 16), (np.uint8, 256)):
        kc = g.integers(0, hi, size=(12, 16, 2, 64)).astype(dtype)
        vc = g.integers(0, hi, size=(12, 16, 2, 64)).astype(dtype)
        k0, v0 = kc.copy(), vc.copy()
        oracle.copy_blocks(kc, vc, [(3, 7), (0, 11), (5, 5), (2, 99), (-1, 4)])
        ek, ev = k0.copy(), v0.copy()
        ek[7], ev[7] = k0[3], v0[3]
        ek[11], ev[11] = k0[0], v0[0]
        assert np.array_equal(kc, ek) and np.array_equal(vc, ev)


def test_copy_on_write_divergence_equals_private_copy():
    """Two sequences share the blocks of a 24-token prefix (the second block half full).
    Before either appends, sequence 1 takes a private copy of the shared partial block
    (copy on write) and points its table there; then each stores its own next token through
    its slots.  Attention for both must equal the result on fully private caches, and the
    shared full block must be untouched."""
    g = torch.Generator().manual_seed(11)
    hq, hkv, d, bs, nb = 4, 2, 64, 16, 8
    prefix = W._randn_bf16(g, 24, hkv, d), W._randn_bf16(g, 24, hkv, d)
    tails = [(W._randn_bf16(g, 1, hkv, d), W._randn_bf16(g, 1, hkv, d)) for _ in range(2)]
    q = W._randn_bf16(g, 2, hq, d)

    def store(kc, vc, bt, b, ctx, rows):
        slots = oracle.slot_mapping(bt[b:b + 1], [0, rows[0].shape[0]], [ctx], bs, nb)
        oracle.kv_store(W.bits(rows[0]), W.bits(rows[1]), kc, vc, slots, bs)

    kc = np.zeros((nb, bs, hkv, d), np.uint16)
    vc = np.zeros((nb, bs, hkv, d), np.uint16)
    shared = np.array([[0, 1, -1], [0, 1, -1]], np.int32)
    store(kc, vc, shared, 0, 24, prefix)                 # the prefix, once, in blocks 0-1
    before = kc[0].copy()
    oracle.copy_blocks(kc, vc, [(1, 5)])                 # copy on write for sequence 1
    bt = np.array([[0, 1, -1], [0, 5, -1]], np.int32)
    for b in range(2):
        store(kc, vc, bt, b, 25, tails[b])
    kp = np.zeros_like(kc)
    vp = np.zeros_like(vc)
    private = np.array([[0, 1, -1], [2, 3, -1]], np.int32)
    for b in range(2):
        store(kp, vp, private, b, 24, prefix)
        store(kp, vp, private, b, 25, tails[b])
    cu = np.array([0, 1, 2], np.int32)
    ctx = np.array([25, 25], np.int32)
    got = oracle.attention(W.bits(q), kc, vc, cu, bt, ctx, d ** -0.5, bs, hkv)
    ref = oracle.attention(W.bits(q), kp, vp, cu, private, ctx, d ** -0.5, bs, hkv)
    assert np.array_equal(got, ref)
    assert np.array_equal(kc[0], before)


# ----------------------------------------------------------------------------- block pool

def test_block_pool_hand_worked_sequence():
    """tests/golden/block_pool.txt: allocations in sequence order from the top of the free
    stack, nothing taken for tokens that fit the blocks held, LIFO reuse of freed blocks, a
    request the pool cannot cover refused whole, double and out-of-range frees rejected."""
    pool = oracle.pool_init(8)
    tables = {}
    steps = {}
    for r in _golden_rows("block_pool.txt"):
        steps.setdefault(r[0], []).append(r)
    for step in sorted(steps, key=int):
        rows = steps[step]
        if rows[0][1] == "free":
            r = rows[0]
            arrow = r.index("->")
            ids = [int(x) for x in r[2:arrow]]
            rej = oracle.pool_free(pool, ids)
            tail = r[arrow + 1:]
            assert int(pool[0]) == int(tail[tail.index(";") + 1])
            assert rej == int(tail[-1])
            continue
        names = [r[2] for r in rows]
        bt = np.full((len(rows), 8), -1, np.int32)
        for i, name in enumerate(names):
            held = tables.get(name, [])
            bt[i, :len(held)] = held
        ctx = np.array([int(r[3]) for r in rows], np.int32)
        cu = np.concatenate([[0], np.cumsum([int(r[4]) for r in rows])]).astype(np.int32)
        rc = oracle.pool_alloc(pool, bt, cu, ctx)
        for i, r in enumerate(rows):
            arrow = r.index("->")
            semi = r.index(";")
            want = r[arrow + 1:semi]
            if want == ["refused"]:
                assert rc == -1
            else:
                assert rc == 0
                got = [int(x) for x in bt[i] if x >= 0]
                assert got == [int(x) for x in want], (r, got)
                tables[names[i]] = got
            assert int(pool[0]) == int(r[semi + 1])


def test_block_pool_invariants_under_random_traffic():
    """Random admissions, growth and completions against a model kept with Python sets:
    no block is ever held by two sequences or held and free at once, every held-or-free id
    is accounted for, every sequence's table covers exactly ceil(L / 16) blocks, and a
    refused request changes nothing."""
    rng = np.random.default_rng(7)
    nb = 64
    pool = oracle.pool_init(nb)
    live = {}          # seq -> (L, table list)
    next_id = 0
    for _ in range(400):
        if live and rng.random() < 0.3:
            s = int(rng.choice(list(live)))
            _, table = live.pop(s)
            assert oracle.pool_free(pool, table) == 0
        else:
            batch = []
            for s in list(live)[:3]:
                batch.append((s, int(rng.integers(1, 40))))
            if rng.random() < 0.6:
                batch.append((next_id, int(rng.integers(1, 90))))
                next_id += 1
            if not batch:
                continue
            bt = np.full((len(batch), 32), -1, np.int32)
            ctx, new = [], []
            for i, (s, n) in enumerate(batch):
                L0, table = live.get(s, (0, []))
                bt[i, :len(table)] = table
                ctx.append(L0 + n)
                new.append(n)
            before = pool.copy()
            cu = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
            rc = oracle.pool_alloc(pool, bt, cu, np.array(ctx, np.int32))
            need = sum(-(-c // 16) - (-(-(c - n) // 16)) for c, n in zip(ctx, new))
            if rc != 0:
                assert need > int(before[0]) or max(-(-c // 16) for c in ctx) > 32
                assert np.array_equal(pool, before)
                continue
            for i, (s, n) in enumerate(batch):
                table = [int(x) for x in bt[i] if x >= 0]
                assert len(table) == -(-ctx[i] // 16)
                live[s] = (ctx[i], table)
        held = [x for _, t in live.values() for x in t]
        free = [int(x) for x in pool[1:1 + int(pool[0])]]
        assert len(set(held)) == len(held) and len(set(free)) == len(free)
        assert not set(held) & set(free) and len(held) + len(free) == nb
        flags = pool[1 + nb:]
        assert all(flags[x] == 1 for x in free) and all(flags[x] == 0 for x in held)
