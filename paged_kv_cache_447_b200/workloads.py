"""Seeded synthetic workloads for the paged KV-cache data plane.

This module only draws inputs: random bf16 tensors, block assignments, slot mappings,
sequence lengths and per-head FP8 scales.  It holds none of the method's arithmetic and
imports neither the CUDA binding nor the oracle, so both sides can take the same inputs
from it.  Everything is generated on the CPU with ``torch.Generator`` (one seed per
workload) and returned as CPU tensors.

Workload shapes (one function each):

* ``tiny``            4 sequences with prompts {5, 17, 33, 60}, 4 q / 2 kv heads, head_dim
                      64, 32 physical blocks in a seeded random order; a prefill step of
                      every prompt token followed by one decode step.
* ``qwen_decode``     Qwen-7B-style MHA decode: batch 64, 32 q = 32 kv heads, head_dim 128,
                      context lengths uniform in [128, 2048].
* ``gqa_decode``      Mistral-7B-style GQA decode: batch 32, 32 q / 8 kv heads, head_dim 128,
                      every sequence 4096 cached tokens, one cache per layer.
* ``shared_prefix``   32 requests whose block tables alias one 2048-token prefix, each with
                      2048 new tokens to prefill; 32 q / 8 kv heads, head_dim 128.
* ``mix``             continuous-batching step: 256 decodes with lognormal context lengths
                      (median 1024, sigma 1, clipped to [1, 32768]) plus 4 chunked prefills
                      of 512 tokens after a prior context from the same law; bf16 or FP8.

Block-size 16, RoPE base 10000 and scale 1/sqrt(head_dim) everywhere.  Values ~ N(0, 1).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

BLOCK_SIZE = 16
ROPE_BASE = 10000.0
FP8_MAX = 448.0


@dataclass
class Step:
    """One call's worth of inputs.  Token rows are grouped by ``cu_seqlens``."""
    name: str
    q: torch.Tensor              # [T, Hq, D] bf16
    k: torch.Tensor              # [T, Hkv, D] bf16 (new keys, not yet rotated)
    v: torch.Tensor              # [T, Hkv, D] bf16
    slot_mapping: torch.Tensor   # [T] int32
    cu_seqlens: torch.Tensor     # [B+1] int32
    context_lens: torch.Tensor   # [B] int32, includes this step's tokens
    block_tables: torch.Tensor   # [B, max_blocks] int32 (unused entries = -1)
    decode_seqs: int = 0         # the first `decode_seqs` sequences have exactly 1 new token

    @property
    def num_tokens(self) -> int:
        return int(self.q.shape[0])

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_new_tokens(self) -> int:
        n = self.cu_seqlens[1:] - self.cu_seqlens[:-1]
        return int(n.max()) if n.numel() else 0

    @property
    def max_context(self) -> int:
        return int(self.context_lens.max()) if self.context_lens.numel() else 0


@dataclass
class Workload:
    name: str
    seed: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    num_blocks: int
    cache_dtype: str             # "bf16" or "fp8"
    k_cache: torch.Tensor        # [NB, 16, Hkv, D] bf16, or uint8 E4M3 codes
    v_cache: torch.Tensor
    steps: list                  # list[Step], applied in order
    max_pos: int                 # RoPE table length
    k_scale: Optional[torch.Tensor] = None   # [Hkv] fp32 (fp8 only)
    v_scale: Optional[torch.Tensor] = None
    layers: int = 1
    block_size: int = BLOCK_SIZE
    rope_base: float = ROPE_BASE
    notes: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


# ----------------------------------------------------------------------------- helpers

def _randn_bf16(g: torch.Generator, *shape) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def _fill_cache(g: torch.Generator, nb: int, hkv: int, d: int, fp8: bool,
                k_scale=None, v_scale=None, nan_fill: bool = False, block_size: int = BLOCK_SIZE):
    shape = (nb, block_size, hkv, d)
    if nan_fill:
        if fp8:
            return (torch.full(shape, 0x7F, dtype=torch.uint8),
                    torch.full(shape, 0x7F, dtype=torch.uint8))
        return (torch.full(shape, float("nan"), dtype=torch.bfloat16),
                torch.full(shape, float("nan"), dtype=torch.bfloat16))
    kc = torch.randn(*shape, generator=g, dtype=torch.float32)
    vc = torch.randn(*shape, generator=g, dtype=torch.float32)
    if not fp8:
        return kc.to(torch.bfloat16), vc.to(torch.bfloat16)
    # Synthetic FP8 cache contents: N(0,1) divided by the head's scale, cast with torch.
    ks = k_scale.view(1, 1, hkv, 1)
    vs = v_scale.view(1, 1, hkv, 1)
    kq = (kc / ks).clamp_(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn).view(torch.uint8)
    vq = (vc / vs).clamp_(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn).view(torch.uint8)
    return kq, vq


def _fp8_scales(k: torch.Tensor, v: torch.Tensor):
    """Per-kv-head scale amax(|x|)/448 over the synthetic new K (resp. V)."""
    hkv = k.shape[1]
    ks = k.float().abs().permute(1, 0, 2).reshape(hkv, -1).amax(dim=1) / FP8_MAX
    vs = v.float().abs().permute(1, 0, 2).reshape(hkv, -1).amax(dim=1) / FP8_MAX
    ks = torch.where(ks > 0, ks, torch.ones_like(ks))
    vs = torch.where(vs > 0, vs, torch.ones_like(vs))
    return ks.to(torch.float32), vs.to(torch.float32)


def blocks_needed(n_tokens: int) -> int:
    return (n_tokens + BLOCK_SIZE - 1) // BLOCK_SIZE


def _assign_blocks(perm: torch.Tensor, counts, max_blocks: int, shared=None) -> torch.Tensor:
    """Block table from a permutation of physical ids.  ``shared`` = list of ids placed
    first in every row (an aliased common prefix)."""
    bt = torch.full((len(counts), max_blocks), -1, dtype=torch.int32)
    cursor = 0
    for b, c in enumerate(counts):
        row = [] if shared is None else list(shared)
        own = c - len(row)
        row += perm[cursor:cursor + own].tolist()
        cursor += own
        bt[b, :len(row)] = torch.tensor(row, dtype=torch.int32)
    return bt


def _slots(bt: torch.Tensor, b: int, positions, block_size: int = BLOCK_SIZE) -> list:
    return [int(bt[b, p // block_size]) * block_size + p % block_size for p in positions]


def _step(name, g, hq, hkv, d, new_counts, ctx_lens, bt, decode_seqs=0,
          block_size: int = BLOCK_SIZE) -> Step:
    T = int(sum(new_counts))
    cu = torch.zeros(len(new_counts) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(new_counts, dtype=torch.int64), 0).to(torch.int32)
    slots = []
    for b, (n, L) in enumerate(zip(new_counts, ctx_lens)):
        slots += _slots(bt, b, range(L - n, L), block_size)
    return Step(name=name, q=_randn_bf16(g, T, hq, d), k=_randn_bf16(g, T, hkv, d),
                v=_randn_bf16(g, T, hkv, d), slot_mapping=torch.tensor(slots, dtype=torch.int32),
                cu_seqlens=cu, context_lens=torch.tensor(ctx_lens, dtype=torch.int32),
                block_tables=bt, decode_seqs=decode_seqs)


# ----------------------------------------------------------------------------- workloads

def tiny(seed: int = 1, nan_fill: bool = False) -> Workload:
    """Prompts {5, 17, 33, 60}: a prefill step of every prompt token, then one decode step
    (one new token per sequence at position L_b, attended with L_b + 1 tokens)."""
    g = torch.Generator().manual_seed(seed)
    hq, hkv, d, nb = 4, 2, 64, 32
    prompts = [5, 17, 33, 60]
    perm = torch.randperm(nb, generator=g)
    counts = [blocks_needed(L + 1) for L in prompts]
    bt = _assign_blocks(perm, counts, max_blocks=max(counts) + 2)
    kc, vc = _fill_cache(g, nb, hkv, d, False, nan_fill=nan_fill)
    pre = _step("tiny-prefill", g, hq, hkv, d, prompts, prompts, bt)
    dec = _step("tiny-decode", g, hq, hkv, d, [1] * 4, [L + 1 for L in prompts], bt,
                decode_seqs=4)
    return Workload("tiny", seed, hq, hkv, d, nb, "bf16", kc, vc, [pre, dec],
                    max_pos=max(prompts) + 1)


def qwen_decode(seed: int = 2, batch: int = 64, lo: int = 128, hi: int = 2048,
                spare_blocks: int = 64, nan_fill: bool = False) -> Workload:
    """Qwen-7B-style MHA decode: 32 q = 32 kv heads, head_dim 128, L_b ~ U[lo, hi]."""
    g = torch.Generator().manual_seed(seed)
    hq = hkv = 32
    d = 128
    lens = torch.randint(lo, hi + 1, (batch,), generator=g).tolist()
    counts = [blocks_needed(L) for L in lens]
    nb = sum(counts) + spare_blocks
    perm = torch.randperm(nb, generator=g)
    bt = _assign_blocks(perm, counts, max_blocks=blocks_needed(hi))
    kc, vc = _fill_cache(g, nb, hkv, d, False, nan_fill=nan_fill)
    st = _step("qwen-decode", g, hq, hkv, d, [1] * batch, lens, bt, decode_seqs=batch)
    return Workload("qwen_decode", seed, hq, hkv, d, nb, "bf16", kc, vc, [st], max_pos=hi,
                    notes={"context": f"U[{lo},{hi}]"})


def gqa_decode(seed: int = 3, batch: int = 32, context: int = 4096, layers: int = 1,
               spare_blocks: int = 16) -> Workload:
    """Mistral-7B-style GQA decode: 32 q / 8 kv heads, head_dim 128, every sequence
    `context` cached tokens.  The returned cache is ONE layer; a multi-layer run keeps
    `layers` distinct copies of it (same values, separate memory)."""
    g = torch.Generator().manual_seed(seed)
    hq, hkv, d = 32, 8, 128
    lens = [context] * batch
    counts = [blocks_needed(L) for L in lens]
    nb = sum(counts) + spare_blocks
    perm = torch.randperm(nb, generator=g)
    bt = _assign_blocks(perm, counts, max_blocks=blocks_needed(context))
    kc, vc = _fill_cache(g, nb, hkv, d, False)
    st = _step("gqa-decode", g, hq, hkv, d, [1] * batch, lens, bt, decode_seqs=batch)
    return Workload("gqa_decode", seed, hq, hkv, d, nb, "bf16", kc, vc, [st], max_pos=context,
                    layers=layers)


def shared_prefix(seed: int = 4, requests: int = 32, prefix: int = 2048, new: int = 2048,
                  hq: int = 32, hkv: int = 8, d: int = 128) -> Workload:
    """Requests whose block tables alias one common prefix of `prefix` tokens (already in
    the cache, keys stored rotated), each prefilling `new` unique tokens causally."""
    assert prefix % BLOCK_SIZE == 0
    g = torch.Generator().manual_seed(seed)
    pb = prefix // BLOCK_SIZE
    own = blocks_needed(new)
    nb = pb + requests * own
    perm = torch.randperm(nb, generator=g)
    shared = perm[:pb].tolist()
    bt = _assign_blocks(perm[pb:], [pb + own] * requests, max_blocks=pb + own, shared=shared)
    kc, vc = _fill_cache(g, nb, hkv, d, False)
    st = _step("shared-prefix-prefill", g, hq, hkv, d, [new] * requests,
               [prefix + new] * requests, bt)
    return Workload("shared_prefix", seed, hq, hkv, d, nb, "bf16", kc, vc, [st],
                    max_pos=prefix + new, notes={"shared_prefix_blocks": shared})


def paged_batch(seed: int, hq: int, hkv: int, d: int, news, ctxs, block_size: int = BLOCK_SIZE,
                fp8: bool = False, decode_seqs: int = 0, spare_blocks: int = 3,
                nan_fill: bool = False) -> Workload:
    """One step over a freshly filled paged cache of any block size / head dim: sequence b
    has ctxs[b] cached tokens, the last news[b] of them new in this step; its blocks come
    from a seeded permutation of the pool.  (Block-size and head-dim variants.)"""
    g = torch.Generator().manual_seed(seed)
    counts = [-(-L // block_size) for L in ctxs]
    nb = sum(counts) + spare_blocks
    perm = torch.randperm(nb, generator=g)
    bt = _assign_blocks(perm, counts, max_blocks=max(counts) + 1)
    st = _step("batch", g, hq, hkv, d, list(news), list(ctxs), bt, decode_seqs=decode_seqs,
               block_size=block_size)
    ks = vs = None
    if fp8:
        ks, vs = _fp8_scales(st.k, st.v)
    kc, vc = _fill_cache(g, nb, hkv, d, fp8, ks, vs, nan_fill=nan_fill, block_size=block_size)
    return Workload("batch", seed, hq, hkv, d, nb, "fp8" if fp8 else "bf16", kc, vc, [st],
                    max_pos=max(ctxs) + 1, k_scale=ks, v_scale=vs, block_size=block_size)


def lognormal_lengths(g: torch.Generator, n: int, median: float = 1024.0, sigma: float = 1.0,
                      lo: int = 1, hi: int = 32768) -> list:
    z = torch.randn(n, generator=g, dtype=torch.float64)
    L = torch.exp(math.log(median) + sigma * z).round().clamp_(lo, hi)
    return [int(x) for x in L.tolist()]


def mix(seed: int = 5, decodes: int = 256, chunks: int = 4, chunk_len: int = 512,
        fp8: bool = False, max_context: int = 32768) -> Workload:
    """Continuous-batching step: `decodes` decode sequences (lognormal context, median 1024,
    sigma 1, clipped to [1, max_context]) followed by `chunks` chunked prefills of
    `chunk_len` tokens whose prior context is drawn from the same law."""
    g = torch.Generator().manual_seed(seed)
    hq, hkv, d = 32, 8, 128
    dec_lens = lognormal_lengths(g, decodes, hi=max_context)
    priors = lognormal_lengths(g, chunks, hi=max_context - chunk_len)
    ctx = dec_lens + [p + chunk_len for p in priors]
    new = [1] * decodes + [chunk_len] * chunks
    counts = [blocks_needed(L) for L in ctx]
    nb = sum(counts) + 16
    perm = torch.randperm(nb, generator=g)
    bt = _assign_blocks(perm, counts, max_blocks=max(counts))
    st = _step("mix", g, hq, hkv, d, new, ctx, bt, decode_seqs=decodes)
    ks = vs = None
    if fp8:
        ks, vs = _fp8_scales(st.k, st.v)
    kc, vc = _fill_cache(g, nb, hkv, d, fp8, ks, vs)
    return Workload("mix_fp8" if fp8 else "mix", seed, hq, hkv, d, nb,
                    "fp8" if fp8 else "bf16", kc, vc, [st], max_pos=max(ctx), k_scale=ks,
                    v_scale=vs, notes={"sum_decode_context": int(sum(dec_lens)),
                                       "chunk_priors": priors})


# ----------------------------------------------------------------------------- helpers

def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bit patterns of a CPU bf16 (-> uint16) or uint8 tensor as numpy."""
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.uint8:
        return t.contiguous().numpy()
    raise TypeError(t.dtype)


def sub_step(st: Step, seqs) -> Step:
    """The inputs of a subset of sequences (token rows and tables re-packed)."""
    seqs = list(seqs)
    rows = []
    cu = [0]
    for b in seqs:
        a, e = int(st.cu_seqlens[b]), int(st.cu_seqlens[b + 1])
        rows += list(range(a, e))
        cu.append(cu[-1] + e - a)
    idx = torch.tensor(rows, dtype=torch.int64)
    sel = torch.tensor(seqs, dtype=torch.int64)
    return Step(name=st.name + "-sub", q=st.q[idx], k=st.k[idx], v=st.v[idx],
                slot_mapping=st.slot_mapping[idx], cu_seqlens=torch.tensor(cu, dtype=torch.int32),
                context_lens=st.context_lens[sel], block_tables=st.block_tables[sel],
                decode_seqs=sum(1 for b in seqs if b < st.decode_seqs))
