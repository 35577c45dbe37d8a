"""Shared test helpers: move a workload to the GPU, run the oracle side, compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from paged_kv_cache_447_b200 import workloads as W

# Tolerances on attention outputs (bf16 inputs, fp32 accumulation, bf16 output):
BF16_MAX_ABS, BF16_MEAN_ABS = 1e-2, 1e-3
FP8_MAX_ABS = 3e-2


def dev(t):
    return None if t is None else t.cuda()


def cache_bits(t: torch.Tensor) -> np.ndarray:
    return W.bits(t.detach().cpu())


def oracle_caches(wl: W.Workload):
    return W.bits(wl.k_cache).copy(), W.bits(wl.v_cache).copy()


def oracle_store(wl: W.Workload, st: W.Step, kc, vc, rope: bool = True):
    tab = oracle.rope_table(wl.max_pos, wl.head_dim, wl.rope_base) if rope else None
    pos = oracle.positions(st.cu_seqlens.numpy(), st.context_lens.numpy()) if rope else None
    fp8 = wl.cache_dtype == "fp8"
    oracle.kv_store(W.bits(st.k), W.bits(st.v), kc, vc, st.slot_mapping.numpy(), wl.block_size,
                    fp8=fp8, k_scale=None if not fp8 else wl.k_scale.numpy(),
                    v_scale=None if not fp8 else wl.v_scale.numpy(), table=tab, pos=pos)


def oracle_attention(wl: W.Workload, st: W.Step, kc, vc, rope: bool = True, rows=None):
    tab = oracle.rope_table(wl.max_pos, wl.head_dim, wl.rope_base) if rope else None
    fp8 = wl.cache_dtype == "fp8"
    return oracle.attention(W.bits(st.q), kc, vc, st.cu_seqlens.numpy(), st.block_tables.numpy(),
                            st.context_lens.numpy(), wl.scale, wl.block_size, wl.n_kv_heads,
                            fp8=fp8, k_scale=None if not fp8 else wl.k_scale.numpy(),
                            v_scale=None if not fp8 else wl.v_scale.numpy(), table=tab, rows=rows)


def compare(got: torch.Tensor, ref: np.ndarray, fp8: bool = False, what: str = ""):
    g = got.detach().float().cpu().numpy().astype(np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    if fp8:
        assert mx <= FP8_MAX_ABS, f"{what}: max-abs {mx:.3e} > {FP8_MAX_ABS}"
    else:
        assert mx <= BF16_MAX_ABS, f"{what}: max-abs {mx:.3e} > {BF16_MAX_ABS}"
        assert mean <= BF16_MEAN_ABS, f"{what}: mean-abs {mean:.3e} > {BF16_MEAN_ABS}"
    return mx, mean


class DeviceWorkload:
    """The workload's cache and RoPE table on the GPU (table built by the library)."""

    def __init__(self, wl: W.Workload):
        import paged_kv_cache_447_b200 as pkv
        self.wl = wl
        self.k_cache = wl.k_cache.cuda()
        self.v_cache = wl.v_cache.cuda()
        self.table = pkv.rope_build_table(wl.max_pos, wl.head_dim, wl.rope_base).cuda()
        self.k_scale = dev(wl.k_scale)
        self.v_scale = dev(wl.v_scale)

    def store(self, st: W.Step, rope: bool = True):
        import paged_kv_cache_447_b200 as pkv
        pkv.kv_store(st.k.cuda(), st.v.cuda(), self.k_cache, self.v_cache, st.slot_mapping.cuda(),
                     k_scale=self.k_scale, v_scale=self.v_scale,
                     rope_cos_sin=self.table if rope else None, cu_seqlens=st.cu_seqlens.cuda(),
                     context_lens=st.context_lens.cuda())

    def decode(self, st: W.Step, rope: bool = True, **kw):
        import paged_kv_cache_447_b200 as pkv
        return pkv.paged_decode_attention(
            st.q.cuda(), self.k_cache, self.v_cache, st.block_tables.cuda(),
            st.context_lens.cuda(), scale=self.wl.scale, k_scale=self.k_scale,
            v_scale=self.v_scale, rope_cos_sin=self.table if rope else None, **kw)

    def prefill(self, st: W.Step, rope: bool = True, **kw):
        import paged_kv_cache_447_b200 as pkv
        return pkv.paged_prefill_attention(
            st.q.cuda(), self.k_cache, self.v_cache, st.cu_seqlens.cuda(), st.block_tables.cuda(),
            st.context_lens.cuda(), st.max_new_tokens, scale=self.wl.scale, k_scale=self.k_scale,
            v_scale=self.v_scale, rope_cos_sin=self.table if rope else None, **kw)
