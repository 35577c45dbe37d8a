"""The allocation-free decode entry point (pkv_paged_decode_attention_noalloc).

Some callers cannot allocate device memory when they run decode attention -- typically an
engine that gave nearly all of the GPU's memory to its KV-block pool at start-up (a later
cudaMalloc may fail), or a latency-critical step where cudaMalloc/cudaFree could
synchronise the device.  For them the library offers a decode entry point without a
workspace argument; it uses a fixed 8 MiB array inside the library's device image.

These tests call it through the C ABI and check that two calls in a row give what the
ordinary (workspace-taking) entry point gives.  Both run the same kernels with the same
launch geometry on the same inputs, so the outputs must be identical bit for bit (which is
within any tolerance): a stale or clobbered scratch array would show up as a difference.
The file is named so that pytest collects it last."""
import pytest
import torch

import paged_kv_cache_447_b200 as pkv
from paged_kv_cache_447_b200 import workloads as W

from helpers import DeviceWorkload

pytestmark = pytest.mark.gpu


def _both(d: DeviceWorkload, st: W.Step):
    wl = d.wl
    q = st.q.cuda()
    bt = st.block_tables.cuda()
    cl = st.context_lens.cuda()
    ref = pkv.paged_decode_attention(q, d.k_cache, d.v_cache, bt, cl, scale=wl.scale,
                                     k_scale=d.k_scale, v_scale=d.v_scale, rope_cos_sin=d.table)
    out = torch.empty_like(q)
    free_before = torch.cuda.mem_get_info()[0]
    pkv.paged_decode_attention_noalloc(q, d.k_cache, d.v_cache, bt, cl, scale=wl.scale,
                                       k_scale=d.k_scale, v_scale=d.v_scale,
                                       rope_cos_sin=d.table, out=out)
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    assert pkv.get_error() == 0
    return ref, out, free_before, free_after


def _same(a: torch.Tensor, b: torch.Tensor):
    assert torch.isfinite(a.float()).all()
    assert torch.equal(a, b), float((a.float() - b.float()).abs().max())


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    # call 1: Qwen-style MHA decode (64 sequences, lengths U[128, 2048])
    d1 = DeviceWorkload(W.qwen_decode(seed=2))
    st1 = d1.wl.steps[0]
    # call 2: the lognormal FP8 decode batch (256 sequences, 8 kv heads, group 4)
    full = W.mix(seed=5, fp8=True)
    st2 = W.sub_step(full.steps[0], range(full.steps[0].decode_seqs))
    wl2 = W.Workload(full.name, full.seed, 32, 8, 128, full.num_blocks, "fp8", full.k_cache,
                     full.v_cache, [st2], full.max_pos, full.k_scale, full.v_scale)
    d2 = DeviceWorkload(wl2)
    for d, st, fp8 in ((d1, st1, False), (d2, st2, True)):
        assert pkv.decode_workspace_bytes(st.num_seqs, d.wl.n_q_heads, d.wl.n_kv_heads,
                                          d.wl.head_dim) <= pkv.NOALLOC_SCRATCH_BYTES
    ref1, out1, _, _ = _both(d1, st1)
    ref2, out2, free_b, free_a = _both(d2, st2)
    _same(out1, ref1)
    _same(out2, ref2)
    # the second call allocated nothing on the device
    assert free_a == free_b
    # and repeating call 1 after call 2 (scratch left holding call 2's data) still matches
    ref1b, out1b, _, _ = _both(d1, st1)
    _same(ref1b, ref1)
    _same(out1b, ref1)


def test_noalloc_rejects_calls_beyond_the_scratch_limit():
    wl = W.tiny(seed=1)
    d = DeviceWorkload(wl)
    st = wl.steps[1]
    # the smallest power-of-two batch (32 q / 4 kv heads, head_dim 128) whose workspace
    # would not fit the built-in array: the call is refused before anything is enqueued
    big_b = 1
    while pkv.decode_workspace_bytes(big_b, 32, 4, 128) <= pkv.NOALLOC_SCRATCH_BYTES:
        big_b *= 2
    q = torch.zeros((big_b, 32, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((4, 16, 4, 128), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((big_b, 1), dtype=torch.int32, device="cuda")
    cl = torch.zeros((big_b,), dtype=torch.int32, device="cuda")
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_decode_attention_noalloc(q, kc, kc, bt, cl, out=torch.empty_like(q))
    assert e.value.code == -8
    # nothing was enqueued and the device is fine
    assert pkv.get_error() == 0
    ref, out, _, _ = _both(d, st)
    _same(out, ref)
