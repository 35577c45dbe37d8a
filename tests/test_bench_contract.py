"""The benchmark's accounting and JSON contract, on the CPU: the algorithmic FLOPs and bytes
the roofline divides by follow the closed forms, the reference arm (the oracle on the host
cores) prints one complete line with our arm's workload config, and the CUDA-path leg is
never entered without a GPU."""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from paged_kv_cache_447_b200 import workloads as W  # noqa: E402


def test_prefill_flops_closed_form_shared_prefix():
    # 32 requests x 2048 new tokens after a 2048-token prefix, 32 q heads, D 128:
    # causal pairs per head per request = 2048 * 2048 + 2048 * 2049 / 2 = 6,292,480
    wl = W.shared_prefix(seed=4)
    st = wl.steps[0]
    pairs = 2048 * 2048 + 2048 * 2049 // 2
    assert pairs == 6_292_480
    assert bench.prefill_flops(st, 32, 128) == 4 * 128 * 32 * 32 * pairs  # 3.299 TFLOP
    assert abs(bench.prefill_flops(st, 32, 128) / 1e12 - 3.299) < 1e-3


def test_prefill_flops_tiny_by_enumeration():
    """Count visible (query, key) pairs one by one on the tiny prompts {5, 17, 33, 60}."""
    wl = W.tiny(seed=1)
    st = wl.steps[0]
    n_pairs = 0
    for b in range(st.num_seqs):
        n = int(st.cu_seqlens[b + 1] - st.cu_seqlens[b])
        L = int(st.context_lens[b])
        for r in range(n):
            pos = L - n + r
            n_pairs += sum(1 for j in range(L) if j <= pos)
    assert bench.prefill_flops(st, wl.n_q_heads, wl.head_dim) == 4 * wl.head_dim * wl.n_q_heads * n_pairs


def test_decode_bytes_qwen():
    wl = W.qwen_decode(seed=2)
    st = wl.steps[0]
    L = [int(x) for x in st.context_lens]
    kv = sum(L) * 32 * 128 * 2 * 2                      # K and V of every cached token
    assert bench.decode_kv_bytes(st, 32, 128, 2) == kv
    blocks = sum((x + 15) // 16 for x in L)
    assert bench.decode_alg_bytes(st, 32, 32, 128, 2) == kv + 2 * 64 * 32 * 128 * 2 + 4 * 64 + 4 * blocks
    # the 16 KiB per cached token of a 32 x 128 bf16 MHA layer (K and V)
    assert bench.decode_kv_bytes(st, 32, 128, 2) // sum(L) == 16384


def test_workload_config_is_shared_by_both_arms():
    for name in ("qwen_decode", "shared_prefix"):
        wl, layers = bench.build_workload(name)
        cfg = bench.workload_config(name, wl, layers, 1)
        assert cfg["workload"] == name and cfg["block_size"] == 16
        assert set(cfg) >= {"batch", "n_q_heads", "n_kv_heads", "head_dim", "layers", "l2",
                            "parallelism"}
    wl, layers = bench.build_workload("gqa_decode")
    assert layers == 32 and bench.workload_config("gqa_decode", wl, layers, 1)["layers"] == 32


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_reference_arm_prints_one_complete_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["value"] > 0 and d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    wl, layers = bench.build_workload("qwen_decode")
    ours = bench.workload_config("qwen_decode", wl, layers, 1)
    assert {k: v for k, v in d["config"].items() if k != "sample"} == ours
