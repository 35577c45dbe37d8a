"""Benchmark of the paged KV-cache data plane on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-suite] [--no-e2e] [--no-cpu-baseline]

A step is one pass of the hot path over one batch: the step's new tokens are stored into
the paged cache (K rotated by RoPE on the way in) and attention runs over the cache (Q
rotated on load).  Decode rows go through the one-launch decode step (store + attention +
split merge in one kernel); prefill rows through kv_store and paged prefill attention.
``--unfused`` runs decode rows as kv_store + paged decode attention (+ its merge kernel)
instead.
The default workload is the Qwen-7B-style MHA decode step (batch 64, 32 heads x 128,
context lengths uniform in [128, 2048]); the headline value is the decode attention's
KV bytes per step divided by the device-timed step time (GB/s).  ``--suite`` (on by
default at N=1) also times the other workloads: GQA decode over 32 layers, the
shared-prefix prefill (TFLOP/s of causal attention) and the continuous-batching mix
(bf16 and FP8).

Under torchrun (N > 1) every rank runs an independent replica of the workload on its
own GPU (no data-path collective: the path shards by sequence); timing is the max over
ranks, the value is the work of all ranks over that time.

``--impl reference`` times the CPU oracle (plain fp64 C, OpenMP) on a bounded sample of
the same workload, on this machine's host cores; it needs no GPU.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from paged_kv_cache_447_b200 import workloads as W  # noqa: E402

METRIC = "paged decode attn KV GB/s (% of HBM peak); prefill TFLOP/s; decode tok/s/layer"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.lines:
            return None
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def timed_region(fn, steps, warmup, stream, dist=None, sampler_index=0, on_timed=None, on_end=None):
    """Run fn() warmup times, then time `steps` calls with CUDA events on `stream`,
    bracketed by a barrier and a device synchronisation; returns (ms total, clocks).
    `on_timed` (if given) is called once between the warm-up and the timed calls; `on_end`
    (if given) after the timed calls, before the end event (to join other streams' work)."""
    for _ in range(warmup):
        fn()
    if on_timed is not None:
        on_timed()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(sampler_index) as cs:
        time.sleep(0.25)
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(steps):
            fn()
        if on_end is not None:
            on_end()
        end.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    return start.elapsed_time(end), cs.summary()


def max_over_ranks(x: float, dist) -> float:
    """Largest value over the ranks (timing: the job ends when its slowest rank ends)."""
    if dist is None:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, ms_local: float, dist=None) -> tuple:
    """Replicas: every rank processes `units_per_rank`; the job's time is the slowest
    rank's.  Returns (units per second of the whole job, job milliseconds)."""
    world = dist.get_world_size() if dist is not None else 1
    ms = max_over_ranks(ms_local, dist)
    return world * units_per_rank / (ms * 1e-3), ms


def decode_kv_bytes(st: W.Step, hkv: int, d: int, esize: int) -> int:
    L = st.context_lens[:st.decode_seqs].long()
    return int(L.sum()) * hkv * d * esize * 2


def decode_alg_bytes(st: W.Step, hq: int, hkv: int, d: int, esize: int) -> int:
    """Bytes decode attention must move: K and V of every cached token of every kv head,
    q and out (bf16), the context lengths and the block-table entries it reads."""
    B = st.decode_seqs
    L = st.context_lens[:B].long()
    blocks = int(((L + 15) // 16).sum())
    return decode_kv_bytes(st, hkv, d, esize) + 2 * B * hq * d * 2 + 4 * B + 4 * blocks


def prefill_flops(st: W.Step, hq: int, d: int) -> float:
    """4 * D flops (QK^T and PV multiply-adds) per visible (query, key) pair per q head."""
    n = (st.cu_seqlens[1:] - st.cu_seqlens[:-1]).long()
    L = st.context_lens.long()
    first = st.decode_seqs
    n, L = n[first:], L[first:]
    pairs = (n * (L - n) + n * (n + 1) // 2).sum()
    return float(4 * d * hq * int(pairs))


def code_sha256(path: str) -> str:
    """sha256 of a C/CUDA source with comments and whitespace removed: it changes when the
    code changes, not when only its comments do."""
    import hashlib
    import re
    src = open(path, encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    src = re.sub(r"\s+", "", src)
    return hashlib.sha256(src.encode()).hexdigest()


def sources_sha256(paths) -> str:
    """code_sha256 over several sources (a kernel and the headers it is built from)."""
    import hashlib
    return hashlib.sha256("".join(code_sha256(os.path.join(ROOT, q)) for q in paths).encode()).hexdigest()


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch (read + write) from the committed ncu record in profiles/, or
    None if there is none for this kernel and workload or the kernel's code has changed
    since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f).get(kernel)
        if not rec or rec.get("workload") != workload:
            return None
        if not sources_sha256(rec["src"]).startswith(rec["code_sha256_prefix"]):
            return None
        return int(rec["dram_bytes_read"]) + int(rec["dram_bytes_write"])
    except (OSError, ValueError, KeyError, TypeError):
        return None


# Suite entries' minimum timed steps (each about 20 ms or more of device time).
SUITE_MIN_STEPS = {"gqa_decode": 8, "shared_prefix": 8, "mix": 50, "mix_fp8": 50, "small_batch": 500,
                   "qwen_decode": 100}


def timed_kernel(wl, decode: bool) -> str:
    """Name of the kernel the bench's attention events bracket for this workload."""
    if not decode:
        return "prefill_kernel"
    g = wl.n_q_heads // wl.n_kv_heads
    if wl.cache_dtype == "fp8" and wl.head_dim == 128 and g in (2, 4, 8) and wl.n_kv_heads % 2 == 0:
        return "decode_tc_kernel"
    return "decode_kernel"


# ----------------------------------------------------------------------------- runner

class Runner:
    """Device buffers of one workload and the step closure (ours)."""

    def __init__(self, wl: W.Workload, layers: int = 1, fused: bool = True):
        import paged_kv_cache_447_b200 as pkv
        self.pkv = pkv
        self.wl = wl
        st = wl.steps[-1]
        self.st = st
        self.layers = layers
        kc = wl.k_cache.cuda()
        vc = wl.v_cache.cuda()
        self.k_caches = [kc] + [kc.clone() for _ in range(layers - 1)]
        self.v_caches = [vc] + [vc.clone() for _ in range(layers - 1)]
        self.table = pkv.rope_build_table(wl.max_pos, wl.head_dim, wl.rope_base).cuda()
        self.k_scale = wl.k_scale.cuda() if wl.k_scale is not None else None
        self.v_scale = wl.v_scale.cuda() if wl.v_scale is not None else None
        # Per-step inputs: views into one flat pinned host buffer and one flat device buffer,
        # so the end-to-end leg moves a step's inputs in one copy (plus one on-device copy).
        names = ["q", "k", "v", "slot_mapping", "cu_seqlens", "context_lens", "block_tables"]
        srcs = {n: getattr(st, n).contiguous() for n in names}
        offs, total = {}, 0
        for n, t in srcs.items():
            offs[n] = total
            total += (t.numel() * t.element_size() + 15) // 16 * 16
        self.host_flat = torch.empty(total, dtype=torch.uint8).pin_memory()
        self.dev_flat = torch.empty(total, dtype=torch.uint8, device="cuda")
        self.stage_flat = [torch.empty_like(self.dev_flat) for _ in range(2)]

        def view(buf, n):
            t = srcs[n]
            nb = t.numel() * t.element_size()
            return buf[offs[n]:offs[n] + nb].view(t.dtype).view(t.shape)

        self.host = {n: view(self.host_flat, n) for n in names}
        self.dev = {n: view(self.dev_flat, n) for n in names}
        for n in names:
            self.host[n].copy_(srcs[n])
            self.dev[n].copy_(srcs[n])
        B = st.decode_seqs
        self.B = B
        self.fused = fused
        if B:
            self.dec_k = self.dev["k"][:B]
            self.dec_v = self.dev["v"][:B]
            # zero-filled once; every decode step leaves its counters at zero
            self.ws_step = pkv.decode_step_workspace(B, wl.n_q_heads, wl.n_kv_heads, wl.head_dim)
            self.dec_bt = self.dev["block_tables"][:B].contiguous()
            self.dec_ctx = self.dev["context_lens"][:B].contiguous()
            self.dec_slots = self.dev["slot_mapping"][:B].contiguous()
            self.dec_cu = torch.arange(B + 1, dtype=torch.int32, device=self.dec_ctx.device)
            # the library's automatic choice: one launch up to one segment per SM
            sms = torch.cuda.get_device_properties(self.dec_ctx.device).multi_processor_count
            self.step_fused = B * wl.n_kv_heads <= sms
            self.ws = torch.empty(pkv.decode_workspace_bytes(B, wl.n_q_heads, wl.n_kv_heads,
                                                             wl.head_dim),
                                  dtype=torch.uint8, device="cuda")
            self.dec_out = torch.empty((B, wl.n_q_heads, wl.head_dim), dtype=torch.bfloat16,
                                       device="cuda")
        P = st.num_seqs - B
        self.P = P
        if P:
            tok0 = int(st.cu_seqlens[B])
            self.pre_q = self.dev["q"][tok0:]
            self.pre_k = self.dev["k"][tok0:]
            self.pre_v = self.dev["v"][tok0:]
            self.pre_slots = self.dev["slot_mapping"][tok0:]
            self.pre_cu = (self.dev["cu_seqlens"][B:] - tok0).contiguous()
            self.pre_bt = self.dev["block_tables"][B:].contiguous()
            self.pre_ctx = self.dev["context_lens"][B:].contiguous()
            self.pre_out = torch.empty_like(self.pre_q)
            self.max_new = int((st.cu_seqlens[B + 1:] - st.cu_seqlens[B:-1]).max())
        self.host_out = [torch.empty((st.num_tokens, wl.n_q_heads, wl.head_dim),
                                     dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        # the end-to-end leg alternates two output sets (a step's result is read back while
        # the next step computes into the other set)
        self.out_sets = [(getattr(self, "dec_out", None), getattr(self, "pre_out", None))]
        self.out_sets.append(tuple(None if t is None else torch.empty_like(t) for t in self.out_sets[0]))
        # one stream per copy direction: on a single stream the read-back of step i would
        # queue the inputs of step i+1 behind step i's compute
        self.h2d_stream, self.d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()
        self.e2e_i = 0
        ev = lambda: [torch.cuda.Event() for _ in range(2)]
        self.ev_loaded, self.ev_stage_free, self.ev_computed, self.ev_out_free = ev(), ev(), ev(), ev()
        self.ev_attn = []  # (start, end) event pairs around the dominant kernel

    def launches_per_step(self) -> int:
        if self.fused:
            # decode step (one launch, or store + attention + merge); store + prefill
            dec = 1 if getattr(self, "step_fused", True) else 3
            n = (dec if self.B else 0) + (2 if self.P else 0)
        else:
            n = 1 + (2 if self.B else 0) + (1 if self.P else 0)  # store, decode + merge, prefill
        return n * self.layers

    def step(self, record: bool = False, dominant: str = "decode"):
        pkv, wl, d = self.pkv, self.wl, self.dev
        s = torch.cuda.current_stream()
        for layer in range(self.layers):
            kc, vc = self.k_caches[layer], self.v_caches[layer]
            if not self.fused:
                pkv.kv_store(d["k"], d["v"], kc, vc, d["slot_mapping"], k_scale=self.k_scale,
                             v_scale=self.v_scale, rope_cos_sin=self.table,
                             cu_seqlens=d["cu_seqlens"], context_lens=d["context_lens"])
            elif self.P:
                pkv.kv_store(self.pre_k, self.pre_v, kc, vc, self.pre_slots, k_scale=self.k_scale,
                             v_scale=self.v_scale, rope_cos_sin=self.table,
                             cu_seqlens=self.pre_cu, context_lens=self.pre_ctx)
            if self.B:
                q = d["q"][:self.B]
                # The decode step runs as one launch for a latency-bound batch and as store +
                # attention + merge otherwise (the library's automatic mode).  The recorded
                # pass times the attention kernels alone: for a split step the store runs
                # first, outside the events.
                split_rec = record and dominant == "decode" and self.fused and not self.step_fused
                if split_rec:
                    pkv.kv_store(self.dec_k, self.dec_v, kc, vc, self.dec_slots, k_scale=self.k_scale,
                                 v_scale=self.v_scale, rope_cos_sin=self.table,
                                 cu_seqlens=self.dec_cu, context_lens=self.dec_ctx)
                if record and dominant == "decode":
                    e0 = torch.cuda.Event(enable_timing=True); e0.record(s)
                if self.fused and not split_rec:
                    pkv.paged_decode_step(q, self.dec_k, self.dec_v, kc, vc, self.dec_bt,
                                          self.dec_ctx, self.ws_step, scale=wl.scale,
                                          k_scale=self.k_scale, v_scale=self.v_scale,
                                          rope_cos_sin=self.table, out=self.dec_out)
                else:
                    pkv.paged_decode_attention(q, kc, vc, self.dec_bt, self.dec_ctx, scale=wl.scale,
                                               k_scale=self.k_scale, v_scale=self.v_scale,
                                               rope_cos_sin=self.table, workspace=self.ws,
                                               out=self.dec_out)
                if record and dominant == "decode":
                    e1 = torch.cuda.Event(enable_timing=True); e1.record(s)
                    self.ev_attn.append((e0, e1))
            if self.P:
                if record and dominant == "prefill":
                    e0 = torch.cuda.Event(enable_timing=True); e0.record(s)
                pkv.paged_prefill_attention(self.pre_q, kc, vc, self.pre_cu, self.pre_bt,
                                            self.pre_ctx, self.max_new, scale=wl.scale,
                                            k_scale=self.k_scale, v_scale=self.v_scale,
                                            rope_cos_sin=self.table, out=self.pre_out)
                if record and dominant == "prefill":
                    e1 = torch.cuda.Event(enable_timing=True); e1.record(s)
                    self.ev_attn.append((e0, e1))

    def e2e_step(self):
        """The same step with its inputs copied from pinned host memory and its attention
        output read back, pipelined as a serving loop would: on copy streams, step i's
        inputs travel while step i-1 computes and step i's output returns while step i+1
        computes.  On the compute stream the step waits for its inputs (then one on-device
        copy puts them in place) and for the read-back of the output set it reuses."""
        b = self.e2e_i & 1
        self.e2e_i += 1
        s, hs, ds = torch.cuda.current_stream(), self.h2d_stream, self.d2h_stream
        hs.wait_event(self.ev_stage_free[b])        # the on-device copy of step i-2 read it
        with torch.cuda.stream(hs):
            self.stage_flat[b].copy_(self.host_flat, non_blocking=True)
            self.ev_loaded[b].record(hs)
        s.wait_event(self.ev_loaded[b])
        self.dev_flat.copy_(self.stage_flat[b], non_blocking=True)
        self.ev_stage_free[b].record(s)
        s.wait_event(self.ev_out_free[b])            # step i-2's output has been read back
        self.dec_out, self.pre_out = self.out_sets[b]
        self.step()
        self.ev_computed[b].record(s)
        ds.wait_event(self.ev_computed[b])
        with torch.cuda.stream(ds):
            off = 0
            for t in self.out_sets[b]:
                if t is not None:
                    self.host_out[b][off:off + t.shape[0]].copy_(t, non_blocking=True)
                    off += t.shape[0]
            self.ev_out_free[b].record(ds)
        self.dec_out, self.pre_out = self.out_sets[0]

    def e2e_finish(self):
        """The timed region ends once the last read-back has landed."""
        torch.cuda.current_stream().wait_stream(self.d2h_stream)

    def e2e_bytes(self):
        h2d = sum(t.numel() * t.element_size() for t in self.host.values())
        d2h = self.host_out[0].numel() * self.host_out[0].element_size()
        return h2d, d2h

    def attn_ms(self) -> float:
        if not self.ev_attn:
            return float("nan")
        torch.cuda.synchronize()
        ts = [a.elapsed_time(b) for a, b in self.ev_attn]
        return sum(ts) / len(ts)


def workload_config(name: str, wl, layers: int, world: int) -> dict:
    """The `config` object of the JSON line (both arms): the workload and its shape."""
    st = wl.steps[-1]
    B = st.decode_seqs
    esize = 1 if wl.cache_dtype == "fp8" else 2
    kv = decode_kv_bytes(st, wl.n_kv_heads, wl.head_dim, esize) * layers if B else 0
    return {"workload": name, "batch": B or (st.num_seqs - B),
            "n_q_heads": wl.n_q_heads, "n_kv_heads": wl.n_kv_heads,
            "head_dim": wl.head_dim, "block_size": 16, "layers": layers,
            "context": wl.notes.get("context", None),
            "l2": f"inputs larger than L2 (KV bytes per step {kv / 1e9:.2f} GB), no flush",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def build_workload(name: str, layers=None):
    if name == "small_batch":
        return W.gqa_decode(seed=6, batch=4, context=4096), 1
    if name == "qwen_decode":
        return W.qwen_decode(seed=2), 1
    if name == "gqa_decode":
        return W.gqa_decode(seed=3), (32 if layers is None else layers)
    if name == "shared_prefix":
        return W.shared_prefix(seed=4), 1
    if name == "mix":
        return W.mix(seed=5), 1
    if name == "mix_fp8":
        return W.mix(seed=5, fp8=True), 1
    raise ValueError(name)


def measure_ours(name, steps, warmup, dist=None, device_index=0, pk=None, e2e=True, layers=None,
                 fused=True):
    wl, layers = build_workload(name, layers)
    r = Runner(wl, layers, fused=fused)
    st = r.st
    # one checked step first: a device error (bounds, a bounded wait that ran out) stops here
    r.step()
    code = r.pkv.get_error()
    if code != 0:
        raise RuntimeError(f"{name}: device error {code} ({r.pkv.strerror(code)}) on the first step")
    esize = 1 if wl.cache_dtype == "fp8" else 2
    dominant = "decode" if r.B else "prefill"
    ms, clocks = timed_region(lambda: r.step(record=True, dominant=dominant), steps, warmup,
                              torch.cuda.current_stream(), dist, device_index,
                              on_timed=r.ev_attn.clear)
    code = r.pkv.get_error()
    assert code == 0, f"device error flag set during the timed region: {code}"
    _, ms = job_throughput(steps, ms, dist)
    world = dist.get_world_size() if dist is not None else 1
    step_ms = ms / steps
    attn_ms = r.attn_ms()
    res = {"workload": name, "step_ms": step_ms, "step_us": step_ms * 1e3, "layers": layers,
           "clocks": clocks, "gpu_launches": r.launches_per_step() * steps,
           "decode_path": ("decode step, " + ("one launch" if getattr(r, "step_fused", False)
                                                  else "store + attention + merge")) if fused
                          else "kv_store + paged_decode_attention"}
    hbm = (pk or FALLBACK_PEAKS)["hbm_gbs"]
    if r.B:
        kv_bytes = decode_kv_bytes(st, wl.n_kv_heads, wl.head_dim, esize) * layers
        alg = decode_alg_bytes(st, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, esize)
        res["decode_kv_bytes_per_step"] = kv_bytes
        res["kv_gbs"] = world * kv_bytes / (step_ms * 1e-3) / 1e9
        res["decode_tok_s_per_layer"] = world * r.B / (step_ms * 1e-3 / layers)
        res["attn_kernel_ms"] = attn_ms
        res["attn_alg_bytes"] = alg
        res["attn_gbs"] = alg / (attn_ms * 1e-3) / 1e9
        res["attn_hbm_frac"] = res["attn_gbs"] / hbm
    if r.P:
        fl = prefill_flops(st, wl.n_q_heads, wl.head_dim) * layers
        res["prefill_flops_per_step"] = fl
        if dominant == "prefill":
            res["attn_kernel_ms"] = attn_ms
            res["prefill_tflops"] = fl / (attn_ms * 1e-3) / 1e12
        res["step_tflops"] = world * fl / (step_ms * 1e-3) / 1e12
    if e2e:
        ms_e, _ = timed_region(r.e2e_step, steps, warmup, torch.cuda.current_stream(), dist,
                               device_index, on_end=r.e2e_finish)
        ms_e = max_over_ranks(ms_e, dist)
        h2d, d2h = r.e2e_bytes()
        res["e2e_step_ms"] = ms_e / steps
        res["e2e_h2d"] = h2d
        res["e2e_d2h"] = d2h
    return res, r


# ----------------------------------------------------------------------------- CPU oracle

def oracle_sample(name: str, step_budget_s: float):
    """A bounded sample of the workload for the CPU oracle: the first n decode sequences
    (or prefill requests), n grown until one oracle pass takes about step_budget_s.
    Returns a closure running one pass and a description."""
    import oracle
    wl, layers = build_workload(name)
    st = wl.steps[-1]
    fp8 = wl.cache_dtype == "fp8"
    esize = 1 if fp8 else 2
    kc0, vc0 = W.bits(wl.k_cache), W.bits(wl.v_cache)
    tab = oracle.rope_table(wl.max_pos, wl.head_dim, wl.rope_base)
    B = st.decode_seqs
    ks = None if not fp8 else wl.k_scale.numpy()
    vs = None if not fp8 else wl.v_scale.numpy()

    def make(seqs):
        sub = W.sub_step(st, seqs)
        pos = oracle.positions(sub.cu_seqlens.numpy(), sub.context_lens.numpy())

        kc, vc = kc0.copy(), vc0.copy()  # the store rewrites the same slots every pass

        def one_pass():
            oracle.kv_store(W.bits(sub.k), W.bits(sub.v), kc, vc, sub.slot_mapping.numpy(), 16,
                            fp8=fp8, k_scale=ks, v_scale=vs, table=tab, pos=pos)
            oracle.attention(W.bits(sub.q), kc, vc, sub.cu_seqlens.numpy(),
                             sub.block_tables.numpy(), sub.context_lens.numpy(), wl.scale, 16,
                             wl.n_kv_heads, fp8=fp8, k_scale=ks, v_scale=vs, table=tab)
        return sub, one_pass

    order = list(range(B)) if B else list(range(st.num_seqs))
    n = 1
    while True:
        sub, one = make(order[:n])
        t0 = time.perf_counter()
        one()
        dt = time.perf_counter() - t0
        if dt >= step_budget_s / 2 or n >= len(order):
            break
        n = min(len(order), max(n + 1, int(n * min(8.0, step_budget_s / max(dt, 1e-4)))))
    if B:
        work, unit = decode_kv_bytes(sub, wl.n_kv_heads, wl.head_dim, esize) / 1e9, "GB/s"
    else:
        work, unit = prefill_flops(sub, wl.n_q_heads, wl.head_dim) / 1e12, "TFLOP/s"
    desc = f"{n} of {len(order)} sequences of one step (one layer), kv_store + attention"
    return one, work, unit, desc


def oracle_step_rate(name: str, budget_s: float = 15.0, steps: int = 3, warmup: int = 1):
    """Time the CPU oracle on a bounded sample of the workload (warm-up passes, then
    `steps` timed passes; each pass sized to about budget_s / (steps + warmup))."""
    import oracle
    per = max(0.05, budget_s / max(1, steps + warmup))
    one, work, unit, desc = oracle_sample(name, per)
    for _ in range(warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(steps):
        one()
    dt = (time.perf_counter() - t0) / steps
    return {"value": work / dt, "unit": unit, "seconds": dt, "sample": desc,
            "cores": oracle.num_threads()}


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen_decode",
                    choices=["qwen_decode", "gqa_decode", "shared_prefix", "mix", "mix_fp8",
                             "small_batch"])
    ap.add_argument("--unfused", action="store_true",
                    help="decode rows as kv_store + paged decode attention (+ merge kernel)")
    ap.add_argument("--no-suite", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="layers of the GQA decode workload (default 32; fewer for profiling)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pk, pk_kind = peaks()

    if args.impl == "reference":
        if rank != 0:
            return
        # the whole --steps/--warmup run of the oracle stays within about two minutes
        r = oracle_step_rate(args.workload, budget_s=120.0, steps=args.steps,
                             warmup=args.warmup)
        line = {"impl": "reference", "metric": METRIC, "value": r["value"], "unit": r["unit"],
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": r["seconds"] * 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": dict(workload_config(args.workload, *build_workload(args.workload, args.layers),
                                               world), sample=r["sample"]),
                "cpu_baseline": {"value": r["value"], "unit": r["unit"], "cores": r["cores"],
                                 "kind": "oracle", "sample": r["sample"]},
                "e2e": {"value": r["value"], "unit": r["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist_mod
        torch.cuda.set_device(local)
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        dist = dist_mod
    else:
        torch.cuda.set_device(0)

    res, runner = measure_ours(args.workload, args.steps, args.warmup, dist, local, pk,
                               e2e=not args.no_e2e, layers=args.layers, fused=not args.unfused)
    wl = runner.wl
    esize = 1 if wl.cache_dtype == "fp8" else 2
    if runner.B:
        value, unit = res["kv_gbs"], "GB/s"
        bound, ach, peak, runit = "hbm", res["attn_gbs"], pk["hbm_gbs"], "GB/s"
    else:
        value, unit = res["step_tflops"], "TFLOP/s"
        bound, ach, peak, runit = ("tensor", res.get("prefill_tflops", float("nan")),
                                   pk["bf16_tflops"], "TFLOP/s")
    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["step_ms"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if esize == 2 else "e4m3",
        "data": "synthetic",
        "config": workload_config(args.workload, wl, res["layers"], world),
        "decode_tok_s_per_layer": res.get("decode_tok_s_per_layer"),
        "roofline": {"bound": bound, "achieved": ach, "peak": peak, "unit": runit,
                     "frac": ach / peak,
                     "traffic": recorded_traffic(timed_kernel(wl, bool(runner.B)), args.workload),
                     "kernel": "paged_decode_attention" if runner.B else "paged_prefill_attention",
                     "peak_source": pk_kind, "kernel_ms": res.get("attn_kernel_ms")},
        "clocks": res["clocks"],
        "gpu_launches": res["gpu_launches"],
    }
    if not args.no_e2e:
        if runner.B:
            ev = world * res["decode_kv_bytes_per_step"] / (res["e2e_step_ms"] * 1e-3) / 1e9
        else:
            ev = world * res["prefill_flops_per_step"] / (res["e2e_step_ms"] * 1e-3) / 1e12
        line["e2e"] = {"value": ev, "unit": unit, "h2d_bytes_per_step": res["e2e_h2d"],
                       "d2h_bytes_per_step": res["e2e_d2h"], "ms_per_step": res["e2e_step_ms"],
                       "pipelining": "each step's inputs copied from pinned host memory and its "
                                     "output read back on two copy streams, overlapping the "
                                     "neighbouring steps' compute"}
    del runner
    torch.cuda.empty_cache()

    if world == 1 and not args.no_suite:
        suite = {}
        runs = [(n, True) for n in ("gqa_decode", "shared_prefix", "mix", "mix_fp8", "small_batch")
                if n != args.workload]
        # the same decode workloads through the three-launch path, for comparison
        runs += [("qwen_decode", False), ("small_batch", False), ("mix_fp8", False)]
        for name, fused in runs:
            key = name if fused else name + "_unfused"
            if name == args.workload and fused != args.unfused:
                continue
            # at least ~20 ms of timed work per entry, so that short steps are not measured
            # over a handful of launches
            n_steps = max(3, args.steps // 4, SUITE_MIN_STEPS.get(name, 3))
            try:
                r, rr = measure_ours(name, n_steps, max(3, min(20, n_steps // 10)), None, 0, pk,
                                     e2e=False, fused=fused)
                del rr
                torch.cuda.empty_cache()
                keep = {k: v for k, v in r.items() if k not in ("clocks",)}
                if r.get("clocks"):
                    keep["clocks"] = {k: r["clocks"][k] for k in ("sm_mhz", "reasons")}
                if "attn_gbs" in r:
                    keep["attn_hbm_frac"] = r["attn_gbs"] / pk["hbm_gbs"]
                if "prefill_tflops" in r:
                    keep["prefill_tensor_frac"] = r["prefill_tflops"] / pk["bf16_tflops"]
                suite[key] = keep
            except Exception as e:  # report, do not hide
                suite[key] = {"error": f"{type(e).__name__}: {e}"}
        line["suite"] = suite

    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        try:
            cb = oracle_step_rate(args.workload, budget_s=15.0, steps=3, warmup=1)
            line["cpu_baseline"] = {"value": cb["value"], "unit": cb["unit"], "cores": cb["cores"],
                                    "kind": "oracle", "sample": cb["sample"]}
        except Exception as e:
            line["cpu_baseline"] = {"error": f"{type(e).__name__}: {e}"}

    if rank == 0:
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
