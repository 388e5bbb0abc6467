#!/usr/bin/env python
"""Benchmark of ragged paged attention on B200 through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload decode|prefill|mixed|sparse] [--no-secondary]

A step is one pass of the whole hot path over one synthetic batch: the fused call
(KV-cache write + attention, with the decode splits merged), plus the block-union table
build for the sparse workload.  Inputs are resident in HBM and larger than L2 (126 MB): the
KV pool rotates over copies (at least three, and together more than twice L2), so that each
step reads memory the previous steps did not touch.  K steps run back to back between two
CUDA events on the stream the kernels run on, with a barrier and a synchronize on both
sides.  The headline line is the decode workload
(Llama-3-8B attention, batch 64, kv_len ~ U[512, 8192]) in HBM GB/s; the prefill, mixed and
sparse workloads are reported as secondary objects on the same line.

Multi-GPU (torchrun, one process per GPU): every rank runs its own independent batch (a
different seed) with no collective on the data path -- weak scaling; the elapsed time is the
max over ranks.  ``--impl reference`` times the fp64 CPU oracle instead, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "paged-attn decode HBM GB/s (% peak) + prefill TFLOP/s (% bf16 peak), 1×B200"

WORKLOAD_TEXT = {
    "decode": "decode-only Llama-3-8B attention: batch 64, q_len=1, Hq=32, Hkv=8, D=128, "
              "page_size=16, kv_len uniform 512-8192, bf16 N(0,1), shuffled pages, 1 new K/V "
              "token written per seq",
    "prefill": "prefill-only: 4 seqs x 4096 prompt tokens, causal, Hq=32, Hkv=8, D=128, "
               "page_size=64, bf16 N(0,1), new K/V for all 16384 tokens scattered into "
               "shuffled pages",
    "mixed": "mixed continuous batch (token budget 2048): 48 decode seqs (kv_len 1024-16384 "
             "uniform) + 2 prefill chunks of 512+976 tokens with prior context 1024 and 8192; "
             "Hq=32, Hkv=8, D=128, page 16, bf16",
    "sparse": "sparse chunked prefill: 1 seq, 2048-query chunk at 128K context, Hq=32, Hkv=8, "
              "D=128, KV-head-major pages of 64, random 64x64 per-head block masks keeping "
              "~25% blocks, Q-block+intra-group union tables",
}

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------------------
# Algorithmic work (bytes that must move, flops that must be done) per workload
# ------------------------------------------------------------------------------------

def visible_pairs(batch, table=None, count=None):
    """Sum over query rows of the number of keys each row sees, per query head."""
    cu = batch.cu_seqlens_q.tolist()
    kv = batch.kv_lens()
    total = 0
    if table is None:
        for b in range(batch.num_seqs):
            q_len = cu[b + 1] - cu[b]
            past = kv[b] - q_len
            if batch.causal:
                total += q_len * past + q_len * (q_len + 1) // 2
            else:
                total += q_len * kv[b]
        return total * batch.num_q_heads
    G = batch.num_q_heads // batch.num_kv_heads
    P = batch.page_size
    for b in range(batch.num_seqs):
        q_len = cu[b + 1] - cu[b]
        past = kv[b] - q_len
        pos = past + np.arange(q_len)
        for g in range(batch.num_kv_heads):
            blocks = np.asarray(table[b, g, :int(count[b, g])], dtype=np.int64)
            starts = blocks * P
            ends = np.minimum(starts + P, kv[b])
            # keys of block k visible to position p: clip(p + 1 - start, 0, end - start)
            vis = np.clip(pos[:, None] + 1 - starts[None, :], 0, (ends - starts)[None, :])
            total += int(vis.sum()) * G
    return total


def work(batch, table=None, count=None):
    D, Hq, Hkv = batch.head_dim, batch.num_q_heads, batch.num_kv_heads
    T = batch.num_tokens
    el = 2  # bf16
    pairs = visible_pairs(batch, table, count)
    flops = 4.0 * D * pairs
    q_o = 2.0 * T * Hq * D * el
    new_kv = 2.0 * 2 * T * Hkv * D * el              # read k_new/v_new + write into the pool
    if table is None:
        kv_read = float(sum(batch.kv_lens())) * Hkv * D * 2 * el
    else:
        kv_read = 0.0
        cnt = np.asarray(count)
        for b, kvl in enumerate(batch.kv_lens()):
            for g in range(Hkv):
                n = int(cnt[b, g])
                blocks = np.asarray(table[b, g, :n], dtype=np.int64)
                keys = np.minimum(blocks * batch.page_size + batch.page_size, kvl) - \
                    blocks * batch.page_size
                kv_read += float(keys.sum()) * D * 2 * el
    return {"flops": flops, "attn_bytes": kv_read + q_o, "step_bytes": kv_read + q_o + new_kv}


# ------------------------------------------------------------------------------------
# Clocks during the timed region (NVML: the counters nvidia-smi prints)
# ------------------------------------------------------------------------------------

class ClockSampler:
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._dev = device_index
        self._thr = None
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self._ok = False

    def _sample(self):
        n = self._nvml
        mhz = n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM)
        try:
            rs = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        except Exception:
            rs = n.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
        self.samples.append(mhz)
        for name, bit in self.REASONS.items():
            if rs & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            time.sleep(self._period)

    def start(self):
        if self._ok:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def stop(self):
        if self._thr is not None:
            self._stop.set()
            self._thr.join()
        if self._ok and not self.samples:
            try:
                self._sample()
            except Exception:
                pass
        return self

    def summary(self):
        if not self._ok:
            return self._nvidia_smi_once()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "source": "nvml"}

    def _nvidia_smi_once(self):
        try:
            out = subprocess.run(
                ["nvidia-smi", f"--id={self._dev}",
                 "--query-gpu=clocks.sm,clocks.max.sm", "--format=csv,noheader,nounits"],
                capture_output=True, text=True, timeout=10).stdout.strip().split(",")
            return {"sm_mhz": float(out[0]), "sm_max_mhz": float(out[1]), "reasons": [],
                    "samples": 1, "source": "nvidia-smi"}
        except Exception:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


# ------------------------------------------------------------------------------------
# GPU side
# ------------------------------------------------------------------------------------

def make_workload(name: str, seed_offset: int = 0):
    from ragged_paged_attention_forward_b200 import workloads as wl
    seeds = {"decode": 1002, "prefill": 1003, "mixed": 1004, "sparse": 1005}
    seed = seeds[name] + seed_offset
    if name == "decode":
        return wl.decode(seed=seed, poison=False, keep_logical=False), None
    if name == "prefill":
        return wl.prefill(seed=seed, poison=False, keep_logical=False), None
    if name == "mixed":
        return wl.mixed(seed=seed, poison=False, keep_logical=False), None
    return wl.sparse(seed=seed, poison=False)


L2_BYTES = 126 << 20


class Runner:
    """Holds one batch on the device and runs steps through the C ABI."""

    def __init__(self, name, batch, mask):
        from ragged_paged_attention_forward_b200 import api
        self.api = api
        self.name = name
        self.batch = batch
        self.mask = mask
        b = batch
        self.d = {k: getattr(b, k).cuda().contiguous() for k in (
            "q", "k_new", "v_new", "k_pool", "v_pool", "block_table", "cu_seqlens_q",
            "seq_lens_k")}
        self.out = torch.empty_like(self.d["q"])
        self.lse = torch.empty(b.num_tokens, b.num_q_heads, dtype=torch.float32, device="cuda")
        self.sparse = mask is not None
        if self.sparse:
            self.mask_d = mask.cuda()
            nkb = mask.shape[-1]
            assert nkb == b.max_blocks
            self.table = torch.empty(b.num_seqs, b.num_kv_heads, nkb, dtype=torch.int32,
                                     device="cuda")
            self.count = torch.empty(b.num_seqs, b.num_kv_heads, dtype=torch.int32,
                                     device="cuda")
        else:
            self.table = self.count = None
        # the KV pool and copies of it, so that consecutive steps read disjoint memory
        pool_bytes = 2 * self.d["k_pool"].numel() * self.d["k_pool"].element_size()
        n = max(3, -(-2 * L2_BYTES // pool_bytes) + 1)
        self.pools = [(self.d["k_pool"], self.d["v_pool"])] + [
            (self.d["k_pool"].clone(), self.d["v_pool"].clone()) for _ in range(n - 1)]
        self.pool_bytes_total = n * pool_bytes
        self.plan = self.make_plan()
        self.ws = torch.empty(max(self.plan.workspace_bytes, 256), dtype=torch.uint8,
                              device="cuda")
        info = self.plan.info()
        self.launches_step = info.launches_forward + (1 if self.sparse else 0)
        self.info = info

    def make_plan(self):
        b = self.batch
        return self.api.rpa_plan(
            num_seqs=b.num_seqs, num_tokens=b.num_tokens, num_q_heads=b.num_q_heads,
            num_kv_heads=b.num_kv_heads, head_dim=b.head_dim, page_size=b.page_size,
            num_pages=b.num_pages, max_blocks_per_seq=b.max_blocks, layout=b.layout,
            causal=b.causal, cu_seqlens_q=b.cu_seqlens_q, seq_lens_k=b.seq_lens_k,
            sparse=self.sparse)

    def tables(self, stream=None):
        if self.sparse:
            self.api.rpa_build_group_tables(self.mask_d, self.batch.num_kv_heads, self.table,
                                            self.count, stream)

    def step(self, fused=True, stream=None, i=0):
        d = self.d
        kp, vp = self.pools[i % len(self.pools)]
        self.tables(stream)
        self.api.rpa_forward(self.plan, d["q"], d["k_new"] if fused else None,
                             d["v_new"] if fused else None, kp, vp,
                             d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"], self.table,
                             self.count, self.batch.scale, self.out, self.lse, self.ws, stream)

    def host_tables(self):
        if not self.sparse:
            return None, None
        self.tables()
        torch.cuda.synchronize()
        return self.table.cpu().numpy(), self.count.cpu().numpy()


def timed_loop(fn, steps, warmup):
    """Mean CUDA-event duration (ms) of fn(i) over `steps` calls run back to back on the
    current stream after `warmup` untimed calls; fn(i) reads the i-th pool copy."""
    stream = torch.cuda.current_stream()
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for i in range(steps):
        fn(warmup + i)
    e.record(stream)
    torch.cuda.synchronize()
    return s.elapsed_time(e) / steps


def e2e_loop(runner, steps, warmup):
    """End to end through the public API: plan on the host, copy the step's inputs from one
    pinned host buffer (one H2D copy), run the fused step, read the output back; the KV pool
    rotates over copies so that no step finds K/V in L2.  Returns (ms list, h2d bytes, d2h
    bytes)."""
    b = runner.batch
    names = ["q", "k_new", "v_new", "block_table", "cu_seqlens_q", "seq_lens_k"]
    srcs = [getattr(b, k).contiguous() for k in names]
    if runner.sparse:
        names.append("mask")
        srcs.append(runner.mask.contiguous())
    offs, total = [], 0
    for t in srcs:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    host = torch.empty(total, dtype=torch.uint8).pin_memory()
    dev = torch.empty(total, dtype=torch.uint8, device="cuda")
    views = {}
    for k, t, o in zip(names, srcs, offs):
        nb = t.numel() * t.element_size()
        host[o:o + nb].copy_(t.view(torch.uint8).reshape(-1))
        views[k] = dev[o:o + nb].view(t.dtype).view(t.shape)
    out_host = torch.empty(runner.out.shape, dtype=runner.out.dtype).pin_memory()
    h2d = total
    d2h = out_host.numel() * out_host.element_size()
    stream = torch.cuda.current_stream()
    pools = runner.pools

    def one(i):
        kp, vp = pools[i % len(pools)]
        plan = runner.make_plan()
        dev.copy_(host, non_blocking=True)
        if runner.sparse:
            runner.api.rpa_build_group_tables(views["mask"], b.num_kv_heads, runner.table,
                                              runner.count)
        runner.api.rpa_forward(plan, views["q"], views["k_new"], views["v_new"], kp, vp,
                               views["block_table"], views["cu_seqlens_q"],
                               views["seq_lens_k"], runner.table, runner.count, b.scale,
                               runner.out, runner.lse, runner.ws)
        out_host.copy_(runner.out, non_blocking=True)
        return plan

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    ms = []
    for i in range(steps):
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(stream)
        plan = one(warmup + i)
        e.record(stream)
        e.synchronize()
        ms.append(s.elapsed_time(e))
        del plan
    return ms, h2d, d2h


def e2e_pipelined(runner, steps, warmup):
    """End to end as a serving loop runs it: every step plans on the host, copies its inputs
    from pinned host memory (one H2D copy on a copy stream), runs the fused step on the
    compute stream and copies the output back (D2H on a second copy stream).  Two device
    input and output buffers let step i+1's H2D and step i-1's D2H overlap step i's kernels,
    and the host plans ahead while the GPU works; the KV pool rotates over copies so that no
    step finds K/V in L2.  Returns (ms per step, h2d bytes, d2h bytes): the time from the
    first step's start to the last step's output landing on the host, divided by the number
    of steps."""
    b = runner.batch
    names = ["q", "k_new", "v_new", "block_table", "cu_seqlens_q", "seq_lens_k"]
    srcs = [getattr(b, k).contiguous() for k in names]
    if runner.sparse:
        names.append("mask")
        srcs.append(runner.mask.contiguous())
    offs, total = [], 0
    for t in srcs:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    host = torch.empty(total, dtype=torch.uint8).pin_memory()
    for t, o in zip(srcs, offs):
        nb = t.numel() * t.element_size()
        host[o:o + nb].copy_(t.view(torch.uint8).reshape(-1))
    devs = [torch.empty(total, dtype=torch.uint8, device="cuda") for _ in range(2)]
    views = []
    for dev in devs:
        v = {}
        for k, t, o in zip(names, srcs, offs):
            nb = t.numel() * t.element_size()
            v[k] = dev[o:o + nb].view(t.dtype).view(t.shape)
        views.append(v)
    outs = [torch.empty_like(runner.out) for _ in range(2)]
    outs_host = [torch.empty(runner.out.shape, dtype=runner.out.dtype).pin_memory()
                 for _ in range(2)]
    h2d = total
    d2h = outs_host[0].numel() * outs_host[0].element_size()
    compute = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]
    pools = runner.pools

    def one(i):
        k = i & 1
        kp, vp = pools[i % len(pools)]
        plan = runner.make_plan()
        up.wait_event(comp_done[k])          # step i-2 has finished reading devs[k]
        with torch.cuda.stream(up):
            devs[k].copy_(host, non_blocking=True)
        h2d_done[k].record(up)
        compute.wait_event(h2d_done[k])
        compute.wait_event(d2h_done[k])      # step i-2's output has left outs[k]
        v = views[k]
        if runner.sparse:
            runner.api.rpa_build_group_tables(v["mask"], b.num_kv_heads, runner.table,
                                              runner.count)
        runner.api.rpa_forward(plan, v["q"], v["k_new"], v["v_new"], kp, vp,
                               v["block_table"], v["cu_seqlens_q"], v["seq_lens_k"],
                               runner.table, runner.count, b.scale, outs[k], runner.lse,
                               runner.ws)
        comp_done[k].record(compute)
        down.wait_event(comp_done[k])
        with torch.cuda.stream(down):
            outs_host[k].copy_(outs[k], non_blocking=True)
        d2h_done[k].record(down)
        return plan

    plans = [one(i) for i in range(warmup)]
    torch.cuda.synchronize()
    plans.clear()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(compute)
    for i in range(steps):
        plans.append(one(warmup + i))
    down.wait_stream(compute)
    end.record(down)
    end.synchronize()
    return start.elapsed_time(end) / steps, h2d, d2h


KERNEL_SOURCES = ("ptx.cuh", "rpa_internal.h")


def kernel_source_sha256(kernel_file: str) -> str:
    """sha256 over the sources a kernel is compiled from (its .cu and the shared headers)."""
    h = hashlib.sha256()
    for name in (kernel_file,) + KERNEL_SOURCES:
        with open(os.path.join(ROOT, "ragged_paged_attention_forward_b200", "csrc", name),
                  "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profile_traffic(kernel_file: str, key: str):
    """DRAM bytes per launch (scaled to the benchmark's workload) from the committed ncu
    summary ``profiles/traffic.json``, or None when the kernel's sources changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)[key]
        if d.get("source_sha256") != kernel_source_sha256(kernel_file):
            return None
        return float(d["dram_bytes_per_launch"])
    except Exception:
        return None


def measure(name, runner, steps, warmup, peaks):
    b = runner.batch
    table, count = runner.host_tables()
    w = work(b, table, count)
    ms = timed_loop(lambda i: runner.step(True, i=i), steps, warmup)
    ams = timed_loop(lambda i: runner.step(False, i=i), steps, warmup)
    res = {"workload": WORKLOAD_TEXT[name], "ms_per_step": ms, "attn_ms": ams,
           "tokens_per_s": b.num_tokens / (ms * 1e-3),
           "step_GBps": w["step_bytes"] / (ms * 1e-3) / 1e9,
           "attn_GBps": w["attn_bytes"] / (ams * 1e-3) / 1e9,
           "attn_TFLOPs": w["flops"] / (ams * 1e-3) / 1e12,
           "flops": w["flops"], "attn_bytes": w["attn_bytes"], "step_bytes": w["step_bytes"],
           "launches_per_step": runner.launches_step,
           "batch_class": int(runner.info.batch_class)}
    t_mem = w["attn_bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_flop = w["flops"] / (peaks["bf16_tflops"] * 1e12)
    res["roofline_frac"] = max(t_mem, t_flop) / (ams * 1e-3)
    res["bound"] = "hbm" if t_mem >= t_flop else "tensor"
    return res


def measure_device_planned_decode(steps, warmup, peaks):
    """The decode step with a device-side plan (rpa_plan_device), captured in CUDA graphs and
    replayed: the planner kernel builds the work lists from the device lengths, then the
    KV write, the decode kernel and the merge run (the tensor-core kernel's CTAs all return
    at once).  One graph per KV-pool copy, replayed in turn, so no step finds K/V in L2."""
    from ragged_paged_attention_forward_b200 import api
    b, _ = make_workload("decode")
    runner = Runner("decode", b, None)
    d = runner.d
    plan = api.rpa_plan_device(num_seqs=b.num_seqs, max_tokens=b.num_tokens,
                               num_q_heads=b.num_q_heads, num_kv_heads=b.num_kv_heads,
                               head_dim=b.head_dim, page_size=b.page_size,
                               num_pages=b.num_pages, max_blocks_per_seq=b.max_blocks,
                               layout=b.layout, causal=b.causal,
                               max_kv_len=int(b.seq_lens_k.max()))
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(d["q"])

    def step(kp, vp):
        api.rpa_forward(plan, d["q"], d["k_new"], d["v_new"], kp, vp, d["block_table"],
                        d["cu_seqlens_q"], d["seq_lens_k"], None, None, b.scale, out, None, ws)

    for kp, vp in runner.pools:  # warm-up outside the capture
        step(kp, vp)
    torch.cuda.synchronize()
    graphs = []
    for kp, vp in runner.pools:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(kp, vp)
        graphs.append(g)
    ms = timed_loop(lambda i: graphs[i % len(graphs)].replay(), steps, warmup)
    table, count = runner.host_tables()
    w = work(b, table, count)
    gbps = w["step_bytes"] / (ms * 1e-3) / 1e9
    info = plan.info()
    res = {"workload": WORKLOAD_TEXT["decode"] + "; device-planned, CUDA-graph replay",
           "ms_per_step": ms, "step_GBps": gbps, "frac_of_hbm": gbps / peaks["hbm_gbs"],
           "launches_per_step": info.launches_forward, "decode_split_keys":
           info.decode_split_keys}
    del graphs
    return res


def measure_decode_kv8(steps, warmup, peaks):
    """The decode step over an e4m3 (fp8) KV cache (rpa_forward_kv8): the same 64 sequences
    as the headline, the context as random finite e4m3 codes with per-KV-head scales, the
    new tokens quantised by the step's fused write.  HBM-bound: algorithmic bytes = K and V
    codes read once (1 byte per element) + Q read and O written (bf16) + the new tokens read
    (bf16) and written (codes).  Timed back to back over rotating pool copies."""
    from ragged_paged_attention_forward_b200 import api
    from ragged_paged_attention_forward_b200 import workloads as wl
    b, _ = make_workload("decode")
    b8, ks, vs = wl.with_kv8_pools(b, seed=1234, poison=False)
    d = {k: getattr(b8, k).cuda().contiguous() for k in (
        "q", "k_new", "v_new", "k_pool", "v_pool", "block_table", "cu_seqlens_q", "seq_lens_k")}
    ks, vs = ks.cuda(), vs.cuda()
    pool_bytes = 2 * d["k_pool"].numel()
    n = max(3, -(-2 * L2_BYTES // pool_bytes) + 1)
    pools = [(d["k_pool"], d["v_pool"])] + [(d["k_pool"].clone(), d["v_pool"].clone())
                                            for _ in range(n - 1)]
    plan = api.rpa_plan(num_seqs=b8.num_seqs, num_tokens=b8.num_tokens,
                        num_q_heads=b8.num_q_heads, num_kv_heads=b8.num_kv_heads,
                        head_dim=b8.head_dim, page_size=b8.page_size, num_pages=b8.num_pages,
                        max_blocks_per_seq=b8.max_blocks, layout=b8.layout, causal=b8.causal,
                        cu_seqlens_q=b8.cu_seqlens_q, seq_lens_k=b8.seq_lens_k)
    ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(d["q"])

    def step(i):
        kp, vp = pools[i % len(pools)]
        api.rpa_forward_kv8(plan, d["q"], d["k_new"], d["v_new"], kp, vp, ks, vs,
                            d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"], b8.scale, out,
                            None, ws)

    ms = timed_loop(step, steps, warmup)
    T, Hq, D = b8.q.shape
    Hkv = b8.num_kv_heads
    kv_read = float(sum(b8.kv_lens())) * Hkv * D * 2
    q_o = 2.0 * T * Hq * D * 2
    new_kv = 2.0 * T * Hkv * D * (2 + 1)
    step_bytes = kv_read + q_o + new_kv
    gbps = step_bytes / (ms * 1e-3) / 1e9
    info = plan.info()
    return {"workload": WORKLOAD_TEXT["decode"] + "; K/V cache as e4m3 codes with per-KV-head "
            "fp32 scales (random finite codes), new tokens quantised in the fused write",
            "ms_per_step": ms, "step_GBps": gbps, "frac_of_hbm": gbps / peaks["hbm_gbs"],
            "step_bytes": step_bytes, "tokens_per_s": T / (ms * 1e-3),
            "launches_per_step": info.launches_forward, "l2": f"{n} pool copies rotate"}


def measure_sparse_ablation(steps, warmup, peaks):
    """Execution-only ablation on the sparse workload (CompactAttention, Fig. 7c): the same
    unioned block mask run (A) through per-group tables -- a pair of query heads per CTA
    sharing every K/V tile -- and (B) block-sparse per query tile and head -- tables built per
    (128-query tile, query head) from the unioned mask written back per head and query block,
    one head per CTA.  Both compute the same attention (bit for bit); only the execution
    differs.  Attention only (tables built once, new tokens already in the pool), back to back
    over rotating pool copies.  (C), for context: block-sparse on the original per-head mask,
    which selects fewer blocks per row and is a different attention."""
    from ragged_paged_attention_forward_b200 import api
    b, mask = make_workload("sparse")
    runner = Runner("sparse", b, mask)
    d = runner.d
    for i in range(len(runner.pools)):  # new tokens into every pool copy
        runner.step(True, i=i)
    runner.tables()
    torch.cuda.synchronize()
    B, Hq, nqb, nkb = mask.shape
    Hkv = b.num_kv_heads
    G = Hq // Hkv
    qbr = b.num_tokens // nqb  # query rows per mask block (one sequence)
    # the unioned mask written back per (head, query block)
    sel = torch.zeros(B, Hkv, nkb + 1, dtype=torch.uint8, device="cuda")
    idx = torch.where(runner.table >= 0, runner.table, torch.full_like(runner.table, nkb))
    sel.scatter_(2, idx.long(), 1)
    union = sel[:, :, :nkb].repeat_interleave(G, dim=1).unsqueeze(2).expand(
        B, Hq, nqb, nkb).contiguous()
    nt = -(-nqb // (128 // qbr))

    def qtiles(m):
        t = torch.empty(B, Hq, nt, nkb, dtype=torch.int32, device="cuda")
        c = torch.empty(B, Hq, nt, dtype=torch.int32, device="cuda")
        api.rpa_build_qtile_tables(m, qbr, t, c)
        return t, c

    tq_u, cq_u = qtiles(union)
    tq_m, cq_m = qtiles(runner.mask_d)
    plan_q = api.rpa_plan(num_seqs=b.num_seqs, num_tokens=b.num_tokens,
                          num_q_heads=b.num_q_heads, num_kv_heads=Hkv, head_dim=b.head_dim,
                          page_size=b.page_size, num_pages=b.num_pages,
                          max_blocks_per_seq=b.max_blocks, layout=b.layout, causal=b.causal,
                          cu_seqlens_q=b.cu_seqlens_q, seq_lens_k=b.seq_lens_k, sparse=2)
    ws_q = torch.empty(max(plan_q.workspace_bytes, 256), dtype=torch.uint8, device="cuda")

    def attend(plan, ws, t, c):
        def f(i):
            kp, vp = runner.pools[i % len(runner.pools)]
            api.rpa_forward(plan, d["q"], None, None, kp, vp, d["block_table"],
                            d["cu_seqlens_q"], d["seq_lens_k"], t, c, b.scale, runner.out,
                            None, ws)
        return f

    ms_a = timed_loop(attend(runner.plan, runner.ws, runner.table, runner.count), steps, warmup)
    ms_b = timed_loop(attend(plan_q, ws_q, tq_u, cq_u), steps, warmup)
    ms_c = timed_loop(attend(plan_q, ws_q, tq_m, cq_m), steps, warmup)
    table, count = runner.host_tables()
    w = work(b, table, count)
    # K/V bytes the CTAs ask for (from L2 or HBM), before the causal cut: every query tile
    # reads each group's table once per CTA of the group -- G/2 CTAs in (A), G in (B)
    kv_tile = float(np.asarray(count).sum()) * b.page_size * b.head_dim * 4
    tiles = -(-b.num_tokens // 128)
    res = {"workload": "sparse workload, same unioned mask: (A) per-group tables, 2 query heads "
                       "per CTA; (B) per-(query tile, query head) tables, 1 head per CTA; (C) "
                       "per-(query tile, query head) tables of the original per-head mask",
           "union_ms": ms_a, "blocksparse_ms": ms_b, "blocksparse_own_mask_ms": ms_c,
           "union_TFLOPs": w["flops"] / (ms_a * 1e-3) / 1e12,
           "blocksparse_TFLOPs": w["flops"] / (ms_b * 1e-3) / 1e12,
           "union_speedup_over_blocksparse": ms_b / ms_a,
           "kv_tile_bytes_union": kv_tile * tiles * (G // 2),
           "kv_tile_bytes_blocksparse": kv_tile * tiles * G}
    return res


def measure_mixed_kv8(steps, warmup, peaks):
    """The mixed workload over e4m3 pools (rpa_forward_kv8 with a kv_e4m3 plan): decode rows
    and the two prefill chunks both on the codes, the tensor-core kernel expanding its tiles
    to f16 itself, after the quantising write.  Timed as the fused step, back to back over
    rotating pool copies."""
    from ragged_paged_attention_forward_b200 import api
    from ragged_paged_attention_forward_b200 import workloads as wl
    b, _ = make_workload("mixed")
    b8, ks, vs = wl.with_kv8_pools(b, seed=4321, poison=False)
    d = {k: getattr(b8, k).cuda().contiguous() for k in (
        "q", "k_new", "v_new", "k_pool", "v_pool", "block_table", "cu_seqlens_q", "seq_lens_k")}
    ks, vs = ks.cuda(), vs.cuda()
    pool_bytes = 2 * d["k_pool"].numel()
    n = max(3, -(-2 * L2_BYTES // pool_bytes) + 1)
    pools = [(d["k_pool"], d["v_pool"])] + [(d["k_pool"].clone(), d["v_pool"].clone())
                                            for _ in range(n - 1)]
    plan = api.rpa_plan(num_seqs=b8.num_seqs, num_tokens=b8.num_tokens,
                        num_q_heads=b8.num_q_heads, num_kv_heads=b8.num_kv_heads,
                        head_dim=b8.head_dim, page_size=b8.page_size, num_pages=b8.num_pages,
                        max_blocks_per_seq=b8.max_blocks, layout=b8.layout, causal=b8.causal,
                        cu_seqlens_q=b8.cu_seqlens_q, seq_lens_k=b8.seq_lens_k, kv_e4m3=True)
    ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(d["q"])

    def step(i):
        kp, vp = pools[i % len(pools)]
        api.rpa_forward_kv8(plan, d["q"], d["k_new"], d["v_new"], kp, vp, ks, vs,
                            d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"], b8.scale, out,
                            None, ws)

    ms = timed_loop(step, steps, warmup)
    w = work(b)
    info = plan.info()
    return {"workload": WORKLOAD_TEXT["mixed"] + "; K/V cache as e4m3 codes with per-KV-head "
            "scales", "ms_per_step": ms, "tokens_per_s": b8.num_tokens / (ms * 1e-3),
            "bf16_equivalent_TFLOPs": w["flops"] / (ms * 1e-3) / 1e12,
            "launches_per_step": info.launches_forward,
            "workspace_MB": plan.workspace_bytes / 1e6}


def measure_prefill_kv8(steps, warmup, peaks):
    """The prefill workload (4 x 4096 causal, page 64) over e4m3 pools: the quantising write
    of the 16384 new tokens, then the persistent tensor-core kernel reading the codes and
    expanding each tile to f16 in shared memory.  Timed as the fused step and as attention
    alone (the pools already written), back to back over rotating pool copies."""
    from ragged_paged_attention_forward_b200 import api
    from ragged_paged_attention_forward_b200 import workloads as wl
    b, _ = make_workload("prefill")
    b8, ks, vs = wl.with_kv8_pools(b, seed=1040, poison=False)
    d = {k: getattr(b8, k).cuda().contiguous() for k in (
        "q", "k_new", "v_new", "k_pool", "v_pool", "block_table", "cu_seqlens_q", "seq_lens_k")}
    ks, vs = ks.cuda(), vs.cuda()
    plan = api.rpa_plan(num_seqs=b8.num_seqs, num_tokens=b8.num_tokens,
                        num_q_heads=b8.num_q_heads, num_kv_heads=b8.num_kv_heads,
                        head_dim=b8.head_dim, page_size=b8.page_size, num_pages=b8.num_pages,
                        max_blocks_per_seq=b8.max_blocks, layout=b8.layout, causal=b8.causal,
                        cu_seqlens_q=b8.cu_seqlens_q, seq_lens_k=b8.seq_lens_k, kv_e4m3=True)
    ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(d["q"])
    # write once, then rotate over copies of the written pools that together pass twice L2
    api.rpa_write_kv8(plan, d["k_new"], d["v_new"], d["k_pool"], d["v_pool"], ks, vs,
                      d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"], None)
    pool_bytes = 2 * d["k_pool"].numel()
    n = max(3, -(-2 * L2_BYTES // pool_bytes) + 1)
    pools = [(d["k_pool"], d["v_pool"])] + [(d["k_pool"].clone(), d["v_pool"].clone())
                                            for _ in range(n - 1)]

    def attn(i):
        kp, vp = pools[i % len(pools)]
        api.rpa_forward_kv8(plan, d["q"], None, None, kp, vp, ks, vs, d["block_table"],
                            d["cu_seqlens_q"], d["seq_lens_k"], b8.scale, out, None, ws)

    def step(i):
        kp, vp = pools[i % len(pools)]
        api.rpa_forward_kv8(plan, d["q"], d["k_new"], d["v_new"], kp, vp, ks, vs,
                            d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"], b8.scale, out,
                            None, ws)

    ms_attn = timed_loop(attn, steps, warmup)
    ms = timed_loop(step, steps, warmup)
    w = work(b)
    peak = peaks["bf16_tflops"]
    return {"workload": WORKLOAD_TEXT["prefill"] + "; K/V cache as e4m3 codes with per-KV-head "
            "scales", "ms_per_step": ms, "attn_ms": ms_attn,
            "attn_TFLOPs": w["flops"] / (ms_attn * 1e-3) / 1e12,
            "attn_frac_of_bf16_peak": w["flops"] / (ms_attn * 1e-3) / 1e12 / peak,
            "launches_per_step": plan.info().launches_forward,
            "note": "the MMAs run kind::f16 on f16 operands (the bf16 and f16 dense peaks are "
                    "the same)"}


def measure_device_planned_decode_kv8(steps, warmup, peaks):
    """The e4m3 decode step with a device plan (kv_e4m3), captured in CUDA graphs and
    replayed (three launches: planner, decode with the quantising write, merge); one graph
    per pool copy, replayed in turn."""
    from ragged_paged_attention_forward_b200 import api
    from ragged_paged_attention_forward_b200 import workloads as wl
    b, _ = make_workload("decode")
    b8, ks, vs = wl.with_kv8_pools(b, seed=1234, poison=False)
    d = {k: getattr(b8, k).cuda().contiguous() for k in (
        "q", "k_new", "v_new", "k_pool", "v_pool", "block_table", "cu_seqlens_q", "seq_lens_k")}
    ks, vs = ks.cuda(), vs.cuda()
    n = max(3, -(-2 * L2_BYTES // (2 * d["k_pool"].numel())) + 1)
    pools = [(d["k_pool"], d["v_pool"])] + [(d["k_pool"].clone(), d["v_pool"].clone())
                                            for _ in range(n - 1)]
    plan = api.rpa_plan_device(num_seqs=b8.num_seqs, max_tokens=b8.num_tokens,
                               num_q_heads=b8.num_q_heads, num_kv_heads=b8.num_kv_heads,
                               head_dim=b8.head_dim, page_size=b8.page_size,
                               num_pages=b8.num_pages, max_blocks_per_seq=b8.max_blocks,
                               layout=b8.layout, causal=b8.causal,
                               max_kv_len=int(b8.seq_lens_k.max()), kv_e4m3=True)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(d["q"])

    def step(kp, vp):
        api.rpa_forward_kv8(plan, d["q"], d["k_new"], d["v_new"], kp, vp, ks, vs,
                            d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"], b8.scale, out,
                            None, ws)

    for kp, vp in pools:
        step(kp, vp)
    torch.cuda.synchronize()
    graphs = []
    for kp, vp in pools:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(kp, vp)
        graphs.append(g)
    ms = timed_loop(lambda i: graphs[i % len(graphs)].replay(), steps, warmup)
    T, Hq, D = b8.q.shape
    step_bytes = float(sum(b8.kv_lens())) * b8.num_kv_heads * D * 2 + 2.0 * T * Hq * D * 2 + \
        2.0 * T * b8.num_kv_heads * D * 3
    res = {"workload": WORKLOAD_TEXT["decode"] + "; e4m3 pools, device-planned, CUDA-graph "
           "replay", "ms_per_step": ms, "step_GBps": step_bytes / (ms * 1e-3) / 1e9,
           "frac_of_hbm": step_bytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
           "launches_per_step": plan.info().launches_forward}
    del graphs
    return res


def measure_input_pass(steps, warmup, peaks):
    """The input pass with rotary embedding (rpa_rotary_write_kv) on the prefill workload's
    16384 new tokens: packed QKV in, RoPE over all 128 dims (split pairs), Q out, K/V
    scattered into the pool.  HBM-bound: algorithmic bytes = the packed input read + Q, K, V
    written + one cos/sin row pair per token.  Timed back to back over rotating copies of
    the input and the pool (together larger than L2)."""
    import numpy as np
    from ragged_paged_attention_forward_b200 import api
    b, _ = make_workload("prefill")
    T, Hq, D = b.q.shape
    Hkv = b.num_kv_heads
    rd = D
    runner = Runner("prefill", b, None)
    d = runner.d
    packed = torch.cat([d["q"].reshape(T, -1), d["k_new"].reshape(T, -1),
                        d["v_new"].reshape(T, -1)], dim=1).contiguous()
    copies = max(3, -(-2 * L2_BYTES // (2 * packed.numel() * 2)) + 1)
    ins = [packed] + [packed.clone() for _ in range(copies - 1)]
    q_outs = [torch.empty_like(d["q"]) for _ in range(copies)]
    max_pos = int(b.seq_lens_k.max()) + 1
    j = np.arange(rd // 2)
    ang = np.arange(max_pos)[:, None] / 10000.0 ** (2.0 * j / rd)[None, :]
    cos = torch.tensor(np.cos(ang), dtype=torch.float32).to(torch.bfloat16).cuda()
    sin = torch.tensor(np.sin(ang), dtype=torch.float32).to(torch.bfloat16).cuda()

    def call(i):
        k = i % copies
        kp, vp = runner.pools[i % len(runner.pools)]
        api.rpa_rotary_write_kv(runner.plan, ins[k], None, None, q_outs[k], kp, vp,
                                d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"],
                                cos, sin, rd, False)

    ms = timed_loop(call, steps, warmup)
    nbytes = 2.0 * T * (Hq + 2 * Hkv) * D * 2 + T * rd * 2
    gbps = nbytes / (ms * 1e-3) / 1e9
    return {"workload": "input pass: 16384 tokens of packed QKV (Hq=32, Hkv=8, D=128), RoPE "
                        "over 128 dims, Q written, K/V scattered into pages of 64",
            "ms": ms, "algorithmic_bytes": nbytes, "GBps": gbps,
            "frac_of_hbm": gbps / peaks["hbm_gbs"], "launches": 1}


def cpu_oracle_baseline(name, batch, target_s=12.0, table=None, count=None):
    """Time the fp64 oracle, as it stands, on a bounded sample of the workload: whole
    sequences (all query heads) until about target_s of CPU work, going over the batch again
    (at most 16 passes) when one pass takes less."""
    from oracle import rpa_oracle as orc
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count() or 1
    cu = batch.cu_seqlens_q.tolist()
    kvl = batch.kv_lens()
    done_bytes = done_flops = 0.0
    elapsed = 0.0
    nseq = 0
    rows_done = 0
    D, Hq, Hkv = batch.head_dim, batch.num_q_heads, batch.num_kv_heads
    passes = 0
    for n in range(16 * batch.num_seqs):
        b = n % batch.num_seqs
        passes = n // batch.num_seqs + 1
        q_len = cu[b + 1] - cu[b]
        if q_len == 0:
            continue
        # rows of this sequence (capped so one sequence stays bounded)
        nrows = min(q_len, 8)
        rows = [(cu[b] + i, h) for i in range(q_len - nrows, q_len) for h in range(Hq)]
        t0 = time.perf_counter()
        orc.attention(batch.q, batch.k_pool, batch.v_pool, batch.block_table,
                      batch.cu_seqlens_q, batch.seq_lens_k, scale=batch.scale,
                      causal=batch.causal, page_size=batch.page_size, layout=batch.layout,
                      num_kv_heads=Hkv, group_table=table, group_count=count, rows=rows)
        elapsed += time.perf_counter() - t0
        past = kvl[b] - q_len
        keys = sum(min(kvl[b], past + i + 1) for i in range(q_len - nrows, q_len))
        done_flops += 4.0 * D * keys * Hq
        done_bytes += float(kvl[b]) * Hkv * D * 2 * 2 + 2.0 * nrows * Hq * D * 2
        nseq += 1
        rows_done += len(rows)
        if elapsed >= target_s:
            break
    return {"elapsed_s": elapsed, "bytes": done_bytes, "flops": done_flops, "threads": threads,
            "sample": f"{nseq} sequences x {Hq} query heads ({passes} pass(es) over the "
                      f"batch), last <=8 query rows each ({rows_done} rows), oracle fp64 numpy"}


def rank_seed_offset(rank: int) -> int:
    """Seed offset of a rank's batch: every rank draws its own independent batch."""
    return 1000 * rank


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The max of a per-rank number over all ranks (the job is as slow as its slowest rank)."""
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbps(world: int, bytes_per_rank_step: float, max_ms_per_step: float) -> float:
    """Aggregate throughput of `world` ranks that each moved `bytes_per_rank_step` per step,
    timed by the slowest rank."""
    return world * bytes_per_rank_step / (max_ms_per_step * 1e-3) / 1e9


def run_gpu(args):
    from ragged_paged_attention_forward_b200 import api  # noqa: F401  (fails loudly if unbuilt)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    peaks, peak_src = load_peaks()

    name = args.workload
    batch, mask = make_workload(name, seed_offset=rank_seed_offset(rank))
    runner = Runner(name, batch, mask)
    table, count = runner.host_tables()
    w = work(batch, table, count)

    # headline: the fused step, K timed steps after W warm-up steps, clocks sampled meanwhile
    for i in range(args.warmup):
        runner.step(True, i=i)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device()).start()
    stream = torch.cuda.current_stream()
    ev_s = torch.cuda.Event(enable_timing=True)
    ev_e = torch.cuda.Event(enable_timing=True)
    t_wall0 = time.perf_counter()
    ev_s.record(stream)
    for i in range(args.steps):
        runner.step(True, i=args.warmup + i)
    ev_e.record(stream)
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall0
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.stop()
    total_ms = max_over_ranks(ev_s.elapsed_time(ev_e), dist, "cuda")
    ms_per_step = total_ms / args.steps
    value = whole_job_gbps(world, w["step_bytes"], ms_per_step)

    # dominant kernel: the attention call alone (decode split + merge for this workload)
    attn_ms = timed_loop(lambda i: runner.step(False, i=i), args.steps, 2)
    attn_gbps = w["attn_bytes"] / (attn_ms * 1e-3) / 1e9
    kernel_file = "decode.cu" if name in ("decode", "mixed") else "prefill.cu"
    bound = "hbm" if name in ("decode", "mixed") else "tensor"
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": attn_gbps, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": attn_gbps / peaks["hbm_gbs"],
                "traffic": profile_traffic(kernel_file, name),
                "algorithmic_bytes_per_launch": w["attn_bytes"],
                "kernel": "rpa_forward attention (split-KV decode + LSE merge)",
                "peak_source": f"{peak_src} (copy bandwidth)"}
    else:
        tf = w["flops"] / (attn_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": tf / peaks["bf16_tflops"],
                "frac_of_sustained": tf / peaks["bf16_tflops_sustained"],
                "traffic": profile_traffic(kernel_file, name),
                "algorithmic_flops_per_launch": w["flops"],
                "kernel": "rpa_forward attention (tcgen05 prefill)",
                "peak_source": f"{peak_src} (cuBLAS bf16 burst)"}

    # end to end through the public API with host buffers: one step at a time (latency) and
    # as a pipelined serving loop (throughput, the reported value)
    e2e_ms, h2d, d2h = e2e_loop(runner, args.steps, 2)
    e2e_ms_mean = max_over_ranks(statistics.mean(e2e_ms), dist, "cuda")
    e2e_serial = whole_job_gbps(world, w["step_bytes"], e2e_ms_mean)
    e2e_pipe_ms, _, _ = e2e_pipelined(runner, args.steps, 4)
    e2e_pipe_ms = max_over_ranks(e2e_pipe_ms, dist, "cuda")
    e2e_val = whole_job_gbps(world, w["step_bytes"], e2e_pipe_ms)

    # planner host time
    t0 = time.perf_counter()
    for _ in range(20):
        runner.make_plan()
    planner_us = (time.perf_counter() - t0) / 20 * 1e6

    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[name], "per_rank_batch": "independent seed per rank",
                   "l2": f"inputs larger than L2: the KV pool rotates over "
                         f"{len(runner.pools)} copies ({runner.pool_bytes_total / 1e9:.2f} GB), "
                         f"so each step reads memory the previous steps did not touch; "
                         f"steps run back to back, no flush",
                   "step": "rpa_forward fused (KV write + attention + LSE merge)"
                           + (" + group-table build" if runner.sparse else ""),
                   "tokens_per_step": batch.num_tokens * world,
                   "tokens_per_s": world * batch.num_tokens / (ms_per_step * 1e-3),
                   "hbm_frac_of_step": value / world / peaks["hbm_gbs"],
                   "planner_host_us": planner_us},
        "roofline": roof,
        "e2e": {"value": e2e_val, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_pipe_ms,
                "includes": "every step: host planner + one pinned H2D copy of q/k_new/v_new/"
                            "block table/lengths + fused step + D2H of out, pipelined over "
                            "two buffers (copy streams overlap the neighbouring steps' kernels)",
                "serial_value": e2e_serial, "serial_ms_per_step": e2e_ms_mean,
                "serial_includes": "the same, one step at a time (each step waits for the "
                                   "previous one's output)"},
        "gpu_launches": runner.launches_step * args.steps,
        "clocks": sampler.summary(),
        "wall_s_timed_region": t_wall,
    }

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_oracle_baseline(name, batch, target_s=args.cpu_seconds, table=table,
                                 count=count)
        line["cpu_baseline"] = {"value": cb["bytes"] / cb["elapsed_s"] / 1e9, "unit": "GB/s",
                                "cores": cb["threads"], "kind": "oracle", "sample": cb["sample"],
                                "elapsed_s": cb["elapsed_s"],
                                "gflops": cb["flops"] / cb["elapsed_s"] / 1e9}

    if not args.no_secondary and world == 1:
        secondary = {}
        del runner
        torch.cuda.empty_cache()
        for other in ("prefill", "mixed", "sparse"):
            if other == name:
                continue
            b2, m2 = make_workload(other)
            r2 = Runner(other, b2, m2)
            res = measure(other, r2, args.steps, args.warmup, peaks)
            if other in ("prefill", "sparse"):
                res["frac_of_bf16_peak"] = res["attn_TFLOPs"] / peaks["bf16_tflops"]
                res["frac_of_bf16_sustained"] = res["attn_TFLOPs"] / peaks[
                    "bf16_tflops_sustained"]
            secondary[other] = res
            del r2, b2
            torch.cuda.empty_cache()
        secondary["input_pass"] = measure_input_pass(args.steps, args.warmup, peaks)
        secondary["decode_kv8"] = measure_decode_kv8(args.steps, args.warmup, peaks)
        secondary["mixed_kv8"] = measure_mixed_kv8(args.steps, args.warmup, peaks)
        secondary["prefill_kv8"] = measure_prefill_kv8(args.steps, args.warmup, peaks)
        secondary["sparse_ablation"] = measure_sparse_ablation(args.steps, args.warmup, peaks)
        secondary["decode_device_planned"] = measure_device_planned_decode(args.steps,
                                                                           args.warmup, peaks)
        secondary["decode_kv8_device_planned"] = measure_device_planned_decode_kv8(
            args.steps, args.warmup, peaks)
        line["secondary"] = secondary
        if "prefill" in secondary:
            line["prefill_TFLOPs"] = secondary["prefill"]["attn_TFLOPs"]
            line["prefill_frac_of_bf16_peak"] = secondary["prefill"]["frac_of_bf16_peak"]
    line["peaks"] = dict(peaks, source=peak_src)
    line["hbm_frac"] = value / world / peaks["hbm_gbs"]
    # one compact object last, so that the end of the line alone holds every workload's
    # figures (attention time, throughput, fraction of the roofline)
    summary = {name: {"attn_ms": round(attn_ms, 5), "roofline_frac": round(roof["frac"], 4)}}
    for k, v in line.get("secondary", {}).items():
        if "attn_ms" in v:
            summary[k] = {"attn_ms": round(v["attn_ms"], 5)}
            for key, out in (("roofline_frac", "roofline_frac"),
                             ("attn_frac_of_bf16_peak", "roofline_frac"),
                             ("attn_TFLOPs", "TFLOPs"), ("attn_GBps", "GBps")):
                if key in v:
                    summary[k][out] = round(v[key], 4 if "frac" in key else 1)
        elif "ms_per_step" in v:
            summary[k] = {"ms_per_step": round(v["ms_per_step"], 5)}
            for key in ("frac_of_hbm", "union_ms", "blocksparse_ms"):
                if key in v:
                    summary[k][key] = round(v[key], 5)
    line["summary"] = summary
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The fp64 CPU oracle, as it stands, on the host cores: each step a bounded sample of
    the workload (rank 0 only)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    name = args.workload
    batch, mask = make_workload(name)
    table = count = None
    if mask is not None:
        from oracle import rpa_oracle as orc
        table, count = orc.build_group_tables(mask, batch.num_kv_heads)
    per_step = max(0.2, min(1.5, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_oracle_baseline(name, batch, target_s=per_step, table=table, count=count)
    tot_bytes = tot_s = 0.0
    last = None
    for _ in range(args.steps):
        last = cpu_oracle_baseline(name, batch, target_s=per_step, table=table, count=count)
        tot_bytes += last["bytes"]
        tot_s += last["elapsed_s"]
    value = tot_bytes / tot_s / 1e9
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot_s / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD_TEXT[name]},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": last["threads"],
                             "kind": "oracle", "sample": last["sample"]},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


CASES = {
    "input_pass": measure_input_pass,
    "decode_kv8": measure_decode_kv8,
    "mixed_kv8": measure_mixed_kv8,
    "prefill_kv8": measure_prefill_kv8,
    "sparse_ablation": measure_sparse_ablation,
    "decode_device_planned": measure_device_planned_decode,
    "decode_kv8_device_planned": measure_device_planned_decode_kv8,
}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="decode", choices=list(WORKLOAD_TEXT))
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--case", default=None, choices=list(CASES),
                    help="time one secondary measurement alone and print its result as one "
                         "JSON line (for launch lists and profiler captures of that case)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.case is not None:
        if not torch.cuda.is_available():
            raise SystemExit("--case needs a CUDA device")
        res = CASES[args.case](args.steps, args.warmup, load_peaks()[0])
        print(json.dumps({"case": args.case, **res}))
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
