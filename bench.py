"""Benchmark: blocked attention with softmax thresholding on B200.

One step = one prefill pass (the library's prefill kernel) over the 32K-token
Llama-3.1-8B-shaped workload (B=1, Hq=32, Hkv=8, d=128, causal, Br=Bc=128,
lambda=1e-3, literal planted-structure generator). `value` is the effective
(dense-equivalent causal) attention TFLOP/s of the whole job, device-timed with
CUDA events; inputs are larger than L2 and L2 is also flushed between steps.

Also reported on the same line: executed TFLOP/s and the tensor roofline of
the prefill kernel, the skip fraction, the lambda = 0 time and the speedup
over it, the same for the calibrated (amplitude 12) structured variant, the
128K prefill, the split-KV decode (GB/s against the HBM roofline), an
end-to-end number through the public API with pinned host buffers, and the
CPU oracle timed on a bounded sample as the CPU baseline.

`--impl reference` times the CPU oracle (the method's plain fp64
restatement) on the same metric and workload, on a bounded sample per step.

Multi-GPU (`--gpus N` under torchrun): the method runs on one GPU and nothing
is exchanged, so each rank runs an independent replica of the workload
(weak scaling); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention effective TFLOP/s & skip % at 32K/128K prefill; decode GB/s"
UNIT = "TFLOP/s"
WORKLOAD = "prefill_32k"
LAMBDA = 1e-3
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------- helpers
def causal_pairs(Lq, Lkv):
    off = Lkv - Lq
    # sum over rows i of min(Lkv, i + off + 1)
    i = np.arange(Lq, dtype=np.int64)
    return int(np.minimum(Lkv, i + off + 1).sum())


def effective_flops(w):
    pairs = causal_pairs(w.Lq, w.Lkv) if w.causal else w.Lq * w.Lkv
    return 4.0 * w.B * w.Hq * w.d * pairs


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


KERNEL_SOURCES = {
    "prefill_32k": ("prefill_sm100.cuh", "ptx_sm100.cuh"),
    "decode_64k": ("decode_sm100.cuh", "ptx_sm100.cuh"),
    "backward_32k": ("bwd_sm100.cuh", "ptx_sm100.cuh"),
    "decode_mla_64k": ("decode_mla_sm100.cuh", "ptx_sm100.cuh"),
}


def code_only(text):
    """C/C++ source without its comments and empty lines, runs of blanks as
    one, so that an edit of the comments or the layout leaves a kernel's hash
    as it was."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"\s+", " ", re.sub(r"//.*$", "", ln)).strip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def kernel_source_hash(kernel_key):
    """Hash of the code (comments stripped) of the source files that make up
    one kernel."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "dynamic_block_sparse_tiled_b200", "csrc")
    for name in KERNEL_SOURCES[kernel_key]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode())
            h.update(code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key):
    """dram bytes per launch recorded from an ncu capture of the current
    kernel sources (profiles/traffic.txt: `key source_hash bytes`), else None."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    cur = kernel_source_hash(kernel_key)
    with open(p) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and parts[0] == kernel_key and parts[1] == cur:
                return float(parts[2])
    return None


class ClockSampler:
    """nvidia-smi samples (every 50 ms) of SM clock and throttle reasons while
    running, each with nvidia-smi's own wall-clock timestamp, so a summary
    can be taken over the time windows of one measurement leg. Entering
    waits for the first sample so the record covers the timed work."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.samples = []  # (wall time, sm MHz, max MHz, set of active reasons)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            t0 = time.monotonic()
            while not self.samples and time.monotonic() - t0 < 10.0 and self.proc.poll() is None:
                time.sleep(0.01)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    @classmethod
    def parse(cls, line, t_read):
        """One csv line -> (wall time, sm MHz, max MHz, reasons) or None."""
        import datetime
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 8:
            return None
        try:
            t = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            t = t_read
        try:
            sm, mx = float(parts[1]), float(parts[2])
        except ValueError:
            return None
        reasons = {n for n, v in zip(cls.REASONS, parts[4:8]) if v.lower() == "active"}
        return (t, sm, mx, reasons)

    def _read(self):
        for line in self.proc.stdout:
            s = self.parse(line, time.time())
            if s is not None:
                self.samples.append(s)

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, windows=None):
        """Median SM clock, max clock and active reasons over the samples that
        fall inside any of `windows` ([(t0, t1)] in time.time() units; all
        samples when None)."""
        sel = [s for s in self.samples
               if windows is None or any(a <= s[0] <= b for a, b in windows)]
        if not sel:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=[], samples=0)
        reasons = set()
        for s in sel:
            reasons |= s[3]
        return dict(sm_mhz=statistics.median(s[1] for s in sel),
                    sm_max_mhz=max(s[2] for s in sel), reasons=sorted(reasons), samples=len(sel))


# ------------------------------------------------------------- GPU side
class Prefill:
    """Device-resident inputs + outputs for one prefill workload."""

    def __init__(self, w, device):
        import torch
        import synth
        self.w = w
        self.torch = torch
        inp = synth.generate(w)
        self.host = inp
        to = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        self.q, self.k, self.v = to(inp.q), to(inp.k), to(inp.v)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32, device=device)
        self.mask = torch.empty((w.B, w.Hq, -(-w.Lq // w.Br), -(-w.Lkv // w.Bc)), dtype=torch.uint8,
                                device=device)

    def run(self, lam, stats=None, stream=None, block_mask=None):
        import dynamic_block_sparse_tiled_b200 as bl
        bl.blasst_fwd_ex(self.q, self.k, self.v, self.o, self.lse, causal=self.w.causal, lam=lam,
                         Br=self.w.Br, Bc=self.w.Bc, skip_mask_out=self.mask, stats_out=stats,
                         stream=stream, block_mask_in=block_mask)


def flush_l2(buf, stream=None):
    """Write a buffer twice the size of L2. On the timed stream: torch's
    side streams do not synchronise with its default stream, so a flush
    issued there would overlap the timed call instead of preceding it."""
    import torch
    if stream is None:
        buf.add_(1)
    else:
        with torch.cuda.stream(stream):
            buf.add_(1)


def time_calls(fn, steps, warmup, stream, flush_buf):
    """Device time (ms) of each call, L2 flushed before each one."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        flush_l2(flush_buf, stream)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    return times


def time_interleaved(arms, rounds, per, warmup, stream, flush_buf):
    """Device time of several arms (same kernel, different settings) measured
    as interleaved blocks: each round times `per` calls of every arm, and
    the arm order alternates between rounds (A B, B A, A B, ...), so a drift
    of clocks or power over the run affects every arm alike. Returns, per
    arm key, the mean of each block (ms) and each block's wall-clock window
    (for the clock record)."""
    import torch
    for _, fn in arms:
        for _ in range(warmup):
            fn()
    torch.cuda.synchronize()
    out = {k: dict(block_ms=[], windows=[]) for k, _ in arms}
    for r in range(rounds):
        for k, fn in (arms if r % 2 == 0 else arms[::-1]):
            t0 = time.time()
            ts = time_calls(fn, per, 0, stream, flush_buf)
            out[k]["block_ms"].append(statistics.mean(ts))
            out[k]["windows"].append((t0, time.time()))
    return out


def kernel_mhz(sd):
    """Mean SM clock while the kernel ran, from its own telemetry (summed CTA
    cycles over summed CTA nanoseconds), or None where the call has none."""
    cyc, ns = sd.get("sm_cycles", 0), sd.get("sm_ns", 0)
    return cyc / ns * 1e3 if cyc > 0 and ns > 0 else None


def arm_summary(t, clk, k_mhz=None):
    """Median block time, the median SM clock over the arm's blocks, and the
    clock-normalised time (ms x MHz = thousands of cycles). With the kernel's
    own clock (``k_mhz``) the cycles use it: the nvidia-smi sampler (every 50
    ms) can miss short blocks or sample between calls."""
    ms = statistics.median(t["block_ms"])
    c = clk.summary(t["windows"]) if clk is not None else dict(sm_mhz=None, reasons=[])
    mhz = k_mhz or c["sm_mhz"]
    kcyc = ms * mhz if mhz else None
    return dict(ms=ms, ms_blocks=t["block_ms"], sm_mhz=c["sm_mhz"], reasons=c["reasons"],
                kernel_mhz=k_mhz, kcycles=kcyc)


def speedups(res, base_key):
    """Speedup of every arm over the base arm: plain and clock-normalised."""
    b = res[base_key]
    for v in res.values():
        v["speedup_vs_lambda0"] = b["ms"] / v["ms"]
        v["speedup_clk"] = (b["kcycles"] / v["kcycles"]) if (b["kcycles"] and v["kcycles"]) else None


def measure_prefill(w, lam, steps, warmup, device, stream, flush_buf, pre=None, block_mask=None):
    import dynamic_block_sparse_tiled_b200 as bl
    pre = pre or Prefill(w, device)
    st = bl.new_stats(device)
    pre.run(lam, stats=st, stream=stream, block_mask=block_mask)
    stream.synchronize()
    rc = bl.blasst_check(stream)
    if rc != 0:
        raise RuntimeError(bl.blasst_status_string(rc))
    sd = bl.stats_dict(st)
    kst = bl.new_stats(device)  # the timed calls' own SM cycles and nanoseconds
    times = time_calls(lambda: pre.run(lam, stream=stream, block_mask=block_mask, stats=kst),
                       steps, warmup, stream, flush_buf)
    mask = pre.mask.cpu().numpy()
    vis = int((mask != 2).sum())
    skip = int((mask == 1).sum())
    return pre, dict(ms=statistics.mean(times), ms_min=min(times), times=times,
                     kernel_mhz=kernel_mhz(bl.stats_dict(kst)),
                     exec_flops=float(sd["mma_flops"]), eff_flops=effective_flops(w),
                     skip_frac=skip / max(vis, 1), tiles_visited=vis, tiles_skipped=skip,
                     v_blocks=sd["v_blocks_loaded"], bytes_loaded=sd["bytes_loaded"])


def measure_decode_mla(w, steps, device, stream, flush_buf, peaks, Bc=64):
    """MLA decode at lambda = 0 and at the workload's lambda: time, executed
    TFLOP/s against the bf16 peak, bytes against the copy bandwidth."""
    import torch
    import synth
    import dynamic_block_sparse_tiled_b200 as bl
    inp = synth.generate(w)
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    q, c = to(inp.q[:, :, 0, :]), to(inp.k[:, 0])
    del inp
    ws = torch.empty(bl.blasst_decode_mla_workspace_bytes(w.B, w.Hq, w.num_splits), dtype=torch.uint8,
                     device=device)
    o = torch.empty((w.B, w.Hq, 512), dtype=torch.bfloat16, device=device)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=device)
    mask = torch.empty((w.B, w.Hq, -(-w.Lkv // Bc)), dtype=torch.uint8, device=device)
    res = {}
    for lam in (0.0, w.lambdas[0]):
        st = bl.new_stats(device)
        bl.blasst_decode_mla(q, c, o, lse, lam=lam, Bc=Bc, num_splits=w.num_splits, workspace=ws,
                             skip_mask_out=mask, stats_out=st, stream=stream)
        stream.synchronize()
        rc = bl.blasst_check(stream)
        if rc != 0:
            raise RuntimeError(bl.blasst_status_string(rc))
        sd = bl.stats_dict(st)
        run = lambda: bl.blasst_decode_mla(q, c, o, lse, lam=lam, Bc=Bc, num_splits=w.num_splits,
                                           workspace=ws, stream=stream)
        ms = statistics.mean(time_calls(run, steps, 3, stream, flush_buf))
        tf = sd["mma_flops"] / (ms * 1e-3) / 1e12
        # algorithmic flops: every visited block's scores once (2 H 64 576),
        # its P V (2 H 64 512) when some head keeps it. The tensor-core
        # kernel forms each score in both CTAs of a pair (the executed count
        # holds it twice); the mma.sync kernel executes exactly these.
        alg_fl = sd["mma_flops"] - (sd["tiles_visited"] * 2 * 64 * 576 if w.Hq % 128 == 0 else 0)
        gbs = sd["bytes_loaded"] / (ms * 1e-3) / 1e9
        res[str(lam)] = dict(ms=ms, executed_tflops=tf, algorithmic_tflops=alg_fl / (ms * 1e-3) / 1e12,
                             gbs=gbs, skip_frac=sd["tiles_skipped"] / max(sd["tiles_visited"], 1))
    base = res["0.0"]["ms"]
    for v in res.values():
        v["speedup_vs_lambda0"] = base / v["ms"]
    top = res[str(w.lambdas[0])]
    # algorithmic bytes of one call: the cache once, the queries, the split
    # partials (O and lse) written by the decode kernel and read by the merge,
    # the merged O and lse
    alg = (w.B * w.Lkv * 576 * 2 + w.B * w.Hq * 576 * 2 + 2 * w.B * w.Hq * w.num_splits * 513 * 4
           + w.B * w.Hq * (512 * 2 + 4))
    hbm_gbs = alg / (top["ms"] * 1e-3) / 1e9
    t_hbm = alg / (peaks["hbm_gbs"] * 1e9)
    t_tc = top["algorithmic_tflops"] / peaks["bf16_tflops"] * top["ms"] * 1e-3
    common = dict(l2_to_sm_gbs=top["gbs"], executed_tflops=top["executed_tflops"],
                  tensor_frac=top["algorithmic_tflops"] / peaks["bf16_tflops"],
                  hbm_frac=hbm_gbs / peaks["hbm_gbs"], algorithmic_bytes=int(alg),
                  traffic=profiled_traffic("decode_mla_64k") if w.name == "decode_mla_64k" else None,
                  note=("tcgen05, 128 heads: two CTAs per (sequence, split), each forms the "
                        "full 576-wide scores and accumulates one 256-column half of the output, "
                        "so the score product runs twice; the call also holds the split merge")
                  if w.Hq % 128 == 0 else
                       ("mma.sync m16n8k16 tiles (16 heads per CTA); the cache is read once from "
                        "HBM, re-read from L2 by each head group"))
    if t_hbm >= t_tc:
        res["roofline"] = dict(bound="hbm", achieved=hbm_gbs, peak=peaks["hbm_gbs"], unit="GB/s",
                               frac=hbm_gbs / peaks["hbm_gbs"], **common)
    else:
        res["roofline"] = dict(bound="tensor", achieved=top["algorithmic_tflops"],
                               peak=peaks["bf16_tflops"], unit="TFLOP/s",
                               frac=top["algorithmic_tflops"] / peaks["bf16_tflops"], **common)
    res["config"] = dict(B=w.B, H=w.Hq, L=w.Lkv, num_splits=w.num_splits, amplitude=w.amp, Bc=Bc)
    return res


def backward_pairs(w, mask):
    """(64-row query tile, 128-key block) pairs the backward computes, from
    the forward's decisions (uint8 [B, Hq, nQt, nKt], 0 = computed)."""
    nT = -(-w.Lq // 64)
    nKb = -(-w.Lkv // 128)
    t = np.arange(nT)
    j = np.arange(nKb)
    qf = (t * 64) // w.Br
    keep = mask == 0                                      # [B, Hq, nQt, nKt]
    if w.Bc == 128:
        kb = keep[:, :, qf][:, :, :, j]
    else:
        k0 = keep[:, :, qf][:, :, :, 2 * j]
        j1 = np.minimum(2 * j + 1, keep.shape[-1] - 1)
        k1 = keep[:, :, qf][:, :, :, j1] & ((2 * j + 1) < keep.shape[-1])[None, None, None, :]
        kb = k0 | k1
    if w.causal:
        vis = (j[None, :] * 128) <= (t[:, None] * 64 + 63 + (w.Lkv - w.Lq))
        kb = kb & vis[None, None]
    return int(kb.sum())


BWD_FLOPS_PER_PAIR = 5 * 2 * 128 * 64 * 128  # S^T, dP^T, dV, dK, dQ^T products
SEL_TAU, SEL_GAMMA = 0.2, 0.9  # selector route threshold and pooled-path coverage


class Backward:
    """Device-resident dO, gradients and workspace for the backward of a
    prefill workload (the forward's outputs come from ``pre``)."""

    def __init__(self, pre, device):
        import torch
        import synth
        import dynamic_block_sparse_tiled_b200 as bl
        w = pre.w
        self.pre = pre
        self.do = torch.from_numpy(synth.grad_output(w).view(np.int16)).view(torch.bfloat16).to(device)
        self.dq = torch.empty((w.B, w.Hq, w.Lq, w.d), dtype=torch.float32, device=device)
        self.dk = torch.empty((w.B, w.Hkv, w.Lkv, w.d), dtype=torch.float32, device=device)
        self.dv = torch.empty_like(self.dk)
        self.ws = torch.empty(bl.blasst_bwd_workspace_bytes(w.B, w.Hq, w.Lq), dtype=torch.uint8,
                              device=device)

    def run(self, stream=None):
        import dynamic_block_sparse_tiled_b200 as bl
        p, w = self.pre, self.pre.w
        bl.blasst_bwd(p.q, p.k, p.v, p.o, self.do, p.lse, self.dq, self.dk, self.dv,
                      causal=w.causal, Br=w.Br, Bc=w.Bc, workspace=self.ws, skip_mask=p.mask,
                      stream=stream)


def measure_backward(w, lam, steps, warmup, device, stream, flush_buf, pre=None, bwd=None):
    """Forward once at ``lam`` (its O, lse and decisions), then time the
    backward with those decisions."""
    import dynamic_block_sparse_tiled_b200 as bl
    pre = pre or Prefill(w, device)
    pre.run(lam, stream=stream)
    bwd = bwd or Backward(pre, device)
    bwd.run(stream=stream)
    stream.synchronize()
    rc = bl.blasst_check(stream)
    if rc != 0:
        raise RuntimeError(bl.blasst_status_string(rc))
    times = time_calls(lambda: bwd.run(stream=stream), steps, warmup, stream, flush_buf)
    mask = pre.mask.cpu().numpy()
    pairs = backward_pairs(w, mask)
    ms = statistics.mean(times)
    flops = pairs * BWD_FLOPS_PER_PAIR
    return pre, bwd, dict(ms=ms, times=times, pairs=pairs, exec_flops=float(flops),
                          executed_tflops=flops / (ms * 1e-3) / 1e12,
                          skip_frac=float((mask == 1).sum()) / max(int((mask != 2).sum()), 1))


class E2EPipeline:
    """Prefill steps through the public API from pinned host buffers, as a
    serving loop runs them: every step uploads its inputs (Q, K, V) host ->
    device, runs the prefill and reads its results (O, lse) back device ->
    host. An upload stream, the compute stream and a readback stream work
    over two sets of device buffers, and each step goes in chunks of one KV
    head group (its g query heads and one K / V head; contiguous slices when
    B = 1), each its own prefill call: the upload of the next chunk and the
    readback of the previous one overlap the prefill of a chunk (the PCIe
    link carries both directions at once), so the pipeline fills and drains
    in one chunk's copies rather than a whole step's. Every step processes
    the same synthetic batch."""

    def __init__(self, w, lam, device, stream):
        import torch
        import synth
        self.w, self.lam, self.stream = w, lam, stream
        self.hq = torch.empty((w.B, w.Hq, w.Lq, w.d), dtype=torch.int16, pin_memory=True)
        self.hk = torch.empty((w.B, w.Hkv, w.Lkv, w.d), dtype=torch.int16, pin_memory=True)
        self.hv = torch.empty_like(self.hk, pin_memory=True)
        synth.generate(w, out_q=self.hq.numpy().view(np.uint16),
                       out_k=self.hk.numpy().view(np.uint16), out_v=self.hv.numpy().view(np.uint16))
        self.dev = [dict(q=torch.empty(self.hq.shape, dtype=torch.bfloat16, device=device),
                         k=torch.empty(self.hk.shape, dtype=torch.bfloat16, device=device),
                         v=torch.empty(self.hv.shape, dtype=torch.bfloat16, device=device),
                         o=torch.empty(self.hq.shape, dtype=torch.bfloat16, device=device),
                         lse=torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32, device=device))
                    for _ in range(2)]
        self.host_out = [dict(o=torch.empty(self.hq.shape, dtype=torch.int16, pin_memory=True),
                              lse=torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32,
                                              pin_memory=True))
                         for _ in range(2)]
        self.up = torch.cuda.Stream(device)
        self.down = torch.cuda.Stream(device)
        self.h2d_bytes = (self.hq.numel() + self.hk.numel() + self.hv.numel()) * 2
        self.d2h_bytes = self.host_out[0]["o"].numel() * 2 + self.host_out[0]["lse"].numel() * 4
        g = w.Hq // w.Hkv
        # (query heads, KV heads) of each chunk: one KV head group each when the
        # slices are contiguous (B = 1), else the whole step
        self.chunks = ([(slice(h * g, (h + 1) * g), slice(h, h + 1)) for h in range(w.Hkv)]
                       if w.B == 1 else [(slice(0, w.Hq), slice(0, w.Hkv))])

    def run(self, n, start_event=None):
        """Enqueue n steps; on return the compute stream waits for the last
        readback (record an event on it to time or join the steps)."""
        import torch
        import dynamic_block_sparse_tiled_b200 as bl
        w, stream, up, down = self.w, self.stream, self.up, self.down
        if start_event is not None:
            up.wait_event(start_event)
            down.wait_event(start_event)
        nc = len(self.chunks)
        computed = [[None] * nc, [None] * nc]  # last prefill of chunk c in buffer set b
        read = [[None] * nc, [None] * nc]      # last readback of chunk c of set b
        for i in range(n):
            b = i % 2
            d, h = self.dev[b], self.host_out[b]
            for c, (qs, ks) in enumerate(self.chunks):
                if computed[b][c] is not None:  # step i-2 has finished reading these inputs
                    up.wait_event(computed[b][c])
                with torch.cuda.stream(up):
                    d["q"][:, qs].view(torch.int16).copy_(self.hq[:, qs], non_blocking=True)
                    d["k"][:, ks].view(torch.int16).copy_(self.hk[:, ks], non_blocking=True)
                    d["v"][:, ks].view(torch.int16).copy_(self.hv[:, ks], non_blocking=True)
                uploaded = torch.cuda.Event()
                uploaded.record(up)
                stream.wait_event(uploaded)
                if read[b][c] is not None:      # step i-2's results have been read back
                    stream.wait_event(read[b][c])
                bl.blasst_fwd_ex(d["q"][:, qs], d["k"][:, ks], d["v"][:, ks], d["o"][:, qs],
                                 d["lse"][:, qs], causal=w.causal, lam=self.lam, Br=w.Br,
                                 Bc=w.Bc, stream=stream)
                computed[b][c] = torch.cuda.Event()
                computed[b][c].record(stream)
                down.wait_event(computed[b][c])
                with torch.cuda.stream(down):
                    h["o"][:, qs].copy_(d["o"][:, qs].view(torch.int16), non_blocking=True)
                    h["lse"][:, qs].copy_(d["lse"][:, qs], non_blocking=True)
                read[b][c] = torch.cuda.Event()
                read[b][c].record(down)
        for evs in read:
            for ev in evs:
                if ev is not None:
                    stream.wait_event(ev)


def measure_e2e(w, lam, steps, warmup, device, stream):
    """Same metric through the public API from pinned host buffers (see
    E2EPipeline): every step's upload and readback inside the timed region,
    which opens before the first upload and closes after the last readback,
    so the pipeline's fill and drain are timed too."""
    import torch
    pipe = E2EPipeline(w, lam, device, stream)
    pipe.run(warmup)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    pipe.run(steps, start_event=e0)
    e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1) / steps
    return dict(value=effective_flops(w) / (ms * 1e-3) / 1e12, unit=UNIT, ms=ms,
                h2d_bytes_per_step=int(pipe.h2d_bytes), d2h_bytes_per_step=int(pipe.d2h_bytes),
                steps=steps,
                chunks=len(pipe.chunks),
                pipelined=("each step in chunks of one KV head group, one prefill call each: the "
                           "next chunk's upload and the previous chunk's readback overlap a chunk's "
                           "prefill (three streams, two device buffer sets); fill and drain timed"))


def block_sparse_pattern(w, sink_blocks=1, band_blocks=8, random_frac=0.1, seed=0):
    """A static block mask shaped like a pre-pass selector's output: every
    query tile keeps the first `sink_blocks` KV blocks, a band of
    `band_blocks` blocks ending at its diagonal, and a seeded random fraction
    of the rest; everything else is excluded (mask 1)."""
    nQt, nKt = -(-w.Lq // w.Br), -(-w.Lkv // w.Bc)
    rng = np.random.default_rng(seed)
    keep = rng.random((w.B, w.Hq, nQt, nKt)) < random_frac
    keep[..., :sink_blocks] = True
    off = w.Lkv - w.Lq
    for qt in range(nQt):
        diag = min(nKt - 1, (min(qt * w.Br + w.Br, w.Lq) - 1 + off) // w.Bc)
        keep[:, :, qt, max(0, diag - band_blocks + 1):diag + 1] = True
    return (~keep).astype(np.uint8)


# ------------------------------------------------------------ lambda legs
def prefill_lambda_leg(w, lams, rounds, per, device, stream, flush_buf, clk, peaks, pre=None):
    """One prefill workload at several lambdas: decisions and counters from
    one call each, then the lambdas timed as interleaved blocks. Reports the
    skip fraction (for workloads with diffuse heads also split into the
    structured and the diffuse heads), executed and effective TFLOP/s, the
    executed fraction of the bf16 peak, and the speedup over lambda = 0,
    plain and clock-normalised."""
    import dynamic_block_sparse_tiled_b200 as bl
    own = pre is None
    pre = pre or Prefill(w, device)
    res = {}
    for lam in lams:
        st = bl.new_stats(device)
        pre.run(lam, stats=st, stream=stream)
        stream.synchronize()
        rc = bl.blasst_check(stream)
        if rc != 0:
            raise RuntimeError(bl.blasst_status_string(rc))
        sd = bl.stats_dict(st)
        m = pre.mask.cpu().numpy()
        vis = m != 2
        r = dict(skip_frac=float((m == 1).sum()) / max(int(vis.sum()), 1),
                 exec_flops=float(sd["mma_flops"]), v_blocks=sd["v_blocks_loaded"])
        if w.diffuse_heads == "upper_half":
            h = w.Hq // 2  # query heads of the diffuse KV heads (contiguous GQA groups)
            r["skip_frac_structured"] = float((m[:, :h] == 1).sum()) / max(int(vis[:, :h].sum()), 1)
            r["skip_frac_diffuse"] = float((m[:, h:] == 1).sum()) / max(int(vis[:, h:].sum()), 1)
        res[lam] = r
    kst = {lam: bl.new_stats(device) for lam in lams}
    t = time_interleaved([(lam, (lambda lam=lam: pre.run(lam, stream=stream, stats=kst[lam])))
                          for lam in lams], rounds, per, 2, stream, flush_buf)
    eff = effective_flops(w)
    for lam in lams:
        r = res[lam]
        r.update(arm_summary(t[lam], clk, kernel_mhz(bl.stats_dict(kst[lam]))))
        r["executed_tflops"] = r["exec_flops"] / (r["ms"] * 1e-3) / 1e12
        r["effective_tflops"] = eff / (r["ms"] * 1e-3) / 1e12
        r["frac"] = r["executed_tflops"] / peaks["bf16_tflops"]
    speedups(res, lams[0])
    if own:
        del pre
    return res


def decode_lambda_leg(w, lam, rounds, per, device, stream, flush_buf, clk, peaks):
    """Split-KV decode at lambda = 0 and at `lam`, interleaved: the fraction
    of (group, block) V fetches made, the bytes the skipped fetches save, and
    the HBM roofline on the bytes each call actually moves."""
    import torch
    import dynamic_block_sparse_tiled_b200 as bl
    import synth
    inp = synth.generate(w)
    to = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    q, k, v = to(inp.q), to(inp.k), to(inp.v)
    del inp
    ws = torch.empty(bl.blasst_decode_workspace_bytes(w.B, w.Hq, w.d, w.num_splits),
                     dtype=torch.uint8, device=device)
    o = torch.empty((w.B, w.Hq, 1, w.d), dtype=torch.bfloat16, device=device)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=device)
    mask = torch.empty((w.B, w.Hq, -(-w.Lkv // w.Bc)), dtype=torch.uint8, device=device)
    lams = (0.0, lam)
    res = {}
    for lm in lams:
        st = bl.new_stats(device)
        bl.blasst_decode(q, k, v, o, lse, lam=lm, Bc=w.Bc, num_splits=w.num_splits, workspace=ws,
                         skip_mask_out=mask, stats_out=st, stream=stream)
        rc = bl.blasst_check(stream)
        if rc != 0:
            raise RuntimeError(bl.blasst_status_string(rc))
        sd = bl.stats_dict(st)
        m = mask.cpu().numpy()
        # algorithmic bytes: K always, V when some head of the group keeps the
        # block, the split partials written then read back by the merge, q, o
        alg = sd["bytes_loaded"] + 2 * ws.numel() + q.numel() * 2 + o.numel() * 2
        res[lm] = dict(bytes=int(alg), skip_frac=float((m == 1).mean()),
                       v_blocks=sd["v_blocks_loaded"],
                       v_fetch_frac=sd["v_blocks_loaded"] / max(1, w.B * w.Hkv * (-(-w.Lkv // w.Bc))))
    t = time_interleaved(
        [(lm, (lambda lm=lm: bl.blasst_decode(q, k, v, o, lse, lam=lm, Bc=w.Bc,
                                              num_splits=w.num_splits, workspace=ws,
                                              stream=stream))) for lm in lams],
        rounds, per, 3, stream, flush_buf)
    for lm in lams:
        r = res[lm]
        r.update(arm_summary(t[lm], clk))
        r["gbs"] = r["bytes"] / (r["ms"] * 1e-3) / 1e9
        r["frac"] = r["gbs"] / peaks["hbm_gbs"]
    speedups(res, 0.0)
    res[lam]["bytes_saved"] = res[0.0]["bytes"] - res[lam]["bytes"]
    return res


def _r(x, n=3):
    """Round for the compact summary line (None passes through)."""
    if x is None:
        return None
    if isinstance(x, float):
        if x == 0.0 or not math.isfinite(x):
            return x
        return float(f"{x:.{n}g}")
    return x


# ------------------------------------------------------------- CPU oracle
def oracle_sample(w, lam, budget_s, seed=0, inputs=None):
    """Time the CPU oracle on a seeded sample of query tiles of workload w,
    sized to about budget_s seconds. Returns effective TFLOP/s of the sample."""
    import oracle
    import synth
    inp = inputs or synth.generate(w)
    nQt = -(-w.Lq // w.Br)
    n_all = w.B * w.Hq * nQt
    rng = np.random.default_rng(seed)
    order = rng.permutation(n_all)

    def eff_of(items):
        tot = 0
        for it in items:
            qt = it % nQt
            r0, r1 = qt * w.Br, min(qt * w.Br + w.Br, w.Lq)
            off = w.Lkv - w.Lq
            rows = np.arange(r0, r1)
            tot += int(np.minimum(w.Lkv, rows + off + 1).sum()) if w.causal else (r1 - r0) * w.Lkv
        return 4.0 * w.d * tot

    nthreads = os.cpu_count() or 1
    # calibrate on a small batch, then run the sized sample
    cal = order[: max(2, nthreads)]
    t0 = time.perf_counter()
    oracle.prefill(inp.q, inp.k, inp.v, causal=w.causal, lam=lam, Br=w.Br, Bc=w.Bc, items=cal)
    tc = time.perf_counter() - t0
    n = int(min(n_all, max(len(cal), len(cal) * budget_s / max(tc, 1e-3))))
    items = order[:n]
    t0 = time.perf_counter()
    oracle.prefill(inp.q, inp.k, inp.v, causal=w.causal, lam=lam, Br=w.Br, Bc=w.Bc, items=items)
    dt = time.perf_counter() - t0
    return dict(value=eff_of(items) / dt / 1e12, unit=UNIT, cores=nthreads, kind="oracle",
                seconds=dt, sample=f"{n} of {n_all} query tiles of {w.name} (seeded), lambda={lam}")


# ------------------------------------------------------------------ main
def run_case(name, lam, calls, overrides=()):
    """Launch one workload's kernel `calls` times with nothing else on the
    GPU (the command an ncu capture wraps); exits non-zero on a device error.
    `overrides` are "field=value" strings applied to the named workload."""
    import torch
    import synth
    import dynamic_block_sparse_tiled_b200 as bl
    ncalls = calls
    backward = name.startswith("backward:")
    select = name.startswith("select:")
    if backward or select:
        name = name.split(":", 1)[1]
    w = synth.CONFIGS[name]
    for ov in overrides:
        key, val = ov.split("=", 1)
        cur = getattr(w, key)
        w = w.replace(**{key: type(cur)(val) if not isinstance(cur, bool) else val == "1"})
    inp = synth.generate(w)
    if w.dtype == "bf16":
        to = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    else:
        to = lambda a: torch.from_numpy(a).cuda()
    q, k, v = to(inp.q), to(inp.k), to(inp.v)
    del inp
    if w.num_splits and w.d == 576:  # MLA-shaped decode: one latent head, values = dims 0-511
        qm, cm = q[:, :, 0, :].contiguous(), k[:, 0].contiguous()
        del q, k, v
        for _ in range(calls):
            bl.attention_decode_mla(qm, cm, lam=lam, num_splits=w.num_splits)
        calls = 0
    if select:
        for _ in range(calls):
            bl.select_blocks(q, k, causal=w.causal, Br=w.Br, Bc=w.Bc, tau=SEL_TAU, gamma=SEL_GAMMA)
        calls = 0
    if backward:
        o, lse, mask = bl.attention_prefill(q, k, v, causal=w.causal, lam=lam, Br=w.Br, Bc=w.Bc,
                                            with_mask=True)
        do = torch.from_numpy(synth.grad_output(w).view(np.int16)).view(torch.bfloat16).cuda()
        for _ in range(calls):
            bl.attention_backward(q, k, v, o, lse, do, causal=w.causal, Br=w.Br, Bc=w.Bc,
                                  skip_mask=mask)
        calls = 0
    for _ in range(calls):
        if w.num_splits:
            bl.attention_decode(q, k, v, lam=lam, Bc=w.Bc, num_splits=w.num_splits)
        else:
            bl.attention_prefill(q, k, v, causal=w.causal, lam=lam, Br=w.Br, Bc=w.Bc)
    torch.cuda.synchronize()
    rc = bl.blasst_check()
    print(json.dumps(dict(case=("backward:" if backward else "select:" if select else "") + name,
                          calls=ncalls,
                          status=bl.blasst_status_string(rc))), flush=True)
    return 0 if rc == 0 else 1


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class Ranks:
    """Host plumbing of the replicas (one process per GPU, nothing exchanged on
    the data path): a barrier with device synchronisation on both sides, and
    device times combined as the maximum over ranks. Every rank makes the same
    calls in the same order."""

    def __init__(self, backend, device):
        self.ws, self.rank, self.local = dist_env()
        self.device = device
        self.cuda = device.type == "cuda"
        if self.ws > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))

    def _sync(self):
        if self.cuda:
            import torch
            torch.cuda.synchronize(self.device)

    def barrier(self):
        self._sync()
        if self.ws > 1:
            import torch.distributed as dist
            dist.barrier()
        self._sync()

    def max(self, x):
        if self.ws == 1:
            return float(x)
        import torch
        import torch.distributed as dist
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def aggregate(self, units_per_rank, ms_per_rank):
        """Whole-job rate: the units all ranks processed over the slowest
        rank's time (units per second)."""
        return self.ws * units_per_rank / (self.max(ms_per_rank) * 1e-3)

    def close(self):
        if self.ws > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


def run_reference(args):
    import synth
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    w = synth.CONFIGS[WORKLOAD]
    inp = synth.generate(w)
    budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(w, LAMBDA, budget / 4, inputs=inp)
    vals, secs = [], []
    for s in range(args.steps):
        r = oracle_sample(w, LAMBDA, budget, seed=s, inputs=inp)
        vals.append(r["value"])
        secs.append(r["seconds"])
    value = statistics.mean(vals)
    line = dict(metric=METRIC, value=value, unit=UNIT, n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=1e3 * statistics.mean(secs), higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                impl="reference",
                config=dict(workload=w.name, B=w.B, Hq=w.Hq, Hkv=w.Hkv, seq_len=w.Lq, d=w.d,
                            causal=w.causal, Br=w.Br, Bc=w.Bc, **{"lambda": LAMBDA},
                            amplitude=w.amp),
                cpu_baseline=dict(value=value, unit=UNIT, cores=r["cores"], kind="oracle",
                                  sample=r["sample"]),
                e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)
    return 0


def leg_static_mask(w, args, device, stream, flush_buf):
    """Static block-sparse input (a selector-shaped mask) on the 32K workload."""
    import torch
    sm_dev = torch.from_numpy(block_sparse_pattern(w)).to(device)
    ps = Prefill(w, device)
    steps = max(3, args.steps // 2)
    ps, s_r = measure_prefill(w, LAMBDA, steps, 3, device, stream, flush_buf, pre=ps,
                              block_mask=sm_dev)
    _, s0_r = measure_prefill(w, LAMBDA, steps, 3, device, stream, flush_buf, pre=ps)
    nvis = s_r["tiles_visited"]
    return dict(pattern="first block + 8-block diagonal band + 10 % seeded random blocks per "
                        "query tile", visited_tiles=nvis,
                visited_frac_of_causal=nvis / max(1, s0_r["tiles_visited"]),
                ms=s_r["ms"], ms_no_mask=s0_r["ms"], speedup_vs_no_mask=s0_r["ms"] / s_r["ms"],
                executed_tflops=s_r["exec_flops"] / (s_r["ms"] * 1e-3) / 1e12)


def leg_selector(args, device, stream, flush_buf, peaks):
    """Pre-pass block selector (CRISP-style) on the literal and calibrated 32K
    workloads, and the forward with and without its mask."""
    import torch
    import synth
    import dynamic_block_sparse_tiled_b200 as bl
    sel = {}
    for wn in (WORKLOAD, WORKLOAD + "_a12"):
        ws_ = synth.CONFIGS[wn]
        ps = Prefill(ws_, device)
        nq, nk = -(-ws_.Lq // ws_.Br), -(-ws_.Lkv // ws_.Bc)
        smask = torch.empty((ws_.B, ws_.Hq, nq, nk), dtype=torch.uint8, device=device)
        sws = torch.empty(bl.blasst_select_workspace_bytes(ws_.B, ws_.Hq, ws_.Hkv, ws_.Lq,
                                                           ws_.Lkv, ws_.d, ws_.Br, ws_.Bc),
                          dtype=torch.uint8, device=device)
        run_sel = lambda: bl.blasst_select_blocks(ps.q, ps.k, smask, causal=ws_.causal,
                                                  Br=ws_.Br, Bc=ws_.Bc, tau=SEL_TAU,
                                                  gamma=SEL_GAMMA, workspace=sws, stream=stream)
        run_sel()
        stream.synchronize()
        t_sel = statistics.mean(time_calls(run_sel, max(5, args.steps), 3, stream, flush_buf))
        causal_tiles = causal_pairs(nq, nk) * ws_.B * ws_.Hq
        nsel = int((smask == 0).sum().item())
        steps = max(3, args.steps // 2)
        ps, m_r = measure_prefill(ws_, LAMBDA, steps, 3, device, stream, flush_buf, pre=ps,
                                  block_mask=smask)
        _, n_r = measure_prefill(ws_, LAMBDA, steps, 3, device, stream, flush_buf, pre=ps)
        sel_bytes = 2.0 * ws_.d * (ws_.B * ws_.Hq * ws_.Lq + ws_.B * ws_.Hkv * ws_.Lkv)
        gbs = sel_bytes / (t_sel * 1e-3) / 1e9
        sel[wn] = dict(selector_ms=t_sel, selected_frac_of_causal=nsel / max(causal_tiles, 1),
                       fwd_ms_with_mask=m_r["ms"], fwd_ms_without=n_r["ms"],
                       speedup_selector_plus_fwd=n_r["ms"] / (t_sel + m_r["ms"]),
                       roofline=dict(bound="hbm", achieved=gbs, peak=peaks["hbm_gbs"],
                                     unit="GB/s", frac=gbs / peaks["hbm_gbs"],
                                     algorithmic="Q and K read once (bf16)"))
        del ps, smask, sws
        torch.cuda.empty_cache()
    return dict(tau=SEL_TAU, gamma=SEL_GAMMA, **sel)


def leg_mla(args, device, stream, flush_buf, peaks):
    """MLA-shaped decode (latent cache, 128 heads), literal and calibrated,
    and the mma.sync kernel on a 112-head shape."""
    import synth
    import dynamic_block_sparse_tiled_b200 as bl
    mla = {}
    for wn in ("decode_mla_64k", "decode_mla_64k_a12"):
        mla[wn] = measure_decode_mla(synth.CONFIGS[wn], max(5, args.steps), device, stream,
                                     flush_buf, peaks)
    base = synth.CONFIGS["decode_mla_64k"]
    mla["decode_mla_64k_h112_mma_sync"] = measure_decode_mla(
        base.replace(name="decode_mla_64k_h112", Hq=112,
                     num_splits=bl.blasst_decode_mla_splits(8, 112, base.Lkv)),
        max(5, args.steps), device, stream, flush_buf, peaks)
    return mla


def leg_backward(w, wa, args, device, stream, flush_buf, peaks):
    """Backward with the forward's decisions held fixed (32K literal at
    lambda = 1e-3; calibrated at lambda = 1e-3 against lambda = 0)."""
    import torch
    steps = max(3, args.steps // 2)
    pb = Prefill(w, device)
    pb, bb, b_l = measure_backward(w, LAMBDA, steps, 3, device, stream, flush_buf, pre=pb)
    del pb, bb
    torch.cuda.empty_cache()
    pb = Prefill(wa, device)
    pb, bb, ba_l = measure_backward(wa, LAMBDA, steps, 3, device, stream, flush_buf, pre=pb)
    _, _, ba_0 = measure_backward(wa, 0.0, steps, 3, device, stream, flush_buf, pre=pb, bwd=bb)
    del pb, bb
    torch.cuda.empty_cache()
    return dict(
        ms=b_l["ms"], pairs=b_l["pairs"], skip_frac=b_l["skip_frac"],
        executed_tflops=b_l["executed_tflops"],
        roofline=dict(bound="tensor", achieved=b_l["executed_tflops"], peak=peaks["bf16_tflops"],
                      unit="TFLOP/s", frac=b_l["executed_tflops"] / peaks["bf16_tflops"],
                      traffic=profiled_traffic("backward_32k"),
                      algorithmic="per computed (64-row tile, 128-key block) pair: 5 products "
                                  "of 2*128*64*128 flops (S^T, dP^T, dV, dK, dQ^T)"),
        a12=dict(ms=ba_l["ms"], ms_lambda0=ba_0["ms"], speedup_vs_lambda0=ba_0["ms"] / ba_l["ms"],
                 skip_frac=ba_l["skip_frac"], executed_tflops=ba_l["executed_tflops"]),
        note="dq, dk, dv in fp32; one call = the row pass (rowsum(dO*O), dq cleared) and the "
             "pair kernel")


def detail(name, obj):
    """A leg's full record, on stderr (stdout carries the one summary line)."""
    def conv(x):
        if isinstance(x, dict):
            return {str(k): conv(v) for k, v in x.items()}
        if isinstance(x, (list, tuple)):
            return [conv(v) for v in x]
        if isinstance(x, (np.integer,)):
            return int(x)
        if isinstance(x, (np.floating,)):
            return float(x)
        return x
    print(json.dumps({"detail": name, **conv(obj)}), file=sys.stderr, flush=True)


def compact_legs(legs):
    """The legs' key figures for the summary line (full records: stderr)."""
    out = {}

    def lam_arm(r, frac=False):
        d = dict(skip=_r(r["skip_frac"]), x=_r(r["speedup_vs_lambda0"]), xc=_r(r["speedup_clk"]))
        if frac:
            d["frac"] = _r(r["frac"])
        for k, kk in (("skip_frac_structured", "skip_s"), ("skip_frac_diffuse", "skip_d")):
            if k in r:
                d[kk] = _r(r[k])
        return d

    for key, lam in (("p32k", LAMBDA), ("p32k_a12", LAMBDA), ("p256k", 1e-3),
                     ("p256k_a12", 1e-3)):
        if key in legs:
            out[key] = lam_arm(legs[key][lam], frac=True)
    for key in ("p128k", "p128k_a12"):
        if key in legs:
            out[key] = {f"{lam:g}": [_r(r["skip_frac"]), _r(r["speedup_vs_lambda0"]),
                                     _r(r["speedup_clk"])]
                        for lam, r in legs[key].items() if lam != 0.0}
    for key in ("dec", "dec_a12"):
        if key in legs:
            r, r0 = legs[key][LAMBDA], legs[key][0.0]
            out[key] = dict(ms=_r(r["ms"]), gbs=_r(r["gbs"], 4), frac=_r(r["frac"]),
                            frac_l0=_r(r0["frac"]), x=_r(r["speedup_vs_lambda0"]),
                            xc=_r(r["speedup_clk"]), skip=_r(r["skip_frac"]),
                            vfetch=_r(r["v_fetch_frac"]), saved_gb=_r(r["bytes_saved"] / 1e9))
    if "mla" in legs:
        rf = legs["mla"]["decode_mla_64k"]["roofline"]
        out["mla"] = dict(ms=_r(legs["mla"]["decode_mla_64k"][str(1e-3)]["ms"]), bound=rf["bound"],
                          frac=_r(rf["frac"]), tensor_frac=_r(rf["tensor_frac"]))
    if "bwd" in legs:
        b = legs["bwd"]
        tr = b["roofline"]["traffic"]
        out["bwd"] = dict(ms=_r(b["ms"]), frac=_r(b["roofline"]["frac"]),
                          traffic_gb=_r(tr / 1e9) if tr else None,
                          a12_x=_r(b["a12"]["speedup_vs_lambda0"]))
    if "sel" in legs:
        s = legs["sel"][WORKLOAD]
        out["sel"] = dict(ms=_r(s["selector_ms"]), frac=_r(s["roofline"]["frac"]))
    if "static" in legs:
        out["static"] = dict(x=_r(legs["static"]["speedup_vs_no_mask"]))
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="blasst", choices=["blasst", "reference"])
    ap.add_argument("--quick", action="store_true",
                    help="headline, its lambda = 0 pair and the end-to-end number only")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--case", default=None,
                    help="profiling driver: run only this workload's kernel --calls times, untimed "
                         "(backward:<workload> runs one forward, then the backward --calls times; "
                         "select:<workload> runs the block selector)")
    ap.add_argument("--calls", type=int, default=4)
    ap.add_argument("--lam", type=float, default=LAMBDA)
    ap.add_argument("--override", action="append", default=[],
                    help="with --case: replace a workload field, e.g. --override B=4")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        return run_reference(args)
    if args.case:
        return run_case(args.case, args.lam, args.calls, args.override)

    import torch
    import synth
    import dynamic_block_sparse_tiled_b200 as bl
    bl.load_library()
    ws, rank, local = dist_env()
    device = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(device)
    ranks = Ranks("nccl", device)
    stream = torch.cuda.Stream(device)
    flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    peaks = load_peaks()
    w = synth.CONFIGS[WORKLOAD]
    wa = synth.CONFIGS[WORKLOAD + "_a12"]
    legs = {}

    with ClockSampler(local) as clk:
        # ---- headline: prefill 32K, lambda 1e-3, literal generator ---------
        pre = Prefill(w, device)
        ranks.barrier()
        t_head = time.time()
        pre, main_r = measure_prefill(w, LAMBDA, args.steps, args.warmup, device, stream,
                                      flush_buf, pre=pre)
        ranks.barrier()
        head_win = [(t_head, time.time())]
        ms = ranks.max(main_r["ms"])
        value = ranks.aggregate(main_r["eff_flops"], main_r["ms"]) / 1e12

        # ---- lambda = 0 against lambda = 1e-3, interleaved, same inputs ----
        legs["p32k"] = prefill_lambda_leg(w, (0.0, LAMBDA), 6, 3, device, stream, flush_buf, clk,
                                          peaks, pre=pre)
        del pre
        torch.cuda.empty_cache()
        # The other legs measure per-GPU properties of the kernels; replicas
        # (N > 1) time the headline and the end-to-end loop only.
        if ws == 1:
            legs["p32k_a12"] = prefill_lambda_leg(wa, (0.0, LAMBDA), 6, 3, device, stream,
                                                  flush_buf, clk, peaks)
            torch.cuda.empty_cache()
        if ws == 1 and not args.quick:
            lam4 = (0.0, 1e-4, 1e-3, 1e-2)
            for key, wn in (("p128k", "prefill_128k"), ("p128k_a12", "prefill_128k_a12")):
                legs[key] = prefill_lambda_leg(synth.CONFIGS[wn], lam4, 4, 1, device, stream,
                                               flush_buf, clk, peaks)
                torch.cuda.empty_cache()
            for key, wn in (("p256k", "prefill_256k"), ("p256k_a12", "prefill_256k_a12")):
                legs[key] = prefill_lambda_leg(synth.CONFIGS[wn], (0.0, 1e-3), 4, 1, device,
                                               stream, flush_buf, clk, peaks)
                torch.cuda.empty_cache()
            for key, wn in (("dec", "decode_64k"), ("dec_a12", "decode_64k_a12")):
                legs[key] = decode_lambda_leg(synth.CONFIGS[wn], LAMBDA, 6, 5, device, stream,
                                              flush_buf, clk, peaks)
                torch.cuda.empty_cache()
            legs["static"] = leg_static_mask(w, args, device, stream, flush_buf)
            torch.cuda.empty_cache()
            legs["sel"] = leg_selector(args, device, stream, flush_buf, peaks)
            legs["mla"] = leg_mla(args, device, stream, flush_buf, peaks)
            torch.cuda.empty_cache()
            legs["bwd"] = leg_backward(w, wa, args, device, stream, flush_buf, peaks)
            torch.cuda.empty_cache()
            if rank == 0:
                d = legs["dec"][LAMBDA]
                legs["dec"]["roofline"] = dict(
                    bound="hbm", achieved=d["gbs"], peak=peaks["hbm_gbs"], unit="GB/s",
                    frac=d["frac"], traffic=profiled_traffic("decode_64k"),
                    peak_source=f"{peaks['source']} hbm_gbs (copy)", vs_8tbs=d["gbs"] / 8000.0)

    # ---- end to end through the public API with host buffers ---------------
    e2e = measure_e2e(w, LAMBDA, max(8, args.steps), 3, device, stream)
    e2e["value"] = ranks.aggregate(effective_flops(w), e2e["ms"]) / 1e12
    e2e.pop("ms")

    exec_tflops = main_r["exec_flops"] / (main_r["ms"] * 1e-3) / 1e12
    roofline = dict(bound="tensor", achieved=exec_tflops, peak=peaks["bf16_tflops"], unit="TFLOP/s",
                    frac=exec_tflops / peaks["bf16_tflops"],
                    traffic=profiled_traffic("prefill_32k"),
                    frac_of_sustained=exec_tflops / peaks["bf16_tflops_sustained"])

    if rank == 0:
        for k, v in legs.items():
            detail(k, v)
        detail("roofline_notes", dict(
            peak_source=f"{peaks['source']} bf16_tflops (burst; the kernel is timed alone)",
            algorithmic="per visited (128-row tile, 128-key block): 2*128*128*128 flops for "
                        "S=QK^T, plus the same for O+=PV when the block is computed",
            e2e_pipelined=e2e.pop("pipelined"), e2e_chunks_per_step=e2e.pop("chunks")))
        cpu = oracle_sample(w, LAMBDA, args.cpu_budget)
        clocks = clk.summary(head_win)
        l0 = legs["p32k"]
        line = dict(
            metric=METRIC, value=value, unit=UNIT, n_gpus=ws, steps=args.steps, warmup=args.warmup,
            ms_per_step=ms, higher_is_better=True, scaling="weak", vs_baseline=None, dtype="bf16",
            data="synthetic", gpu_launches=args.steps,
            config=dict(workload=w.name, B=w.B, Hq=w.Hq, Hkv=w.Hkv, seq_len=w.Lq, d=w.d,
                        causal=w.causal, Br=w.Br, Bc=w.Bc, amplitude=w.amp,
                        parallelism=f"replicas{ws}", l2="flushed between steps; inputs > L2",
                        **{"lambda": LAMBDA}),
            roofline=roofline,
            cpu_baseline={k: cpu[k] for k in ("value", "unit", "cores", "kind", "sample")},
            e2e=e2e, clocks=dict({k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
                                 sm_mhz_kernel=_r(main_r["kernel_mhz"], 4)),
            skip_frac=main_r["skip_frac"], executed_tflops=exec_tflops,
            ms_lambda0=l0[0.0]["ms"], speedup_vs_lambda0=l0[LAMBDA]["speedup_vs_lambda0"],
            speedup_vs_lambda0_clk=l0[LAMBDA]["speedup_clk"],
            legs=compact_legs(legs))
        for k in ("value", "ms_per_step", "executed_tflops", "ms_lambda0", "speedup_vs_lambda0",
                  "speedup_vs_lambda0_clk"):
            line[k] = _r(line[k], 4)
        for k in ("achieved", "frac", "frac_of_sustained"):
            line["roofline"][k] = _r(line["roofline"][k], 4)
        line["e2e"]["value"] = _r(line["e2e"]["value"], 4)
        line["e2e"].pop("steps", None)
        line["cpu_baseline"]["value"] = _r(line["cpu_baseline"]["value"], 4)
        print(json.dumps(line, separators=(",", ":")), flush=True)
    ranks.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
