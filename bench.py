#!/usr/bin/env python
"""Benchmark of the Gemma self-attention forward (libgattn) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Default workload: the largest single-GPU configuration, the Gemma-4-12b-shaped
global K=V prefill (batch 1, seq 32768, 16 query heads, 1 KV head, head_dim 512,
partial RoPE 0.25, plain-weight QK-norm, full causal), metric "attention prefill
TFLOP/s" on effective (visible-pair) FLOPs.  A step is one gattn_prefill call
(query/key prologue + tensor-core attention kernel) on inputs already resident
in HBM; L2 is flushed (256 MiB write) before every step and the flush is outside
the per-step CUDA-event timing.  Decode workloads report KV GB/s on algorithmic
bytes; the default line also carries both Gemma-4 decode layers (local and
global K=V, batch 64), each timed the same way, under "decode".

Under torchrun (N>1) every rank runs its own replica of the workload on its own
GPU (independent problems, no collective on the data path: weak scaling); the
time is the maximum over ranks.  ``--impl reference`` times the float64 CPU
oracle instead (rank 0 only), on a bounded sample per step.

``--sweep FILE`` runs every workload (or those of ``--sweep-workloads``) in turn and
appends each one's JSON line to FILE; workloads FILE already holds for the same arm
are skipped, so an interrupted sweep resumes where it stopped.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

PREFILL_WL = {
    "gemma1_2b_mqa_b4_s2048": W.GEMMA1_MQA,
    "gemma2_2b_local_s256": W.GEMMA2_LOCAL,
    "gemma3_1b_local_w512_b2_s8192": W.GEMMA3_LOCAL,
    "gemma3_1b_global_b2_s8192": W.GEMMA3_GLOBAL,
    "gemma4_12b_global_keqv_s32768": W.GEMMA4_GLOBAL,
    "gemma3_1b_global_b8_s4096_leftpad": W.GEMMA3_GLOBAL_LEFTPAD,
}
DECODE_WL = {w.name: w for w in (W.GEMMA4_DECODE_LOCAL, W.GEMMA4_DECODE_GLOBAL,
                                 W.GEMMA4_DECODE_GLOBAL_NORM, W.GEMMA4_DECODE_LOCAL_INT8,
                                 W.GEMMA4_DECODE_LOCAL_TK, W.GEMMA4_DECODE_LOCAL_INT8_TK,
                                 W.GEMMA4_DECODE_GLOBAL_INT8)}
CHUNK_WL = {w.name: w for w in (W.GEMMA3_GLOBAL_CHUNK, W.GEMMA3_GLOBAL_CHUNK_TK)}
HEADLINE = "gemma4_12b_global_keqv_s32768"
# decode layers measured alongside the headline prefill (their own timed steps)
HEADLINE_DECODE = ("gemma4_12b_decode_local_b64", "gemma4_12b_decode_global_keqv_b64")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---- work counts -------------------------------------------------------------------------

def visible_pairs(S: int, window: int) -> int:
    """Visible (query, key) pairs of one causal sequence of S tokens."""
    if window <= 0 or window >= S:
        return S * (S + 1) // 2
    return window * (window + 1) // 2 + (S - window) * window


def row_visible(i, window):
    i = np.asarray(i, dtype=np.int64)
    return i + 1 if window <= 0 else np.minimum(i + 1, window)


def prefill_flops(wl: W.PrefillWorkload, seq_range=None) -> float:
    """Q K^T and P V multiply-adds (2 FLOPs each) over the visible pairs; a padded batch
    counts each sequence's valid tokens only."""
    L = wl.layer
    if seq_range is None:
        return 4.0 * L.head_dim * L.num_heads * wl.batch * visible_pairs(wl.seq, L.window)
    pairs = sum(visible_pairs(int(hi) - int(lo), L.window) for lo, hi in seq_range.tolist() if hi > lo)
    return 4.0 * L.head_dim * L.num_heads * pairs


def chunk_flops(wl: W.ChunkWorkload, rows=None) -> float:
    """Q K^T and P V FLOPs of the chunk rows ``rows`` (default all): row i is token prefix + i."""
    L = wl.layer
    rows = np.arange(wl.chunk) if rows is None else np.asarray(rows, dtype=np.int64)
    return 4.0 * L.head_dim * L.num_heads * wl.batch * float(row_visible(wl.prefix + rows, L.window).sum())


def rows_flops(wl: W.PrefillWorkload, d, rows) -> float:
    """FLOPs of the query rows ``rows`` of every sequence (padding rows count nothing)."""
    L = wl.layer
    rows = np.asarray(rows, dtype=np.int64)
    sr = d.get("seq_range")
    if sr is None:
        return 4.0 * L.head_dim * L.num_heads * wl.batch * float(row_visible(rows, L.window).sum())
    total = 0.0
    for lo, hi in sr.tolist():
        r = rows[(rows >= lo) & (rows < hi)]
        total += float(row_visible(r - lo, L.window).sum())
    return 4.0 * L.head_dim * L.num_heads * total


def decode_bytes(layer: W.Layer, seq_lens, int8: bool = False) -> float:
    """Bytes a decode step must move: the visible cache rows (bf16, or int8 codes plus one
    fp32 scale per row and kv head), the query and the output."""
    n = np.asarray(seq_lens, dtype=np.int64)
    if layer.window > 0:
        n = np.minimum(n, layer.window)
    per_row = layer.num_kv_heads * (layer.head_dim + 4 if int8 else layer.head_dim * 2)
    kv = n.sum() * per_row * (1 if layer.k_eq_v else 2)
    qo = len(n) * layer.num_heads * layer.head_dim * 2 * 2
    return float(kv + qo)


# ---- environment helpers ---------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 100 ms while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.uuid}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 7:
                self.rows.append(parts)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[3 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(self.rows)}


def source_hash(*paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(name: str, kernel_src):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current kernel."""
    p = os.path.join(ROOT, "profiles", f"{name}.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    if rec.get("source_hash") != source_hash(*kernel_src):
        return None
    return rec.get("dram_bytes_per_launch")


# ---- distributed plumbing ---------------------------------------------------------------------

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def reduce_max(x: float, device) -> float:
    """Maximum of a float over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ---- the two arms ---------------------------------------------------------------------------

def make_prefill(wl, dev):
    from gemma_family_decoder_b200 import AttentionLayer, LayerSpec
    d = W.prefill_inputs(wl)
    layer = AttentionLayer(LayerSpec.of(wl.layer), wl.seq, d["w_q"], d["w_k"], device=dev)
    host = {k: d[k].pin_memory() for k in ("q", "k", "v", "positions", "seq_range") if d[k] is not None}
    devt = {k: t.to(dev) for k, t in host.items()}
    out = torch.empty_like(devt["q"])
    host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    ws = layer.prefill_workspace(wl.batch, wl.seq, dev)

    def step(src=devt):
        layer.prefill(src["q"], src["k"], src.get("v"), src["positions"], out=out, workspace=ws,
                      seq_range=src.get("seq_range"))

    return dict(layer=layer, host=host, dev=devt, out=out, host_out=host_out, ws=ws, step=step,
                work=prefill_flops(wl, d["seq_range"]), unit="TFLOP/s", scale=1e12,
                metric="attention prefill TFLOP/s (effective FLOPs)", bound="tensor",
                launches=2 if (wl.layer.rot_dim or wl.layer.qk_norm) else 1,
                kernel_src=(dominant_prefill_src(wl.layer, d["seq_range"] is not None),
                            "gemma_family_decoder_b200/csrc/kernels/common.cuh"),
                oracle=lambda: d)


def dominant_prefill_src(L: W.Layer, padded: bool) -> str:
    """Source of the attention kernel a whole-prompt prefill runs: the SM-pair kernel for
    head_dim 512 with an even number of query heads per kv head, else the single-SM one."""
    G = L.num_heads // L.num_kv_heads
    if L.head_dim == 512 and G % 2 == 0 and not padded:
        return "gemma_family_decoder_b200/csrc/prefill_pair.cu"
    return "gemma_family_decoder_b200/csrc/prefill.cu"


def make_chunk(wl, dev):
    from gemma_family_decoder_b200 import AttentionLayer, LayerSpec
    d = W.chunk_inputs(wl)
    spec = dataclasses.replace(LayerSpec.of(wl.layer), keys_transformed=wl.keys_transformed)
    layer = AttentionLayer(spec, d["max_len"], d["w_q"], d["w_k"], device=dev)
    host = {k: d[k].pin_memory() for k in ("q", "k_new", "v_new", "prefix_lens") if d[k] is not None}
    devt = {k: t.to(dev) for k, t in host.items()}
    k_cache = d["k_cache"].to(dev)
    v_cache = None if d["v_cache"] is None else d["v_cache"].to(dev)
    if wl.keys_transformed:
        # the cached prefix as the library's append writes it: keys normed and rotated
        full_k = torch.zeros_like(k_cache)
        full_v = torch.zeros_like(v_cache)
        layer.kv_append(k_cache[:, :wl.prefix].contiguous(), v_cache[:, :wl.prefix].contiguous(), full_k, full_v,
                        torch.zeros(wl.batch, dtype=torch.int32, device=dev))
        k_cache, v_cache = full_k, full_v
    out = torch.empty_like(devt["q"])
    host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    ws = layer.prefill_chunk_workspace(wl.batch, wl.chunk, d["max_len"], dev)

    def step(src=devt):
        # append the chunk's rows to the cache, then attend (rewriting the same rows every step)
        layer.prefill_chunk(src["q"], k_cache, v_cache, src["prefix_lens"], k_new=src["k_new"], v_new=src.get("v_new"),
                            out=out, workspace=ws)

    prep = bool(wl.layer.rot_dim or wl.layer.qk_norm)
    return dict(layer=layer, host=host, dev=devt, out=out, host_out=host_out, ws=ws, step=step,
                work=chunk_flops(wl), unit="TFLOP/s", scale=1e12,
                metric="attention prefill TFLOP/s (effective FLOPs)", bound="tensor",
                launches=4 if prep else 2,
                kernel_src=("gemma_family_decoder_b200/csrc/prefill.cu",
                            "gemma_family_decoder_b200/csrc/kernels/common.cuh"))


def dominant_decode_src(L: W.Layer, int8: bool = False) -> str:
    """Source of the split kernel a decode layer runs (the step's dominant kernel): the
    tensor-core one for K=V with 8 or 16 query heads per kv head (bf16 or int8 caches),
    the CUDA-core one for 1, 2 or 4, else the split kernel in the prologue/combine file."""
    G = L.num_heads // L.num_kv_heads
    if L.k_eq_v and G in (8, 16):
        return "gemma_family_decoder_b200/csrc/decode_tc.cu"
    if G in (1, 2, 4):
        return "gemma_family_decoder_b200/csrc/decode_simt.cu"
    return "gemma_family_decoder_b200/csrc/prep_decode.cu"


def make_decode(wl, dev):
    from gemma_family_decoder_b200 import AttentionLayer, LayerSpec
    dq = W.decode_inputs(wl)
    L = wl.layer
    lens = dq["seq_lens"]
    shape = (wl.batch, wl.max_len, L.num_kv_heads, L.head_dim)
    k = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
    v = None if L.k_eq_v else torch.zeros(shape, dtype=torch.bfloat16, device=dev)
    for b in range(wl.batch):
        n = int(lens[b])
        lo = 0 if L.window == 0 else max(0, n - L.window)
        rows = W.decode_cache_rows(wl, b, n - lo, lo)
        k[b, lo:n] = rows["k"].to(dev)
        if v is not None:
            v[b, lo:n] = rows["v"].to(dev)
    spec = dataclasses.replace(LayerSpec.of(L), keys_transformed=wl.keys_transformed)
    layer = AttentionLayer(spec, wl.max_len, dq["w_q"], dq["w_k"], device=dev)
    if wl.keys_transformed:
        # the same rows as the library's append writes them: keys normed and rotated
        kt = torch.zeros_like(k)
        v_scratch = torch.empty_like(v[:1])  # the append's value copy, not needed here
        for b in range(wl.batch):
            n = int(lens[b])
            lo = 0 if L.window == 0 else max(0, n - L.window)
            layer.kv_append(k[b:b + 1, lo:n].contiguous(), v[b:b + 1, lo:n].contiguous(), kt[b:b + 1], v_scratch,
                            torch.tensor([lo], dtype=torch.int32, device=dev))
        del v_scratch
        k = kt
    host = {"q": dq["q"].pin_memory(), "seq_lens": lens.pin_memory()}
    devt = {"q": host["q"].to(dev), "seq_lens": host["seq_lens"].to(dev), "k": k, "v": v}
    out = torch.empty_like(devt["q"])
    host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    ws = layer.decode_workspace(wl.batch, wl.max_len, dev)

    if wl.kv_int8:
        from gemma_family_decoder_b200 import kv_quantize
        kq, ks = kv_quantize(k)
        vq, vs = (None, None) if v is None else kv_quantize(v)
        del k, v
        devt.update(k=None, v=None, kq=kq, ks=ks, vq=vq, vs=vs)

        def step(src=devt):
            layer.decode_int8(src["q"], devt["kq"], devt["ks"], devt["vq"], devt["vs"], src["seq_lens"], out=out,
                              workspace=ws)
    else:
        def step(src=devt):
            layer.decode(src["q"], devt["k"], devt["v"], src["seq_lens"], out=out, workspace=ws)

    return dict(layer=layer, host=host, dev=devt, out=out, host_out=host_out, ws=ws, step=step,
                work=decode_bytes(L, lens.numpy(), wl.kv_int8), unit="GB/s", scale=1e9,
                metric="decode KV GB/s (algorithmic bytes)", bound="hbm", launches=2,
                kernel_src=(dominant_decode_src(L, wl.kv_int8), "gemma_family_decoder_b200/csrc/kernels/common.cuh"))


def make_runner(name, args, dev):
    is_prefill = name in PREFILL_WL
    is_chunk = name in CHUNK_WL
    wl = PREFILL_WL[name] if is_prefill else CHUNK_WL[name] if is_chunk else DECODE_WL[name]
    if args.len_hi and not is_prefill and not is_chunk:
        # a smaller cache for profiling; with a window no longer than the
        # shortest sequence the work per step is the same
        wl = dataclasses.replace(wl, len_hi=max(wl.len_lo, args.len_hi))
    if args.seq and is_prefill:
        # a shorter prompt of the same layer, for profiling captures
        wl = dataclasses.replace(wl, seq=args.seq)
    R = make_prefill(wl, dev) if is_prefill else make_chunk(wl, dev) if is_chunk else make_decode(wl, dev)
    R.update(wl=wl, is_prefill=is_prefill, is_chunk=is_chunk)
    return R


class L2Flush:
    """A write larger than L2 evicts the inputs; the read that follows drains the
    write's dirty lines, so that their write-back to HBM does not overlap the timed step."""

    def __init__(self, dev):
        self.w = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        self.r = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.sink)


def time_steps(R, args, dev, flush, K):
    """W warm-up steps, then K timed steps (each one CUDA-graph replay of the library
    call, L2 flushed before each outside its events), then the main kernel's own time on
    eager calls from the library's profile events around its launch.  Returns the per-step
    times, the kernel times, the clock summary and the wall time of the timed loop."""
    from gemma_family_decoder_b200 import check, set_profile_events
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush()
        R["step"]()
    torch.cuda.synchronize()
    st = check(R["ws"])
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    kev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    for e in kev:  # torch creates the CUDA event at its first record; the library re-records it
        e.record(stream)
    torch.cuda.synchronize()
    graph = None
    if not args.eager:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            R["step"]()
        torch.cuda.synchronize()
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for i in range(K):
        flush()
        ev[i][0].record(stream)
        if graph is not None:
            graph.replay()
        else:
            R["step"]()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    wall = time.perf_counter() - wall0
    sampler.stop()
    st = check(R["ws"])
    if st != 0:
        raise RuntimeError(f"device status {st} after the timed steps")
    step_ms = [e[0].elapsed_time(e[1]) for e in ev]
    kern_ms = []
    for i in range(min(K, 200)):
        flush()
        set_profile_events(kev[0], kev[1])
        R["step"]()
        set_profile_events(None, None)
        torch.cuda.synchronize()
        kern_ms.append(kev[0].elapsed_time(kev[1]))
    del graph
    return step_ms, kern_ms, sampler.summary(), wall


def roofline(R, name, kern_mean, clocks=None, timed_kernel_ms=0.0):
    """The dominant kernel against its roofline.  A tensor-bound kernel is compared with
    the measured bf16 GEMM rate of the same regime: the burst figure for a kernel timed
    alone, the sustained figure (the GEMM back to back under the 1 kW cap) once the timed
    steps keep the tensor cores busy long enough to reach the power cap (at least 100 ms of
    kernel time with sw_power_cap seen during the timed region); the other fraction is
    reported beside it."""
    peaks, peak_src = load_peaks()
    achieved = R["work"] / (kern_mean / 1e3) / R["scale"]
    extra = {}
    if R["bound"] == "tensor":
        burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
        capped = bool(clocks) and "sw_power_cap" in (clocks.get("reasons") or []) and timed_kernel_ms >= 100.0
        peak, which = (sustained, "bf16_tflops_sustained: power-capped, long step") if capped else \
            (burst, "bf16_tflops burst")
        extra = {"frac_of_burst": round(achieved / burst, 4), "frac_of_sustained": round(achieved / sustained, 4)}
        peak_unit = "TFLOP/s"
    else:
        peak, which = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]), "hbm_gbs copy"
        peak_unit = "GB/s"
    return {"bound": R["bound"], "achieved": round(achieved, 3), "peak": peak,
            "unit": peak_unit, "frac": round(achieved / peak, 4), "traffic": profiled_traffic(name, R["kernel_src"]),
            "peak_source": f"{peak_src} ({which})", **extra, "kernel_ms": round(kern_mean, 5)}


def run_ours(args, world, rank, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    name = args.workload
    R = make_runner(name, args, dev)
    wl, is_prefill, is_chunk = R["wl"], R["is_prefill"], R["is_chunk"]
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()
    K = args.steps
    step_ms, kern_ms, clocks, wall = time_steps(R, args, dev, flush, K)
    total_ms = reduce_max(sum(step_ms), dev)

    # end to end through the public call: pinned host inputs in, result out, every step
    E = max(3, min(K, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h2d = sum(t.numel() * t.element_size() for t in R["host"].values())
    d2h = R["out"].numel() * R["out"].element_size()
    scratch = {k: torch.empty_like(t, device=dev) for k, t in R["host"].items()}
    for it in range(E + 2):
        if it == 2:
            barrier()
            torch.cuda.synchronize()
            e0.record(stream)
        for k2, t in R["host"].items():
            scratch[k2].copy_(t, non_blocking=True)
        R["step"](scratch if is_prefill else dict(scratch))
        R["host_out"].copy_(R["out"], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1), dev) / E
    del scratch

    unit, scale = R["unit"], R["scale"]
    value = R["work"] * world * K / (total_ms / 1e3) / scale
    result = {
        "metric": R["metric"], "value": round(value, 3), "unit": unit, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(total_ms / K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": name, "l2": "flushed before every step (256 MiB write, then a 256 MiB read "
                   "that drains the write's dirty lines), outside the per-step CUDA-event time",
                   "step": "eager library call" if args.eager else "CUDA-graph replay of the library call",
                   **({"len_hi": wl.len_hi} if args.len_hi and not is_prefill and not is_chunk else {}),
                   **({"seq": wl.seq} if args.seq and is_prefill else {}),
                   "parallelism": f"replicas{world}"},
        "roofline": roofline(R, name, statistics.mean(kern_ms), clocks, statistics.mean(kern_ms) * K),
        "e2e": {"value": round(R["work"] * world / (e2e_ms / 1e3) / scale, 3), "unit": unit,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": R["launches"] * K,
        "clocks": clocks,
        "wall_s_timed_region": round(wall, 3),
    }
    del R
    torch.cuda.empty_cache()
    if name == HEADLINE and not (args.no_decode or args.seq):
        # the decode target is measured in the same run: each layer its own timed steps
        result["decode"] = []
        for dn in HEADLINE_DECODE:
            D = make_runner(dn, args, dev)
            d_steps, d_kern, d_clocks, _ = time_steps(D, args, dev, flush, K)
            d_total = reduce_max(sum(d_steps), dev)
            result["decode"].append({
                "workload": dn, "metric": D["metric"],
                "value": round(D["work"] * world * K / (d_total / 1e3) / D["scale"], 3), "unit": D["unit"],
                "ms_per_step": round(d_total / K, 5),
                "roofline": roofline(D, dn, statistics.mean(d_kern), d_clocks, statistics.mean(d_kern) * K),
                "gpu_launches": D["launches"] * K, "clocks": d_clocks})
            del D
            torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(name, budget_s=args.cpu_budget)
    return result


# ---- the float64 oracle on the host cores ---------------------------------------------------------

def _oracle_prefill_rows(wl, d, rows):
    import oracle as O
    O.attention_prefill(d["q"], d["k"], d["v"], d["positions"], wl.layer, w_q=d["w_q"],
                        w_k=d["w_k"], rows=rows, seq_range=d.get("seq_range"))


def _oracle_cache(wl, ks, vs, firsts):
    """The oracle's cache rows per batch row (None where left out): bf16 as drawn (keys
    transformed by the oracle for a transformed-key workload), or, for an int8 workload,
    the oracle's own codes and scales of them."""
    import oracle as O
    if wl.keys_transformed:
        ks = [None if r is None else O.transform_keys(r, np.arange(firsts[b], firsts[b] + len(r)), wl.layer)
              for b, r in enumerate(ks)]
    if not wl.kv_int8:
        return dict(k=ks, v=vs)

    def q8(rows):
        cs = [None if r is None else O.kv_quantize(r.float().numpy() if torch.is_tensor(r) else np.asarray(r))
              for r in rows]
        return [None if c is None else c[0] for c in cs], [None if c is None else c[1] for c in cs]

    kc, ksc = q8(ks)
    vc, vsc = (None, None) if wl.layer.k_eq_v else q8(vs)
    return dict(kc=kc, ks=ksc, vc=vc, vs=vsc)


def _oracle_decode(wl, dq, cache, batches, firsts):
    import oracle as O
    L = wl.layer
    if wl.kv_int8:
        return O.attention_decode_int8(dq["q"], cache["kc"], cache["ks"], cache["vc"], cache["vs"], dq["seq_lens"],
                                       L, w_q=dq["w_q"], w_k=dq["w_k"], batches=batches, first_rows=firsts,
                                       keys_transformed=wl.keys_transformed)
    return O.attention_decode(dq["q"], cache["k"], None if L.k_eq_v else cache["v"], dq["seq_lens"], L,
                              w_q=dq["w_q"], w_k=dq["w_k"], batches=batches, first_rows=firsts,
                              keys_transformed=wl.keys_transformed)


def _oracle_chunk(wl, d, rows):
    import oracle as O
    kc = d["k_cache"].clone()
    kc[:, wl.prefix:] = d["k_new"]
    vc = None
    if d["v_cache"] is not None:
        vc = d["v_cache"].clone()
        vc[:, wl.prefix:] = d["v_new"]
    return O.attention_prefill_chunk(d["q"], kc, vc, d["prefix_lens"], wl.layer, w_q=d["w_q"], w_k=d["w_k"],
                                     rows=rows)


# The oracle runs in a process pool over independent units (query-row blocks of a
# prompt, batch rows of a decode step) on the host's cores, one BLAS thread per
# worker.  Workers are started with "spawn" (never fork a process that has
# touched CUDA) and get the inputs through torch shared memory; the pool size is
# the core count, capped by the host memory the float64 oracle needs per worker.

_POOL = {}


def _pool_init(kind, name, data):
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except Exception:
        pass
    torch.set_num_threads(1)
    _POOL.update(kind=kind, name=name, data=data)


def _pool_task(arg):
    kind, name, data = _POOL["kind"], _POOL["name"], _POOL["data"]
    if kind == "prefill":
        _oracle_prefill_rows(PREFILL_WL[name], data, arg)
    elif kind == "chunk":
        _oracle_chunk(CHUNK_WL[name], data, arg)
    else:
        wl = DECODE_WL[name]
        _oracle_decode(wl, data["dq"], data["cache"], arg, data["firsts"])
    return len(arg)


def _shared(x):
    """Tensors (also inside dicts and lists) moved to shared memory for the workers."""
    if torch.is_tensor(x):
        return x.share_memory_()
    if isinstance(x, dict):
        return {k: _shared(v) for k, v in x.items()}
    if isinstance(x, (list, tuple)):
        return type(x)(_shared(v) for v in x)
    return x


def _pool_size(per_worker_bytes: float) -> int:
    n = os.cpu_count() or 1
    try:
        import psutil
        avail = psutil.virtual_memory().available
        n = min(n, int(avail * 0.6 // max(per_worker_bytes, 1.0)))
    except Exception:
        pass
    return max(1, n)


class OraclePool:
    """A spawn-context process pool holding one workload's inputs."""

    def __init__(self, name):
        import concurrent.futures as cf
        import torch.multiprocessing as tmp
        if name in CHUNK_WL:
            wl = CHUNK_WL[name]
            kind, data = "chunk", W.chunk_inputs(wl)
            per = 8.0 * 4 * sum(t.numel() for t in data.values() if torch.is_tensor(t))
        elif name in PREFILL_WL:
            wl = PREFILL_WL[name]
            kind, data = "prefill", W.prefill_inputs(wl)
            per = 8.0 * 2 * sum(t.numel() for t in data.values() if torch.is_tensor(t))
        else:
            wl = DECODE_WL[name]
            dq = W.decode_inputs(wl)
            lens = dq["seq_lens"].numpy()
            L = wl.layer
            ks, vs, firsts = [], [], []
            for b in range(wl.batch):
                n = int(lens[b])
                lo = 0 if L.window == 0 else max(0, n - L.window)
                rows = W.decode_cache_rows(wl, b, n - lo, lo)
                ks.append(rows["k"])
                vs.append(rows["v"])
                firsts.append(lo)
            cache = _oracle_cache(wl, ks, vs, firsts)
            kind, data = "decode", dict(dq=dq, cache=cache, firsts=firsts)
            per = 8.0 * 4 * max(int(n) for n in lens) * L.num_kv_heads * L.head_dim
        self.kind, self.name, self.wl, self.data = kind, name, wl, data
        self.workers = _pool_size(per + 256e6)
        self.ex = cf.ProcessPoolExecutor(self.workers, mp_context=tmp.get_context("spawn"), initializer=_pool_init,
                                         initargs=(kind, name, _shared(data)))
        # start every worker (initializer, imports, first-call costs) before any timing
        first = np.array([0]) if kind != "decode" else [0]
        list(self.ex.map(_pool_task, [first] * self.workers))

    def run(self, tasks):
        """Wall seconds to run every task, spread over the pool."""
        t0 = time.perf_counter()
        list(self.ex.map(_pool_task, tasks))
        return time.perf_counter() - t0

    def close(self):
        self.ex.shutdown()


def _row_tasks(rows, nchunks):
    """Interleaved row blocks, so that causal costs spread evenly over the blocks."""
    rows = np.asarray(rows)
    return [rows[i::nchunks] for i in range(min(nchunks, len(rows))) if len(rows[i::nchunks])]


def cpu_baseline(name, budget_s=15.0):
    """The oracle timed on a strided sample of query rows (prefill, chunk) or on the batch rows
    (decode) of the workload, over a process pool on the host cores."""
    pool = OraclePool(name)
    try:
        P = pool.workers
        if pool.kind in ("prefill", "chunk"):
            wl = pool.wl
            n_all = wl.seq if pool.kind == "prefill" else wl.chunk
            # pilot: one block of rows on one worker sizes the sample to about the budget
            pilot = np.unique(np.linspace(0, n_all - 1, min(n_all, 8)).astype(np.int64))
            t_pilot = pool.run([pilot])
            per_row = t_pilot / len(pilot)
            n = int(max(P, min(n_all, budget_s * P / max(per_row, 1e-9))))
            rows = np.unique(np.linspace(0, n_all - 1, n).astype(np.int64))
            dt = pool.run(_row_tasks(rows, 2 * P))
            if pool.kind == "prefill":
                work = rows_flops(wl, pool.data, rows)
                what = f"query rows of {n_all}, all {wl.batch} sequences and {wl.layer.num_heads} heads"
            else:
                work = chunk_flops(wl, rows)
                what = f"chunk rows of {n_all}, all {wl.batch} sequences and {wl.layer.num_heads} heads"
            return {"value": round(work / dt / 1e12, 6), "unit": "TFLOP/s", "cores": P, "kind": "oracle",
                    "sample": f"{len(rows)} evenly spaced {what}, in {min(2 * P, len(rows))} blocks over {P} "
                              f"worker processes, one BLAS thread each ({dt:.1f} s wall, float64 numpy)"}
        wl = pool.wl
        lens = pool.data["dq"]["seq_lens"].numpy()
        dt = pool.run([[b] for b in range(wl.batch)])
        work = decode_bytes(wl.layer, lens, wl.kv_int8)
        return {"value": round(work / dt / 1e9, 4), "unit": "GB/s", "cores": P, "kind": "oracle",
                "sample": f"all {wl.batch} batch rows, one per task over {P} worker processes, one BLAS thread "
                          f"each ({dt:.1f} s wall, float64 numpy)"}
    finally:
        pool.close()


def run_reference(args, world, rank):
    """The oracle as the reference arm: each step is a bounded sample of the same workload,
    spread over a process pool on the host cores."""
    if rank != 0:
        return None
    name = args.workload
    budget = float(os.environ.get("GATTN_REF_BUDGET_S", "120"))
    n_steps = args.steps + args.warmup
    pool = OraclePool(name)
    try:
        P = pool.workers
        wl = pool.wl
        rng = np.random.default_rng(0)
        work, dt = 0.0, 0.0
        if pool.kind in ("prefill", "chunk"):
            n_all = wl.seq if pool.kind == "prefill" else wl.chunk
            per_row = pool.run([np.array([n_all - 1])])
            rows_per_step = int(max(1, min(n_all, budget * P / n_steps / max(per_row, 1e-9))))
            for i in range(n_steps):
                rows = np.sort(rng.choice(n_all, size=rows_per_step, replace=False))
                el = pool.run(_row_tasks(rows, 2 * P))
                if i >= args.warmup:
                    dt += el
                    work += rows_flops(wl, pool.data, rows) if pool.kind == "prefill" else chunk_flops(wl, rows)
            value, unit = work / dt / 1e12, "TFLOP/s"
            sample = (f"{rows_per_step} random {'query' if pool.kind == 'prefill' else 'chunk'} rows of {n_all} per "
                      f"step, all sequences and heads, over {P} worker processes (one BLAS thread each)")
            metric = "attention prefill TFLOP/s (effective FLOPs)"
        else:
            lens = pool.data["dq"]["seq_lens"].numpy()
            per_step = min(wl.batch, P)
            for i in range(n_steps):
                bs = [int(b) for b in rng.choice(wl.batch, size=per_step, replace=False)]
                el = pool.run([[b] for b in bs])
                if i >= args.warmup:
                    dt += el
                    work += decode_bytes(wl.layer, lens[bs], wl.kv_int8)
            value, unit = work / dt / 1e9, "GB/s"
            sample = f"{per_step} random batch rows per step, one per task over {P} worker processes"
            metric = "decode KV GB/s (algorithmic bytes)"
    finally:
        pool.close()
    return {"impl": "reference", "metric": metric, "value": round(value, 6), "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / max(args.steps, 1) * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": name},
            "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": P, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(PREFILL_WL) + sorted(CHUNK_WL) + sorted(DECODE_WL))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode layers measured with the headline")
    ap.add_argument("--eager", action="store_true", help="time eager library calls instead of a graph replay")
    ap.add_argument("--len-hi", type=int, default=0,
                    help="decode: draw sequence lengths up to this (and size the cache for it); for profiling")
    ap.add_argument("--seq", type=int, default=0,
                    help="prefill: a prompt of this many tokens instead of the workload's; for profiling")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work")
    ap.add_argument("--sweep", default="", help="append every workload's JSON line to this file, skipping those "
                                                  "it already holds (resume)")
    ap.add_argument("--sweep-workloads", default="", help="comma-separated workloads for --sweep (default: all)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.sweep:
        return sweep(args, ap)
    run_one(args)


def sweep_done(path: str, impl: str) -> set:
    """Workloads whose line for this arm is already in the sweep file (unparsable lines,
    e.g. one cut short by an interrupted run, do not count)."""
    done = set()
    if os.path.exists(path):
        with open(path) as f:
            for line in f:
                try:
                    rec = json.loads(line)
                except ValueError:
                    continue
                if rec.get("impl", "ours") == impl and "config" in rec:
                    done.add(rec["config"].get("workload"))
    return done


def sweep(args, ap):
    names = [n for n in args.sweep_workloads.split(",") if n] or \
        sorted(PREFILL_WL) + sorted(CHUNK_WL) + sorted(DECODE_WL)
    known = set(PREFILL_WL) | set(CHUNK_WL) | set(DECODE_WL)
    for n in names:
        if n not in known:
            ap.error(f"unknown workload {n}")
    done = sweep_done(args.sweep, args.impl)  # read once, so every rank skips the same ones
    for n in names:
        if n in done:
            print(f"sweep: {n} already in {args.sweep}, skipped", file=sys.stderr)
            continue
        args.workload = n
        res = run_one(args, emit=False)
        if res is not None:
            line = json.dumps(res)
            print(line, flush=True)
            with open(args.sweep, "a+b") as f:  # one write per line, on a fresh line
                f.seek(0, os.SEEK_END)
                lead = b""
                if f.tell() > 0:
                    f.seek(-1, os.SEEK_END)
                    lead = b"" if f.read(1) == b"\n" else b"\n"  # after a line cut short
                f.write(lead + line.encode() + b"\n")


def run_one(args, emit=True):
    """One workload on this arm; rank 0 returns (and by default prints) its JSON line."""
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores only; other ranks have no work
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        if res is not None and emit:
            print(json.dumps(res), flush=True)
        return res
    world, rank, local = dist_setup()
    if world != args.gpus and rank == 0:
        print(f"note: WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)
    try:
        res = run_ours(args, world, rank, local)
        if rank != 0:
            res = None
        if res is not None and emit:
            print(json.dumps(res), flush=True)
        return res
    finally:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
