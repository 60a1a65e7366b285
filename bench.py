"""Benchmark of the Gemma 4 attention layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-extra-prefill] [--no-decode] [--decode-only]
                    [--decode-batch B] [--no-kv-single] [--no-qkv] [--no-vision]
                    [--no-e2e] [--no-cpu-baseline]

Headline: prefill attention TFLOP/s counting unmasked FLOPs only
(4 * d * sum_i |I_i| * Hq * B; 2d for QK^T and 2d for PV per allowed pair) on
the E2B-shaped sliding layer (B 1, T 8192, 8 query heads on 1 KV head, head
dim 256, window 512), one g4attn_prefill call (prologue included) per step.
The same JSON line carries the other prefill workloads under "prefill" (the
12B-shaped multimodal sliding layer and the 31B-shaped K=V global layer at
head_dim 512, each with its own roofline and CPU baseline), and the second
half of the metric, decode KV-cache GB/s on the 26B-A4B-shaped step (64
sequences, cache lengths uniform in [4096, 131072]; a sliding layer on a
1024-slot rolling cache, a K=V global layer and a KV-shared layer reading it),
under "decode" (with the same step over a single-tensor K=V cache under
"kv_single").  Two more legs: "qkv_prologue", the QKV projection with the
prologue in its epilogue on the E2B-shaped prompt (TFLOP/s of the
projection, cuBLAS's projection alone timed beside it), and "vision", the
vision tower's bidirectional attention shape through g4attn_attend.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launching stream; L2 is flushed (a 256 MiB write) before every timed
prefill step, outside the events; the decode step reads ~36 GB, far more than
L2.  Barrier + synchronize on both sides; the maximum over ranks is reported.
With N > 1 every rank runs its own instance (independent sequences, no
collective on the data path): weak scaling.  NVML clock samples (every
~0.2 ms) are taken over every timed region.

--impl reference times the float64 CPU oracle (the only other implementation
of this layer) on the same workload and metric, on a bounded row sample.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from attention_prologue_b200 import g4attn as G  # noqa: E402
from attention_prologue_b200 import workloads as W  # noqa: E402

METRIC = "prefill attn TFLOP/s (unmasked) & decode KV-cache GB/s, % of B200 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# algorithmic work

def allowed_pairs(w: W.PrefillWorkload, ids: torch.Tensor | None) -> int:
    """sum over sequences and rows of |I_i| (keys each query sees)."""
    L, T = w.layer, w.T
    i = np.arange(T, dtype=np.int64)
    if L.layer_type == W.GLOBAL:
        return int(w.B * (i + 1).sum())
    total = 0
    for b in range(w.B):
        lo = np.maximum(0, i - L.window + 1)
        hi = i.copy()
        if ids is not None:
            row = ids[b].cpu().numpy()
            t = 0
            while t < T:
                if row[t] < 0:
                    t += 1
                    continue
                e = t
                while e + 1 < T and row[e + 1] == row[t]:
                    e += 1
                lo[t:e + 1] = np.minimum(lo[t:e + 1], t)
                hi[t:e + 1] = e
                t = e + 1
        total += int((hi - lo + 1).sum())
    return total


def prefill_flops(w: W.PrefillWorkload, ids) -> float:
    return 4.0 * w.layer.head_dim * w.layer.num_heads * allowed_pairs(w, ids)


def decode_bytes(L: W.LayerShape, lens, es=2, tensors=2) -> float:
    """K and V bytes of the keys the new tokens attend to (P = len, after the
    append) plus q, out and the appended K/V; tensors=1: a single-tensor cache
    of a K=V layer (V alone, K rebuilt from it)."""
    n = np.asarray(lens, np.int64) + 1
    if L.layer_type == W.SLIDING:
        n = np.minimum(n, L.window)
    kv = float(n.sum()) * L.num_kv_heads * L.head_dim * tensors * es
    return kv + len(lens) * L.head_dim * es * (2 * L.num_heads + tensors * L.num_kv_heads)


# ---------------------------------------------------------------------------
# environment

def profile_field(profile: str, row: str):
    """A number from a committed ncu summary under profiles/ (the table row
    `| row | value |`), or None if the summary or row is missing or the
    kernel source has changed since the counters were taken (the summary
    records the source's sha256)."""
    path = os.path.join(ROOT, "profiles", profile)
    if not os.path.exists(path):
        return None
    import hashlib
    fields = {}
    for line in open(path):
        if line.startswith(("kernel source:", "source_sha256:")):
            k, v = line.split(":", 1)
            fields[k] = v.strip()
        elif line.startswith(f"| {row} |"):
            fields["value"] = line.split("|")[2].strip()
    src = os.path.join(ROOT, fields.get("kernel source", ""))
    if "value" not in fields or not os.path.isfile(src):
        return None
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != fields.get("source_sha256"):
            return None
    return float(fields["value"])


def profiled_traffic(profile: str, workload: str, bench_workload: str):
    """DRAM bytes per launch of a kernel captured on this very workload."""
    if workload != bench_workload:
        return None
    return profile_field(profile, "traffic_bytes_per_launch")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML while running."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.0002, paused: bool = False):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._paused = paused
        self._period = period_s
        self._index = index
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            if self._paused:
                time.sleep(self._period)
                continue
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def pause(self):
        """Stop sampling (between timed regions) until resume()."""
        self._paused = True

    def resume(self):
        self._paused = False

    def summary(self, ms_per_step: float | None = None):
        if not self.samples:
            return None
        mhz = float(statistics.median(self.samples))
        out = {"sm_mhz": mhz, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
               "samples": len(self.samples)}
        if ms_per_step is not None:  # SM clock cycles per step at the median clock
            out["mcycles_per_step"] = ms_per_step * mhz / 1e3
        return out


def visible_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        try:
            return int(vis.split(",")[local_rank])
        except ValueError:
            return local_rank
    return local_rank


class Dist:
    """One process per GPU (RANK / WORLD_SIZE / LOCAL_RANK / MASTER_* from the
    launcher). NCCL on GPUs; gloo with CPU tensors when asked (the host-logic
    tests run two CPU ranks). Collectives carry only timings."""

    def __init__(self, backend: str | None = None, timeout_s: float = 120.0):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.device = "cpu"
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            backend = backend or "nccl"
            timeout = datetime.timedelta(seconds=timeout_s)
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                self.device = "cuda"
                dist.init_process_group("nccl", timeout=timeout,
                                        device_id=torch.device("cuda", self.local))
            else:
                dist.init_process_group(backend, timeout=timeout)
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def job_rate(world: int, units_per_step: float, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the units every rank processed (weak scaling:
    the same per rank) over the slowest rank's time."""
    return world * units_per_step * steps / (max_ms * 1e-3)


def desc_of(L: W.LayerShape, dtype=torch.bfloat16) -> G.LayerDesc:
    return G.make_desc(L.layer_type, L.num_heads, L.num_kv_heads, L.head_dim, window=L.window,
                       rotary_fraction=L.rotary_fraction, rope_theta=L.rope_theta,
                       k_eq_v=L.k_eq_v, softmax_scale=L.scale, rms_eps=L.rms_eps, dtype=dtype,
                       logit_softcap=L.logit_softcap)


def made_events(n):
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in ev:  # torch creates the CUDA event on first record
        e.record()
    torch.cuda.synchronize()
    return ev


# ---------------------------------------------------------------------------
# prefill

# committed ncu summaries of the attention kernel, by workload: (file, the
# workload the capture ran, how its traffic maps onto a full launch)
PROFILES = {
    W.E2B_SLIDING.name: ("attn_sm100_e2b_sliding.md", "same"),
    W.G12B_SLIDING_MM.name: ("attn_sm100_12b_sliding_mm.md", "same"),
    W.G31B_GLOBAL.name: ("attn_pair_31b_global.md", "same"),
}


def prefill_traffic(w: W.PrefillWorkload):
    """DRAM bytes per launch of the attention kernel on this workload, from a
    committed capture of the same kernel source on the same workload."""
    prof = PROFILES.get(w.name)
    if prof is None:
        return None
    return profile_field(prof[0], "traffic_bytes_per_launch")


def bench_prefill(args, dist: Dist, pk: dict, w: W.PrefillWorkload, clk: ClockSampler,
                  e2e: bool, steps: int):
    """One g4attn_prefill call per step on workload w (CUDA graph replay),
    then the attention kernel alone (events the library records around it),
    then optionally the same call end to end from pinned host memory."""
    dev = torch.device("cuda", dist.local)
    inp = W.prefill_inputs(w, dev, seed=dist.rank)
    d = desc_of(w.layer)
    out = torch.empty_like(inp["q_raw"])
    ws = torch.empty(G.g4attn_prefill_workspace_size(d, w.B, w.T), dtype=torch.uint8, device=dev)
    flops = prefill_flops(w, inp["image_block_ids"])
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        G.g4attn_prefill(d, inp["q_raw"], inp["k_raw"], inp["v_raw"], inp["q_norm_w"],
                         inp["k_norm_w"], inp["image_block_ids"], out=out, workspace=ws,
                         stream=stream)

    for _ in range(args.warmup):
        step()
    K = steps
    s0, s1, a0, a1 = (made_events(K) for _ in range(4))
    # One step as a CUDA graph (the library's launches of one g4attn_prefill
    # call), replayed K times: no host launch gaps inside the timed steps.
    graph = None
    if not args.no_graph:
        torch.cuda.synchronize()
        n0 = G.g4attn_launch_count()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            G.g4attn_prefill(d, inp["q_raw"], inp["k_raw"], inp["v_raw"], inp["q_norm_w"],
                             inp["k_norm_w"], inp["image_block_ids"], out=out, workspace=ws)
        per_step_launches = G.g4attn_launch_count() - n0
        for _ in range(args.warmup):
            graph.replay()
    torch.cuda.synchronize()
    dist.barrier()
    launches0 = G.g4attn_launch_count()
    n_clk = len(clk.samples)
    clk.resume()
    torch.cuda.synchronize()
    dist.barrier()
    for i in range(K):
        flush.fill_(i & 0xFF)
        s0[i].record(stream)
        if graph is None:
            step()
        else:
            graph.replay()
        s1[i].record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clk_steps = len(clk.samples) - n_clk
    launches = (G.g4attn_launch_count() - launches0 if graph is None
                else per_step_launches * K)
    step_ms = [s0[i].elapsed_time(s1[i]) for i in range(K)]
    # the dominant kernel alone: the library records a0/a1 around its
    # attention launch on the call's stream (eager calls, same L2 flushing)
    for i in range(K):
        flush.fill_(i & 0xFF)
        G.g4attn_time_next_attention(a0[i], a1[i])
        step()
    torch.cuda.synchronize()
    clk.pause()
    attn_ms = [a0[i].elapsed_time(a1[i]) for i in range(K)]
    total_ms = dist.max(sum(step_ms))
    value = job_rate(dist.world, flops, K, total_ms) / 1e12
    attn_avg = statistics.mean(attn_ms)
    achieved = flops / (attn_avg * 1e-3) / 1e12
    status = G.g4attn_get_device_status()
    if status != G.G4ATTN_OK:
        raise RuntimeError(f"device status after prefill: {G.g4attn_status_string(status)}")

    peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    kernel = "attn_pair_kernel" if w.layer.head_dim == 512 else "attn_sm100_kernel"
    res = dict(
        metric="prefill attn TFLOP/s (unmasked)", value=value, unit="TFLOP/s",
        ms_per_step=total_ms / K, steps=K, flops=flops, launches=launches,
        clock_samples_in_steps=clk_steps,
        roofline={"bound": "tensor", "kernel": f"{kernel} (g4attn_prefill)",
                  "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                  "frac": achieved / peak, "traffic": prefill_traffic(w),
                  "algorithmic_per_launch": flops, "avg_launch_ms": attn_avg},
        e2e=None, inputs=inp, workload=w, graph=graph is not None)
    if not e2e:
        del flush, ws, graph
        return res

    # end to end: host (pinned) inputs -> device, prefill, output -> host,
    # every step, pipelined as a serving loop runs it: step i's inputs go in
    # on one copy stream while step i - 1 computes, and step i - 1's output
    # comes back on another (two device buffer sets; PCIe carries the two
    # directions at once).  Timed from the first input copy to the last
    # output copy; the L2 flush before each prefill stays inside.
    host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in inp.items()}
    host_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    dev_in = [{k: (torch.empty_like(v) if v is not None else None) for k, v in inp.items()}
              for _ in range(2)]
    dev_out = [torch.empty_like(out) for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = host_out[0].numel() * host_out[0].element_size()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready, in_free, done, out_free = ([torch.cuda.Event() for _ in range(2)] for _ in range(4))

    def e2e_steps(n, t0=None, t1=None):
        if t0 is not None:
            t0.record(s_in)
        for i in range(n):
            j = i & 1
            if i >= 2:
                s_in.wait_event(in_free[j])  # the prefill of step i - 2 has read dev_in[j]
            with torch.cuda.stream(s_in):
                for k, v in host.items():
                    if v is not None:
                        dev_in[j][k].copy_(v, non_blocking=True)
            in_ready[j].record(s_in)
            stream.wait_event(in_ready[j])
            if i >= 2:
                stream.wait_event(out_free[j])  # step i - 2's output has left dev_out[j]
            with torch.cuda.stream(stream):
                flush.fill_(i & 0xFF)
                x = dev_in[j]
                G.g4attn_prefill(d, x["q_raw"], x["k_raw"], x["v_raw"], x["q_norm_w"],
                                 x["k_norm_w"], x["image_block_ids"], out=dev_out[j],
                                 workspace=ws, stream=stream)
            in_free[j].record(stream)
            done[j].record(stream)
            s_out.wait_event(done[j])
            with torch.cuda.stream(s_out):
                host_out[j].copy_(dev_out[j], non_blocking=True)
            out_free[j].record(s_out)
        if t1 is not None:
            t1.record(s_out)

    e2e_steps(max(2, args.warmup))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    clk.resume()
    e2e_steps(K, e0, e1)
    torch.cuda.synchronize()
    clk.pause()
    e2e_ms = dist.max(e0.elapsed_time(e1))
    e2e_value = job_rate(dist.world, flops, K, e2e_ms) / 1e12
    res["e2e"] = {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                  "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / K,
                  "copies": "pinned host -> device and device -> host every step, two-deep "
                            "pipeline over a copy-in and a copy-out stream"}
    del flush, ws, graph
    return res


def public_prefill(res: dict) -> dict:
    """A prefill leg as it goes into the JSON line (no tensors)."""
    w = res["workload"]
    out = {k: v for k, v in res.items() if k not in ("inputs", "workload", "graph", "e2e")}
    out["workload"] = w.name
    out["config"] = {"global_batch": w.B, "seq_len": w.T,
                     "heads": [w.layer.num_heads, w.layer.num_kv_heads],
                     "head_dim": w.layer.head_dim, "window": w.layer.window,
                     "image_blocks": [w.n_blocks, w.block_len] if w.n_blocks else None,
                     "k_eq_v": w.layer.k_eq_v}
    return out


# ---------------------------------------------------------------------------
# decode

def bench_decode(args, dist: Dist, pk: dict, clk: ClockSampler):
    from dataclasses import replace
    w = W.A4B_DECODE if not args.decode_batch else replace(W.A4B_DECODE, batch=args.decode_batch)
    dev = torch.device("cuda", dist.local)
    lens = W.decode_lengths(w, seed=dist.rank)
    g = torch.Generator(device=dev)
    g.manual_seed(1000 + dist.rank)
    S, Gl = w.sliding, w.global_
    X = replace(Gl, softmax_scale=Gl.scale)  # KV-shared layer: own queries, G's cache
    s_tok = W.decode_token_inputs(S, w.batch, g, dev, w.dtype)
    g_tok = W.decode_token_inputs(Gl, w.batch, g, dev, w.dtype)
    x_tok = W.decode_token_inputs(X, w.batch, g, dev, w.dtype, with_kv=False)
    s_cache = G.KVCache.allocate(w.batch, S.num_kv_heads, w.sliding_capacity, S.head_dim,
                                 rolling=True, device=dev)
    g_cache = G.KVCache.allocate(w.batch, Gl.num_kv_heads, w.global_capacity, Gl.head_dim,
                                 device=dev)
    W.fill_cache(s_cache.k, s_cache.v, lens, True, g)
    W.fill_cache(g_cache.k, g_cache.v, lens, False, g)
    lens_dev = torch.as_tensor(lens, dtype=torch.int32, device=dev)
    ds, dg, dx = desc_of(S), desc_of(Gl), desc_of(X)
    outs = {k: torch.empty_like(t["q_raw"]) for k, t in (("s", s_tok), ("g", g_tok), ("x", x_tok))}
    ws_s = torch.empty(G.g4attn_decode_workspace_size(ds, s_cache), dtype=torch.uint8, device=dev)
    ws_g = torch.empty(G.g4attn_decode_workspace_size(dg, g_cache), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    nbytes = decode_bytes(S, lens) + decode_bytes(Gl, lens) + decode_bytes(X, lens)

    def reset():
        s_cache.len.copy_(lens_dev)
        g_cache.len.copy_(lens_dev)

    def step(ev=None):
        G.g4attn_cache_append(ds, s_cache, s_tok["k_raw"], s_tok["v_raw"], s_tok["k_norm_w"], stream)
        G.g4attn_decode(ds, s_cache, s_tok["q_raw"], s_tok["q_norm_w"], outs["s"], ws_s, stream)
        G.g4attn_cache_append(dg, g_cache, g_tok["k_raw"], None, g_tok["k_norm_w"], stream)
        if ev:
            G.g4attn_time_next_attention(*ev)
        G.g4attn_decode(dg, g_cache, g_tok["q_raw"], g_tok["q_norm_w"], outs["g"], ws_g, stream)
        G.g4attn_decode(dx, g_cache, x_tok["q_raw"], x_tok["q_norm_w"], outs["x"], ws_g, stream)

    for _ in range(args.warmup):
        reset()
        step()
    K = args.steps
    s0, s1, a0, a1 = (made_events(K) for _ in range(4))
    torch.cuda.synchronize()
    dist.barrier()
    launches0 = G.g4attn_launch_count()
    n_clk = len(clk.samples)
    clk.resume()
    for i in range(K):
        reset()
        s0[i].record(stream)
        step((a0[i], a1[i]))
        s1[i].record(stream)
    torch.cuda.synchronize()
    clk.pause()
    clk_steps = len(clk.samples) - n_clk
    dist.barrier()
    launches = G.g4attn_launch_count() - launches0
    total_ms = dist.max(sum(s0[i].elapsed_time(s1[i]) for i in range(K)))
    status = G.g4attn_get_device_status()
    if status != G.G4ATTN_OK:
        raise RuntimeError(f"device status after decode: {G.g4attn_status_string(status)}")
    g_ms = statistics.mean(a0[i].elapsed_time(a1[i]) for i in range(K))
    g_split_bytes = decode_bytes(Gl, lens)
    peak = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    achieved = g_split_bytes / (g_ms * 1e-3) / 1e9
    # DRAM traffic of the global layer's split kernel, from a capture of the
    # same kernel source on this very step (64 sequences, rank 0's lengths)
    traffic = (profile_field("decode_mma_26b_a4b_global.md", "traffic_bytes_per_launch")
               if w.batch == 64 and dist.rank == 0 else None)
    res = {"metric": "decode KV-cache GB/s", "value": job_rate(dist.world, nbytes, K, total_ms) / 1e9,
           "unit": "GB/s", "ms_per_step": total_ms / K, "bytes_per_step": nbytes,
           "workload": w.name if w.batch == 64 else f"{w.name}-b{w.batch}", "batch": w.batch, "len_range": [w.len_lo, w.len_hi],
           "layers": ["sliding 16/8 d256 w1024 rolling 1024", "global K=V 16/2 d512",
                      "KV-shared global 16/2 d512"],
           "roofline": {"bound": "hbm", "kernel": "decode split-KV (global layer)",
                        "achieved": achieved, "peak": peak, "unit": "GB/s",
                        "frac": achieved / peak, "frac_of_8000": achieved / 8000.0,
                        "traffic": traffic, "algorithmic_per_launch": g_split_bytes,
                        "avg_launch_ms": g_ms},
           "gpu_launches": launches, "clock_samples_in_steps": clk_steps, "cpu_baseline": None}
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = decode_cpu_baseline(w, lens, (S, s_tok, s_cache), (Gl, g_tok, g_cache),
                                                  (X, x_tok))
    if not args.no_kv_single:
        # the same step with the global layer's cache stored as V alone (the
        # K=V single-tensor cache): the global and KV-shared layers read half
        # the bytes; the sliding layer is unchanged
        del g_cache
        torch.cuda.empty_cache()
        sg = G.KVCache.allocate(w.batch, Gl.num_kv_heads, w.global_capacity, Gl.head_dim,
                                device=dev, single=True, k_norm_w=g_tok["k_norm_w"])
        W.fill_cache(sg.k, sg.k, lens, False, g)

        def step1(ev=None):
            G.g4attn_cache_append(ds, s_cache, s_tok["k_raw"], s_tok["v_raw"], s_tok["k_norm_w"],
                                  stream)
            G.g4attn_decode(ds, s_cache, s_tok["q_raw"], s_tok["q_norm_w"], outs["s"], ws_s, stream)
            G.g4attn_cache_append(dg, sg, g_tok["k_raw"], None, g_tok["k_norm_w"], stream)
            if ev:
                G.g4attn_time_next_attention(*ev)
            G.g4attn_decode(dg, sg, g_tok["q_raw"], g_tok["q_norm_w"], outs["g"], ws_g, stream)
            G.g4attn_decode(dx, sg, x_tok["q_raw"], x_tok["q_norm_w"], outs["x"], ws_g, stream)

        for _ in range(args.warmup):
            s_cache.len.copy_(lens_dev)
            sg.len.copy_(lens_dev)
            step1()
        torch.cuda.synchronize()
        dist.barrier()
        clk.resume()
        for i in range(K):
            s_cache.len.copy_(lens_dev)
            sg.len.copy_(lens_dev)
            s0[i].record(stream)
            step1((a0[i], a1[i]))
            s1[i].record(stream)
        torch.cuda.synchronize()
        clk.pause()
        dist.barrier()
        t1 = dist.max(sum(s0[i].elapsed_time(s1[i]) for i in range(K)))
        status = G.g4attn_get_device_status()
        if status != G.G4ATTN_OK:
            raise RuntimeError(f"device status after decode: {G.g4attn_status_string(status)}")
        g1_ms = statistics.mean(a0[i].elapsed_time(a1[i]) for i in range(K))
        g1_bytes = decode_bytes(Gl, lens, tensors=1)
        n1 = decode_bytes(S, lens) + g1_bytes + decode_bytes(X, lens, tensors=1)
        res["kv_single"] = {
            "metric": "decode KV-cache GB/s", "cache": "global layer: single-tensor K=V cache",
            "value": job_rate(dist.world, n1, K, t1) / 1e9, "unit": "GB/s",
            "ms_per_step": t1 / K, "bytes_per_step": n1,
            "speedup_vs_two_tensor_step": (total_ms / K) / (t1 / K),
            "roofline": {"bound": "hbm", "kernel": "decode split-KV (global layer, K rebuilt)",
                         "achieved": g1_bytes / (g1_ms * 1e-3) / 1e9, "peak": peak,
                         "unit": "GB/s", "frac": g1_bytes / (g1_ms * 1e-3) / 1e9 / peak,
                         "traffic": (profile_field("decode_mma_26b_a4b_global_single.md",
                                                   "traffic_bytes_per_launch")
                                     if w.batch == 64 and dist.rank == 0 else None),
                         "algorithmic_per_launch": g1_bytes, "avg_launch_ms": g1_ms}}
        del sg
        g_cache = None
    del g_cache, s_cache
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------------------
# the QKV projection with the prologue in its epilogue, and the vision shape

def timed(fn, K, flush, stream, ev=None):
    """Device ms of K calls of fn (L2 flushed before each), from events on
    `stream`; ev: events the library records around its dominant kernel."""
    s0, s1 = made_events(K), made_events(K)
    torch.cuda.synchronize()
    for i in range(K):
        flush.fill_(i & 0xFF)
        s0[i].record(stream)
        if ev is not None:
            G.g4attn_time_next_attention(ev[0][i], ev[1][i])
        fn()
        s1[i].record(stream)
    torch.cuda.synchronize()
    return [s0[i].elapsed_time(s1[i]) for i in range(K)]


def bench_qkv(args, dist: Dist, pk: dict, clk: ClockSampler, steps: int):
    """g4attn_qkv_prologue on the E2B-shaped layer's prompt (x [1, 8192, 1536]
    -> 8 query heads, K and V of 256: the raw projections stay in TMEM), and
    the same projection by cuBLAS (torch.matmul to bf16 raw, no prologue)
    timed beside it.  Unit: the projection's FLOPs, 2 * tokens * rows of W *
    hidden."""
    w = W.E2B_SLIDING
    L, hidden = w.layer, W.HIDDEN[w.name]
    dev = torch.device("cuda", dist.local)
    inp = W.projection_inputs(L, w.B, w.T, hidden, dev, seed=dist.rank)
    d = desc_of(L)
    cache = G.KVCache.allocate(w.B, L.num_kv_heads, w.T, L.head_dim, device=dev)
    q_hat = torch.empty(w.B, w.T, L.num_heads, L.head_dim, dtype=torch.bfloat16, device=dev)
    n_rows = inp["w_qkv"].shape[0]
    flops = 2.0 * w.B * w.T * n_rows * hidden
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    raw = torch.empty(w.B * w.T, n_rows, dtype=torch.bfloat16, device=dev)
    x2 = inp["x"].view(w.B * w.T, hidden)

    def fused():
        G.g4attn_qkv_prologue(d, 0, inp["x"], inp["w_qkv"], inp["q_norm_w"], inp["k_norm_w"],
                              cache, q_hat=q_hat, stream=stream)

    def cublas():
        torch.matmul(x2, inp["w_qkv"].t(), out=raw)

    for _ in range(args.warmup):
        fused()
        cublas()
    dist.barrier()
    clk.resume()
    n0 = G.g4attn_launch_count()
    f_ms = timed(fused, steps, flush, stream)
    launches = G.g4attn_launch_count() - n0
    c_ms = timed(cublas, steps, flush, stream)
    clk.pause()
    dist.barrier()
    status = G.g4attn_get_device_status()
    if status != G.G4ATTN_OK:
        raise RuntimeError(f"device status after qkv: {G.g4attn_status_string(status)}")
    total = dist.max(sum(f_ms))
    avg = statistics.mean(f_ms)
    peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    achieved = flops / (avg * 1e-3) / 1e12
    res = {"metric": "QKV projection + prologue TFLOP/s", "unit": "TFLOP/s",
           "value": job_rate(dist.world, flops, steps, total) / 1e12,
           "ms_per_step": total / steps, "steps": steps, "flops": flops, "launches": launches,
           "workload": f"{w.name}: x [{w.B}, {w.T}, {hidden}] -> {n_rows} rows of W",
           "roofline": {"bound": "tensor", "kernel": "qkv_pair_kernel<256> (CTA pairs)",
                        "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                        "frac": achieved / peak,
                        "traffic": profile_field("qkv_pair_e2b.md", "traffic_bytes_per_launch"),
                        "algorithmic_per_launch": flops, "avg_launch_ms": avg},
           "cublas_projection_only": {"ms": statistics.mean(c_ms),
                                      "tflops": flops / (statistics.mean(c_ms) * 1e-3) / 1e12,
                                      "note": "torch.matmul to bf16 raw q/k/v, no prologue"},
           "cpu_baseline": None}
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = qkv_cpu_baseline(w, inp, hidden)
    del raw, flush, cache, q_hat
    return res


def qkv_cpu_baseline(w, inp, hidden, target_s=5.0):
    """The oracle's projection (float64 matmul) and prologue on the first
    tokens of the prompt, sized to about target_s."""
    import oracle
    oracle.build()
    ol = oracle_layer_of(w.layer)
    cpu = {k: v.cpu() for k, v in inp.items() if v is not None}
    n_rows = cpu["w_qkv"].shape[0]
    n = 256
    while True:
        t0 = time.perf_counter()
        oracle.qkv_prologue(ol, cpu["x"][:, :n], cpu["w_qkv"], cpu["q_norm_w"], cpu["k_norm_w"])
        secs = time.perf_counter() - t0
        if secs > target_s / 4 or n >= w.T:
            break
        n = min(w.T, n * 4)
    flops = 2.0 * n * n_rows * hidden
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": oracle.default_threads(),
            "kind": "oracle",
            "sample": f"the first {n} tokens of the prompt: float64 numpy matmul (x W^T) and the "
                      f"C prologue, {secs:.1f} s"}


def bench_vision(args, dist: Dist, pk: dict, clk: ClockSampler, steps: int):
    """The vision-tower attention shape through g4attn_attend (bidirectional,
    scale 1.0, 8 images of up to 2520 patches with per-image padding, 16
    heads of 64): unmasked TFLOP/s = 4 d Hq T sum_b n_b (every row sees the
    n_b valid patches of its image)."""
    w = W.VISION_BIDIR
    L = w.layer
    dev = torch.device("cuda", dist.local)
    inp = W.vision_inputs(w, dev, seed=dist.rank)
    d = desc_of(L)
    cache = G.KVCache.allocate(w.B, L.num_kv_heads, w.T, L.head_dim, device=dev)
    cache.k.copy_(inp["k_hat"])
    cache.v.copy_(inp["v_hat"])
    out = torch.empty_like(inp["q_hat"])
    ws = torch.empty(G.g4attn_attend_workspace_size(d, w.B, w.T, 0), dtype=torch.uint8,
                     device=dev)
    flops = 4.0 * L.head_dim * L.num_heads * w.T * float(inp["valid"].sum())
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        G.g4attn_attend(d, 0, inp["q_hat"], cache, attention_mask=inp["attention_mask"],
                        out=out, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    a0, a1 = made_events(steps), made_events(steps)
    dist.barrier()
    clk.resume()
    n0 = G.g4attn_launch_count()
    s_ms = timed(step, steps, flush, stream, ev=(a0, a1))
    launches = G.g4attn_launch_count() - n0
    clk.pause()
    dist.barrier()
    status = G.g4attn_get_device_status()
    if status != G.G4ATTN_OK:
        raise RuntimeError(f"device status after vision: {G.g4attn_status_string(status)}")
    total = dist.max(sum(s_ms))
    attn = statistics.mean(a0[i].elapsed_time(a1[i]) for i in range(steps))
    peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    achieved = flops / (attn * 1e-3) / 1e12
    res = {"metric": "prefill attn TFLOP/s (unmasked)", "unit": "TFLOP/s",
           "value": job_rate(dist.world, flops, steps, total) / 1e12,
           "ms_per_step": total / steps, "steps": steps, "flops": flops, "launches": launches,
           "workload": w.name,
           "config": {"images": w.B, "patch_budget": w.T, "heads": [L.num_heads, L.num_kv_heads],
                      "head_dim": L.head_dim, "softmax_scale": L.scale,
                      "valid_patches": [int(n) for n in inp["valid"]],
                      "step": "one g4attn_attend call (eager)"},
           "roofline": {"bound": "tensor", "kernel": "attn_sm100_kernel<64> (g4attn_attend)",
                        "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                        "frac": achieved / peak,
                        "traffic": profile_field("attn_sm100_vision.md", "traffic_bytes_per_launch"),
                        "algorithmic_per_launch": flops, "avg_launch_ms": attn},
           "cpu_baseline": None}
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = vision_cpu_baseline(w, inp)
    del cache, out, ws, flush
    return res


def vision_cpu_baseline(w, inp, target_s=5.0):
    """The oracle's attention of every `stride`-th patch row of every image."""
    import oracle
    oracle.build()
    threads = oracle.default_threads()
    ol = oracle_layer_of(w.layer)
    qh = inp["q_hat"].double().cpu().numpy()
    kh = inp["k_hat"].double().cpu().numpy().transpose(0, 2, 1, 3)
    vh = inp["v_hat"].double().cpu().numpy().transpose(0, 2, 1, 3)
    keep = inp["attention_mask"].cpu().numpy()
    stride = 256
    while True:
        rows = list(range(0, w.T, stride))
        t0 = time.perf_counter()
        oracle.attend_rows(ol, qh, kh, vh, 0, None, rows, threads, attention_mask=keep)
        secs = time.perf_counter() - t0
        if secs > target_s / 4 or stride == 1:
            break
        stride = max(1, stride // 4)
    flops = 4.0 * w.layer.head_dim * w.layer.num_heads * len(rows) * float(inp["valid"].sum())
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{w.name}: {rows_phrase(stride)} of every image, all heads, {secs:.1f} s; "
                      f"float64 C, {threads} threads"}


def decode_cpu_baseline(w, lens, s_state, g_state, x_state, n_global_seqs=4):
    """The float64 oracle's decode of the same step on the host cores: the
    sliding layer for every sequence, the global and KV-shared layers for a
    few sequences (copying a 131072-position cache to the host is ~0.5 GB per
    sequence); GB/s = the attended cache bytes of what was computed / its
    time.  The caches hold the new token already (the step appended it)."""
    import oracle
    oracle.build()
    threads = oracle.default_threads()
    S, s_tok, s_cache = s_state
    Gl, g_tok, g_cache = g_state
    X, x_tok = x_state
    post = np.asarray(lens, np.int64) + 1  # after the append

    def olayer(L):
        return oracle.Layer(layer_type=L.layer_type, window=L.window,
                            rotary_fraction=L.rotary_fraction, rope_theta=L.rope_theta,
                            k_eq_v=L.k_eq_v, num_heads=L.num_heads,
                            num_kv_heads=L.num_kv_heads, head_dim=L.head_dim,
                            softmax_scale=L.scale, rms_eps=L.rms_eps)

    secs, nbytes = 0.0, 0.0
    # sliding layer, all sequences (rolling cache of `window` slots)
    ck, cv = s_cache.k.cpu(), s_cache.v.cpu()
    t0 = time.perf_counter()
    oracle.decode(olayer(S), s_tok["q_raw"].cpu(), s_tok["q_norm_w"].cpu(), ck, cv,
                  s_cache.capacity, True, post, nthreads=threads)
    secs += time.perf_counter() - t0
    nbytes += decode_bytes(S, lens)
    # global and KV-shared layers: the first n sequences
    sel = list(range(n_global_seqs))
    n_max = int(post[sel].max())
    ck = g_cache.k[sel][:, :, :n_max].cpu()
    cv = g_cache.v[sel][:, :, :n_max].cpu()
    for L, tok in ((Gl, g_tok), (X, x_tok)):
        t0 = time.perf_counter()
        oracle.decode(olayer(L), tok["q_raw"][sel].cpu(), tok["q_norm_w"].cpu(), ck, cv, n_max,
                      False, post[sel], nthreads=threads)
        secs += time.perf_counter() - t0
        nbytes += decode_bytes(L, np.asarray(lens)[sel])
    return {"value": nbytes / secs / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{w.name}: sliding layer all {w.batch} sequences, global and KV-shared "
                      f"layers the first {n_global_seqs} sequences ({nbytes / 1e9:.2f} GB of "
                      f"attended K/V, {secs:.1f} s); float64 C, {threads} threads"}


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and the reference arm)

def row_pairs(w: W.PrefillWorkload, ids, rows) -> float:
    """sum over sequences and the given rows of |I_i| (image blocks included)."""
    L, T = w.layer, w.T
    i = np.asarray(rows, np.int64)
    if L.layer_type == W.GLOBAL:
        return float(w.B * (i + 1).sum())
    total = 0
    for b in range(w.B):
        lo = np.maximum(0, i - L.window + 1)
        hi = i.copy()
        if ids is not None:
            row = ids[b].cpu().numpy()
            for n, r in enumerate(rows):
                if row[r] >= 0:
                    s = r
                    while s > 0 and row[s - 1] == row[r]:
                        s -= 1
                    e = r
                    while e + 1 < T and row[e + 1] == row[r]:
                        e += 1
                    lo[n] = min(lo[n], s)
                    hi[n] = e
        total += int((hi - lo + 1).sum())
    return float(total)


def oracle_layer_of(L: W.LayerShape):
    import oracle
    return oracle.Layer(layer_type=L.layer_type, window=L.window,
                        rotary_fraction=L.rotary_fraction, rope_theta=L.rope_theta,
                        k_eq_v=L.k_eq_v, num_heads=L.num_heads, num_kv_heads=L.num_kv_heads,
                        head_dim=L.head_dim, softmax_scale=L.scale, rms_eps=L.rms_eps)


def cpu_inputs(inp: dict) -> dict:
    return {k: (v.cpu() if v is not None else None) for k, v in inp.items()}


def oracle_sample(w: W.PrefillWorkload, cpu: dict, stride: int, threads: int, kv=None):
    """Oracle on every `stride`-th query row (all heads, all sequences), plus
    its key/value prologue charged pro rata.  Returns (TFLOP/s, seconds,
    rows, (khat, vhat))."""
    import oracle
    ol = oracle_layer_of(w.layer)
    t0 = time.perf_counter()
    if kv is None:
        kv = oracle.prefill_kv(ol, cpu["k_raw"], cpu["v_raw"], cpu["k_norm_w"], threads)
    t_kv = time.perf_counter() - t0
    kh, vh = kv
    rows = list(range(0, w.T, stride))
    ids = cpu["image_block_ids"]
    t0 = time.perf_counter()
    oracle.prefill_rows(ol, cpu["q_raw"], cpu["q_norm_w"], kh, vh,
                        None if ids is None else ids.numpy(), rows, threads)
    t_rows = time.perf_counter() - t0
    flops = 4.0 * w.layer.head_dim * w.layer.num_heads * row_pairs(w, ids, rows)
    secs = t_rows + t_kv * len(rows) / w.T
    return flops / secs / 1e12, secs, len(rows), kv


def pick_stride(w, cpu, threads, target_s):
    """Row stride whose sample takes about target_s seconds (calibrated on a
    64-row probe; returns the probe's key/value prologue for reuse)."""
    probe = max(1, w.T // 64)
    _, secs, n, kv = oracle_sample(w, cpu, probe, threads)
    per_row = secs / n
    return max(1, int(math.ceil(w.T * per_row / target_s))), kv


def rows_phrase(stride: int) -> str:
    return "every query row" if stride == 1 else f"every {stride}th query row"


def cpu_baseline(w, inp, target_s=10.0):
    import oracle
    oracle.build()
    threads = oracle.default_threads()
    cpu = cpu_inputs(inp)
    stride, kv = pick_stride(w, cpu, threads, target_s)
    v, secs, n, _ = oracle_sample(w, cpu, stride, threads)
    return {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{w.name}: {rows_phrase(stride)} ({n} rows x {w.layer.num_heads} heads x "
                      f"{w.B} sequences, {secs:.1f} s) plus the K/V prologue charged pro rata; "
                      f"TFLOP/s of the unmasked pairs of those rows; float64 C, {threads} threads"}


def run_reference(args, dist: Dist):
    if dist.rank != 0:
        return 0
    import oracle
    oracle.build()
    w = W.E2B_SLIDING
    cpu = cpu_inputs(W.prefill_inputs(w, "cpu", seed=0))
    threads = oracle.default_threads()
    per_step = min(10.0, 150.0 / max(1, args.steps + args.warmup))
    stride, kv = pick_stride(w, cpu, threads, per_step)
    for _ in range(args.warmup):
        oracle_sample(w, cpu, stride, threads)
    vals, secs = [], 0.0
    for _ in range(args.steps):
        v, s, n, _ = oracle_sample(w, cpu, stride, threads)
        vals.append(v)
        secs += s
    value = float(np.mean(vals))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "global_batch": w.B, "seq_len": w.T,
                       "heads": [w.layer.num_heads, w.layer.num_kv_heads],
                       "head_dim": w.layer.head_dim, "window": w.layer.window},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": f"{rows_phrase(stride)} of {w.name}, all heads"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # 200 steps: the headline prefill's timed region (~15 ms) then spans many
    # NVML clock samples; the other legs take at most as many steps as
    # --extra-steps (the 31B global layer runs ~50 ms a step)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--extra-steps", type=int, default=10,
                    help="timed steps of the other prefill workloads and of decode (at most "
                         "--steps)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=W.E2B_SLIDING.name,
                    choices=[n for n in W.PREFILL_WORKLOADS if not n.startswith("tiny")])
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override the prefill workload's prompt length (profiling runs)")
    ap.add_argument("--no-extra-prefill", action="store_true",
                    help="only the headline prefill workload")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-only", action="store_true")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="sequences of the decode step (default: the workload's 64)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-kv-single", action="store_true",
                    help="skip the decode step over a single-tensor K=V cache")
    ap.add_argument("--no-qkv", action="store_true",
                    help="skip the fused QKV projection + prologue leg")
    ap.add_argument("--no-vision", action="store_true",
                    help="skip the vision-tower (bidirectional) attention leg")
    ap.add_argument("--no-graph", action="store_true", help="time eager calls, not a CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    dist = Dist() if args.impl == "ours" else None
    if args.impl == "reference":
        class _D:  # reference arm: CPU only, rank 0 prints
            rank = int(os.environ.get("RANK", "0"))
        return run_reference(args, _D())

    torch.cuda.set_device(dist.local)
    G.lib()  # fail loudly if the CUDA library is missing
    pk, pk_src = peaks()
    extra_steps = max(1, min(args.steps, args.extra_steps))
    want_cpu = dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline
    with ClockSampler(visible_index(dist.local), paused=True) as clk:
        if args.decode_only:
            dec = bench_decode(args, dist, pk, clk)
            dec["roofline"]["peak_source"] = f"{pk_src}: hbm_gbs"
            dec["clocks"] = clk.summary(dec["ms_per_step"])
            if dist.rank == 0:
                line = {"metric": METRIC, "value": dec["value"], "unit": "GB/s",
                        "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
                        "ms_per_step": dec["ms_per_step"], "higher_is_better": True,
                        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                        "data": "synthetic",
                        "config": {"workload": dec["workload"],
                                   "global_batch": dec["batch"] * dist.world},
                        "roofline": dec["roofline"], "cpu_baseline": dec["cpu_baseline"],
                        "e2e": None, "gpu_launches": dec["gpu_launches"], "clocks": dec["clocks"],
                        "decode": dec}
                print(json.dumps(line), flush=True)
            dist.close()
            return 0

        # the headline workload
        w = W.PREFILL_WORKLOADS[args.workload]
        if args.seq_len:  # a shorter prompt of the same layer (profiling runs)
            w = W.scaled_down(w, T=args.seq_len)
        pre = bench_prefill(args, dist, pk, w, clk, e2e=not args.no_e2e, steps=args.steps)
        head_clocks = clk.summary(pre["ms_per_step"])
        cpu = cpu_baseline(pre["workload"], pre["inputs"]) if want_cpu else None
        pre.pop("inputs")
        # the other prefill workloads (their own roofline and CPU baseline)
        legs = {}
        if not args.no_extra_prefill and not args.seq_len:
            for name, ow in W.PREFILL_WORKLOADS.items():
                if name.startswith("tiny") or name == w.name:
                    continue
                torch.cuda.empty_cache()
                res = bench_prefill(args, dist, pk, ow, clk, e2e=False, steps=extra_steps)
                res["roofline"]["peak_source"] = f"{pk_src}: bf16_tflops (burst)"
                res["cpu_baseline"] = cpu_baseline(ow, res["inputs"]) if want_cpu else None
                res.pop("inputs")
                legs[name] = public_prefill(res)
                del res
                torch.cuda.empty_cache()
        dec = None
        if not args.no_decode:
            dargs = argparse.Namespace(**{**vars(args), "steps": extra_steps})
            dec = bench_decode(dargs, dist, pk, clk)
            dec["roofline"]["peak_source"] = f"{pk_src}: hbm_gbs"
        qkv = vis = None
        if not args.no_qkv and not args.seq_len:
            torch.cuda.empty_cache()
            qkv = bench_qkv(args, dist, pk, clk, extra_steps)
            qkv["roofline"]["peak_source"] = f"{pk_src}: bf16_tflops (burst)"
        if not args.no_vision and not args.seq_len:
            torch.cuda.empty_cache()
            vis = bench_vision(args, dist, pk, clk, extra_steps)
            vis["roofline"]["peak_source"] = f"{pk_src}: bf16_tflops (burst)"
    roof = dict(pre["roofline"])
    roof["peak_source"] = f"{pk_src}: bf16_tflops (burst)"
    clocks = head_clocks or {}
    clocks = dict(clocks, samples_in_headline_steps=pre["clock_samples_in_steps"],
                  samples_all_timed_regions=len(clk.samples)) if clocks else None
    line = {"metric": METRIC, "value": pre["value"], "unit": "TFLOP/s", "n_gpus": dist.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": pre["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "global_batch": w.B * dist.world, "seq_len": w.T,
                       "heads": [w.layer.num_heads, w.layer.num_kv_heads],
                       "head_dim": w.layer.head_dim, "window": w.layer.window,
                       "parallelism": f"replicas{dist.world}",
                       "l2": "flushed (256 MiB write) before every timed prefill step",
                       "step": "one g4attn_prefill call replayed as a CUDA graph" if pre["graph"]
                               else "one g4attn_prefill call (eager)",
                       "unmasked_gflop_per_step": pre["flops"] / 1e9},
            "roofline": roof, "cpu_baseline": cpu, "e2e": pre["e2e"],
            "gpu_launches": pre["launches"], "clocks": clocks, "prefill": legs, "decode": dec,
            "qkv_prologue": qkv, "vision": vis}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
