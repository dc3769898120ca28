#!/usr/bin/env python
"""Benchmark of the RIPE verification step on B200.

A step is one verification pass of a draft block through every loop and recurrent layer
(for r in 0..R-1, for layer in 0..L-1: append plane r of the block, verify at loop r),
followed by the accept / rollback commit with window eviction -- every step of the hot
path -- captured once as a CUDA graph and replayed.  Inputs are resident in HBM before the
timed region; the per-step accepted lengths are drawn uniform on {0..B} from a seed.

Headline workload (the largest single-GPU configuration): long-context GQA verify, 4 recurrent
layers, 32 query / 8 kv heads x 128, R = 32, T = 32768, W = 64, B = 8, batch 8, planes
approaching the deepest at 0.85 per loop.  The same step is timed with the deepest-plane-only
layout, and the full cache on one layer (four layers would hold 137 GB).

With one GPU the same line also carries, as extra keys (``--extras``):
  huginn        the Huginn-shaped workload (55 MHA heads x 96, T = 1024, batch 1): the three
                layouts, warm and cold verify launches, the wavefront call and the draft phase;
  sweep         the window/block sweep, T = 4096, batch 4, one layer: all 15 (W, B) points;
  streaming     batch 16, Huginn heads, T0 = 512, 1000 decoding steps with ragged accepted
                lengths, append / verify / commit with eviction inside every step;
  fixed_memory  the largest batch of each layout whose cache fits a KV budget (20 GB) and its
                verification throughput (Huginn shape).

Prints one JSON line (rank 0).  Multi-GPU: one process per GPU (torchrun); every rank runs
its own replica of the workload (independent sequences, no collective in the data path);
times are the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "verify-attn GB/s (% of HBM peak) and verified tokens/s, RIPE vs full cache"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_L2_BYTES = 126 * 1024 * 1024

CONFIGS = {
    "long_gqa": dict(N=8, L=4, Hq=32, kvH=8, d=128, R=32, T=32768, W=64, B=8, rho=0.85,
                     workload="Long-context GQA: 4 recurrent layers, 32 q / 8 kv heads x 128, R=32, "
                              "T=32768, W=64, B=8, batch 8, rho 0.85"),
    "gqa64": dict(N=8, L=4, Hq=64, kvH=8, d=128, R=32, T=32768, W=64, B=8, rho=0.85,
                  workload="Long-context GQA, 64 query rows per kv head: 4 recurrent layers, 64 q / 8 kv "
                           "heads x 128, R=32, T=32768, W=64, B=8, batch 8, rho 0.85"),
    "huginn": dict(N=1, L=4, Hq=55, kvH=55, d=96, R=32, T=1024, W=64, B=8, rho=0.88,
                   workload="Huginn-shaped verify: 4 recurrent layers, 55 MHA heads x 96, R=32, "
                            "T=1024, W=64, B=8, batch 1, rho 0.88"),
    "sweep": dict(N=4, L=1, Hq=55, kvH=55, d=96, R=32, T=4096, W=64, B=8, rho=0.81,
                  workload="Window/block sweep point: 1 layer, 55 MHA heads x 96, R=32, T=4096, "
                           "W=64, B=8, batch 4, rho 0.81"),
    "streaming": dict(N=16, L=4, Hq=55, kvH=55, d=96, R=32, T=512, W=64, B=8, rho=0.88, max_T=8192,
                      steps=1000,
                      workload="Streaming decode: batch 16, 4 layers, 55 MHA heads x 96, R=32, W=64, B=8, "
                               "T0=512, 1000 steps, accepted length U{0..8} per sequence and step"),
    "tiny": dict(N=1, L=1, Hq=2, kvH=2, d=64, R=4, T=128, W=16, B=4, rho=0.88,
                 workload="Tiny RIPE check: 1 layer, 2 heads x 64, R=4, T=128, W=16, B=4, batch 1"),
}
SWEEP_W = (0, 8, 64, 256, 4096)
SWEEP_B = (4, 8, 16)
EXTRAS = ("huginn", "gqa64", "sweep", "streaming", "fixed_memory")
FIXED_MEMORY_GB = 20.0


# ------------------------------------------------------------------ accounting
def dual_keys(T, W, B, R, r, mode=0):
    """Window keys read at the deepest plane by later queries of the block (query window)."""
    if mode != 0 or r == R - 1:
        return 0
    D = max(0, T - W)
    return max(0, min(T, T + B - 1 - W) - D)


def verify_bytes(cfg, T_list, r):
    """Algorithmic bytes of one verify call: one plane per key read (K and V), the extra
    deepest-plane reads of the query window, the queries and the outputs."""
    row = 4 * cfg["kvH"] * cfg["d"]               # K + V, bf16, all kv heads, one position
    keys = sum(T + cfg["B"] + dual_keys(T, cfg["W"], cfg["B"], cfg["R"], r) for T in T_list)
    qo = 2 * len(T_list) * cfg["B"] * cfg["Hq"] * cfg["d"] * 2
    return keys * row + qo


DRAFT_LOOPS = 4  # draft depth of the timed draft phase: loops 0..3 of 32
DRAFT_SINK, DRAFT_WINDOW = 4, 256  # windowed draft attention: attention sink and sliding window


def draft_bytes(cfg, T_list, r, j, W):
    """Algorithmic bytes of one draft step (block position j at loop r): one plane per key
    t <= T + j, the deepest-plane reads of window keys older than W for that query, the
    query and the output."""
    row = 4 * cfg["kvH"] * cfg["d"]
    keys = sum(T + j + 1 + dual_keys(T, W, j + 1, cfg["R"], r) for T in T_list)
    return keys * row + 2 * len(T_list) * cfg["Hq"] * cfg["d"] * 2


def _code_only(text):
    """C/C++/CUDA source without comments and blank-run whitespace (comment edits do not
    change what a capture measured)."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(" ".join(line.split()) for line in text.splitlines() if line.strip())


def draft_window_bytes(cfg, T_list, r, j, W, sink, window):
    """Bytes one windowed draft step reads: the sink and window keys of the deepest-plane
    region, the window ring up to the query, the dual window keys, the query and the output."""
    row = 4 * cfg["kvH"] * cfg["d"]
    keys = 0
    for T in T_list:
        D = max(0, T - W)
        se = min(sink, D)
        dw0 = min(max(T + j - window, se), D)
        keys += se + (D - dw0) + (T + j + 1 - D) + dual_keys(T, W, j + 1, cfg["R"], r)
    return keys * row + 2 * len(T_list) * cfg["Hq"] * cfg["d"] * 2


# The sources that make each verify kernel (its translation unit, the shared headers and the host
# code that sizes its launch): an ncu capture stands for that kernel while they hash the same.
KERNEL_SOURCES = {
    "ripe_verify_kernel": ("ripe_verify.cu", "ripe_verify.cuh", "ripe_common.cuh"),
    "ripe_verify_tc_kernel": ("ripe_verify_tc.cu", "ripe_verify.cu", "ripe_verify.cuh", "ripe_common.cuh"),
}


def sources_digest(kernel="ripe_verify_kernel"):
    """sha256 over the code of a verify kernel's CUDA sources and the C header, comments removed
    (ties an ncu capture to a kernel version)."""
    import hashlib
    h = hashlib.sha256()
    files = [os.path.join(ROOT, "self_speculative_decode_b200", "csrc", f) for f in KERNEL_SOURCES[kernel]]
    files += [os.path.join(ROOT, "include", "ripe.h")]
    for path in files:
        with open(path, encoding="utf-8") as f:
            h.update(os.path.basename(path).encode() + b"\0" + _code_only(f.read()).encode())
    return h.hexdigest()


def captured_traffic(config, kernel=None):
    """DRAM bytes per verify launch from the committed ncu summary for this workload and kernel (the
    one the library runs now unless given), if the kernel's sources still hash to the captured ones."""
    kernel = kernel or verify_kernel_name(CONFIGS[config])
    path = os.path.join(ROOT, "profiles", "ripe_verify_traffic.txt")
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if "=" in line and not line.lstrip().startswith("#"):
                    k, v = line.split("=", 1)
                    kv[k.strip()] = v.strip()
        key = f"{config}.{kernel}"
        if kv.get(f"{kernel}.sources_sha256") != sources_digest(kernel) or f"{key}.bytes_per_launch" not in kv:
            return None
        return {"bytes_per_launch": float(kv[f"{key}.bytes_per_launch"]),
                "T": int(kv[f"{key}.T"]) if f"{key}.T" in kv else None,
                "algorithmic_bytes": float(kv[f"{key}.algorithmic_bytes"])
                if f"{key}.algorithmic_bytes" in kv else None}
    except Exception:
        return None


def traffic_for(config, alg_bytes, kernel=None):
    """DRAM bytes per timed verify launch: the captured launch's bytes, scaled by algorithmic bytes
    from the captured launch (the committed prefix length) to the timed ones (a few blocks longer;
    a launch's traffic grows with the key rows it reads)."""
    t = captured_traffic(config, kernel)
    if not t:
        return None
    if t["algorithmic_bytes"]:
        return t["bytes_per_launch"] * alg_bytes / t["algorithmic_bytes"]
    return t["bytes_per_launch"]


def traffic_basis(config, kernel=None):
    t = captured_traffic(config, kernel)
    if not t:
        return "no ncu capture of these sources for this workload and kernel"
    return (f"ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch at T = {t['T']} (cold L2), "
            "scaled by algorithmic bytes to the timed launches")


def verify_kernel_name(cfg):
    """The verify kernel that serves this workload's launches: the tcgen05 consumer only when the
    process selected it (ripe_set_verify_consumer, or RIPE_VERIFY_CONSUMER=tc) and the launch has
    more than 8 query rows per kv head."""
    from self_speculative_decode_b200 import ripe
    rows = cfg["B"] * cfg["Hq"] // cfg["kvH"]
    tc = rows > 8 and ripe.ripe_get_verify_consumer() == ripe.RIPE_CONSUMER_TC
    return "ripe_verify_tc_kernel" if tc else "ripe_verify_kernel"


def wave_loops(cfg):
    """A diagonal wavefront: block position j at loop R-1-4j (older positions deeper)."""
    return [max(0, cfg["R"] - 1 - 4 * j) for j in range(cfg["B"])]


def wave_bytes(cfg, T_list, W):
    """Algorithmic bytes of one wavefront call: the deepest region once, the window ring once
    per distinct loop, the dual window keys, queries and outputs."""
    loops = wave_loops(cfg)
    nl = len(set(loops))
    row = 4 * cfg["kvH"] * cfg["d"]
    keys = 0
    for T in T_list:
        D = max(0, T - W)
        dual = max(0, min(T, T + cfg["B"] - 1 - W) - D)
        keys += D + nl * (T + cfg["B"] - D) + dual
    return keys * row + 2 * len(T_list) * cfg["B"] * cfg["Hq"] * cfg["d"] * 2


def step_bytes(cfg, T_start, acc_rows):
    """Verify bytes of every step, from the committed lengths each step starts with."""
    T = list(T_start)
    out = []
    for row in acc_rows:
        out.append(sum(verify_bytes(cfg, T, r) for r in range(cfg["R"])) * cfg["L"])
        T = [t + int(a) for t, a in zip(T, row)]
    return out, T


def l2_note(per_call_bytes, step_distinct_bytes, l2_bytes):
    """Whether the timed launches can be served from L2, from the bytes they touch."""
    mb = 1e-6
    if per_call_bytes > l2_bytes:
        return (f"each verify launch reads {per_call_bytes * mb:.0f} MB > L2 {l2_bytes * mb:.0f} MB: "
                f"warm and cold launches both stream from HBM")
    if step_distinct_bytes > l2_bytes:
        return (f"a launch reads {per_call_bytes * mb:.1f} MB < L2 {l2_bytes * mb:.0f} MB; a step touches "
                f"{step_distinct_bytes * mb:.0f} MB > L2, so back-to-back (warm) launches are partly served "
                f"from L2: the HBM-bound figure is roofline_cold (L2 flushed before every launch)")
    return (f"a step touches {step_distinct_bytes * mb:.0f} MB <= L2 {l2_bytes * mb:.0f} MB: warm launches are "
            f"served largely from L2; roofline_cold flushes L2 before every launch")


def step_distinct_bytes(cfg, T, W, layers):
    """Distinct cache bytes one step reads: every layer's deepest region once, and the window
    ring (window + block) of every loop."""
    row = 4 * cfg["kvH"] * cfg["d"] * cfg["N"]
    D = max(0, T - W)
    return layers * row * (D + cfg["R"] * (T + cfg["B"] - D))


# ------------------------------------------------------------------ fixed-memory model
def fit_batch(kv_bytes_per_sequence, budget_bytes, cap=1024):
    """Largest batch whose key/value regions fit the budget (at most ``cap`` sequences)."""
    if kv_bytes_per_sequence <= 0:
        raise ValueError("kv_bytes_per_sequence must be positive")
    return int(min(budget_bytes // kv_bytes_per_sequence, cap))


def two_point_cost_model(t1_ms, tn_ms, n):
    """Step time t(N) = a + b N through (1, t1) and (n, tn); returns (a, b)."""
    b = (tn_ms - t1_ms) / (n - 1) if n > 1 else 0.0
    return t1_ms - b, b


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def l2_bytes():
    import torch
    try:
        return int(torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size)
    except Exception:
        return FALLBACK_L2_BYTES


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples during the timed region (read-only queries)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,utilization.gpu")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons, loaded = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    clk, cmax, util = float(parts[1]), float(parts[2]), float(parts[9])
                except ValueError:
                    continue
                smax = cmax
                if util < 1:       # keep the samples taken while the GPU was busy with the benchmark
                    continue
                loaded += 1
                sm.append(clk)
                for name, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "samples": loaded, "reasons": sorted(reasons)}


def gpu_id(index):
    """nvidia-smi identifier of a torch device (its UUID, robust to CUDA_VISIBLE_DEVICES)."""
    import torch
    try:
        u = str(torch.cuda.get_device_properties(index).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(index)


# ------------------------------------------------------------------ GPU workload
class Workload:
    """One cache with a loaded prefix, the step's inputs in HBM, and its CUDA graphs.

    ``replicate``: draw the planes for that many sequences and repeat them over the batch (for
    large batches whose timing does not depend on the values; see fixed_memory)."""

    def __init__(self, cfg, layout, total_steps, seed, device, fused=False, replicate=None, max_T=None):
        import torch
        from self_speculative_decode_b200.ripe import RipeCache
        from self_speculative_decode_b200.synth import PlaneSource, acceptance_draws

        self.cfg, self.layout, self.device = cfg, layout, device
        self.fused = fused
        N, L, Hq, kvH, d, R, T, B = (cfg[k] for k in ("N", "L", "Hq", "kvH", "d", "R", "T", "B"))
        self.max_T = max_T or T + B * (total_steps + 4)
        W = {"ripe": cfg["W"], "full": self.max_T, "deepest": 0}[layout]
        self.W = W
        self.cache = RipeCache(N, L, Hq, kvH, d, R, W, self.max_T, B)
        Ng = N if not replicate else min(N, replicate)
        reps = -(-N // Ng)

        def rep(x):
            return x if Ng == N else x.repeat((reps,) + (1,) * (x.dim() - 1))[:N].contiguous()

        for layer in range(L):
            src = PlaneSource(Ng, kvH, d, R, T, cfg["rho"], seed, layer=layer, backend="torch", device=device)
            for pl in range(R):
                self.cache.load_prefix(layer, pl, [T] * N, rep(src.plane(pl, "K")), rep(src.plane(pl, "V")))
            src.release()
        bf = torch.bfloat16
        self.q = torch.empty((L, R, N, B, Hq, d), dtype=bf, device=device)
        self.k = torch.empty((L, R, N, B, kvH, d), dtype=bf, device=device)
        self.v = torch.empty_like(self.k)
        self.out = torch.empty_like(self.q)
        for layer in range(L):
            src = PlaneSource(Ng, kvH, d, R, T, cfg["rho"], seed, layer=layer, backend="torch", device=device)
            for r in range(R):
                self.k[layer, r] = rep(src.block(0, r, B, "K"))
                self.v[layer, r] = rep(src.block(0, r, B, "V"))
                self.q[layer, r] = rep(src.queries(r, B, Hq))
        draws = acceptance_draws(seed, total_steps + 2, N, B)
        self.acc_host = draws
        self.acc_table = torch.tensor(draws, dtype=torch.int32, device=device)
        self.acc = torch.zeros(N, dtype=torch.int32, device=device)
        torch.cuda.synchronize()
        self.T0 = T

    def _appends_and_verifies(self, verify_only=False):
        c, cfg = self.cache, self.cfg
        for r in range(cfg["R"]):
            for layer in range(cfg["L"]):
                if verify_only:
                    c.verify_attn(layer, r, self.q[layer, r], out=self.out[layer, r])
                elif self.fused:  # append plane r of the block and verify at loop r: one launch
                    c.append_verify(layer, r, self.k[layer, r], self.v[layer, r], self.q[layer, r],
                                    out=self.out[layer, r])
                else:
                    c.append_block(layer, r, self.k[layer, r], self.v[layer, r])
                    c.verify_attn(layer, r, self.q[layer, r], out=self.out[layer, r])

    def append_all(self):
        for r in range(self.cfg["R"]):
            for layer in range(self.cfg["L"]):
                self.cache.append_block(layer, r, self.k[layer, r], self.v[layer, r])

    def capture(self):
        import torch
        c = self.cache
        # put the block in place so the verify-only graph can be captured, then both graphs
        self.append_all()
        torch.cuda.synchronize()
        n0 = c.launch_count()
        self.g_verify = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_verify):
            self._appends_and_verifies(verify_only=True)
        self.launches_verify = c.launch_count() - n0
        n0 = c.launch_count()
        self.g_step = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_step):
            self._appends_and_verifies()
            c.commit_device(self.acc)
        self.launches_step = c.launch_count() - n0
        torch.cuda.synchronize()

    def run_steps(self, first, count):
        for i in range(first, first + count):
            self.acc.copy_(self.acc_table[i], non_blocking=True)
            self.g_step.replay()

    def close(self):
        assert self.cache.device_error() == 0, "device error word set"
        self.cache.close()


def time_region(fn, sync_group):
    import torch
    torch.cuda.synchronize()
    if sync_group:
        import torch.distributed as dist
        dist.barrier()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record()
    fn()
    e.record()
    torch.cuda.synchronize()
    if sync_group:
        import torch.distributed as dist
        dist.barrier()
    return s.elapsed_time(e)  # ms


def max_over_ranks(x, dist_on, device="cuda"):
    """The slowest rank's time: every multi-GPU number is taken as the max over ranks."""
    if not dist_on:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(per_rank_bytes, max_ms, world):
    """Whole-job GB/s of replicas: every rank moves per_rank_bytes; the job takes the slowest rank's time."""
    return world * per_rank_bytes / (max_ms * 1e-3) / 1e9


class L2Flush:
    """Empties L2 of the timed kernel's data before a cold launch: a 512 MB buffer is written,
    then read back, so that L2 ends up holding clean lines of the flush buffer (a write alone
    would leave ~L2-size of dirty lines that the timed kernel would have to write back)."""

    def __init__(self, device, nbytes=512 * 1024 * 1024):
        import torch
        self.buf = torch.empty(nbytes // 4, dtype=torch.float32, device=device)
        self.acc = torch.empty((), dtype=torch.float32, device=device)

    def __call__(self, i):
        import torch
        self.buf.fill_(float(i))
        torch.sum(self.buf, dim=0, out=self.acc)


def verify_launch_timing(wl, reps, dist_on, peak, cold_calls=32):
    """The dominant kernel alone: the step's R*L verify launches back to back as a CUDA graph
    (warm: consecutive launches may find data in L2), and single launches with L2 flushed before
    each (cold).  Leaves the block appended."""
    import torch
    cfg = wl.cfg
    calls = cfg["R"] * cfg["L"]
    T_now = wl.cache.sync_lengths()
    wl.append_all()
    vbytes = sum(verify_bytes(cfg, T_now, r) for r in range(cfg["R"])) * cfg["L"] / calls
    wl.g_verify.replay()
    vms = max_over_ranks(time_region(lambda: [wl.g_verify.replay() for _ in range(reps)], dist_on), dist_on)
    warm_us = vms * 1e3 / (reps * calls)
    flush = L2Flush(wl.device)
    evs = []
    for i in range(min(calls, cold_calls)):
        r, layer = (i * 7) % cfg["R"], i % cfg["L"]
        flush(i)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        wl.cache.verify_attn(layer, r, wl.q[layer, r], out=wl.out[layer, r])
        b.record()
        evs.append((a, b, verify_bytes(cfg, T_now, r)))
    torch.cuda.synchronize()
    del flush
    cold_us = sum(a.elapsed_time(b) for a, b, _ in evs) * 1e3 / len(evs)
    cold_bytes = sum(x for _, _, x in evs) / len(evs)
    cold_us = max_over_ranks(cold_us, dist_on)
    return {"T": T_now, "warm": {"us_per_launch": warm_us, "bytes_per_launch": vbytes,
                                 "gbs": vbytes / (warm_us * 1e-6) / 1e9,
                                 "frac": vbytes / (warm_us * 1e-6) / 1e9 / peak},
            "cold": {"us_per_launch": cold_us, "bytes_per_launch": cold_bytes,
                     "gbs": cold_bytes / (cold_us * 1e-6) / 1e9,
                     "frac": cold_bytes / (cold_us * 1e-6) / 1e9 / peak, "launches": len(evs)}}


def bench_layout(cfg, layout, args, seed, device, dist_on, peak, want_extras, launches=True, replicate=None):
    import torch
    # warm-up + timed steps, then the per-call and the graph end-to-end steps
    wl = Workload(cfg, layout, args.warmup + 3 * args.steps + 2, seed, device, fused=args.append == "fused",
                  replicate=replicate)
    wl.capture()
    N = cfg["N"]
    res = {}
    wl.run_steps(0, args.warmup)
    T_start = wl.cache.sync_lengths()
    ms = time_region(lambda: wl.run_steps(args.warmup, args.steps), dist_on)
    ms = max_over_ranks(ms, dist_on)
    rows = wl.acc_host[args.warmup:args.warmup + args.steps]
    per_step, T_end = step_bytes(cfg, T_start, rows)
    T_check = wl.cache.sync_lengths()
    assert T_check == T_end, (T_check, T_end)
    nbytes = sum(per_step)
    res.update(ms_per_step=ms / args.steps, bytes_per_step=nbytes / args.steps,
               gbs=nbytes / (ms * 1e-3) / 1e9,
               verified_tokens_per_s=N * cfg["B"] * args.steps / (ms * 1e-3),
               accepted_tokens_per_s=float(rows.sum()) / (ms * 1e-3),
               T_range=[min(T_start), max(T_end)], launches_per_step=wl.launches_step)
    if launches:
        res["verify"] = verify_launch_timing(wl, max(3, args.steps), dist_on, peak)
    if want_extras:
        res["draft"] = draft_timing(wl, args, dist_on)
        res["e2e"] = e2e_per_call(wl, args, dist_on)
        res["e2e_graph"] = e2e_graph(wl, args, dist_on)
    if layout in ("ripe", "full") and launches:
        res["wave"] = wave_timing(wl, args, dist_on)
    wl.close()
    del wl
    torch.cuda.empty_cache()
    return res


def wave_timing(wl, args, dist_on):
    """One wavefront call per layer (block positions at different loops), as a CUDA graph."""
    import torch
    cfg, c = wl.cfg, wl.cache
    if c.stats()["block_len"] == 0:
        wl.append_all()
    loops = wave_loops(cfg)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for layer in range(cfg["L"]):
            c.verify_attn_wave(layer, loops, wl.q[layer, 0], out=wl.out[layer, 0])
    reps = max(3, args.steps)
    g.replay()
    ms = max_over_ranks(time_region(lambda: [g.replay() for _ in range(reps)], dist_on), dist_on)
    T_now = c.sync_lengths()
    us = ms * 1e3 / (reps * cfg["L"])
    nbytes = wave_bytes(cfg, T_now, wl.W)
    return dict(us_per_call=us, bytes_per_call=nbytes, gbs=nbytes / (us * 1e-6) / 1e9, loops=loops)


def draft_timing(wl, args, dist_on):
    """The draft phase of one block as a CUDA graph: for each block position j, every layer at
    loops 0 .. DRAFT_LOOPS-1 writes plane r of position j and attends its query (B = 1)."""
    import torch
    cfg, c = wl.cfg, wl.cache
    if c.stats()["block_len"]:          # a verification block is in flight: drop it first
        c.commit([0] * cfg["N"])
    L, B, rd = cfg["L"], cfg["B"], min(DRAFT_LOOPS, cfg["R"])
    dk = [[[wl.k[layer, r][:, j:j + 1].contiguous() for j in range(B)] for r in range(rd)] for layer in range(L)]
    dv = [[[wl.v[layer, r][:, j:j + 1].contiguous() for j in range(B)] for r in range(rd)] for layer in range(L)]
    dq = [[[wl.q[layer, r][:, j:j + 1].contiguous() for j in range(B)] for r in range(rd)] for layer in range(L)]
    dout = torch.empty_like(dq[0][0][0])
    n0 = c.launch_count()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for j in range(B):
            for layer in range(L):
                for r in range(rd):
                    c.draft_attn(layer, r, j, dk[layer][r][j], dv[layer][r][j], dq[layer][r][j], out=dout)
    launches = c.launch_count() - n0
    # the same phase with windowed draft attention (attention sink + sliding window)
    gw = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gw):
        for j in range(B):
            for layer in range(L):
                for r in range(rd):
                    c.draft_attn(layer, r, j, dk[layer][r][j], dv[layer][r][j], dq[layer][r][j], out=dout,
                                 sink=DRAFT_SINK, window=DRAFT_WINDOW)
    reps = max(3, args.steps)
    g.replay()
    gw.replay()
    ms = max_over_ranks(time_region(lambda: [g.replay() for _ in range(reps)], dist_on), dist_on)
    msw = max_over_ranks(time_region(lambda: [gw.replay() for _ in range(reps)], dist_on), dist_on)
    T_now = c.sync_lengths()            # the next append_block ends the draft phase
    nbytes = sum(draft_bytes(cfg, T_now, r, j, wl.W) for j in range(B) for r in range(rd)) * L
    wbytes = sum(draft_window_bytes(cfg, T_now, r, j, wl.W, DRAFT_SINK, DRAFT_WINDOW)
                 for j in range(B) for r in range(rd)) * L
    phase_ms, wphase_ms = ms / reps, msw / reps
    return dict(loops=rd, calls_per_block=launches, ms_per_block=phase_ms,
                us_per_call=phase_ms * 1e3 / launches, bytes_per_call=nbytes / launches,
                gbs=nbytes / (phase_ms * 1e-3) / 1e9,
                drafted_tokens_per_s=cfg["N"] * B / (phase_ms * 1e-3),
                windowed={"sink": DRAFT_SINK, "window": DRAFT_WINDOW, "ms_per_block": wphase_ms,
                          "us_per_call": wphase_ms * 1e3 / launches, "bytes_per_call": wbytes / launches,
                          "gbs": wbytes / (wphase_ms * 1e-3) / 1e9,
                          "drafted_tokens_per_s": cfg["N"] * B / (wphase_ms * 1e-3)})


def _pinned_like(t):
    import torch
    h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
    h.copy_(t)
    return h


def e2e_per_call(wl, args, dist_on):
    """Steps driven call by call through the public API (RipeCache.append_block / verify_attn /
    commit, no graph), with host buffers: every step copies its queries and block planes from
    pinned host memory to the device and its outputs back.  Two device input/output sets and two
    copy streams let the copies of one step overlap the work of the previous one."""
    import torch
    cfg, c = wl.cfg, wl.cache
    if c.stats()["block_len"]:
        c.commit([0] * cfg["N"])
    hq, hk, hv = _pinned_like(wl.q), _pinned_like(wl.k), _pinned_like(wl.v)
    ho = torch.empty(wl.out.shape, dtype=wl.out.dtype, pin_memory=True)
    bufs = [(wl.q, wl.k, wl.v, wl.out),
            (torch.empty_like(wl.q), torch.empty_like(wl.k), torch.empty_like(wl.v), torch.empty_like(wl.out))]
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    up_done, comp_done, down_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    first = args.warmup + args.steps
    steps = args.steps
    acc = [list(map(int, row)) for row in wl.acc_host[first:first + steps]]
    T_start = c.sync_lengths()
    L, R = cfg["L"], cfg["R"]

    def upload(b):
        q, k, v, _ = bufs[b]
        with torch.cuda.stream(up):
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            up_done[b].record(up)

    def run():
        up.wait_stream(comp)
        down.wait_stream(comp)
        upload(0)
        if steps > 1:
            upload(1)
        for i in range(steps):
            b = i % 2
            q, k, v, out = bufs[b]
            comp.wait_event(up_done[b])
            if i >= 2:
                comp.wait_event(down_done[b])
            for r in range(R):
                for layer in range(L):
                    c.append_block(layer, r, k[layer, r], v[layer, r])
                    c.verify_attn(layer, r, q[layer, r], out=out[layer, r])
            c.commit(acc[i])
            comp_done[b].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(comp_done[b])
                ho.copy_(out, non_blocking=True)
                down_done[b].record(down)
            if i + 2 < steps:
                up.wait_event(comp_done[b])
                upload(b)
        comp.wait_event(down_done[(steps - 1) % 2])

    ms = max_over_ranks(time_region(run, dist_on), dist_on)
    per_step, T_end = step_bytes(cfg, T_start, acc)
    assert c.sync_lengths() == T_end
    h2d = hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2 + cfg["N"] * 4
    return dict(value=sum(per_step) / (ms * 1e-3) / 1e9, unit="GB/s", ms_per_step=ms / steps,
                h2d_bytes_per_step=h2d, d2h_bytes_per_step=ho.numel() * 2,
                path="RipeCache.append_block / verify_attn per call, RipeCache.commit with host lengths; "
                     "pinned host copies in and out every step, overlapped with the previous step")


def e2e_graph(wl, args, dist_on):
    """The captured step replayed with host buffers: pinned host -> device copies of the step's
    queries and block planes, the graph, and the outputs copied back, all on one stream."""
    import torch
    c = wl.cache
    if c.stats()["block_len"]:
        c.commit([0] * wl.cfg["N"])
    hq, hk, hv = _pinned_like(wl.q), _pinned_like(wl.k), _pinned_like(wl.v)
    ho = torch.empty(wl.out.shape, dtype=wl.out.dtype, pin_memory=True)
    ha = torch.tensor(wl.acc_host, dtype=torch.int32).pin_memory()
    first = args.warmup + 2 * args.steps
    T_start = c.sync_lengths()

    def run():
        for i in range(first, first + args.steps):
            wl.q.copy_(hq, non_blocking=True)
            wl.k.copy_(hk, non_blocking=True)
            wl.v.copy_(hv, non_blocking=True)
            wl.acc.copy_(ha[i], non_blocking=True)
            wl.g_step.replay()
            ho.copy_(wl.out, non_blocking=True)

    ms = max_over_ranks(time_region(run, dist_on), dist_on)
    per_step, T_end = step_bytes(wl.cfg, T_start, wl.acc_host[first:first + args.steps])
    assert c.sync_lengths() == T_end      # graph replays leave the host copy of T behind
    h2d = hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2 + wl.cfg["N"] * 4
    return dict(value=sum(per_step) / (ms * 1e-3) / 1e9, unit="GB/s", ms_per_step=ms / args.steps,
                h2d_bytes_per_step=h2d, d2h_bytes_per_step=ho.numel() * 2,
                path="captured step (CUDA graph) replayed; pinned host copies in and out on the same stream")


def layout_summary(res, peak):
    out = {x: res[x] for x in ("ms_per_step", "gbs", "verified_tokens_per_s", "bytes_per_step", "T_range")}
    out["pct_of_hbm_peak"] = 100.0 * res["gbs"] / peak
    if "verify" in res:
        v = res["verify"]
        out["verify_warm_us"], out["verify_cold_us"] = v["warm"]["us_per_launch"], v["cold"]["us_per_launch"]
        out["frac_warm"], out["frac_cold"] = v["warm"]["frac"], v["cold"]["frac"]
    return out


# ------------------------------------------------------------------ extras
def huginn_extra(args, device, peak, l2):
    cfg = CONFIGS["huginn"]
    sub = argparse.Namespace(**vars(args))
    res = {lay: bench_layout(cfg, lay, sub, args.seed, device, False, peak, want_extras=(lay == "ripe"))
           for lay in ("ripe", "full", "deepest")}
    m = res["ripe"]
    v = m["verify"]
    out = {"workload": cfg["workload"],
           "layouts": {k: layout_summary(r, peak) for k, r in res.items()},
           "roofline": {"achieved": v["warm"]["gbs"], "frac": v["warm"]["frac"], "launch_us": v["warm"]["us_per_launch"],
                        "bytes_per_launch": v["warm"]["bytes_per_launch"],
                        "traffic": traffic_for("huginn", v["warm"]["bytes_per_launch"])},
           "roofline_cold": {"achieved": v["cold"]["gbs"], "frac": v["cold"]["frac"],
                             "launch_us": v["cold"]["us_per_launch"]},
           "l2": l2_note(v["warm"]["bytes_per_launch"], step_distinct_bytes(cfg, v["T"][0], cfg["W"], cfg["L"]), l2),
           "full_over_ripe_latency": res["full"]["ms_per_step"] / m["ms_per_step"]}
    wr, wf = res["ripe"]["wave"], res["full"]["wave"]
    out["wavefront"] = {
        "loops": wr["loops"], "ripe_us": wr["us_per_call"], "full_us": wf["us_per_call"],
        "latency_ratio_full_over_ripe": wf["us_per_call"] / wr["us_per_call"],
        "bytes_ratio_full_over_ripe": wf["bytes_per_call"] / wr["bytes_per_call"],
        "ripe_gbs": wr["gbs"], "full_gbs": wf["gbs"]}
    d = m["draft"]
    out["draft_phase"] = dict(d, pct_of_hbm_peak=100.0 * d["gbs"] / peak, cycle_ms=d["ms_per_block"] + m["ms_per_step"])
    out["e2e_per_call"] = m["e2e"]
    return out


def gqa64_extra(args, device, peak, l2):
    """Long-context GQA with 64 query rows per kv head (8 q heads per kv head), RIPE layout, on each
    consumer of such launches: the mma.sync kernel (the library's default) and the tcgen05 kernel.
    Per consumer: the step, each verify launch warm and cold against the roofline, the wavefront call."""
    from self_speculative_decode_b200 import ripe
    cfg = CONFIGS["gqa64"]
    sub = argparse.Namespace(**vars(args))
    out = {"workload": cfg["workload"], "consumers": {}}
    for name, consumer in (("mma", ripe.RIPE_CONSUMER_MMA), ("tc", ripe.RIPE_CONSUMER_TC)):
        prev = ripe.ripe_set_verify_consumer(consumer)
        try:
            kernel = verify_kernel_name(cfg)
            m = bench_layout(cfg, "ripe", sub, args.seed, device, False, peak, want_extras=False)
        finally:
            ripe.ripe_set_verify_consumer(prev)
        v = m["verify"]
        out["consumers"][name] = {
            "kernel": kernel, "layouts": {"ripe": layout_summary(m, peak)},
            "roofline": {"achieved": v["warm"]["gbs"], "frac": v["warm"]["frac"],
                         "launch_us": v["warm"]["us_per_launch"], "bytes_per_launch": v["warm"]["bytes_per_launch"],
                         "traffic": traffic_for("gqa64", v["warm"]["bytes_per_launch"], kernel),
                         "traffic_basis": traffic_basis("gqa64", kernel)},
            "roofline_cold": {"achieved": v["cold"]["gbs"], "frac": v["cold"]["frac"],
                              "launch_us": v["cold"]["us_per_launch"]},
            "wavefront": {"loops": m["wave"]["loops"], "ripe_us": m["wave"]["us_per_call"], "ripe_gbs": m["wave"]["gbs"]}}
        out["l2"] = l2_note(v["warm"]["bytes_per_launch"], step_distinct_bytes(cfg, v["T"][0], cfg["W"], cfg["L"]), l2)
    c = out["consumers"]
    out["tc_over_mma_launch"] = c["tc"]["roofline"]["launch_us"] / c["mma"]["roofline"]["launch_us"]
    return out


def sweep_extra(args, device, peak):
    """All 15 (W, B) points of the window/block sweep on one layer: per-launch verify latency
    (warm, and cold with L2 flushed), the step, and the wavefront call; the full cache's step
    and wavefront call per B.  The planes are drawn once and loaded into every cache."""
    import torch
    from self_speculative_decode_b200.ripe import RipeCache
    from self_speculative_decode_b200.synth import PlaneSource, acceptance_draws
    base = CONFIGS["sweep"]
    N, Hq, kvH, d, R, T = (base[k] for k in ("N", "Hq", "kvH", "d", "R", "T"))
    steps, warm = 5, 3
    Bmax = max(SWEEP_B)
    src = PlaneSource(N, kvH, d, R, T, base["rho"], args.seed + 77, backend="torch", device=device)
    planes = [(src.plane(pl, "K"), src.plane(pl, "V")) for pl in range(R)]
    src.release()
    blocks = [(src.block(0, pl, Bmax, "K"), src.block(0, pl, Bmax, "V")) for pl in range(R)]
    queries = {B: [src.queries(pl, B, Hq) for pl in range(R)] for B in SWEEP_B}
    points = []

    def one(W_layout, B, with_launches):
        cfg = dict(base, W=W_layout, B=B)
        max_T = T + B * (warm + steps + 6)
        Wc = min(W_layout, max_T)
        acc = acceptance_draws(args.seed + 78 + B, warm + steps + 2, N, B)
        c = RipeCache(N, 1, Hq, kvH, d, R, Wc, max_T, B)
        for pl in range(R):
            c.load_prefix(0, pl, [T] * N, planes[pl][0], planes[pl][1])
        kb = [blocks[pl][0][:, :B].contiguous() for pl in range(R)]
        vb = [blocks[pl][1][:, :B].contiguous() for pl in range(R)]
        out = torch.empty((R, N, B, Hq, d), dtype=torch.bfloat16, device=device)
        acc_dev = torch.tensor(acc, dtype=torch.int32, device=device)
        a_cur = torch.zeros(N, dtype=torch.int32, device=device)
        for pl in range(R):
            c.append_block(0, pl, kb[pl], vb[pl])
        Tn = c.sync_lengths()
        res = {}
        # the block in flight: the R verify launches of a step, and the wavefront call
        gv = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gv):
            for r in range(R):
                c.verify_attn(0, r, queries[B][r], out=out[r])
        gw = torch.cuda.CUDAGraph()
        loops = wave_loops(cfg)
        with torch.cuda.graph(gw):
            c.verify_attn_wave(0, loops, queries[B][0], out=out[0])
        if with_launches:
            gv.replay()
            ms = time_region(lambda: [gv.replay() for _ in range(steps)], False)
            vb_call = sum(verify_bytes(cfg, Tn, r) for r in range(R)) / R
            us = ms * 1e3 / (steps * R)
            flush = L2Flush(device)
            evs = []
            for i, r in enumerate((0, 9, 18, 27, 31)):
                flush(i)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                c.verify_attn(0, r, queries[B][r], out=out[r])
                e1.record()
                evs.append((e0, e1, verify_bytes(cfg, Tn, r)))
            torch.cuda.synchronize()
            del flush
            cold_us = sum(e0.elapsed_time(e1) for e0, e1, _ in evs) * 1e3 / len(evs)
            cold_b = sum(x for _, _, x in evs) / len(evs)
            res.update(verify_warm_us=us, verify_bytes=vb_call, frac_warm=vb_call / (us * 1e-6) / 1e9 / peak,
                       verify_cold_us=cold_us, frac_cold=cold_b / (cold_us * 1e-6) / 1e9 / peak)
        gw.replay()
        ms = time_region(lambda: [gw.replay() for _ in range(steps)], False)
        wus = ms * 1e3 / steps
        res.update(wave_us=wus, wave_gbs=wave_bytes(cfg, Tn, Wc) / (wus * 1e-6) / 1e9)
        c.commit([0] * N)
        # the step: R x (append + verify) + commit with eviction
        gs = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gs):
            for r in range(R):
                c.append_block(0, r, kb[r], vb[r])
                c.verify_attn(0, r, queries[B][r], out=out[r])
            c.commit_device(a_cur)
        for i in range(warm):
            a_cur.copy_(acc_dev[i])
            gs.replay()
        T0 = c.sync_lengths()

        def run():
            for i in range(warm, warm + steps):
                a_cur.copy_(acc_dev[i], non_blocking=True)
                gs.replay()

        ms = time_region(run, False)
        per, T1 = step_bytes(cfg, T0, acc[warm:warm + steps])
        assert c.sync_lengths() == T1
        res.update(step_ms=ms / steps, step_gbs=sum(per) / (ms * 1e-3) / 1e9)
        assert c.device_error() == 0
        del gv, gs, gw
        c.close()
        return res

    full = {}
    for B in SWEEP_B:
        full[B] = one(10 ** 9, B, False)
        for W in SWEEP_W:
            r = one(W, B, True)
            r.update(W=W, B=B, full_step_ms=full[B]["step_ms"], full_wave_us=full[B]["wave_us"],
                     full_over_ripe_step=full[B]["step_ms"] / r["step_ms"],
                     full_over_ripe_wave=full[B]["wave_us"] / r["wave_us"])
            points.append(r)
    del planes, blocks
    torch.cuda.empty_cache()
    return {"workload": "Window/block sweep: 1 layer, 55 MHA heads x 96, R=32, T=4096, batch 4, rho 0.81; "
                        "W in {0, 8, 64, 256, 4096} x B in {4, 8, 16}",
            "points": points,
            "note": "verify_*: the R verify launches of a step back to back (warm) or one at a time after an "
                    "L2 flush (cold); step: R x (append + verify) + commit/evict as a CUDA graph; wave: one call "
                    "with block position j at loop R-1-4j; full_*: the full cache at the same B"}


def streaming_extra(args, device, peak, steps=None):
    """Streaming decode with cache maintenance: every step appends plane r of a block of 8 for
    every loop and layer, verifies it, and commits an accepted length drawn U{0..8} per sequence
    (window eviction inside the commit).  The step is captured once as a CUDA graph: the kernels
    read the committed lengths from the device, so the same graph serves every step while the
    sequences grow apart."""
    import numpy as np
    import torch
    cfg = CONFIGS["streaming"]
    steps = steps or cfg["steps"]
    warm = 3
    wl = Workload(cfg, "ripe", warm + steps + 2, args.seed + 5, device, max_T=cfg["max_T"])
    wl.capture()
    wl.run_steps(0, warm)
    T_start = wl.cache.sync_lengths()
    ms = time_region(lambda: wl.run_steps(warm, steps), False)
    rows = wl.acc_host[warm:warm + steps]
    per_step, T_end = step_bytes(cfg, T_start, rows)
    assert wl.cache.sync_lengths() == T_end
    nbytes = sum(per_step)
    T_end_arr = np.array(T_end)
    out = {"workload": cfg["workload"], "steps": steps, "warmup": warm, "ms": ms,
           "ms_per_step_mean": ms / steps, "gbs": nbytes / (ms * 1e-3) / 1e9,
           "pct_of_hbm_peak": 100.0 * nbytes / (ms * 1e-3) / 1e9 / peak,
           "verified_tokens_per_s": cfg["N"] * cfg["B"] * steps / (ms * 1e-3),
           "accepted_tokens_per_s": float(rows.sum()) / (ms * 1e-3),
           "T_start": [min(T_start), max(T_start)],
           "T_final": {"min": int(T_end_arr.min()), "mean": float(T_end_arr.mean()), "max": int(T_end_arr.max())},
           "launches_per_step": wl.launches_step,
           "note": "accepted tokens/s include append, commit and window eviction; the same resident "
                   "block inputs every step (timing does not depend on their values)"}
    wl.close()
    del wl
    torch.cuda.empty_cache()
    return out


def fixed_memory(cfg, args, device, peak, budget_gb, steps=5, warmup=3):
    """Throughput at a fixed KV-memory budget: the largest batch of each layout whose cache fits,
    its verification step measured at that batch and at batch 1, and the two-point cost model
    t_step(N) = a + b * N.  Attention only: per-step costs outside this path (weights) are not in a.
    Large batches repeat the planes of four drawn sequences (timing does not depend on values)."""
    import torch
    from self_speculative_decode_b200.ripe import RipeCache
    sub = argparse.Namespace(**dict(vars(args), steps=steps, warmup=warmup, append="separate"))
    budget = budget_gb * 1e9
    total_steps = warmup + 2 * steps + 2
    max_T = cfg["T"] + cfg["B"] * (total_steps + 4)
    out = {}
    for layout in ("full", "ripe", "deepest"):
        W = {"ripe": cfg["W"], "full": max_T, "deepest": 0}[layout]
        probe = RipeCache(1, cfg["L"], cfg["Hq"], cfg["kvH"], cfg["d"], cfg["R"], W, max_T, cfg["B"])
        per_seq = probe.stats()["kv_bytes"]
        probe.close()
        n_max = fit_batch(per_seq, budget)
        res = {"kv_bytes_per_sequence": per_seq, "batch": n_max, "kv_gb": n_max * per_seq / 1e9}
        if n_max < 1:
            out[layout] = res
            continue
        for tag, n in (("n1", 1), ("nmax", n_max)):
            r = bench_layout(dict(cfg, N=n), layout, sub, args.seed, device, False, peak, want_extras=False,
                             launches=False, replicate=4)
            res[tag] = {k: r[k] for k in ("ms_per_step", "gbs", "verified_tokens_per_s", "accepted_tokens_per_s")}
            torch.cuda.empty_cache()
        a, b = two_point_cost_model(res["n1"]["ms_per_step"], res["nmax"]["ms_per_step"], n_max)
        res["cost_model_ms"] = {"a": a, "b_per_sequence": b}
        out[layout] = res
    full = out["full"].get("nmax", {}).get("verified_tokens_per_s")
    for layout, res in out.items():
        if full and "nmax" in res:
            res["throughput_over_full"] = res["nmax"]["verified_tokens_per_s"] / full
    return {"budget_gb": budget_gb, "workload": cfg["workload"], "steps": steps, "warmup": warmup,
            "layouts": out,
            "note": "largest batch whose KV cache fits the budget, verification steps timed as in the main "
                    "benchmark (CUDA graph, CUDA events); attention only"}


def profile_calls(cfg, args, device):
    """A few verify calls of one layer of the workload, nothing else: the launch ncu captures."""
    import torch
    one = dict(cfg, L=1)
    wl = Workload(one, "ripe", 1, args.seed, device)
    wl.append_all()
    for i in range(args.profile_calls):
        wl.cache.verify_attn(0, 0, wl.q[0, 0], out=wl.out[0, 0])
    torch.cuda.synchronize()
    T = wl.cache.sync_lengths()
    wl.close()
    print(json.dumps({"profile_calls": args.profile_calls, "workload": one["workload"] + " (1 layer)",
                      "T": T, "algorithmic_bytes_per_call": verify_bytes(one, T, 0)}))


def profile_step(cfg, args, device, layout):
    """Eager steps of the workload (no graph) for a launch-by-launch ncu capture: per step
    R*L x (append + verify) + commit/evict, with host-side accepted lengths."""
    import torch
    wl = Workload(cfg, layout, args.profile_steps + 2, args.seed, device)
    for i in range(args.profile_steps):
        wl._appends_and_verifies()
        wl.cache.commit(list(map(int, wl.acc_host[i])))
    torch.cuda.synchronize()
    T = wl.cache.sync_lengths()
    wl.close()
    print(json.dumps({"profile_steps": args.profile_steps, "layout": layout, "workload": cfg["workload"], "T": T}))


# ------------------------------------------------------------------ CPU oracle
class OracleSample:
    """A bounded sample of the workload for the CPU oracle: the first sequence and (at most) the
    first two kv heads with their query heads, layer 0, verify calls at loops 0..3 and R-1."""

    def __init__(self, cfg, seed=0, loops=4, seqs=1, heads=2):
        import numpy as np
        from oracle import ripe_oracle as orc
        from self_speculative_decode_b200.synth import PlaneSource
        self.orc = orc
        N, kvH, d, R, T, B, W = (cfg[k] for k in ("N", "kvH", "d", "R", "T", "B", "W"))
        self.Ns, self.kvHs = min(N, seqs), min(kvH, heads)
        g = cfg["Hq"] // kvH
        self.g, self.B, self.R, self.W = g, B, R, W
        self.cfg = dict(cfg, N=self.Ns, kvH=self.kvHs, Hq=self.kvHs * g)
        src = PlaneSource(self.Ns, self.kvHs, d, R, T + B, cfg["rho"], seed)
        keep_planes = set(range(min(loops, R))) | {R - 1}
        oc = orc.OracleCache(self.Ns, 1, self.kvHs, d, R, W, T + B, value_planes=keep_planes)
        for pl in range(R):
            keep = pl in keep_planes
            oc.load_prefix(0, pl, [T] * self.Ns, src.plane(pl, "K") if keep else None,
                           src.plane(pl, "V") if keep else None)
        for pl in range(R):
            if pl in keep_planes:
                kp, vp = src.plane(pl, "K"), src.plane(pl, "V")
                oc.append(0, pl, np.ascontiguousarray(kp[:, :, T:T + B].transpose(0, 2, 1, 3)),
                          np.ascontiguousarray(vp[:, :, T:T + B].transpose(0, 2, 1, 3)))
            else:
                oc.append(0, pl, None, None, B=B)
        self.T = oc.T.copy()
        self.inputs = [(r, oc.verify_inputs(0, r)[:4], orc.bf16_to_f64(src.queries(r, B, self.kvHs * g)))
                       for r in sorted(keep_planes)]
        self.calls = 0

    def run(self, seconds):
        """Oracle verify calls until ``seconds`` of oracle time; returns (GB/s, calls, seconds, threads)."""
        spent, calls, nbytes = 0.0, 0, 0
        while spent < seconds:
            r, (Kr, Vr, Kl, Vl), q = self.inputs[self.calls % len(self.inputs)]
            t0 = time.perf_counter()
            self.orc.verify(self.T, self.B, r, self.R, self.W, self.g, Kr, Vr, Kl, Vl, q)
            spent += time.perf_counter() - t0
            calls += 1
            self.calls += 1
            nbytes += verify_bytes(self.cfg, list(self.T), r)
        threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
        return nbytes / spent / 1e9, calls, spent, threads

    def describe(self, calls, seconds):
        return (f"{calls} oracle verify calls of layer 0 (loops 0-3 and {self.R - 1}) on {self.Ns} sequence(s) x "
                f"{self.kvHs} kv head(s) of the workload, {seconds:.1f} s of oracle time")


def run_reference(args, cfg, rank):
    """The oracle as the reference arm: each step is one bounded sample of the workload."""
    if rank != 0:
        return
    samp = OracleSample(cfg, seed=args.seed)
    per_step = []
    calls_total = 0
    for i in range(args.warmup + args.steps):
        gbs, calls, sec, threads = samp.run(0.5)
        if i >= args.warmup:
            per_step.append((gbs, sec, calls))
            calls_total += calls
    value = sum(g * s for g, s, _ in per_step) / sum(s for _, s, _ in per_step)
    ms = sum(s for _, s, _ in per_step) / len(per_step) * 1e3
    sample = samp.describe(calls_total, sum(s for _, s, _ in per_step)) + ", about 0.5 s per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg["workload"], "layout": "ripe", "parallelism": "cpu oracle, OpenMP"},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ripe", choices=["ripe", "reference"])
    ap.add_argument("--config", default="long_gqa", choices=sorted(CONFIGS))
    ap.add_argument("--layouts", default=None,
                    help="comma list of ripe, full, deepest (default: all three; long_gqa: the full cache "
                         "on one layer)")
    ap.add_argument("--extras", default=None,
                    help=f"comma list of {', '.join(EXTRAS)} or 'none' (default: all of them with one GPU, "
                         f"none with several)")
    ap.add_argument("--streaming-steps", type=int, default=None)
    ap.add_argument("--profile-calls", type=int, default=0,
                    help="only run this many verify calls of layer 0 (for ncu captures) and exit")
    ap.add_argument("--profile-steps", type=int, default=0,
                    help="only run this many eager steps (no graph) of --profile-layout and exit")
    ap.add_argument("--profile-layout", default="ripe", choices=["ripe", "full", "deepest"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--fixed-memory-gb", type=float, default=0.0,
                    help="only run the fixed-memory throughput comparison at this KV budget and exit")
    ap.add_argument("--append", default="separate", choices=["separate", "fused"],
                    help="block append as its own launch before each verify, or inside it (ripe_append_verify)")
    ap.add_argument("--seed", type=int, default=0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = CONFIGS[args.config]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, cfg, rank)
        return

    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_on = world > 1
    if dist_on:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    from self_speculative_decode_b200 import ripe
    ripe.lib()
    peak, peak_kind = hbm_peak()
    l2 = l2_bytes()

    if args.profile_calls:
        profile_calls(cfg, args, device)
        return
    if args.profile_steps:
        profile_step(cfg, args, device, args.profile_layout)
        return
    if args.fixed_memory_gb:
        print(json.dumps(fixed_memory(cfg, args, device, peak, args.fixed_memory_gb)), flush=True)
        return
    if args.layouts is None:
        args.layouts = "ripe,deepest,full"
    layouts = [x for x in args.layouts.split(",") if x]
    if args.extras is None:
        extras = list(EXTRAS) if world == 1 else []
    else:
        extras = [] if args.extras == "none" else [x for x in args.extras.split(",") if x]
    results = {}
    clocks = ClockSampler(gpu_id(local))
    clocks.start()
    time.sleep(0.3)  # nvidia-smi needs a moment before its first sample
    layout_cfg = {}
    for lay in layouts:
        lc = cfg
        if lay == "full" and args.config == "long_gqa":
            lc = dict(cfg, L=1)   # four layers of the full cache would need 137 GB
        layout_cfg[lay] = lc
        results[lay] = bench_layout(lc, lay, args, args.seed + 1000 * rank, device, dist_on, peak,
                                    want_extras=(lay == layouts[0]))
    extra_out = {}
    for name in extras:
        if name == "huginn" and args.config != "huginn":
            extra_out["huginn"] = huginn_extra(args, device, peak, l2)
        elif name == "gqa64" and args.config != "gqa64":
            extra_out["gqa64"] = gqa64_extra(args, device, peak, l2)
        elif name == "sweep":
            extra_out["sweep"] = sweep_extra(args, device, peak)
        elif name == "streaming":
            extra_out["streaming"] = streaming_extra(args, device, peak, args.streaming_steps)
        elif name == "fixed_memory":
            extra_out["fixed_memory"] = fixed_memory(CONFIGS["huginn"], args, device, peak, FIXED_MEMORY_GB)
    clock_rec = clocks.stop()
    main_l = layouts[0]
    m = results[main_l]
    v = m["verify"]
    value = job_throughput(m["bytes_per_step"] * args.steps, m["ms_per_step"] * args.steps, world)
    T_bench = v["T"]
    traffic_val = traffic_for(args.config, v["warm"]["bytes_per_launch"])
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg["workload"], "layout": main_l,
                   "step": ("R*L x (append plane r + verify at loop r" +
                            (", one launch" if args.append == "fused" else ", two launches") +
                            ") + commit/evict, CUDA graph"),
                   "T_range": m["T_range"],
                   "l2": l2_note(v["warm"]["bytes_per_launch"],
                                 step_distinct_bytes(cfg, T_bench[0], cfg["W"], cfg["L"]), l2),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "pct_of_hbm_peak": 100.0 * m["gbs"] / peak,
        "verified_tokens_per_s": m["verified_tokens_per_s"] * world,
        "accepted_tokens_per_s": m["accepted_tokens_per_s"] * world,
        "layouts": {k: dict(layout_summary(r, peak), layers=layout_cfg[k]["L"]) for k, r in results.items()},
        "roofline": {"bound": "hbm", "achieved": v["warm"]["gbs"], "peak": peak, "unit": "GB/s",
                     "frac": v["warm"]["frac"], "traffic": traffic_val, "peak_kind": peak_kind,
                     "kernel": verify_kernel_name(cfg), "launch_us": v["warm"]["us_per_launch"],
                     "bytes_per_launch": v["warm"]["bytes_per_launch"], "T": T_bench,
                     "traffic_basis": traffic_basis(args.config),
                     "note": "R*L verify launches back to back as in the step"},
        "roofline_cold": {"achieved": v["cold"]["gbs"], "frac": v["cold"]["frac"],
                          "launch_us": v["cold"]["us_per_launch"], "note": "L2 flushed before each launch"},
        "e2e": m["e2e"],
        "e2e_graph": m["e2e_graph"],
        "gpu_launches": m["launches_per_step"] * args.steps,
        "clocks": dict(clock_rec, window="every layout's warm-up, timed steps, per-launch and end-to-end "
                                         "timing, and the extras"),
    }
    if "full" in results and main_l == "ripe":
        lf = layout_cfg["full"]["L"]
        line["full_over_ripe_latency_per_layer"] = (results["full"]["ms_per_step"] / lf) / (m["ms_per_step"] / cfg["L"])
        if "wave" in results["full"]:
            wr, wf = results["ripe"]["wave"], results["full"]["wave"]
            line["wavefront"] = {
                "loops": wr["loops"], "ripe_us": wr["us_per_call"], "full_us": wf["us_per_call"],
                "latency_ratio_full_over_ripe": wf["us_per_call"] / wr["us_per_call"],
                "bytes_ratio_full_over_ripe": wf["bytes_per_call"] / wr["bytes_per_call"],
                "ripe_gbs": wr["gbs"], "full_gbs": wf["gbs"],
                "note": "one call per layer verifies every block position at its own loop; the deepest "
                        "region is read once for all loops, the window once per loop"}
    if "draft" in m:
        d = m["draft"]
        line["draft_phase"] = dict(d, pct_of_hbm_peak=100.0 * d["gbs"] / peak,
                                   cycle_ms=d["ms_per_block"] + m["ms_per_step"],
                                   note=f"draft-then-verify: B positions drafted one at a time at loops "
                                        f"0..{d['loops'] - 1} of every layer (ripe_draft_attn, B=1 decode "
                                        f"shape), then the step verifies the block at all R loops; a read-only "
                                        f"stream can exceed the copy-measured peak slightly")
    line.update(extra_out)
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        samp = OracleSample(cfg, seed=args.seed)
        gbs, calls, sec, threads = samp.run(args.cpu_seconds)
        line["cpu_baseline"] = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": samp.describe(calls, sec)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
