#!/usr/bin/env python
"""Benchmark of the RIPE verification step on B200.

A step is one verification pass of a draft block through every loop and recurrent layer
(for r in 0..R-1, for layer in 0..L-1: append plane r of the block, verify at loop r),
followed by the accept / rollback commit with window eviction -- every step of the hot
path -- captured once as a CUDA graph and replayed.  Inputs are resident in HBM before the
timed region; the per-step accepted lengths are drawn uniform on {0..B} from a seed.

Default workload: Huginn-shaped verify (4 recurrent layers, 55 MHA heads x 96, R = 32,
T = 1024, W = 64, B = 8, batch 1, planes approaching the deepest at 0.88 per loop).
The same step is also timed with the full-cache and deepest-plane-only layouts.

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

CONFIGS = {
    "huginn": dict(N=1, L=4, Hq=55, kvH=55, d=96, R=32, T=1024, W=64, B=8, rho=0.88,
                   workload="Huginn-shaped verify: 4 recurrent layers, 55 MHA heads x 96, R=32, "
                            "T=1024, W=64, B=8, batch 1, rho 0.88"),
    "long_gqa": dict(N=8, L=4, Hq=32, kvH=8, d=128, R=32, T=32768, W=64, B=8, rho=0.85,
                     workload="Long-context GQA: 4 recurrent layers, 32 q / 8 kv heads x 128, R=32, "
                              "T=32768, W=64, B=8, batch 8, rho 0.85"),
    "sweep": dict(N=4, L=1, Hq=55, kvH=55, d=96, R=32, T=4096, W=64, B=8, rho=0.81,
                  workload="Window/block sweep point: 1 layer, 55 MHA heads x 96, R=32, T=4096, "
                           "W=64, B=8, batch 4, rho 0.81"),
    "tiny": dict(N=1, L=1, Hq=2, kvH=2, d=64, R=4, T=128, W=16, B=4, rho=0.88,
                 workload="Tiny RIPE check: 1 layer, 2 heads x 64, R=4, T=128, W=16, B=4, batch 1"),
}


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
    qo = 2 * cfg["N"] * cfg["B"] * cfg["Hq"] * cfg["d"] * 2
    return keys * row + qo


DRAFT_LOOPS = 4  # draft depth of the timed draft phase: loops 0..3 of 32
DRAFT_SINK, DRAFT_WINDOW = 4, 256  # windowed draft attention: attention sink and sliding window


def draft_bytes(cfg, T_list, r, j, W):
    """Algorithmic bytes of one draft step (block position j at loop r): one plane per key
    t <= T + j, the deepest-plane reads of window keys older than W for that query, the
    query and the output."""
    row = 4 * cfg["kvH"] * cfg["d"]
    keys = sum(T + j + 1 + dual_keys(T, W, j + 1, cfg["R"], r) for T in T_list)
    return keys * row + 2 * cfg["N"] * cfg["Hq"] * cfg["d"] * 2


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
    return keys * row + 2 * cfg["N"] * cfg["Hq"] * cfg["d"] * 2


def sources_digest():
    """sha256 over the code of the library's CUDA sources and C header, comments removed
    (ties an ncu capture to a kernel version)."""
    import glob
    import hashlib
    h = hashlib.sha256()
    files = sorted(glob.glob(os.path.join(ROOT, "self_speculative_decode_b200", "csrc", "*.cu*")))
    files += [os.path.join(ROOT, "include", "ripe.h")]
    for path in files:
        with open(path, encoding="utf-8") as f:
            h.update(os.path.basename(path).encode() + b"\0" + _code_only(f.read()).encode())
    return h.hexdigest()


def captured_traffic(config):
    """DRAM bytes per verify launch from the committed ncu summary, if it matches these sources."""
    path = os.path.join(ROOT, "profiles", "ripe_verify_traffic.txt")
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if "=" in line and not line.lstrip().startswith("#"):
                    k, v = line.split("=", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("sources_sha256") != sources_digest() or f"{config}.bytes_per_launch" not in kv:
            return None
        return float(kv[f"{config}.bytes_per_launch"])
    except Exception:
        return None


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
    return keys * row + 2 * cfg["N"] * cfg["B"] * cfg["Hq"] * cfg["d"] * 2


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


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
                                          "--format=csv,noheader,nounits", "-lms", "20"],
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
                "samples": loaded, "reasons": sorted(reasons),
                "window": "every layout's warm-up, timed steps, per-launch and end-to-end timing"}


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
    """One cache with a loaded prefix, the step's inputs in HBM, and its CUDA graphs."""

    def __init__(self, cfg, layout, total_steps, seed, device, fused=False):
        import torch
        from self_speculative_decode_b200.ripe import RipeCache
        from self_speculative_decode_b200.synth import PlaneSource, acceptance_draws

        self.cfg, self.layout, self.device = cfg, layout, device
        self.fused = fused
        N, L, Hq, kvH, d, R, T, B = (cfg[k] for k in ("N", "L", "Hq", "kvH", "d", "R", "T", "B"))
        self.max_T = T + B * (total_steps + 4)
        W = {"ripe": cfg["W"], "full": self.max_T, "deepest": 0}[layout]
        self.W = W
        self.cache = RipeCache(N, L, Hq, kvH, d, R, W, self.max_T, B)
        for layer in range(L):
            src = PlaneSource(N, kvH, d, R, T, cfg["rho"], seed, layer=layer, backend="torch", device=device)
            for pl in range(R):
                self.cache.load_prefix(layer, pl, [T] * N, src.plane(pl, "K"), src.plane(pl, "V"))
            src.release()
        bf = torch.bfloat16
        self.q = torch.empty((L, R, N, B, Hq, d), dtype=bf, device=device)
        self.k = torch.empty((L, R, N, B, kvH, d), dtype=bf, device=device)
        self.v = torch.empty_like(self.k)
        self.out = torch.empty_like(self.q)
        for layer in range(L):
            src = PlaneSource(N, kvH, d, R, T, cfg["rho"], seed, layer=layer, backend="torch", device=device)
            for r in range(R):
                self.k[layer, r] = src.block(0, r, B, "K")
                self.v[layer, r] = src.block(0, r, B, "V")
                self.q[layer, r] = src.queries(r, B, Hq)
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

    def capture(self):
        import torch
        c = self.cache
        # put the block in place so the verify-only graph can be captured, then both graphs
        for r in range(self.cfg["R"]):
            for layer in range(self.cfg["L"]):
                c.append_block(layer, r, self.k[layer, r], self.v[layer, r])
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


def step_bytes(cfg, T_start, acc_rows):
    """Verify bytes of every step, from the committed lengths each step starts with."""
    T = list(T_start)
    out = []
    for row in acc_rows:
        out.append(sum(verify_bytes(cfg, T, r) for r in range(cfg["R"])) * cfg["L"])
        T = [t + int(a) for t, a in zip(T, row)]
    return out, T


def bench_layout(cfg, layout, args, seed, device, dist_on, want_extras):
    import torch
    wl = Workload(cfg, layout, args.warmup + 2 * args.steps + 2, seed, device, fused=args.append == "fused")
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
    if want_extras:
        res["draft"] = draft_timing(wl, args, dist_on)
    nbytes = sum(per_step)
    res.update(ms_per_step=ms / args.steps, bytes_per_step=nbytes / args.steps,
               gbs=nbytes / (ms * 1e-3) / 1e9,
               verified_tokens_per_s=N * cfg["B"] * args.steps / (ms * 1e-3),
               accepted_tokens_per_s=float(rows.sum()) / (ms * 1e-3),
               T_range=[min(T_start), max(T_end)], launches_per_step=wl.launches_step)
    if want_extras:
        # dominant kernel: verify, the same R*L launches as in the step, back to back (graph)
        calls = cfg["R"] * cfg["L"]
        reps = max(3, args.steps)
        T_now = wl.cache.sync_lengths()
        # a real block at the current lengths for the verify-only launches below
        for r in range(cfg["R"]):
            for layer in range(cfg["L"]):
                wl.cache.append_block(layer, r, wl.k[layer, r], wl.v[layer, r])
        vbytes = sum(verify_bytes(cfg, T_now, r) for r in range(cfg["R"])) * cfg["L"] / calls
        vms = time_region(lambda: [wl.g_verify.replay() for _ in range(reps)], dist_on)
        res["verify_warm"] = dict(us_per_launch=vms * 1e3 / (reps * calls), bytes_per_launch=vbytes)
        # cold: L2 flushed (a 512 MB write) before every launch, each launch bracketed by events
        flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
        evs = []
        for i in range(min(calls, 64)):
            r, layer = divmod(i, cfg["L"])
            flush.fill_(float(i))
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            wl.cache.verify_attn(layer, r % cfg["R"], wl.q[layer, r % cfg["R"]], out=wl.out[layer, r % cfg["R"]])
            b.record()
            evs.append((a, b, verify_bytes(cfg, T_now, r % cfg["R"])))
        torch.cuda.synchronize()
        tot_ms = sum(a.elapsed_time(b) for a, b, _ in evs)
        res["verify_cold"] = dict(us_per_launch=tot_ms * 1e3 / len(evs),
                                  bytes_per_launch=sum(x for _, _, x in evs) / len(evs))
        del flush
        res["e2e"] = e2e_steps(wl, args, dist_on)
    if layout in ("ripe", "full"):
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
        for r in range(cfg["R"]):
            for layer in range(cfg["L"]):
                c.append_block(layer, r, wl.k[layer, r], wl.v[layer, r])
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
    T_now = c.sync_lengths()
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


def e2e_steps(wl, args, dist_on):
    """The same steps through the public API with host buffers: pinned host -> device copies of
    the step's queries and block planes, the step, and the outputs copied back, all timed."""
    import torch
    hq = torch.empty(wl.q.shape, dtype=wl.q.dtype, pin_memory=True)
    hk = torch.empty(wl.k.shape, dtype=wl.k.dtype, pin_memory=True)
    hv = torch.empty(wl.v.shape, dtype=wl.v.dtype, pin_memory=True)
    ho = torch.empty(wl.out.shape, dtype=wl.out.dtype, pin_memory=True)
    hq.copy_(wl.q)
    hk.copy_(wl.k)
    hv.copy_(wl.v)
    ha = torch.tensor(wl.acc_host, dtype=torch.int32).pin_memory()
    first = args.warmup + args.steps
    T_start = wl.cache.sync_lengths()

    def run():
        for i in range(first, first + args.steps):
            wl.q.copy_(hq, non_blocking=True)
            wl.k.copy_(hk, non_blocking=True)
            wl.v.copy_(hv, non_blocking=True)
            wl.acc.copy_(ha[i], non_blocking=True)
            wl.g_step.replay()
            ho.copy_(wl.out, non_blocking=True)

    ms = max_over_ranks(time_region(run, dist_on), dist_on)
    per_step, _ = step_bytes(wl.cfg, T_start, wl.acc_host[first:first + args.steps])
    h2d = hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2 + wl.cfg["N"] * 4
    return dict(value=sum(per_step) / (ms * 1e-3) / 1e9, unit="GB/s", ms_per_step=ms / args.steps,
                h2d_bytes_per_step=h2d, d2h_bytes_per_step=ho.numel() * 2)


def fixed_memory(cfg, args, device):
    """Throughput at a fixed KV-memory budget: the largest batch of each layout whose cache fits in
    args.fixed_memory_gb, its verification step measured at that batch and at batch 1, and the
    two-point cost model t_step(N) = a + b * N.  Attention only: per-step costs outside this path
    (weights) are not in a, which is why the gain at fixed memory here is the batch ratio's effect
    on a only."""
    import torch
    from self_speculative_decode_b200.ripe import RipeCache
    budget = args.fixed_memory_gb * 1e9
    total_steps = args.warmup + 2 * args.steps + 2
    max_T = cfg["T"] + cfg["B"] * (total_steps + 4)
    out = {}
    for layout in ("full", "ripe", "deepest"):
        W = {"ripe": cfg["W"], "full": max_T, "deepest": 0}[layout]
        probe = RipeCache(1, cfg["L"], cfg["Hq"], cfg["kvH"], cfg["d"], cfg["R"], W, max_T, cfg["B"])
        per_seq = probe.stats()["kv_bytes"]
        probe.close()
        n_max = int(min(budget // per_seq, 1024))
        res = {"kv_bytes_per_sequence": per_seq, "batch": n_max, "kv_gb": n_max * per_seq / 1e9}
        if n_max < 1:
            out[layout] = res
            continue
        for tag, n in (("n1", 1), ("nmax", n_max)):
            r = bench_layout(dict(cfg, N=n), layout, args, args.seed, device, False, want_extras=False)
            res[tag] = {k: r[k] for k in ("ms_per_step", "gbs", "verified_tokens_per_s", "accepted_tokens_per_s")}
            torch.cuda.empty_cache()
        t1, tn = res["n1"]["ms_per_step"], res["nmax"]["ms_per_step"]
        b = (tn - t1) / (n_max - 1) if n_max > 1 else 0.0
        res["cost_model_ms"] = {"a": t1 - b, "b_per_sequence": b}
        out[layout] = res
    full = out["full"].get("nmax", {}).get("verified_tokens_per_s")
    for layout, res in out.items():
        if full and "nmax" in res:
            res["throughput_over_full"] = res["nmax"]["verified_tokens_per_s"] / full
    print(json.dumps({"fixed_memory_gb": args.fixed_memory_gb, "workload": cfg["workload"],
                      "steps": args.steps, "warmup": args.warmup, "layouts": out,
                      "note": "largest batch whose KV cache fits the budget, verification steps timed as "
                              "in the main benchmark (CUDA graph, CUDA events); attention only"}), flush=True)


def profile_calls(cfg, args, device):
    """A few verify calls of one layer of the workload, nothing else: the launch ncu captures."""
    import torch
    one = dict(cfg, L=1)
    wl = Workload(one, "ripe", 1, args.seed, device)
    for r in range(one["R"]):
        wl.cache.append_block(0, r, wl.k[0, r], wl.v[0, r])
    for i in range(args.profile_calls):
        wl.cache.verify_attn(0, 0, wl.q[0, 0], out=wl.out[0, 0])
    torch.cuda.synchronize()
    wl.close()
    print(json.dumps({"profile_calls": args.profile_calls, "workload": one["workload"] + " (1 layer)"}))


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(cfg, seconds, seed=0, loops=4):
    """Time the CPU oracle on verify calls of layer 0 (loops 0..loops-1 and the deepest),
    repeating until `seconds` of oracle time; returns (GB/s, calls, seconds, threads)."""
    import numpy as np
    from oracle import ripe_oracle as orc
    from self_speculative_decode_b200.synth import PlaneSource

    N, kvH, d, R, T, B, W = (cfg[k] for k in ("N", "kvH", "d", "R", "T", "B", "W"))
    g = cfg["Hq"] // kvH
    src = PlaneSource(N, kvH, d, R, T + B, cfg["rho"], seed)
    oc = orc.OracleCache(N, 1, kvH, d, R, W, T + B, value_planes=set(range(loops)) | {R - 1})
    for pl in range(R):
        keep = pl < loops or pl == R - 1
        k = src.plane(pl, "K") if keep else None
        v = src.plane(pl, "V") if keep else None
        oc.load_prefix(0, pl, [T] * N, k, v)
    for pl in range(R):
        keep = pl < loops or pl == R - 1
        if keep:
            kp, vp = src.plane(pl, "K"), src.plane(pl, "V")
            kb = np.ascontiguousarray(kp[:, :, T:T + B].transpose(0, 2, 1, 3))
            vb = np.ascontiguousarray(vp[:, :, T:T + B].transpose(0, 2, 1, 3))
            oc.append(0, pl, kb, vb)
        else:
            oc.append(0, pl, None, None, B=B)
    inputs = [(r, oc.verify_inputs(0, r)[:4], src.queries(r, B, cfg["Hq"])) for r in list(range(loops)) + [R - 1]]
    spent, calls, nbytes = 0.0, 0, 0
    while spent < seconds:
        r, (Kr, Vr, Kl, Vl), q = inputs[calls % len(inputs)]
        qf = orc.bf16_to_f64(q)
        t0 = time.perf_counter()
        orc.verify(oc.T, B, r, R, W, g, Kr, Vr, Kl, Vl, qf)
        spent += time.perf_counter() - t0
        calls += 1
        nbytes += verify_bytes(cfg, [T] * N, r)
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return nbytes / spent / 1e9, calls, spent, threads


def run_reference(args, cfg, rank):
    """The oracle as the reference arm: each step is one bounded sample of the workload."""
    if rank != 0:
        return
    per_step = []
    calls_total = 0
    for i in range(args.warmup + args.steps):
        gbs, calls, sec, threads = oracle_sample(cfg, 0.5, seed=i)
        if i >= args.warmup:
            per_step.append((gbs, sec, calls))
            calls_total += calls
    value = sum(g * s for g, s, _ in per_step) / sum(s for _, s, _ in per_step)
    ms = sum(s for _, s, _ in per_step) / len(per_step) * 1e3
    sample = (f"{calls_total} oracle verify calls of layer 0 (loops 0-3 and {cfg['R'] - 1}), "
              f"about 0.5 s of oracle time per step")
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
    ap.add_argument("--config", default="huginn", choices=sorted(CONFIGS))
    ap.add_argument("--layouts", default=None,
                    help="comma list of ripe, full, deepest (default: all three; long_gqa: ripe,deepest)")
    ap.add_argument("--profile-calls", type=int, default=0,
                    help="only run this many verify calls of layer 0 (for ncu captures) and exit")
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

    if args.profile_calls:
        profile_calls(cfg, args, device)
        return
    if args.fixed_memory_gb:
        fixed_memory(cfg, args, device)
        return
    if args.layouts is None:
        # the full cache of the long-context config needs R * T * 4 layers (137 GB): not by default
        args.layouts = "ripe,deepest" if args.config == "long_gqa" else "ripe,full,deepest"
    layouts = [x for x in args.layouts.split(",") if x]
    results = {}
    clocks = ClockSampler(gpu_id(local))
    clocks.start()
    time.sleep(0.3)  # nvidia-smi needs a moment before its first sample
    for lay in layouts:
        results[lay] = bench_layout(cfg, lay, args, args.seed + 1000 * rank, device, dist_on,
                                    want_extras=(lay == layouts[0]))
    clock_rec = clocks.stop()
    main_l = layouts[0]
    m = results[main_l]
    peak, peak_kind = hbm_peak()
    warm = m["verify_warm"]
    cold = m["verify_cold"]
    achieved = warm["bytes_per_launch"] / (warm["us_per_launch"] * 1e-6) / 1e9
    achieved_cold = cold["bytes_per_launch"] / (cold["us_per_launch"] * 1e-6) / 1e9
    value = job_throughput(m["bytes_per_step"] * args.steps, m["ms_per_step"] * args.steps, world)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg["workload"], "layout": main_l,
                   "step": ("R*L x (append plane r + verify at loop r" +
                            (", one launch" if args.append == "fused" else ", two launches") +
                            ") + commit/evict, CUDA graph"),
                   "T_range": m["T_range"], "l2": "inputs larger than L2 (every step reads the whole cache)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "pct_of_hbm_peak": 100.0 * m["gbs"] / peak,
        "verified_tokens_per_s": m["verified_tokens_per_s"] * world,
        "accepted_tokens_per_s": m["accepted_tokens_per_s"] * world,
        "layouts": {k: {x: v[x] for x in ("ms_per_step", "gbs", "verified_tokens_per_s", "bytes_per_step")}
                    for k, v in results.items()},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": captured_traffic(args.config), "peak_kind": peak_kind,
                     "kernel": "ripe_verify_kernel", "launch_us": warm["us_per_launch"],
                     "note": "R*L verify launches back to back as in the step (L2 warm)"},
        "roofline_cold": {"achieved": achieved_cold, "frac": achieved_cold / peak,
                          "launch_us": cold["us_per_launch"], "note": "L2 flushed before each launch"},
        "e2e": m["e2e"],
        "gpu_launches": m["launches_per_step"] * args.steps,
        "clocks": clock_rec,
    }
    if "full" in results and main_l == "ripe":
        line["full_over_ripe_latency"] = results["full"]["ms_per_step"] / m["ms_per_step"]
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
                                        f"shape), then the step verifies the block at all R loops")
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        gbs, calls, sec, threads = oracle_sample(cfg, args.cpu_seconds)
        line["cpu_baseline"] = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": f"{calls} oracle verify calls of layer 0 (loops 0-3 and "
                                          f"{cfg['R'] - 1}), {sec:.1f} s of oracle time"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
