#!/usr/bin/env python
"""Benchmark of the WKV operator (libwkv.so) on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
wkv_forward over the workload's [B, T, C] sequence (chunked scan or
sequential kernel, as dispatched), then one batched wkv_step decode token for
the B streams from the returned state. Metric: WKV channel-steps per second
(B*T*C + B*C per step), and the forward kernel's achieved HBM bandwidth against
the measured B200 copy bandwidth.

The headline workload is `long` (B=1, T=65536, C=2048 fp32, 1.6 GB per
forward), the largest single-GPU configuration. At N=1 the same JSON line also
carries one sub-record per other workload ("workloads": layer 8x1024x768 fp32,
mixed 16x4096x4096 bf16, the 256-step batched decode of 4096 streams x 768,
small 1x64x768, the backward pass on layer and long, and the RWKV-v6
matrix-state forward 8x1024x12x64 in fp32 and bf16), each with its own
throughput, roofline fraction, clocks and CPU-oracle baseline.

    python bench.py [--gpus N --steps K --warmup W] [--workload long]
    python -m torch.distributed.run --nproc-per-node N bench.py --gpus N ...
    python bench.py --impl reference ...     # the float64 CPU oracle, timed

Each rank processes its own batch (seed = rank): the work per GPU is fixed as N
grows (weak scaling) and no collective touches the data path; ranks only meet
at the barriers around the timed region and for the max-over-ranks timing.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import ctypes
import glob
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "WKV channel-steps/sec (B*T*C per s) and achieved HBM GB/s vs B200 peak"
UNIT = "channel-steps/s"
FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------------------
# distributed plumbing (also exercised on CPU with gloo by the tests)
# ---------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def dist_init(backend: str, timeout_s: float = 120.0):
    import datetime

    import torch.distributed as dist
    if not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def max_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def throughput(units_per_step: int, steps: int, local_ms: float, device=None):
    """Whole-job throughput: units of all ranks over the slowest rank's time.

    Every rank processes its own batch (weak scaling), so the job's units are
    units_per_step * steps * world_size, and the job takes as long as its
    slowest rank. Returns (value per second, max milliseconds over ranks)."""
    import torch.distributed as dist
    world = dist.get_world_size() if (dist.is_available() and dist.is_initialized()) else 1
    ms = max_over_ranks(local_ms, device)
    return units_per_step * steps * world / (ms / 1e3), ms


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and str(device).startswith("cuda"):
            dist.barrier(device_ids=[int(str(device).split(":")[1])])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# workload bookkeeping
# ---------------------------------------------------------------------------

def workload_desc(wl):
    return (f"wkv_forward {wl.kv_dtype} B={wl.B} T={wl.T} C={wl.C}"
            f"{' (state in)' if wl.state != 'zero' else ''} + 1 wkv_step decode token")


def decode_desc(wl):
    return (f"batched decode: wkv_step over {wl.B} streams x C={wl.C} fp32, state from a {wl.T}-token "
            f"prefix (wkv_forward), {wl.decode_steps} steps with fresh k, v")


def workload(args, name=None, override=False):
    """The named workload (the headline's when name is None), with B and/or T
    overridden for profiling runs (the headline, or with override)."""
    import dataclasses

    from wkv_recurrence_b200 import inputs as I
    wl = I.WORKLOADS[name or args.workload]
    if (name is None or override) and (args.batch or args.tokens):
        wl = dataclasses.replace(wl, B=args.batch or wl.B, T=args.tokens or wl.T)
    return wl


def units_per_step(wl) -> int:
    return wl.B * wl.T * wl.C + wl.B * wl.C


def forward_bytes(wl) -> int:
    """Algorithmic HBM bytes of one wkv_forward launch: k, v read once, out
    written once, w and u read once, the state read (if any) and written once."""
    kv_es = 2 if wl.kv_dtype == "bf16" else 4
    out_es = 2 if wl.out_dtype == "bf16" else 4
    n = wl.B * wl.T * wl.C
    state = 12 * wl.B * wl.C
    return n * (2 * kv_es + out_es) + state * (2 if wl.state != "zero" else 1) + 8 * wl.C


def step_bytes(wl) -> int:
    """One wkv_step over B x C: k, v, out and the 3-word state read and written (fp32)."""
    return 36 * wl.B * wl.C + 8 * wl.C


KERNEL_NAMES = {1: "wkv_fwd_seq", 2: "wkv_fwd_chunk", 3: "wkv_tile_totals+scan+replay", 4: "wkv_fwd_pipe",
                5: "wkv_fwd_cluster"}


def forward_kernel_name(wl, options) -> str:
    """The kernel that wkv_forward launches for this workload, as the library
    itself reports it."""
    import torch
    import wkv_recurrence_b200 as W
    kv = torch.bfloat16 if wl.kv_dtype == "bf16" else torch.float32
    return KERNEL_NAMES[W.forward_kernel(wl.B, wl.T, wl.C, kv, options)]


def launches_per_step(wl, options) -> int:
    """Kernel launches of one step: the forward's (as the library reports them
    for this shape and options) and one decode launch."""
    import torch
    import wkv_recurrence_b200 as W
    kv = torch.bfloat16 if wl.kv_dtype == "bf16" else torch.float32
    return W.forward_launches(wl.B, wl.T, wl.C, kv, options) + 1


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_digest() -> str:
    """Hash of the kernels and of the code that chooses and launches them (tile
    shapes, stages and grids change the traffic a capture records)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "wkv_recurrence_b200", "csrc")
    for p in sorted(glob.glob(os.path.join(csrc, "*.cuh")) + glob.glob(os.path.join(csrc, "*.cu"))):
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """(DRAM bytes per launch, XU pipe use in % of its peak or None) recorded
    by an ncu capture under profiles/, if it was taken on the current kernel
    sources (else (None, None)). The XU pipe (ex2, rcp) is the path's second
    ceiling after HBM."""
    digest = source_digest()
    for p in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        with open(p) as f:
            for line in f:
                m = re.match(r"traffic:\s*kernel=(\S+)\s+workload=(\S+)\s+source=(\S+)\s+bytes_per_launch=(\d+)"
                             r"(?:\s+xu_pct=([0-9.]+))?", line.strip())
                if m and m.group(1) == kernel and m.group(2) == workload and m.group(3) == digest:
                    return int(m.group(4)), (float(m.group(5)) if m.group(5) else None)
    return None, None


class L2Flusher:
    """Evicts everything a step touched from L2, outside the timed region.

    Writing a buffer of twice the L2 size evicts the step's inputs and outputs,
    but leaves L2 full of dirty lines, which the next timed step would then pay
    for by writing them back to HBM while it reads its own inputs (about its
    own input size again in extra DRAM traffic). Reading a second 2x-L2
    buffer right after turns those into clean lines, so the timed step moves
    only its own bytes.
    """
    DESCRIPTION = ("flushed between timed steps: a 2x-L2 buffer is written, then another 2x-L2 buffer "
                   "is read, so no data of the step stays in L2 and no dirty lines are left to write back")

    def __init__(self, l2_bytes: int, device):
        import torch
        n = max(2 * l2_bytes, 256 << 20) // 4
        self.wbuf = torch.empty(n, dtype=torch.float32, device=device)
        self.rbuf = torch.ones(n, dtype=torch.float32, device=device)
        self.sink = torch.empty(1, dtype=torch.float32, device=device)

    def __call__(self):
        self.wbuf.zero_()
        self.sink.copy_(self.rbuf.sum().view(1))


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.reader = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.reader.join(timeout=5)
        rows = []
        for line in list(self.lines):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, val in zip(names, r[5:9]) if val.lower() == "active"})
        busy = [x for x in sm if smax and x >= 0.5 * max(smax)] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def _to_dev(x, device, as_bf16=False):
    import numpy as np
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x.view(np.int16) if as_bf16 else x)).to(device)
    return t.view(torch.bfloat16) if as_bf16 else t


def _timed_graph(g, n_rep, stream, device):
    """Milliseconds of n_rep back-to-back replays of graph g, by CUDA events on
    `stream`, bracketed by a barrier and a synchronize on both sides."""
    import torch
    barrier(device)
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n_rep):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    return e0.elapsed_time(e1)


def _capture(items, body, stream, device):
    """A CUDA graph of body(item, stream handle) for every item, captured on a
    side stream."""
    import torch
    side = torch.cuda.Stream(device)
    side.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        h = ctypes.c_void_p(side.cuda_stream)
        with torch.cuda.graph(g, stream=side):
            for it in items:
                body(it, h)
    stream.wait_stream(side)
    torch.cuda.synchronize(device)
    return g


def measure_forward(wl, args, options, device, rank, world, headline):
    """Throughput of the step (forward + one decode token) on workload wl, the
    forward's roofline, and (headline only) the end-to-end number through the
    public API. Returns the record (a dict) on every rank."""
    import numpy as np
    import torch

    import wkv_recurrence_b200 as W
    from wkv_recurrence_b200 import inputs as I

    k, v = I.draw_kv(wl, seed=rank)
    w, u = I.draw_w(wl, seed=0), I.draw_u(wl, seed=0)
    st = I.draw_state(wl, seed=rank)
    k1, v1 = I.draw_decode_token(wl, 0, seed=rank)
    bf16 = wl.kv_dtype == "bf16"
    out_dtype = torch.bfloat16 if wl.out_dtype == "bf16" else torch.float32
    Wt, U = _to_dev(w, device), _to_dev(u, device)
    S_in = None if st is None else tuple(_to_dev(s, device) for s in st)
    # R independent buffer sets (inputs, outputs, states), used in turn, so
    # that a step never finds its inputs in L2: R sets together exceed 2.5x L2
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    set_bytes = forward_bytes(wl) + step_bytes(wl)
    R = int(min(8, max(2, -(-int(2.5 * l2) // set_bytes))))
    sets = []
    for _ in range(R):
        d = dict(K=_to_dev(k, device, bf16), V=_to_dev(v, device, bf16), K1=_to_dev(k1, device),
                 V1=_to_dev(v1, device), out=torch.empty(wl.B, wl.T, wl.C, dtype=out_dtype, device=device),
                 state=tuple(torch.empty(wl.B, wl.C, device=device) for _ in range(3)),
                 out1=torch.empty(wl.B, wl.C, device=device))
        sets.append(d)
    ws = W.make_workspace(wl.B, wl.T, wl.C, options=options, device=device)
    stream = torch.cuda.current_stream(device)
    # arguments checked and marshalled once; each call below is one C-ABI call
    for d in sets:
        d["fwd"] = W.PreparedForward(d["K"], d["V"], Wt, U, S_in, out=d["out"], state_out=d["state"],
                                     workspace=ws, options=options)
        d["dec"] = W.PreparedStep(d["state"], d["K1"], d["V1"], Wt, U, out=d["out1"])

    def one_step(d=sets[0], strm=None):
        d["fwd"](strm)
        d["dec"](strm)

    warm = max(3, args.warmup)
    for i in range(warm):
        one_step(sets[i % R])
    torch.cuda.synchronize(device)
    if W.query_status(ws) != 0:
        raise RuntimeError("device-side wait timed out during warm-up")
    g_step = _capture(sets, lambda d, h: one_step(d, h), stream, device)
    g_fwd = _capture(sets, lambda d, h: d["fwd"](h), stream, device)
    for g in (g_step, g_fwd):
        g.replay()
    torch.cuda.synchronize(device)
    n_rep = max(1, -(-args.steps // R))
    K_steps = n_rep * R

    sampler = ClockSampler(torch.cuda.current_device()) if not args.no_clocks else None
    if sampler:
        sampler.start()
    t_wall0 = time.perf_counter()
    total_ms = _timed_graph(g_step, n_rep, stream, device)
    t_wall = time.perf_counter() - t_wall0
    fwd_total_ms = _timed_graph(g_fwd, n_rep, stream, device)
    clocks = sampler.stop() if sampler else None
    if W.query_status(ws) != 0:
        raise RuntimeError("device-side wait timed out during the timed steps")
    value, total_ms_max = throughput(units_per_step(wl), K_steps, total_ms, device)

    # roofline of the dominant kernel (the forward launch), back to back
    peak, peak_kind = measured_peaks()
    fwd_mean_ms = max_over_ranks(fwd_total_ms / K_steps, device)
    algo = forward_bytes(wl)
    achieved = algo / (fwd_mean_ms / 1e3) / 1e9
    kernel_name = forward_kernel_name(wl, options)
    traffic, xu_pct = recorded_traffic(kernel_name, wl.name)

    # the same forward timed alone after an L2 flush (launch latency included)
    flusher = L2Flusher(l2, device)
    cold = []
    for i in range(10):
        flusher()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        sets[i % R]["fwd"]()
        e1.record(stream)
        cold.append((e0, e1))
    torch.cuda.synchronize(device)
    cold_ms = statistics.median(a.elapsed_time(b) for a, b in cold)
    del flusher

    # end to end through the public API: pinned host -> device, compute, device -> host
    e2e = None
    if headline and not args.no_e2e:
        K, V, K1, V1, out, out1, state = (sets[0][x] for x in ("K", "V", "K1", "V1", "out", "out1", "state"))
        pin = lambda x: torch.from_numpy(np.ascontiguousarray(x)).pin_memory()  # noqa: E731
        hk = pin(k.view(np.int16) if bf16 else k)
        hv = pin(v.view(np.int16) if bf16 else v)
        hk1, hv1 = pin(k1), pin(v1)
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        hout1 = torch.empty(out1.shape).pin_memory()
        hst = tuple(torch.empty(wl.B, wl.C).pin_memory() for _ in range(3))
        n_e2e = max(3, min(K_steps, args.e2e_steps))

        # the forward through the host-resident entry point: the library streams
        # segments of k, v in and of out back while it computes
        hk_t = hk.view(torch.bfloat16) if bf16 else hk
        hv_t = hv.view(torch.bfloat16) if bf16 else hv
        host_buf = torch.zeros(W.forward_host_buffer_size(wl.B, wl.T, wl.C, hk_t.dtype, out_dtype),
                               dtype=torch.uint8, device=device)

        def e2e_step():
            W.forward_host(hk_t, hv_t, Wt, U, S_in, out=hout, state_out=state, buffer=host_buf)
            K1.copy_(hk1, non_blocking=True)
            V1.copy_(hv1, non_blocking=True)
            sets[0]["dec"]()
            hout1.copy_(out1, non_blocking=True)
            for hh, s in zip(hst, state):
                hh.copy_(s, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(device)
        barrier(device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(device)
        barrier(device)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), device)
        h2d = k.nbytes + v.nbytes + k1.nbytes + v1.nbytes
        d2h = hout.numel() * hout.element_size() + hout1.numel() * 4 + 3 * wl.B * wl.C * 4
        e2e = {"value": units_per_step(wl) * n_e2e * world / (e2e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": n_e2e,
               "ms_per_step": e2e_ms / n_e2e}

    rec = {
        "workload": workload_desc(wl), "name": wl.name, "B": wl.B, "T": wl.T, "C": wl.C,
        "kv_dtype": wl.kv_dtype, "out_dtype": wl.out_dtype,
        "value": value, "unit": UNIT, "steps": K_steps, "warmup": warm, "ms_per_step": total_ms_max / K_steps,
        "forward_value": wl.B * wl.T * wl.C / (fwd_mean_ms / 1e3) * world,
        "roofline": {"bound": "hbm", "kernel": kernel_name, "achieved": achieved, "peak": peak,
                     "peak_source": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "xu_pipe_pct_of_peak": xu_pct, "algorithmic_bytes": algo,
                     "launch_ms": fwd_mean_ms},
        "forward_ms": {"back_to_back": fwd_total_ms / K_steps, "cold_after_l2_flush": cold_ms},
        "gpu_launches": launches_per_step(wl, options) * K_steps,
        "clocks": clocks, "wall_s_timed_region": t_wall, "buffer_sets": R,
        "l2": (f"inputs larger than L2: steps rotate over {R} separate buffer sets "
               f"({R * set_bytes / 2**20:.0f} MiB in total, L2 is {l2 / 2**20:.0f} MiB), so every step reads "
               "inputs that are not in L2; steps run back to back from a CUDA graph"),
        "e2e": e2e,
    }
    del sets, ws, g_step, g_fwd
    torch.cuda.empty_cache()
    return rec


def measure_decode(wl, args, device):
    """The batched decode workload: the per-step time of wkv_step over
    S streams x C channels, with the state of every stream built by a T-token
    prefix through wkv_forward. Steps rotate over 4 independent sets of stream
    states, and the k, v of each step are one of the workload's drawn decode
    steps, so that neither a step's state nor its tokens are still in L2 from
    an earlier launch. N=1 only."""
    import torch

    import wkv_recurrence_b200 as W
    from wkv_recurrence_b200 import inputs as I

    S, C = wl.B, wl.C
    w, u = I.draw_w(wl), I.draw_u(wl)
    Wt, U = _to_dev(w, device), _to_dev(u, device)
    # the prefix, in slices of streams to bound host memory
    base = tuple(torch.empty(S, C, device=device) for _ in range(3))
    slab = 512
    for s0 in range(0, S, slab):
        kp, vp = I.draw_kv_rows(wl, range(s0, min(S, s0 + slab)))
        W.forward(_to_dev(kp, device), _to_dev(vp, device), Wt, U,
                  state_out=tuple(x[s0:s0 + slab] for x in base))
        torch.cuda.synchronize(device)
        del kp, vp
    n_tok = wl.decode_steps
    toks = []
    for j in range(n_tok):
        kd, vd = I.draw_decode_token(wl, j)
        toks.append((_to_dev(kd, device), _to_dev(vd, device)))
    R = 4
    sets = [tuple(x.clone() for x in base) for _ in range(R)]
    out = [torch.empty(S, C, device=device) for _ in range(R)]
    stream = torch.cuda.current_stream(device)
    # launch n = (step j of set r, n = R*j + r) takes token buffer n mod n_tok:
    # each set takes fresh tokens every step, and a token buffer is read again
    # only n_tok launches later
    calls = []
    for j in range(n_tok):
        for r in range(R):
            kd, vd = toks[(R * j + r) % n_tok]
            calls.append(W.PreparedStep(sets[r], kd, vd, Wt, U, out=out[r]))
    for c in calls[:max(3, args.warmup)]:
        c()
    torch.cuda.synchronize(device)
    g = _capture(calls, lambda c, h: c(h), stream, device)
    g.replay()
    torch.cuda.synchronize(device)
    n_rep = max(1, -(-args.steps // len(calls)))
    sampler = ClockSampler(torch.cuda.current_device()) if not args.no_clocks else None
    if sampler:
        sampler.start()
    ms = _timed_graph(g, n_rep, stream, device)
    clocks = sampler.stop() if sampler else None
    launches = n_rep * len(calls)
    step_ms = ms / launches
    peak, peak_kind = measured_peaks()
    algo = step_bytes(wl)
    achieved = algo / (step_ms / 1e3) / 1e9
    traffic, xu_pct = recorded_traffic("wkv_step_kernel", "decode")
    rec = {
        "workload": decode_desc(wl), "name": "decode", "S": S, "C": C, "prefix_T": wl.T, "steps_per_stream": n_tok,
        "value": S * C / (step_ms / 1e3), "unit": UNIT, "steps": launches, "ms_per_step": step_ms,
        "roofline": {"bound": "hbm", "kernel": "wkv_step_kernel", "achieved": achieved, "peak": peak,
                     "peak_source": peak_kind, "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                     "xu_pipe_pct_of_peak": xu_pct, "algorithmic_bytes": algo, "launch_ms": step_ms},
        "gpu_launches": launches, "clocks": clocks,
        "l2": (f"{R} independent sets of stream states are stepped in turn and the k, v of each launch are one "
               f"of {n_tok} drawn decode steps ({n_tok * 2 * S * C * 4 / 2**30:.1f} GiB), so a launch reads "
               "state and tokens last touched at least 3 launches (340 MB of traffic) earlier; launches run "
               "back to back from a CUDA graph"),
    }
    del g, calls, sets, toks, base
    torch.cuda.empty_cache()
    return rec


def measure_backward(wl, args, device):
    """wkv_backward over workload wl with g ~ N(0, 1): per-call time in a CUDA
    graph, buffer sets rotated so that no call finds its inputs in L2.
    Algorithmic bytes: k, v, g read and dk, dv written once (20 B per
    channel-step in fp32), w, u read and dw, du written, the state in read and
    its gradient written."""
    import torch

    import wkv_recurrence_b200 as W
    from wkv_recurrence_b200 import _abi
    from wkv_recurrence_b200 import inputs as I

    k, v = I.draw_kv(wl)
    w, u = I.draw_w(wl), I.draw_u(wl)
    st = I.draw_state(wl)
    g = I.draw_r_rows(wl, range(wl.B))
    bf16 = wl.kv_dtype == "bf16"
    n = wl.B * wl.T * wl.C
    kv_es = 2 if bf16 else 4
    algo = n * (2 * kv_es + 4 + 8) + 16 * wl.C + (24 * wl.B * wl.C if st is not None else 0)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    R = int(min(6, max(2, -(-int(2.5 * l2) // algo))))
    Wt, U = _to_dev(w, device), _to_dev(u, device)
    S_in = None if st is None else tuple(_to_dev(x, device) for x in st)
    ws_bytes = _abi.lib().wkv_backward_workspace_size(wl.B, wl.T, wl.C)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
    L = _abi.lib()
    P = ctypes.c_void_p
    sets = []
    for _ in range(R):
        d = dict(K=_to_dev(k, device, bf16), V=_to_dev(v, device, bf16), G=_to_dev(g, device),
                 dk=torch.empty(wl.B, wl.T, wl.C, device=device), dv=torch.empty(wl.B, wl.T, wl.C, device=device),
                 dw=torch.empty(wl.C, device=device), du=torch.empty(wl.C, device=device),
                 ds=tuple(torch.empty(wl.B, wl.C, device=device) for _ in range(3)))
        d["sin"] = None if S_in is None else _abi.wkv_cstate(*(x.data_ptr() for x in S_in))
        d["sout"] = _abi.wkv_state(*(x.data_ptr() for x in d["ds"]))
        sets.append(d)

    def call(d, h=None):
        code = L.wkv_backward(wl.B, wl.T, wl.C, P(d["K"].data_ptr()), P(d["V"].data_ptr()),
                              _abi.WKV_BF16 if bf16 else _abi.WKV_F32, P(Wt.data_ptr()), P(U.data_ptr()),
                              ctypes.byref(d["sin"]) if d["sin"] is not None else None, P(d["G"].data_ptr()),
                              P(d["dk"].data_ptr()), P(d["dv"].data_ptr()), P(d["dw"].data_ptr()),
                              P(d["du"].data_ptr()), ctypes.byref(d["sout"]), P(ws.data_ptr()), ws_bytes,
                              h if h is not None else P(torch.cuda.current_stream(device).cuda_stream))
        if code:
            _abi.check(code, "wkv_backward")

    stream = torch.cuda.current_stream(device)
    for i in range(max(3, args.warmup)):
        call(sets[i % R])
    torch.cuda.synchronize(device)
    g_bwd = _capture(sets, call, stream, device)
    g_bwd.replay()
    torch.cuda.synchronize(device)
    n_rep = max(1, -(-max(1, args.steps // 20) // R))
    sampler = ClockSampler(torch.cuda.current_device()) if not args.no_clocks else None
    if sampler:
        sampler.start()
    ms = _timed_graph(g_bwd, n_rep, stream, device)
    clocks = sampler.stop() if sampler else None
    call_ms = ms / (n_rep * R)
    peak, peak_kind = measured_peaks()
    achieved = algo / (call_ms / 1e3) / 1e9
    traffic, xu_pct = recorded_traffic("wkv_backward", wl.name)
    launches = 6 if wl.T > 32 else 4
    rec = {
        "workload": f"wkv_backward {wl.kv_dtype} B={wl.B} T={wl.T} C={wl.C} (gradients of sum(g * wkv), "
                    f"g ~ N(0, 1){', state in' if st is not None else ''})",
        "name": f"backward_{wl.name}", "value": n / (call_ms / 1e3), "unit": UNIT, "steps": n_rep * R,
        "ms_per_step": call_ms,
        "roofline": {"bound": "hbm", "kernel": "wkv_backward (6 launches)", "achieved": achieved, "peak": peak,
                     "peak_source": peak_kind, "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                     "xu_pipe_pct_of_peak": xu_pct, "algorithmic_bytes": algo, "launch_ms": call_ms},
        "gpu_launches": launches * n_rep * R, "clocks": clocks, "buffer_sets": R,
        "l2": f"calls rotate over {R} separate buffer sets ({R * algo / 2**20:.0f} MiB of algorithmic traffic)",
    }
    del g_bwd, sets, ws
    torch.cuda.empty_cache()
    return rec


# fp32 SIMT peak of a B200 for the matrix-state kernel's roofline: 148 SMs x
# 128 fp32 lanes x 2 flops per fused multiply-add x the 1965 MHz maximum clock
V6_FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def measure_v6(wl, args, device):
    """wkv_v6_forward over the v6 workload: per-call time in a CUDA graph over
    rotating buffer sets. Roofline: fp32 instruction issue, 5 D^2 flops per
    (token, head) (update: a product and a fused multiply-add per state entry;
    readout: a fused multiply-add per entry) against the fp32 SIMT peak; HBM
    bytes (r, w, k, v read, y written) reported beside it."""
    import torch

    import wkv_recurrence_b200 as W
    from wkv_recurrence_b200 import inputs as I

    r, w, k, v = I.draw_v6(wl)
    bf16 = wl.kv_dtype == "bf16"
    n = wl.B * wl.T * wl.H * wl.D
    es = 2 if bf16 else 4
    hbm = n * (3 * es + 4 + (2 if wl.out_dtype == "bf16" else 4))
    flops = 5 * wl.B * wl.T * wl.H * wl.D * wl.D
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    R = int(min(6, max(2, -(-int(2.5 * l2) // hbm))))
    out_dtype = torch.bfloat16 if wl.out_dtype == "bf16" else torch.float32
    sets = []
    for _ in range(R):
        sets.append(dict(r=_to_dev(r, device, bf16), w=_to_dev(w, device), k=_to_dev(k, device, bf16),
                         v=_to_dev(v, device, bf16),
                         y=torch.empty(wl.B, wl.T, wl.H, wl.D, dtype=out_dtype, device=device),
                         s=torch.empty(wl.B, wl.H, wl.D, wl.D, device=device)))
    stream = torch.cuda.current_stream(device)
    ws = torch.zeros(256, dtype=torch.uint8, device=device)

    def call(d, h=None):
        # on the current stream: the capture's side stream while capturing
        W.v6_forward(d["r"], d["w"], d["k"], d["v"], None, out=d["y"], state_out=d["s"], workspace=ws)

    for i in range(max(3, args.warmup)):
        call(sets[i % R])
    torch.cuda.synchronize(device)
    g6 = _capture(sets, call, stream, device)
    g6.replay()
    torch.cuda.synchronize(device)
    n_rep = max(1, -(-max(1, args.steps // 20) // R))
    sampler = ClockSampler(torch.cuda.current_device()) if not args.no_clocks else None
    if sampler:
        sampler.start()
    ms = _timed_graph(g6, n_rep, stream, device)
    clocks = sampler.stop() if sampler else None
    call_ms = ms / (n_rep * R)
    tflops = flops / (call_ms / 1e3) / 1e12
    peak, peak_kind = measured_peaks()
    traffic, _ = recorded_traffic("wkv6_fwd", wl.name)
    rec = {
        "workload": f"wkv_v6_forward {wl.kv_dtype} B={wl.B} T={wl.T} H={wl.H} D={wl.D} (matrix-valued state, "
                    "zero state in, state out)",
        "name": wl.name, "value": n / (call_ms / 1e3), "unit": "channel-steps/s (B*T*H*D per s)",
        "steps": n_rep * R, "ms_per_step": call_ms,
        "roofline": {"bound": "alu", "kernel": "wkv6_fwd", "achieved": tflops, "peak": V6_FP32_PEAK_TFLOPS,
                     "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x 1965 MHz", "unit": "TFLOP/s",
                     "frac": tflops / V6_FP32_PEAK_TFLOPS, "traffic": traffic, "algorithmic_flops": flops,
                     "hbm_achieved_gbs": hbm / (call_ms / 1e3) / 1e9, "hbm_frac_of_measured": hbm / (call_ms / 1e3) / 1e9 / peak,
                     "launch_ms": call_ms},
        "gpu_launches": n_rep * R, "clocks": clocks, "buffer_sets": R,
    }
    del g6, sets
    torch.cuda.empty_cache()
    return rec


def run_ours(args):
    import torch

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        dist_init("nccl")
    options = json.loads(args.options) if args.options else None
    if args.part:
        # one sub-record alone (profiling): printed as its own JSON line
        from wkv_recurrence_b200 import inputs as I
        if args.part.startswith("backward_"):
            rec = measure_backward(workload(args, args.part[len("backward_"):], override=True), args, device)
        else:
            rec = measure_v6(I.V6_WORKLOADS[args.part], args, device)
        if rank == 0:
            print(json.dumps(rec), flush=True)
        return
    wl = workload(args)
    main = measure_forward(wl, args, options, device, rank, world, headline=True)

    subs = {}
    if world == 1 and not args.no_sub:
        for name in ("layer", "mixed", "decode", "small"):
            if name == wl.name:
                continue
            swl = workload(args, name)
            if name == "decode":
                subs[name] = measure_decode(swl, args, device)
            else:
                subs[name] = measure_forward(swl, args, None, device, rank, world, headline=False)
        from wkv_recurrence_b200 import inputs as I
        for name in ("layer", "long"):
            subs[f"backward_{name}"] = measure_backward(workload(args, name), args, device)
        subs["v6"] = measure_v6(I.V6_WORKLOADS["v6"], args, device)
        subs["v6_bf16"] = measure_v6(I.V6_WORKLOADS["v6_bf16"], args, device)

    if rank == 0 and world == 1 and not args.no_cpu:
        main["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_seconds, one_core_s=args.cpu_seconds / 2)
        for name, rec in subs.items():
            if name.startswith("backward_") or name.startswith("v6"):
                continue
            rec["cpu_baseline"] = cpu_baseline(workload(args, name), budget_s=args.cpu_seconds / 3,
                                               one_core_s=args.cpu_seconds / 4, decode=(name == "decode"))
        for name in ("layer", "long"):
            subs[f"backward_{name}"]["cpu_baseline"] = cpu_baseline_backward(workload(args, name),
                                                                             budget_s=args.cpu_seconds / 3)
        from wkv_recurrence_b200 import inputs as I
        for name in ("v6", "v6_bf16"):
            subs[name]["cpu_baseline"] = cpu_baseline_v6(I.V6_WORKLOADS[name], budget_s=args.cpu_seconds / 4)

    if rank == 0:
        bf16 = wl.kv_dtype == "bf16"
        line = {
            "metric": METRIC, "value": main["value"], "unit": UNIT, "n_gpus": world, "steps": main["steps"],
            "warmup": main["warmup"], "ms_per_step": main["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32" if not bf16 else "bf16-io/f32",
            "data": "synthetic (seeded numpy draws of the workload's distributions)",
            "config": {"workload": main["workload"], "name": wl.name, "B": wl.B, "T": wl.T, "C": wl.C,
                       "kv_dtype": wl.kv_dtype, "out_dtype": wl.out_dtype, "global_batch": wl.B * world,
                       "seq_len": wl.T, "parallelism": f"dp{world}" if world > 1 else "single",
                       "l2": main["l2"], "options": options or "auto"},
            "roofline": main["roofline"], "forward_ms": main["forward_ms"],
            "forward_value": main["forward_value"],
            "cpu_baseline": main.get("cpu_baseline"), "e2e": main["e2e"], "gpu_launches": main["gpu_launches"],
            "clocks": main["clocks"], "wall_s_timed_region": main["wall_s_timed_region"],
            "buffer_sets": main["buffer_sets"],
            "workloads": subs,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# the CPU oracle, timed (cpu_baseline leg, and the reference arm)
# ---------------------------------------------------------------------------

def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _oracle_sample(wl, rows, cols, seed=0):
    from wkv_recurrence_b200 import inputs as I
    k, v = I.draw_kv_rows(wl, range(rows), seed=seed)
    k, v = k[:, :, :cols].copy(), v[:, :, :cols].copy()
    w, u = I.draw_w(wl)[:cols].copy(), I.draw_u(wl)[:cols].copy()
    st = I.draw_state(wl, rows=range(rows), seed=seed)
    if st is not None:
        st = tuple(s[:, :cols].copy() for s in st)
    k1, v1 = I.draw_decode_token(wl, 0, rows=range(rows), seed=seed)
    return k, v, w, u, st, k1[:, :cols].copy(), v1[:, :cols].copy()


def _oracle_step(O, sample, threads):
    k, v, w, u, st, k1, v1 = sample
    _, s = O.recurrence_forward(k, v, w, u, st, threads=threads)
    O.recurrence_step(s, k1, v1, w, u)


def _pick_sample(wl, max_units):
    """Largest (rows, channels) slice of the workload with at most max_units channel-steps."""
    rows = wl.B
    cols = wl.C
    per = wl.T + 1
    while rows * cols * per > max_units and rows > 1:
        rows = max(1, rows // 2)
    while rows * cols * per > max_units and cols > 16:
        cols = max(16, cols // 2)
    return rows, cols


def _set_oracle_threads(O, n):
    """The oracle's OpenMP thread count for the calls that follow (a tiny
    forward with an explicit count sets it for the process)."""
    import numpy as np
    z = np.zeros((1, 1, 1), np.float32)
    O.recurrence_forward(z, z, np.zeros(1, np.float32), np.zeros(1, np.float32), threads=n)


def _rate(O, wl, budget_s, threads, decode):
    """Channel-steps per second of the oracle on a slice of wl sized to about
    budget_s of CPU work with `threads` threads; and the slice's description."""
    from wkv_recurrence_b200 import inputs as I
    _set_oracle_threads(O, threads)
    if decode:
        # one decode step of every stream in a slice, from a state drawn by a short prefix
        rows = min(wl.B, 64)
        sample = _oracle_sample(wl, rows, wl.C)
        _, st = O.recurrence_forward(sample[0][:, :16], sample[1][:, :16], sample[2], sample[3])
        kd, vd = I.draw_decode_token(wl, 0, rows=range(rows))
        reps = 0
        t0 = time.perf_counter()
        while True:
            _, st = O.recurrence_step(st, kd, vd, sample[2], sample[3])
            reps += 1
            if time.perf_counter() - t0 >= budget_s:
                break
        dt = time.perf_counter() - t0
        return rows * wl.C * reps / dt, (f"float64 C recurrence step on streams 0..{rows - 1} (all {wl.C} "
                                         f"channels), {reps} decode steps, {dt:.1f} s")
    rows, cols = _pick_sample(wl, 2_000_000)
    sample = _oracle_sample(wl, rows, cols)
    t0 = time.perf_counter()
    _oracle_step(O, sample, threads)
    rate = rows * cols * (wl.T + 1) / max(time.perf_counter() - t0, 1e-6)
    rows, cols = _pick_sample(wl, max(2_000, int(rate * budget_s / 3)))
    sample = _oracle_sample(wl, rows, cols)
    reps = 0
    t0 = time.perf_counter()
    while True:
        _oracle_step(O, sample, threads)
        reps += 1
        if time.perf_counter() - t0 >= budget_s or reps >= 50:
            break
    dt = time.perf_counter() - t0
    return (rows * cols * (wl.T + 1) * reps / dt,
            f"float64 C recurrence on rows 0..{rows - 1}, channels 0..{cols - 1} of the {wl.name} workload "
            f"(T={wl.T}, plus one decode token), {reps} repetition(s), {dt:.1f} s")


def cpu_baseline(wl, budget_s=10.0, one_core_s=5.0, decode=False):
    """The float64 oracle timed on this host's cores (OpenMP over channels),
    and on one core, on a bounded slice of the workload."""
    from oracle import oracle as O
    O.build()
    _set_oracle_threads(O, 0)
    cores = os.cpu_count() or 1
    value, sample = _rate(O, wl, budget_s, cores, decode)
    one, one_sample = _rate(O, wl, one_core_s, 1, decode)
    _set_oracle_threads(O, cores)
    return {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
            "value_1core": one, "sample_1core": one_sample, "cpu_model": cpu_model()}


def cpu_baseline_backward(wl, budget_s=3.0):
    """The float64 oracle backward on a slice of the workload, all host cores."""
    import numpy as np

    from oracle import oracle as O
    from wkv_recurrence_b200 import inputs as I
    O.build()
    cores = os.cpu_count() or 1
    _set_oracle_threads(O, cores)
    rows = 1
    cols = min(wl.C, 256)
    T = min(wl.T, 4096)
    k, v = I.draw_kv_rows(wl, range(rows), T=T)
    k, v = k[:, :, :cols].copy(), v[:, :, :cols].copy()
    w, u = I.draw_w(wl)[:cols].copy(), I.draw_u(wl)[:cols].copy()
    g = np.random.default_rng(0).normal(size=k.shape)
    reps = 0
    t0 = time.perf_counter()
    while True:
        O.recurrence_backward(k, v, w, u, g, threads=cores)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": rows * T * cols * reps / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"float64 C backward recurrence on row 0, channels 0..{cols - 1}, tokens 0..{T - 1} of the "
                      f"{wl.name} workload, {reps} repetition(s), {dt:.1f} s", "cpu_model": cpu_model()}


def cpu_baseline_v6(wl, budget_s=3.0):
    """The float64 numpy oracle of the matrix-valued state on a slice of the workload."""
    from oracle import v6_oracle as V
    from wkv_recurrence_b200 import inputs as I
    T = 64
    r, w, k, v = I.draw_v6(wl, T=T)
    reps = 0
    t0 = time.perf_counter()
    while True:
        V.recurrence(r, w, k, v, kv_dtype=wl.kv_dtype)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": wl.B * T * wl.H * wl.D * reps / dt, "unit": "channel-steps/s (B*T*H*D per s)",
            "cores": 1, "kind": "oracle",
            "sample": f"float64 numpy recurrence on tokens 0..{T - 1} of every head of the {wl.name} workload, "
                      f"{reps} repetition(s), {dt:.1f} s", "cpu_model": cpu_model()}


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return
    from oracle import oracle as O
    O.build()
    wl = workload(args)
    steps, warm = args.steps, max(3, args.warmup)
    budget = float(args.reference_seconds)
    cores = os.cpu_count() or 1
    # size each step so that warm-up + timed steps take about `budget` seconds
    rows, cols = _pick_sample(wl, 200_000)
    sample = _oracle_sample(wl, rows, cols)
    t0 = time.perf_counter()
    _oracle_step(O, sample, cores)
    rate = rows * cols * (wl.T + 1) / max(time.perf_counter() - t0, 1e-6)
    per_step = max(2_000, int(rate * budget / (steps + warm)))
    rows, cols = _pick_sample(wl, per_step)
    sample = _oracle_sample(wl, rows, cols)
    for _ in range(warm):
        _oracle_step(O, sample, cores)
    t0 = time.perf_counter()
    for _ in range(steps):
        _oracle_step(O, sample, cores)
    dt = time.perf_counter() - t0
    units = rows * cols * (wl.T + 1) * steps
    value = units / dt
    desc = (f"float64 C recurrence (OpenMP) per step on rows 0..{rows - 1}, channels 0..{cols - 1} of the "
            f"{wl.name} workload (T={wl.T}) plus one decode token")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": warm, "ms_per_step": dt / steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(wl), "name": wl.name, "B": wl.B, "T": wl.T, "C": wl.C},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": desc, "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long", help="tiny|small|layer|decode|long|mixed (the headline)")
    ap.add_argument("--options", default="", help='JSON wkv_options, e.g. {"kernel": 2, "chunk_len": 64}')
    ap.add_argument("--batch", type=int, default=0, help="override B of the workload (profiling)")
    ap.add_argument("--tokens", type=int, default=0, help="override T of the workload (profiling)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--reference-seconds", type=float, default=60.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-sub", action="store_true", help="headline workload only (no per-workload sub-records)")
    ap.add_argument("--part", choices=["backward_layer", "backward_long", "v6", "v6_bf16"], default="",
                    help="measure this sub-record alone and print it (profiling)")
    ap.add_argument("--no-clocks", action="store_true")
    args = ap.parse_args(argv)
    _, _, world = dist_env()
    if world != args.gpus and args.impl == "ours" and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
