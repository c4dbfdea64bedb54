#!/usr/bin/env python
"""Benchmark of the W8A8 quantized Linear on B200.

One step = the int W8A8 DiT MLP block, forward and input gradient, at
M = 4608 tokens (4096 image + 512 text), hidden 3072, MLP 12288:
    Y1  = Lin(X,   W1)    3072 -> 12288        quantize_rows + int8 GEMM
    Y2  = Lin(Y1,  W2)    12288 -> 3072        quantize_rows + int8 GEMM
    dX2 = Q(dY2) Q(W2)    dgrad                quantize_rows + int8 GEMM (MN-major W)
    dX1 = Q(dX2) Q(W1)    dgrad                quantize_rows + int8 GEMM (MN-major W)
with the weights quantized tensor-wise once, outside the timed region.
Metric: TOPS = 4 * 2*M*N*K / step time (quant + GEMM + epilogue).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs the same per-GPU workload on its own seeded
tokens (weak scaling, no data-path collective); the step time is the max over
ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W8A8 linear TOPS (quant+GEMM+epilogue) at DiT shapes; % of int8/fp8 TC peak"
UNIT = "TOPS"
M_TOK, HID, MLP = 4608, 3072, 12288
OPS_PER_GEMM = 2 * M_TOK * HID * MLP
OPS_PER_STEP = 4 * OPS_PER_GEMM
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic of one launch of the dominant kernel from an ncu capture, keyed
# by the hash of the kernel source it was taken on (null when they differ).
GEMM_TRAFFIC = {"source_sha": "bc0ebb1129955a71", "bytes_per_launch": 122957312,
                "note": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one up-proj launch "
                        "(bench.py --case up): 52.08 MB read + 70.88 MB written"}


def gemm_source_sha() -> str:
    h = hashlib.sha256()
    for f in ("gemm_pair.cuh", "gemm.cuh", "device.cuh"):
        with open(os.path.join(ROOT, "w8a8_quantized_linear_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region, filtered
    to one GPU by UUID (or by index when the UUID is unknown)."""
    QUERY = ("uuid,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, uuid: str, index: str):
        self.uuid = (uuid or "").lower().replace("gpu-", "")
        self.index = index
        self.proc = None
        self.out = ""

    def __enter__(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="w8a8_clocks_", suffix=".csv")
        os.close(fd)
        try:   # -f: nvidia-smi writes (and flushes) every sample to the file itself
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.QUERY, "--format=csv,noheader,nounits",
                                          "-lms", "200", "-f", self.path],
                                         stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.5)   # first sample before the timed region
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
        try:
            with open(self.path) as fh:
                self.out = fh.read()
            os.unlink(self.path)
        except OSError:
            self.out = ""

    def parse(self, text):
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        rows = [[c.strip() for c in r] for r in csv.reader(io.StringIO(text or "")) if len(r) >= 9]
        mine = [r for r in rows if self.uuid and r[0].lower().replace("gpu-", "") == self.uuid]
        if not mine:
            mine = [r for r in rows if r[1] == self.index]
        sm = [num(r[2]) for r in mine if num(r[2]) is not None]
        mx = [num(r[3]) for r in mine if num(r[3]) is not None]
        pw = [num(r[4]) for r in mine if num(r[4]) is not None]
        reasons = sorted({self.NAMES[i] for r in mine for i in range(4) if r[5 + i].lower() == "active"})
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        load = [v for v in sm if v >= 0.3 * max(mx or sm)] or sm
        return {"sm_mhz": statistics.median(load), "sm_mhz_min": min(load), "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None, "reasons": reasons, "samples": len(mine)}

    def summary(self):
        return self.parse(self.out)


def gpu_identity(torch, dev):
    """(uuid, nvidia-smi index) of a torch device."""
    uuid = ""
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    vis = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    idx = dev.index or 0
    index = vis[idx] if idx < len(vis) and vis[idx].isdigit() else str(idx)
    return uuid, index


# ----------------------------------------------------------------------------- ranks
def rank_workload(rank: int):
    """Per-rank step inputs: every rank quantizes its own seeded tokens (the
    path shards by tokens) against the same weights."""
    import workloads
    wl = workloads.dit_mlp()
    if rank > 0:
        wl["x"] = workloads.with_outlier_channels((M_TOK, HID), 1.0, 21 + 1000 * rank)
        wl["dy2"] = workloads.normal((M_TOK, HID), 1e-3, 24 + 1000 * rank)
    return wl


def max_over_ranks(value: float, dist, device) -> float:
    """The largest of the ranks' values (timings are taken as the slowest
    rank's); the identity without a process group."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- oracle (CPU)
def oracle_chain_rows(orc, wl, W1r, s1r, W2r, s2r, rows):
    """The step on the CPU oracle for a subset of token rows (every step is
    row-local).  Returns the int ops of the sample."""
    import workloads
    x = workloads.to_u16(wl["x"])[rows]
    dy = workloads.to_u16(wl["dy2"])[rows]
    r1 = orc.linear_fwd(x, W1r, s1r)
    orc.linear_fwd(r1["y"], W2r, s2r)
    g2 = orc.linear_dgrad(dy, W2r, s2r)
    orc.linear_dgrad(g2["y"], W1r, s1r)
    return 4 * 2 * len(rows) * HID * MLP


def oracle_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def time_oracle(orc, wl, W1r, s1r, W2r, s2r, target_s):
    import numpy as np
    probe = np.arange(16)
    t0 = time.perf_counter()
    oracle_chain_rows(orc, wl, W1r, s1r, W2r, s2r, probe)
    dt = time.perf_counter() - t0
    n = int(min(M_TOK, max(16, 16 * target_s / max(dt, 1e-3))))
    rows = np.linspace(0, M_TOK - 1, n).astype(np.int64)
    t0 = time.perf_counter()
    ops = oracle_chain_rows(orc, wl, W1r, s1r, W2r, s2r, rows)
    dt = time.perf_counter() - t0
    return ops / dt / 1e12, n, dt


def oracle_weights(orc, wl):
    import workloads
    W1r, s1r = orc.quantize_weight(workloads.to_u16(wl["w1"]), orc.INT8, orc.TENSOR)
    W2r, s2r = orc.quantize_weight(workloads.to_u16(wl["w2"]), orc.INT8, orc.TENSOR)
    return W1r, s1r, W2r, s2r


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import oracle as orc
    import workloads
    orc.build()
    wl = workloads.dit_mlp()
    W1r, s1r, W2r, s2r = oracle_weights(orc, wl)
    import numpy as np
    # size each step so that warmup + steps end within about two minutes
    probe = np.arange(8)
    t0 = time.perf_counter()
    oracle_chain_rows(orc, wl, W1r, s1r, W2r, s2r, probe)
    per_row = (time.perf_counter() - t0) / 8
    budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(min(M_TOK, max(8, budget / max(per_row, 1e-6))))
    rows = np.linspace(0, M_TOK - 1, n).astype(np.int64)
    for _ in range(args.warmup):
        oracle_chain_rows(orc, wl, W1r, s1r, W2r, s2r, rows)
    t0 = time.perf_counter()
    ops = 0
    for _ in range(args.steps):
        ops += oracle_chain_rows(orc, wl, W1r, s1r, W2r, s2r, rows)
    dt = time.perf_counter() - t0
    value = ops / dt / 1e12
    sample = "%d of %d token rows per step (row-local step), all 4 GEMMs with quantize + epilogue" % (n, M_TOK)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
            "data": "synthetic", "config": workload_config(),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config():
    return {"workload": "int W8A8 DiT MLP block fwd+dgrad (up 3072->12288, down 12288->3072, "
                        "dgrad through both), tensor-wise int8 W, token-wise int8 activations",
            "M": M_TOK, "hidden": HID, "mlp": MLP, "global_batch_tokens_per_gpu": M_TOK,
            "parallelism": "token-sharded replicas", "l2": "flushed between timed steps: 256 MiB written, then read back (outside the step's events)"}


# ----------------------------------------------------------------------------- ours
def run_ours(args, rank, world, local_rank):
    import torch
    import workloads
    import w8a8_quantized_linear_b200 as w8
    from w8a8_quantized_linear_b200 import _build

    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        dist = dist_mod
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if rank == 0:
        _build.build()
    if dist is not None:
        dist.barrier()
    w8.lib()

    wl = rank_workload(rank)
    X = wl["x"].to(dev)
    dY2 = wl["dy2"].to(dev)
    W1q, s1 = w8.quantize_weight(wl["w1"].to(dev), "int8", "tensor")
    W2q, s2 = w8.quantize_weight(wl["w2"].to(dev), "int8", "tensor")
    # pre-allocated codes, scales, outputs (no allocation inside the step)
    u8 = lambda *s: torch.empty(*s, dtype=torch.int8, device=dev)
    f32 = lambda *s: torch.empty(*s, dtype=torch.float32, device=dev)
    b16 = lambda *s: torch.empty(*s, dtype=torch.bfloat16, device=dev)
    xq1, sx1, Y1 = u8(M_TOK, HID), f32(M_TOK), b16(M_TOK, MLP)
    xq2, sx2, Y2 = u8(M_TOK, MLP), f32(M_TOK), b16(M_TOK, HID)
    gq2, sg2, dX2 = u8(M_TOK, HID), f32(M_TOK), b16(M_TOK, MLP)
    gq1, sg1, dX1 = u8(M_TOK, MLP), f32(M_TOK), b16(M_TOK, HID)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    E = lambda: torch.cuda.Event(enable_timing=True)

    KERNELS = [lambda: w8.quantize_rows(X, "int8", out=xq1, scale=sx1),
               lambda: w8.qgemm_fwd(xq1, sx1, W1q, s1, out=Y1),
               lambda: w8.quantize_rows(Y1, "int8", out=xq2, scale=sx2),
               lambda: w8.qgemm_fwd(xq2, sx2, W2q, s2, out=Y2),
               lambda: w8.quantize_rows(dY2, "int8", out=gq2, scale=sg2),
               lambda: w8.qgemm_dgrad(gq2, sg2, W2q, s2, out=dX2),
               lambda: w8.quantize_rows(dX2, "int8", out=gq1, scale=sg1),
               lambda: w8.qgemm_dgrad(gq1, sg1, W1q, s1, out=dX1)]

    def step(ev, per_kernel=False):
        """The step's 8 launches between events ev[0] and ev[-1]; with
        per_kernel, an event after each launch as well (ev has 9 entries).
        Without them consecutive launches may overlap (programmatic dependent
        launch), so the timed steps record only the two ends."""
        ev[0].record(stream)
        for k, fn in enumerate(KERNELS):
            fn()
            if per_kernel:
                ev[k + 1].record(stream)
        if not per_kernel:
            ev[-1].record(stream)

    def flush_l2(i):
        flush.fill_(i & 0xFF)          # L2 flush (write, then read back so that no dirty
        return flush.view(torch.int64).sum()   # lines are left for the step), outside the step's events

    for i in range(args.warmup):
        flush_l2(i)
        step([E(), E()])
    torch.cuda.synchronize()
    assert w8.device_status() == 0, "device-side error during warm-up"

    events = [[E(), E()] for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(*gpu_identity(torch, dev)) as clk:
        wall0 = time.perf_counter()
        for i in range(args.steps):
            flush_l2(i)
            step(events[i])
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
        # the per-kernel split, from as many steps again with an event after
        # every launch (same inputs and launches; L2 flushed the same way)
        kev = [[E() for _ in range(9)] for _ in range(args.steps)]
        for i in range(args.steps):
            flush_l2(i)
            step(kev[i], per_kernel=True)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    step_ms = [ev[0].elapsed_time(ev[-1]) for ev in events]
    gemm_ms = [ev[k - 1].elapsed_time(ev[k]) for ev in kev for k in (2, 4, 6, 8)]
    quant_ms = [ev[k - 1].elapsed_time(ev[k]) for ev in kev for k in (1, 3, 5, 7)]
    total_ms = max_over_ranks(sum(step_ms), dist, dev)
    ms_per_step = total_ms / args.steps
    value = world * OPS_PER_STEP * args.steps / (total_ms * 1e-3) / 1e12
    assert w8.device_status() == 0, "device-side error during the timed steps"

    # ---- end to end: pinned host inputs -> public API -> pinned host results.
    # Three streams, double-buffered device inputs and outputs: the copies of
    # step i + 1's inputs and of step i - 1's results overlap step i's
    # compute.  Dependencies are per tensor: the forward waits only for X,
    # the input gradient only for dY; Y2 leaves as soon as the forward is
    # done; an input buffer is refilled once its one reader has finished.
    # Every step copies all of its inputs in and all of its results out.
    e2e = None
    if args.e2e_steps > 0:
        hx = wl["x"].pin_memory()
        hdy = wl["dy2"].pin_memory()
        hy2 = [torch.empty((M_TOK, HID), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        hdx1 = [torch.empty((M_TOK, HID), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        ws = torch.empty(w8.workspace_bytes(w8.OP_LINEAR_FWD, M_TOK, MLP, MLP), dtype=torch.uint8, device=dev)
        Xd = [torch.empty_like(X) for _ in range(2)]
        dYd = [torch.empty_like(dY2) for _ in range(2)]
        Y2d = [torch.empty_like(Y2) for _ in range(2)]
        dX1d = [torch.empty_like(dX1) for _ in range(2)]
        s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        ev = lambda: torch.cuda.Event()
        x_in, dy_in = [ev(), ev()], [ev(), ev()]             # inputs landed
        x_read, dy_read = [ev(), ev()], [ev(), ev()]         # inputs consumed
        y2_done, dx1_done = [ev(), ev()], [ev(), ev()]       # results computed
        y2_out, dx1_out = [ev(), ev()], [ev(), ev()]         # results copied out

        def e2e_steps(n, first):
            for i in range(n):
                b = i & 1
                reuse = not (first and i < 2)                 # buffer b was used two steps ago
                with torch.cuda.stream(s_in):
                    if reuse:
                        s_in.wait_event(x_read[b])
                    Xd[b].copy_(hx, non_blocking=True)
                    x_in[b].record(s_in)
                    if reuse:
                        s_in.wait_event(dy_read[b])
                    dYd[b].copy_(hdy, non_blocking=True)
                    dy_in[b].record(s_in)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(x_in[b])
                    if reuse:
                        s_cmp.wait_event(y2_out[b])
                    w8.linear_fwd(Xd[b], W1q, s1, out=Y1, ws=ws)
                    x_read[b].record(s_cmp)
                    w8.linear_fwd(Y1, W2q, s2, out=Y2d[b], ws=ws)
                    y2_done[b].record(s_cmp)
                    s_cmp.wait_event(dy_in[b])
                    if reuse:
                        s_cmp.wait_event(dx1_out[b])
                    w8.linear_dgrad(dYd[b], W2q, s2, out=dX2, ws=ws)
                    dy_read[b].record(s_cmp)
                    w8.linear_dgrad(dX2, W1q, s1, out=dX1d[b], ws=ws)
                    dx1_done[b].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(y2_done[b])
                    hy2[b].copy_(Y2d[b], non_blocking=True)
                    y2_out[b].record(s_out)
                    s_out.wait_event(dx1_done[b])
                    hdx1[b].copy_(dX1d[b], non_blocking=True)
                    dx1_out[b].record(s_out)

        e2e_steps(3, True)
        torch.cuda.synchronize()
        a, b = E(), E()
        a.record(s_in)
        e2e_steps(args.e2e_steps, False)
        s_in.wait_stream(s_out)
        s_in.wait_stream(s_cmp)
        b.record(s_in)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b), dist, dev)
        e2e = {"value": world * OPS_PER_STEP * args.e2e_steps / (e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": hx.numel() * 2 + hdy.numel() * 2,
               "d2h_bytes_per_step": hy2[0].numel() * 2 + hdx1[0].numel() * 2,
               "ms_per_step": e_ms / args.e2e_steps, "steps": args.e2e_steps,
               "api": "w8a8_linear_fwd x2 + w8a8_linear_dgrad x2 per step; pinned host buffers; "
                      "copies in and out timed, overlapped with compute across steps (3 streams, "
                      "per-tensor dependencies)"}

    if rank != 0:
        return 0

    peaks, src = load_peaks()
    # int8 dense = 2 x bf16 dense (4.5 vs 2.25 PFLOP/s nominal).  The timed
    # region lasts tens of milliseconds, so the burst figure applies; the
    # sustained fraction is reported beside it.
    int8_peak = 2.0 * peaks["bf16_tflops"]
    gemm_avg = statistics.mean(gemm_ms)
    achieved = OPS_PER_GEMM / (gemm_avg * 1e-3) / 1e12
    sha = gemm_source_sha()
    traffic = GEMM_TRAFFIC["bytes_per_launch"] if GEMM_TRAFFIC["source_sha"] == sha else None
    roofline = {"bound": "tensor", "kernel": "gemm_pair_kernel<i8> (tcgen05 cta_group::2 kind::i8, fused epilogue)",
                "achieved": achieved, "peak": int8_peak, "unit": "TFLOP/s", "frac": achieved / int8_peak,
                "traffic": traffic,
                "peak_source": "%s: 2 x bf16_tflops (burst; int8 dense = 2x bf16 dense nominal)" % src,
                "frac_of_sustained": achieved / (2.0 * peaks["bf16_tflops_sustained"]),
                "gemm_ms_avg": gemm_avg, "quantize_ms_avg": statistics.mean(quant_ms),
                "quantize_share": sum(quant_ms) / (sum(quant_ms) + sum(gemm_ms)),
                "per_kernel_events": "separate steps with an event after every launch (launches then "
                                     "cannot overlap); their sum per step: %.4f ms" %
                                     ((sum(quant_ms) + sum(gemm_ms)) / args.steps)}
    clocks = clk.summary()

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic", "config": workload_config(),
            "roofline": roofline, "e2e": e2e, "clocks": clocks, "gpu_launches": 8 * args.steps,
            "wall_s_timed_region": wall}
    if args.cpu_baseline and world == 1:
        import oracle as orc
        orc.build()
        W1r, s1r, W2r, s2r = oracle_weights(orc, wl)
        v, n, dt = time_oracle(orc, wl, W1r, s1r, W2r, s2r, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": oracle_cores(), "kind": "oracle",
                                "sample": "%d of %d token rows of the same step (row-local), %.1f s" % (n, M_TOK, dt)}
    if args.extras and world == 1:
        with ClockSampler(*gpu_identity(torch, dev)) as clk_x:
            line["extras"] = extras(w8, torch, workloads, dev, peaks, src)
        line["extras"]["clocks"] = clk_x.summary()   # over all extras: a dip shows in sm_mhz_min
    # the compact per-row summary goes last, so that a reader keeping only the
    # end of the line still sees every row's number
    line["rows"] = summary_rows(line)
    print(json.dumps(line), flush=True)
    return 0


def _g3(v):
    """A number rounded to 3 significant digits (None passes through)."""
    return None if v is None else float("%.3g" % v)


def summary_rows(line):
    """One short entry per row of the hot path: microseconds, and the
    fraction of the roofline the row is bound by (HBM copy bandwidth, or the
    8-bit / bf16 tensor peak), taken from the headline and the extras."""
    rf = line["roofline"]
    rows = {"headline_dit_mlp_fwd_dgrad": {"TOPS": _g3(line["value"]), "ms": _g3(line["ms_per_step"]),
                                           "gemm_frac": _g3(rf["frac"]), "e2e_TOPS": _g3((line.get("e2e") or {}).get("value"))}}
    x = line.get("extras")
    if not x:
        return rows
    us = lambda d: _g3(d["ms"] * 1e3)
    bw = lambda d: {"us": us(d), "hbm_frac": _g3(d["hbm_frac"])}
    rows["a1_quantize_rows_4608x12288"] = bw(x["quantize_rows_4608x12288"])
    rows["a2_quantize_weight_tensor_12288x3072"] = {"us": us(x["quantize_weight_tensor_12288x3072"]),
                                                    "GBps": _g3(x["quantize_weight_tensor_12288x3072"]["GB/s"])}
    rows["a3_q8_0_quantize_2^28"] = bw(x["q8_0_quantize_2^28"])
    rows["a3_q8_0_dequantize_2^28"] = bw(x["q8_0_dequantize_2^28"])
    rows["a4_q8_0_to_axis_int8_12288x3072"] = bw(x["q8_0_to_axis_int8_12288x3072"])
    rows["f2_q8_0_to_axis_e4m3_12288x3072"] = bw(x["q8_0_to_axis_e4m3_12288x3072"])
    d = x["int_w8a8_fwd_tiny_256x512x512"]
    rows["cfg1_int_tiny_256x512x512"] = {"us": us(d)}
    d = x["float_w8a8_fwd_4096x3072x3072"]
    rows["cfg2_float_w8a8_4096x3072x3072"] = {"us": us(d), "TOPS": _g3(d["TOPS"]), "gemm_us": _g3(d["gemm_ms"] * 1e3),
                                              "gemm_frac_fp8": _g3(d["gemm_frac_fp8_burst"])}
    d = x["svdquant_r32_fwd_4608x3072x3072"]
    rows["cfg4_svdquant_int8_r32"] = {"us": us(d), "frac_int8": _g3(d["frac_int8_burst"])}
    d = x["svdquant_e4m3_r32_fwd_4608x3072x3072"]
    rows["f4_svdquant_e4m3_r32"] = {"us": us(d), "frac_fp8": _g3(d["frac_fp8_burst"])}
    for key, name in (("gguf_a8_int_fwd_sweep_N12288_K3072", "cfg5_gguf_a8_int"),
                      ("gguf_a8_float_fwd_sweep_N12288_K3072", "f2_gguf_a8_float")):
        rows[name] = {m: [us(v), _g3(v["roofline_frac"])] for m, v in x[key].items()}
    rows["cfg5_format"] = "M: [us, roofline_frac]"
    wo = x["weight_only_fwd_4608x12288x3072"]
    wd = x["weight_only_dgrad_4608x12288x3072"]
    rows["f3_weight_only_frac_bf16"] = {k: [_g3(wo[k]["frac_bf16_burst"]), _g3(wd[k]["frac_bf16_burst"])]
                                        for k in ("bf16_gemm", "float8", "gguf")}
    rows["f3_format"] = "[fwd, dgrad] at 4608x12288x3072"
    rows["a3_dequant_bf16_12288x3072_hbm_frac"] = {"e4m3": _g3(x["dequantize_e4m3_bf16_12288x3072"]["hbm_frac"]),
                                                   "q8_0": _g3(x["q8_0_dequantize_bf16_12288x3072"]["hbm_frac"])}
    f1 = x["dit_mlp_fwd_gelu_4608x3072x12288"]
    rows["f1_mlp_fwd_gelu_us"] = {k: us(v) for k, v in f1.items()}
    return rows


def run_case(args):
    """One quantize + GEMM pair of the step, or one other kernel of the path,
    warmup + steps times (profiling)."""
    import torch
    import workloads
    import w8a8_quantized_linear_b200 as w8
    dev = torch.device("cuda", 0)
    if args.case in ("requant", "gguf_m1", "gguf_m64", "svdq", "requant_e4m3", "gguf_f_m1", "gguf_f_m4608",
                     "svdq_e4m3", "wo_float8", "wo_gguf", "gguf_m512", "q8_0_quant", "q8_0_dequant",
                     "float_w8a8", "float_w8a8_int8"):
        return run_other_case(args, torch, workloads, w8, dev)
    wl = workloads.dit_mlp()
    if args.case in ("up", "dgrad_up"):
        wq, sw = w8.quantize_weight(wl["w1"].to(dev), "int8", "tensor")      # [12288, 3072]
    else:
        wq, sw = w8.quantize_weight(wl["w2"].to(dev), "int8", "tensor")      # [3072, 12288]
    if args.case == "up":
        x = wl["x"].to(dev)
        fn = lambda xq, s: w8.qgemm_fwd(xq, s, wq, sw)
    elif args.case == "down":
        x = workloads.normal((M_TOK, MLP), 0.5, 25).to(dev)
        fn = lambda xq, s: w8.qgemm_fwd(xq, s, wq, sw)
    elif args.case == "dgrad_down":
        x = wl["dy2"].to(dev)
        fn = lambda xq, s: w8.qgemm_dgrad(xq, s, wq, sw)
    else:
        x = workloads.normal((M_TOK, MLP), 1e-3, 26).to(dev)
        fn = lambda xq, s: w8.qgemm_dgrad(xq, s, wq, sw)
    for _ in range(args.warmup + args.steps):
        xq, s = w8.quantize_rows(x, "int8")
        fn(xq, s)
    torch.cuda.synchronize()
    assert w8.device_status() == 0
    print("case %s ok" % args.case)
    return 0


def run_other_case(args, torch, workloads, w8, dev):
    """requant / requant_e4m3: Q8_0 -> axis int8 / e4m3 of the 12288 x 3072
    GGUF weight; gguf_m1 / gguf_m64 / gguf_m512: the GGUF A8 int forward at M = 1 / 64 / 512;
    gguf_f_m1 / gguf_f_m4608: the GGUF A8 float forward at M = 1 / 4608;
    svdq / svdq_e4m3: the SVDQuant r = 32 forward at 4608 x 3072 x 3072 with
    an int8 / e4m3 residual; wo_float8 / wo_gguf: the weight-only forwards
    on the DiT up-projection (dequantize to bf16, then the bf16 Linear);
    float_w8a8 / float_w8a8_int8: the float W8A8 forward with bias at 4096 x
    3072 x 3072 (e4m3), and the same shape with int8 codes."""
    if args.case in ("q8_0_quant", "q8_0_dequant"):
        # the standalone Q8_0 quantize / dequantize, 2^26 fp32 values (256 MiB,
        # twice the L2; the bench extras time 2^28)
        n = 1 << 26
        xf = workloads.q8_0_standalone(n).to(dev)
        blk = w8.q8_0_quantize(xf)
        yf = torch.empty_like(xf)
        fn = (lambda: w8.q8_0_quantize(xf, out=blk)) if args.case == "q8_0_quant" else \
            (lambda: w8.q8_0_dequantize(blk, n, out=yf))
    elif args.case in ("wo_float8", "wo_gguf"):
        g = workloads.gguf_q8_0(M=M_TOK)
        x = g["x"].to(dev)
        if args.case == "wo_float8":
            wq, sw = w8.quantize_weight(g["w_f32"].to(torch.bfloat16).to(dev), "e4m3", "tensor")
            fn = lambda: w8.float8_linear_fwd(x, wq, sw)
        else:
            blk = w8.q8_0_quantize(g["w_f32"].reshape(-1).to(dev))
            fn = lambda: w8.gguf_linear_fwd(x, blk, MLP)
    elif args.case in ("float_w8a8", "float_w8a8_int8"):
        d = workloads.float_w8a8()
        qt = "e4m3" if args.case == "float_w8a8" else "int8"
        wq, sw = w8.quantize_weight(d["w"].to(dev), qt, "tensor")
        x, bias = d["x"].to(dev), d["bias"].to(dev)
        fn = lambda: w8.linear_fwd(x, wq, sw, bias=bias)
    elif args.case in ("svdq", "svdq_e4m3"):
        d = workloads.svdquant()
        prep = w8.svdq_prepare(d["w"].to(dev), d["r"], "e4m3" if args.case == "svdq_e4m3" else "int8")
        x = d["x"].to(dev)
        fn = lambda: w8.svdq_linear_fwd(x, prep["rq"], prep["r_scale"], prep["l1"], prep["l2"])
    else:
        g = workloads.gguf_q8_0(M=4608 if args.case == "gguf_f_m4608" else 512)
        N, K = g["w_f32"].shape
        blk = w8.q8_0_quantize(g["w_f32"].reshape(-1).to(dev))
        if args.case == "requant":
            fn = lambda: w8.q8_0_to_axis_int8(blk, N, K)
        elif args.case == "requant_e4m3":
            fn = lambda: w8.q8_0_to_axis_e4m3(blk, N, K)
        elif args.case.startswith("gguf_f_m"):
            wq, sw = w8.q8_0_to_axis_e4m3(blk, N, K)
            x = g["x"][:int(args.case[len("gguf_f_m"):])].to(dev)
            fn = lambda: w8.linear_fwd(x, wq, sw)
        else:
            wq, sw = w8.q8_0_to_axis_int8(blk, N, K)
            x = g["x"][:{"gguf_m1": 1, "gguf_m64": 64, "gguf_m512": 512}[args.case]].to(dev)
            fn = lambda: w8.linear_fwd(x, wq, sw)
    for _ in range(args.warmup + args.steps):
        fn()
    torch.cuda.synchronize()
    assert w8.device_status() == 0
    print("case %s ok" % args.case)
    return 0


L2_BYTES = 126 << 20


def _nsets(set_bytes):
    """Copies of a buffer set to rotate through so that each is touched once
    per cycle over at least 3x the L2 size (no set is L2-resident when used)."""
    return max(2, -(-3 * L2_BYTES // max(1, int(set_bytes))))


def _time_rot(fns, reps, torch, stream):
    """Mean GPU time of one call.  The calls, cycling through ``fns`` (each on
    its own buffers), are captured once in a CUDA graph, and the graph is
    replayed between two events on the launching stream: host-side launch
    cost is left out, as in a captured model step (every call of the library
    is stream-ordered and capturable).  The fastest of three replays."""
    for f in fns:
        f()
    torch.cuda.synchronize()
    n = max(reps, len(fns))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            fns[i % len(fns)]()
    g.replay()
    torch.cuda.synchronize()
    E = lambda: torch.cuda.Event(enable_timing=True)
    best = None
    for _ in range(3):   # the fastest of three replays (clock and scheduling noise)
        a, b = E(), E()
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        t = a.elapsed_time(b) / n
        best = t if best is None or t < best else best
    del g
    return best


def _gemm_roof_ms(M, N, K, hbm_gbs, tops):
    """Roofline time of a W8A8 forward in ms: the slower of streaming its
    bytes (8-bit weight, bf16 activations in and out, 8-bit codes written and
    read) at the copy bandwidth and its 2MNK operations at the 8-bit peak."""
    nbytes = N * K + M * K * 2 + M * K * 2 + M * N * 2
    return max(nbytes / (hbm_gbs * 1e9), 2.0 * M * N * K / (tops * 1e12)) * 1e3


def extras(w8, torch, workloads, dev, peaks, src):
    """The other rows of the hot path, each timed on its own: mean over reps
    launched back to back, rotating through copies of the inputs and outputs
    whose footprint is at least 3x the L2 size."""
    out = {}
    stream = torch.cuda.current_stream(dev)
    hbm = peaks["hbm_gbs"]
    tc8 = 2.0 * peaks["bf16_tflops"]
    nbytes = lambda *ts: sum(t.numel() * t.element_size() for t in ts)
    # token-wise quantize (K1) at 4608 x 12288
    x0 = workloads.normal((M_TOK, MLP), 1.0, 5).to(dev)
    sets = []
    for i in range(_nsets(nbytes(x0) * 1.5)):
        x = x0.clone()
        q = torch.empty((M_TOK, MLP), dtype=torch.int8, device=dev)
        s = torch.empty(M_TOK, dtype=torch.float32, device=dev)
        sets.append(lambda x=x, q=q, s=s: w8.quantize_rows(x, "int8", out=q, scale=s))
    ms = _time_rot(sets, 30, torch, stream)
    gbs = (x0.numel() * 3 + M_TOK * 4) / (ms * 1e-3) / 1e9
    out["quantize_rows_4608x12288"] = {"ms": ms, "GB/s": gbs, "hbm_frac": gbs / hbm}
    del x0, sets
    # DiT MLP forward with GELU between the projections: the down-projection's
    # quantizer reduces each row itself, or takes the row absmax that the
    # up-projection's epilogue gathered (same codes, same output)
    wl = workloads.dit_mlp()
    w1q, s1 = w8.quantize_weight(wl["w1"].to(dev), "int8", "tensor")
    w2q, s2 = w8.quantize_weight(wl["w2"].to(dev), "int8", "tensor")
    xm0 = wl["x"].to(dev)
    res = {}
    for name, fused in (("unfused", False), ("fused_absmax", True)):
        sets = []
        for i in range(_nsets(nbytes(xm0) + M_TOK * MLP * 3 + M_TOK * HID * 2)):
            xm = xm0.clone()
            y1 = torch.empty((M_TOK, MLP), dtype=torch.bfloat16, device=dev)
            y2 = torch.empty((M_TOK, HID), dtype=torch.bfloat16, device=dev)
            a1 = torch.empty(M_TOK, dtype=torch.int32, device=dev)
            ws1 = torch.empty(w8.workspace_bytes(0, M_TOK, MLP, HID), dtype=torch.uint8, device=dev)
            ws2 = torch.empty(w8.workspace_bytes(0, M_TOK, HID, MLP), dtype=torch.uint8, device=dev)
            if fused:
                def fn(xm=xm, y1=y1, y2=y2, a1=a1, ws1=ws1, ws2=ws2):
                    w8.linear_fwd_ex(xm, w1q, s1, act="gelu", y_amax=a1, out=y1, ws=ws1)
                    w8.linear_fwd_ex(y1, w2q, s2, x_amax=a1, out=y2, ws=ws2)
            else:
                def fn(xm=xm, y1=y1, y2=y2, ws1=ws1, ws2=ws2):
                    w8.linear_fwd_ex(xm, w1q, s1, act="gelu", out=y1, ws=ws1)
                    w8.linear_fwd(y1, w2q, s2, out=y2, ws=ws2)
            sets.append(fn)
        ms = _time_rot(sets, 10, torch, stream)
        res[name] = {"ms": ms, "TOPS": 2 * 2 * M_TOK * MLP * HID / ms / 1e9}
        del sets
    out["dit_mlp_fwd_gelu_4608x3072x12288"] = res
    del xm0, w1q, w2q
    # the tiny int W8A8 forward (256 x 512 x 512): latency-bound, reported
    # without a bar
    d = workloads.int_tiny()
    wqt, swt = w8.quantize_weight(d["w"].to(dev), "int8", "tensor")
    sets = []
    for i in range(4):
        xt = d["x"].to(dev).clone()
        yt = torch.empty((256, 512), dtype=torch.bfloat16, device=dev)
        wst = torch.empty(w8.workspace_bytes(0, 256, 512, 512), dtype=torch.uint8, device=dev)
        sets.append(lambda xt=xt, yt=yt, wst=wst: w8.linear_fwd(xt, wqt, swt, out=yt, ws=wst))
    ms = _time_rot(sets, 50, torch, stream)
    out["int_w8a8_fwd_tiny_256x512x512"] = {"ms": ms, "TOPS": 2 * 256 * 512 * 512 / ms / 1e9,
                                            "note": "inputs L2-resident (1 MB); launch- and latency-bound"}
    del sets
    # float W8A8 forward (e4m3, bias) 4096 x 3072 x 3072
    d = workloads.float_w8a8()
    wq0, sw = w8.quantize_weight(d["w"].to(dev), "e4m3", "tensor")
    xx0, bb = d["x"].to(dev), d["bias"].to(dev)
    xq0, sx0 = w8.quantize_rows(xx0, "e4m3")
    fsets, gsets = [], []
    for i in range(_nsets(nbytes(xx0, wq0) + 4096 * 3072 * 2)):
        xx, wq, xq = xx0.clone(), wq0.clone(), xq0.clone()
        y = torch.empty((4096, 3072), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(w8.workspace_bytes(0, 4096, 3072, 3072), dtype=torch.uint8, device=dev)
        fsets.append(lambda xx=xx, wq=wq, y=y, ws=ws: w8.linear_fwd(xx, wq, sw, bias=bb, out=y, ws=ws))
        gsets.append(lambda xq=xq, wq=wq, y=y: w8.qgemm_fwd(xq, sx0, wq, sw, bias=bb, out=y))
    ms = _time_rot(fsets, 30, torch, stream)
    gms = _time_rot(gsets, 30, torch, stream)
    ops = 2 * 4096 * 3072 * 3072
    out["float_w8a8_fwd_4096x3072x3072"] = {"ms": ms, "TOPS": ops / ms / 1e9, "gemm_ms": gms,
                                            "gemm_TOPS": ops / gms / 1e9, "gemm_frac_fp8_burst": ops / gms / 1e9 / tc8}
    del fsets, gsets
    # SVDQuant r=32, 4608 x 3072 x 3072
    d = workloads.svdquant()
    prep0 = w8.svdq_prepare(d["w"].to(dev), d["r"])
    xx0 = d["x"].to(dev)
    sets = []
    for i in range(_nsets(nbytes(xx0, prep0["rq"]) + M_TOK * 3072 * 2)):
        xx = xx0.clone()
        rq, l1, l2 = prep0["rq"].clone(), prep0["l1"].clone(), prep0["l2"].clone()
        y = torch.empty((M_TOK, 3072), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(w8.workspace_bytes(2, M_TOK, 3072, 3072, 32), dtype=torch.uint8, device=dev)
        sets.append(lambda xx=xx, rq=rq, l1=l1, l2=l2, y=y, ws=ws:
                    w8.svdq_linear_fwd(xx, rq, prep0["r_scale"], l1, l2, out=y, ws=ws))
    ms = _time_rot(sets, 30, torch, stream)
    ops = 2 * M_TOK * 3072 * 3072
    out["svdquant_r32_fwd_4608x3072x3072"] = {"ms": ms, "TOPS_main": ops / ms / 1e9,
                                              "frac_int8_burst": ops / ms / 1e9 / tc8,
                                              "lowrank_GFLOP": 2 * 2 * M_TOK * 3072 * 32 / 1e9}
    del sets, prep0
    # the same with an e4m3 residual (float W8A8 + SVDQuant)
    prep0 = w8.svdq_prepare(d["w"].to(dev), d["r"], "e4m3")
    sets = []
    for i in range(_nsets(nbytes(xx0, prep0["rq"]) + M_TOK * 3072 * 2)):
        xx = xx0.clone()
        rq, l1, l2 = prep0["rq"].clone(), prep0["l1"].clone(), prep0["l2"].clone()
        y = torch.empty((M_TOK, 3072), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(w8.workspace_bytes(2, M_TOK, 3072, 3072, 32), dtype=torch.uint8, device=dev)
        sets.append(lambda xx=xx, rq=rq, l1=l1, l2=l2, y=y, ws=ws:
                    w8.svdq_linear_fwd(xx, rq, prep0["r_scale"], l1, l2, out=y, ws=ws))
    ms = _time_rot(sets, 30, torch, stream)
    out["svdquant_e4m3_r32_fwd_4608x3072x3072"] = {"ms": ms, "TOPS_main": ops / ms / 1e9,
                                                   "frac_fp8_burst": ops / ms / 1e9 / tc8,
                                                   "lowrank_GFLOP": 2 * 2 * M_TOK * 3072 * 32 / 1e9}
    del sets, prep0
    # GGUF Q8_0: standalone quantize / dequantize of 2^28 fp32 (each 1.3 GB of traffic)
    n = 1 << 28
    xf0 = workloads.q8_0_standalone(n).to(dev)
    qsets, dsets = [], []
    for i in range(2):
        xf = xf0 if i == 0 else xf0.clone()
        blk = torch.empty(w8.q8_0_bytes(n), dtype=torch.uint8, device=dev)
        w8.q8_0_quantize(xf, out=blk)
        yf = torch.empty_like(xf)
        qsets.append(lambda xf=xf, blk=blk: w8.q8_0_quantize(xf, out=blk))
        dsets.append(lambda blk=blk, yf=yf: w8.q8_0_dequantize(blk, n, out=yf))
    nb = w8.q8_0_bytes(n)
    ms = _time_rot(qsets, 10, torch, stream)
    gbs = (4 * n + nb) / (ms * 1e-3) / 1e9
    out["q8_0_quantize_2^28"] = {"ms": ms, "GB/s": gbs, "hbm_frac": gbs / hbm}
    ms = _time_rot(dsets, 10, torch, stream)
    gbs = (4 * n + nb) / (ms * 1e-3) / 1e9
    out["q8_0_dequantize_2^28"] = {"ms": ms, "GB/s": gbs, "hbm_frac": gbs / hbm}
    del xf0, qsets, dsets
    # requant Q8_0 -> axis int8 (K10), 12288 x 3072
    g = workloads.gguf_q8_0(M=max(workloads.GGUF_MS))
    wb0 = w8.q8_0_quantize(g["w_f32"].reshape(-1).to(dev))
    wq0, sw = w8.q8_0_to_axis_int8(wb0, MLP, HID)
    sets = []
    for i in range(_nsets(nbytes(wb0, wq0))):
        wb = wb0.clone()
        q = torch.empty_like(wq0)
        s = torch.empty(MLP, dtype=torch.float32, device=dev)
        sets.append(lambda wb=wb, q=q, s=s: w8.q8_0_to_axis_int8(wb, MLP, HID, out=q, scale=s))
    ms = _time_rot(sets, 30, torch, stream)
    gbs = (wb0.numel() + MLP * HID + MLP * 4) / (ms * 1e-3) / 1e9
    out["q8_0_to_axis_int8_12288x3072"] = {"ms": ms, "GB/s": gbs, "hbm_frac": gbs / hbm}
    del sets
    # GGUF A8 float: Q8_0 -> axis e4m3 (same traffic as the int8 requant); the
    # e4m3 forward sweep, one weight scale per output column, runs below
    wq0e, swe = w8.q8_0_to_axis_e4m3(wb0, MLP, HID)
    sets = []
    for i in range(_nsets(nbytes(wb0, wq0))):
        wb = wb0.clone()
        q = torch.empty_like(wq0e)
        s = torch.empty(MLP, dtype=torch.float32, device=dev)
        sets.append(lambda wb=wb, q=q, s=s: w8.q8_0_to_axis_e4m3(wb, MLP, HID, out=q, scale=s))
    ms = _time_rot(sets, 30, torch, stream)
    gbs = (wb0.numel() + MLP * HID + MLP * 4) / (ms * 1e-3) / 1e9
    out["q8_0_to_axis_e4m3_12288x3072"] = {"ms": ms, "GB/s": gbs, "hbm_frac": gbs / hbm}
    del sets
    # tensor-wise weight quantization (load time), 12288 x 3072
    wt0 = workloads.normal((MLP, HID), 0.02, 9).to(dev)
    sets = [lambda wt=(wt0 if i == 0 else wt0.clone()): w8.quantize_weight(wt, "int8", "tensor")
            for i in range(_nsets(nbytes(wt0) * 1.5))]
    ms = _time_rot(sets, 30, torch, stream)
    out["quantize_weight_tensor_12288x3072"] = {"ms": ms, "GB/s": wt0.numel() * 3 / (ms * 1e-3) / 1e9}
    del sets, wt0
    # the weight-only types' two dequantizations alone (12288 x 3072 weight -> bf16)
    wq8, sw8 = w8.quantize_weight(g["w_f32"].to(torch.bfloat16).to(dev), "e4m3", "tensor")
    wgg = w8.q8_0_quantize(g["w_f32"].reshape(-1).to(dev))
    sets_e, sets_g = [], []
    for i in range(_nsets(MLP * HID * 3)):
        wq, blk = wq8.clone(), wgg.clone()
        ye = torch.empty((MLP, HID), dtype=torch.bfloat16, device=dev)
        yg = torch.empty(MLP * HID, dtype=torch.bfloat16, device=dev)
        sets_e.append(lambda wq=wq, ye=ye: w8.dequantize_e4m3_bf16(wq, sw8, out=ye))
        sets_g.append(lambda blk=blk, yg=yg: w8.q8_0_dequantize_bf16(blk, MLP * HID, out=yg))
    ms = _time_rot(sets_e, 30, torch, stream)
    gbs = MLP * HID * 3 / (ms * 1e-3) / 1e9
    out["dequantize_e4m3_bf16_12288x3072"] = {"ms": ms, "GB/s": gbs, "hbm_frac": gbs / hbm}
    ms = _time_rot(sets_g, 30, torch, stream)
    gbs = (wgg.numel() + MLP * HID * 2) / (ms * 1e-3) / 1e9
    out["q8_0_dequantize_bf16_12288x3072"] = {"ms": ms, "GB/s": gbs, "hbm_frac": gbs / hbm}
    del sets_e, sets_g
    # GGUF A8 int and float forward sweeps over M, interleaved so that the
    # few-token points (latency-bound) run before the large products: kernels
    # timed after several long power-capped GEMMs ran up to 25-40 % slower for
    # seconds, so the bandwidth- and latency-bound lines above come first too.
    # The weight is rotated, so that small M streams it from HBM as in a model.
    sweeps = {"int8": {}, "e4m3": {}}
    xg = g["x"].to(dev)
    for M in workloads.GGUF_MS:
        xm0 = xg[:M].contiguous()
        for qt, wqq, sww in (("int8", wq0, sw), ("e4m3", wq0e, swe)):
            sets = []
            for i in range(_nsets(nbytes(xm0, wqq) + M * MLP * 2)):
                xm, wq = xm0.clone(), wqq.clone()
                y = torch.empty((M, MLP), dtype=torch.bfloat16, device=dev)
                ws = torch.empty(w8.workspace_bytes(0, M, MLP, HID), dtype=torch.uint8, device=dev)
                sets.append(lambda xm=xm, wq=wq, y=y, ws=ws, sww=sww: w8.linear_fwd(xm, wq, sww, out=y, ws=ws))
            ms = _time_rot(sets, 30, torch, stream)
            sweeps[qt][str(M)] = {"ms": ms, "TOPS": 2 * M * MLP * HID / ms / 1e9,
                                  "weight_GB/s": MLP * HID / (ms * 1e-3) / 1e9,
                                  "roofline_frac": _gemm_roof_ms(M, MLP, HID, hbm, tc8) / ms}
            del sets
    out["gguf_a8_int_fwd_sweep_N12288_K3072"] = sweeps["int8"]
    out["gguf_a8_float_fwd_sweep_N12288_K3072"] = sweeps["e4m3"]
    # weight-only types (float8, GGUF) on the DiT up-projection: the weight
    # dequantized to bf16 in the workspace, then the bf16 Linear
    tcb = peaks["bf16_tflops"]
    xb0 = workloads.normal((M_TOK, HID), 1.0, 5).to(dev)
    wb0 = g["w_f32"].to(torch.bfloat16).to(dev)
    ops = 2 * M_TOK * MLP * HID   # wq8, sw8, wgg: quantized above from the same weight
    wsz = w8.workspace_bytes(w8.OP_WEIGHT_ONLY_FWD, M_TOK, MLP, HID)
    res = {}
    for name, mk in (("bf16_gemm", lambda xx, ws: (lambda: w8.bf16_linear_fwd(xx, wb0, ws=ws))),
                     ("float8", lambda xx, ws: (lambda: w8.float8_linear_fwd(xx, wq8, sw8, ws=ws))),
                     ("gguf", lambda xx, ws: (lambda: w8.gguf_linear_fwd(xx, wgg, MLP, ws=ws)))):
        sets = []
        for i in range(_nsets(nbytes(xb0) + M_TOK * MLP * 2)):
            sets.append(mk(xb0.clone(), torch.empty(max(wsz, 16), dtype=torch.uint8, device=dev)))
        ms = _time_rot(sets, 20, torch, stream)
        res[name] = {"ms": ms, "TFLOPS": ops / ms / 1e9, "frac_bf16_burst": ops / ms / 1e9 / tcb}
        del sets
    out["weight_only_fwd_4608x12288x3072"] = res
    # their input gradients through the same weight: dY [4608, 12288] -> dX [4608, 3072]
    dy0 = workloads.normal((M_TOK, MLP), 1e-3, 7).to(dev)
    wsd = w8.workspace_bytes(w8.OP_WEIGHT_ONLY_DGRAD, M_TOK, MLP, HID)
    res = {}
    for name, mk in (("bf16_gemm", lambda dd, ws: (lambda: w8.bf16_linear_dgrad(dd, wb0, ws=ws))),
                     ("float8", lambda dd, ws: (lambda: w8.float8_linear_dgrad(dd, wq8, sw8, ws=ws))),
                     ("gguf", lambda dd, ws: (lambda: w8.gguf_linear_dgrad(dd, wgg, HID, ws=ws)))):
        sets = []
        for i in range(_nsets(nbytes(dy0) + M_TOK * HID * 2)):
            sets.append(mk(dy0.clone(), torch.empty(max(wsd, 16), dtype=torch.uint8, device=dev)))
        ms = _time_rot(sets, 20, torch, stream)
        res[name] = {"ms": ms, "TFLOPS": ops / ms / 1e9, "frac_bf16_burst": ops / ms / 1e9 / tcb}
        del sets
    out["weight_only_dgrad_4608x12288x3072"] = res
    del dy0
    del xb0, wb0
    out["peaks"] = {"source": src, "hbm_gbs": hbm, "int8_burst_tops": tc8}
    out["method"] = ("mean over the reps of one CUDA-graph replay (no host launch cost), rotating through "
                     ">= 3x L2 of input/output copies; the fastest of three replays")
    assert w8.device_status() == 0
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-extras", dest="extras", action="store_false")
    ap.add_argument("--case", choices=["up", "down", "dgrad_down", "dgrad_up", "requant", "gguf_m1", "gguf_m64", "svdq",
                                       "requant_e4m3", "gguf_f_m1", "gguf_f_m4608", "svdq_e4m3", "wo_float8",
                                       "wo_gguf", "gguf_m512", "q8_0_quant", "q8_0_dequant", "float_w8a8",
                                       "float_w8a8_int8"],
                    default=None, help="run only one of the step's four quantize+GEMM pairs, or one other kernel "
                                       "of the path (for profiling), no JSON")
    args = ap.parse_args()
    if args.warmup < 3 and not args.case:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.case:
        return run_case(args)
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
