#!/usr/bin/env python
"""Benchmark of the Mamba-2 SSD layer on B200: chunked scan (prefill) and decode step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one ssd_chunk_scan_fwd over the 2.7B-layer workload (batch 4, seqlen 8192, 80
heads x 64, dstate 128, bf16 x/B/C, fp32 initial state): every row of the hot path from the
log-decay cumsums to y and the final state.  The decode row is timed in the same run on its own
workload (1000 ssd_step calls, batch 256, 80 x 64 x 128 fp32 state) and reported under
"decode".  Inputs are synthetic (ssd_inputs, seed 1002 / 1004) and resident in HBM; they are
larger than L2 (126 MB), so no flush is needed between steps.  One JSON line on stdout (rank 0).

With N > 1 (torchrun, one process per GPU) every rank runs the same workload on its own GPU
(the layer shards over batch rows and heads with no exchange): weak scaling, no collective on
the data path; times are the max over ranks.

--impl reference runs the float64 CPU oracle (the plain sequential recurrence) on the host
cores, each step a bounded sample of the same workload (batch row 0: 80 heads x 64 channels
x 8192 tokens), and reports the same metric.

--profile scan|decode|backward runs only W + K calls of that workload (backward: the gradients
at the 130M-layer shape) and prints nothing else: the command the launch lists and ncu captures
under profiles/ were taken with.

--glue times the block steps around the layer at the 2.7B shape (short convolution + SiLU over
the 5376 x/B/C channels, dt softplus, SiLU output gate over y) and prints one JSON line with
each kernel's HBM bytes, time and bandwidth against the measured copy peak.

--selective times the selective scan with a per-state transition (the first Mamba
generation's layer) on the same x and y as the scan workload (batch 4, seqlen 8192, 5120
channels) with 16 states per channel, and prints one JSON line: tokens/s, the ex2 rate against
the SFU peak that bounds it, and its HBM bandwidth.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import ssd_inputs  # noqa: E402

METRIC = "SSD scan tokens/s per layer at 2.7B shape, % roofline; decode steps/s"
SCAN_CFG = 2
DECODE_CFG = 4


def scan_bytes(c, y_bytes=4):
    """Algorithmic bytes of one scan: every input read once, y (float32) written once,
    init/final state."""
    tok = c["batch"] * c["seqlen"]
    es = 2 if c["io"] == "bf16" else 4
    x = tok * c["nheads"] * c["headdim"] * es
    y = tok * c["nheads"] * c["headdim"] * y_bytes
    bc = 2 * tok * c["ngroups"] * c["dstate"] * es
    dt = tok * c["nheads"] * 4
    st = c["batch"] * c["nheads"] * c["headdim"] * c["dstate"] * 4
    init = st if c["init"] != "zeros" else 0
    return x + y + bc + dt + 2 * c["nheads"] * 4 + init + st


def scan_flops(c):
    """Causal tensor-core work per token: G(Q+1)N + H[(Q+1)P + 4NP]."""
    Q, N, P, H, G = c["chunk"], c["dstate"], c["headdim"], c["nheads"], c["ngroups"]
    return c["batch"] * c["seqlen"] * (G * (Q + 1) * N + H * ((Q + 1) * P + 4 * N * P))


def step_bytes(c, y_bytes=4):
    es = 2
    st = c["batch"] * c["nheads"] * c["headdim"] * c["dstate"] * 4
    x = c["batch"] * c["nheads"] * c["headdim"] * es
    y = c["batch"] * c["nheads"] * c["headdim"] * y_bytes
    bc = 2 * c["batch"] * c["ngroups"] * c["dstate"] * es
    return 2 * st + x + y + bc + c["batch"] * c["nheads"] * 4 + 2 * c["nheads"] * 4


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per scan call and per decode step,
# from ncu captures of `python bench.py --profile ...` (profiles/), each with the hash of the
# device-code headers of its kernels (KERNEL_SOURCES[kind]) it was taken on: reported only while
# those sources match.
KERNEL_SOURCES = {"scan": ("ssd_common.cuh", "tc_prims.cuh", "tc_kernels.cuh"),
                  "decode": ("ssd_common.cuh", "step_kernels.cuh")}
# scan: from the 4 x 2048-token capture, per-block reads x4 plus the initial state, and y x4 plus
# the final state less the y still dirty in L2 when the kernel exits (50.0 MB; read 373.8 MB,
# write 631.6 MB; profiles/scan_walk_2p7b_ncu.md)
MEASURED_TRAFFIC = {"scan": (1005360384, "9d08bbd559aa2e21"),
                    "decode": (1290920192, "98855f81fa05bee0")}


def kernel_source_hash(kind):
    import hashlib
    d = os.path.join(ROOT, "mamba_ssd_scan_03_b200", "csrc")
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kind]:
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def measured_traffic(kind):
    nbytes, src = MEASURED_TRAFFIC[kind]
    return nbytes if nbytes is not None and src == kernel_source_hash(kind) else None


# B200 HBM3e bandwidth from the spec sheet (8 TB/s): a second denominator next to the measured
# copy bandwidth, which a read-heavy kernel can exceed (a fraction above 1.0 against the measured
# copy only says that the copy is not a ceiling).
SPEC_HBM_GBS = 8000.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


class Clocks:
    """nvidia-smi sampling during the timed region (started before, stopped after)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        time.sleep(0.25)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [v.strip() for v in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def to_dev(a, bf16, dev):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if bf16:
        t = t.view(torch.bfloat16)
    return t.to(dev)


def device_scan_inputs(c, dev, seed):
    """Inputs of a scan workload drawn on the device with a seeded torch generator, with the
    distributions of the workload recipe (x ~ N(0,1); dt = softplus(N(-2, 0.5)); A = -exp(U(ln 1,
    ln 16)); B, C ~ N(0,1)/sqrt(N); D ~ N(0,1); init N(0, 0.1) or zeros).  Used only for timing
    keys, whose kernels' time does not depend on the values; the headline workload and every
    parity test use ssd_inputs."""
    import torch
    g = torch.Generator(device=dev).manual_seed(seed)
    Bt, L, H, P, G, N = (c["batch"], c["seqlen"], c["nheads"], c["headdim"], c["ngroups"],
                         c["dstate"])
    rn = lambda *shape: torch.randn(*shape, generator=g, device=dev)  # noqa: E731
    t = {"x": rn(Bt, L, H, P).to(torch.bfloat16),
         "dt": torch.nn.functional.softplus(-2.0 + 0.5 * rn(Bt, L, H)),
         "A": -torch.exp(torch.rand(H, generator=g, device=dev) * np.log(16.0)),
         "B": (rn(Bt, L, G, N) / np.sqrt(N)).to(torch.bfloat16),
         "C": (rn(Bt, L, G, N) / np.sqrt(N)).to(torch.bfloat16),
         "D": rn(H),
         "init": 0.1 * rn(Bt, H, P, N) if c.get("init") == "normal0.1" else None}
    return t


def timed_after_flush(once, flush, steps):
    """Device time of `steps` calls of once(), each right behind an L2 flush (a write of
    `flush`), timed with CUDA events.  Every step is queued before the first is waited for, so
    the device runs flush, call, flush, call ... back to back and the host's time to validate
    and launch a call (which a small call does not hide) is not counted; eight more flushes
    ahead of the first give the host its lead."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for _ in range(8):
        flush.zero_()
    for e0, e1 in evs:
        flush.zero_()
        e0.record()
        once()
        e1.record()
    torch.cuda.synchronize()
    return [e0.elapsed_time(e1) for e0, e1 in evs]


def time_scan(c, dev, seed, y_dtype, steps, warmup, hbm):
    """Mean time of one ssd_chunk_scan_fwd over a device-seeded workload, each call timed alone
    with CUDA events after an L2 flush (a 256 MB write), and its roofline figures."""
    import torch
    import mamba_ssd_scan_03_b200 as ssd
    t = device_scan_inputs(c, dev, seed)
    y = torch.empty(t["x"].shape, dtype=y_dtype, device=dev)
    fin = torch.empty((c["batch"], c["nheads"], c["headdim"], c["dstate"]), dtype=torch.float32,
                      device=dev)
    ws = torch.empty(max(1, ssd.workspace_size(c["batch"], c["seqlen"], c["nheads"], c["headdim"],
                                               c["dstate"], c["ngroups"], c["chunk"])),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def once():
        ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], c["chunk"],
                           init_state=t["init"], workspace=ws, out=y, final_out=fin)

    for _ in range(warmup):
        once()
    times = timed_after_flush(once, flush, steps)
    assert ssd.device_status() == 0
    ms = statistics.mean(times)
    nbytes = scan_bytes(c, 2 if y_dtype == torch.bfloat16 else 4)
    gbs = nbytes / (ms * 1e-3) / 1e9
    tok = c["batch"] * c["seqlen"]
    info = ssd.plan_info(c["batch"], c["seqlen"], c["nheads"], c["headdim"], c["dstate"],
                         c["ngroups"], c["chunk"])
    del t, y, fin, ws, flush
    torch.cuda.empty_cache()
    return {"ms": round(ms, 5), "tokens_per_s": round(tok / (ms * 1e-3), 1),
            "ns_per_token": round(ms * 1e6 / tok, 4), "algorithmic_bytes": nbytes,
            "achieved_gbs": round(gbs, 1), "frac": round(gbs / hbm, 4),
            "frac_spec": round(gbs / SPEC_HBM_GBS, 4),
            "y_dtype": "bf16" if y_dtype == torch.bfloat16 else "f32", "plan": info,
            "steps": steps, "l2": "flushed before every timed call (256 MB write)"}


def time_backward(c, dev, seed, steps, warmup, hbm):
    """Mean time of one ssd_chunk_scan_bwd (all seven gradients) over a device-seeded workload,
    each call timed alone after an L2 flush."""
    import torch
    import mamba_ssd_scan_03_b200 as ssd
    t = device_scan_inputs(c, dev, seed)
    g = torch.Generator(device=dev).manual_seed(seed + 7)
    dy = torch.randn(t["x"].shape, generator=g, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ws = torch.empty(max(1, ssd.load().ssd_chunk_scan_bwd_workspace_size(
        c["batch"], c["seqlen"], c["nheads"], c["headdim"], c["dstate"], c["ngroups"], 1)),
        dtype=torch.uint8, device=dev)

    def once():
        ssd.chunk_scan_bwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], dy,
                           init_state=t["init"], workspace=ws)

    for _ in range(warmup):
        once()
    times = timed_after_flush(once, flush, steps)
    assert ssd.device_status() == 0
    ms = statistics.mean(times)
    tok = c["batch"] * c["seqlen"]
    del t, dy, flush, ws
    torch.cuda.empty_cache()
    flops = 2 * backward_fmas(c)
    achieved = flops / (ms * 1e-3) / 1e12
    return {"ms": round(ms, 5), "tokens_per_s": round(tok / (ms * 1e-3), 1),
            "kernels": "float32 CUDA cores (cumsum, chunk states, state pass, adjoint summaries, "
                       "adjoint pass, per-chunk gradients, group and head sums: 8 launches)",
            "roofline": {"bound": "fp32 fma", "flops": flops, "achieved_tflops": round(achieved, 2),
                         "peak_tflops": round(FP32_TFLOPS, 1), "frac": round(achieved / FP32_TFLOPS, 4),
                         "peak_src": "148 SMs x 128 FMA/clk x 2 flops x 1965 MHz (nominal)"},
            "steps": steps, "l2": "flushed before every timed call (256 MB write)"}


# float32 FMAs the backward kernels perform (chunks of 64 tokens): the chunk and adjoint summaries
# (P N Q each), and per chunk the C.B and x.dy tables, the per-token products (M^T dy over
# tau >= t: about Q/2 + 2 terms, B R, C H) and the dB / dC products (N2^T C and K2 B over about
# Q/2 + 2 terms, x R, dy H), as the kernels tile them
FP32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def backward_fmas(c):
    Q = 64
    P, N = c["headdim"], c["dstate"]
    half = Q // 2 + 2
    per_chunk = (2 * P * N * Q + Q * Q * N + Q * Q * P + Q * P * half + 2 * Q * P * N +
                 2 * Q * N * half + 2 * Q * N * P)
    nc = (c["seqlen"] + Q - 1) // Q
    return per_chunk * c["batch"] * nc * c["nheads"]


def scan_extras(dev, hbm, steps=5, warmup=3):
    """The other scan workloads: the 130M-layer and million-token shapes, the 2.7B layer with
    bf16 y, and the length sweep at the 2.7B layer's heads (batch 1)."""
    import torch
    out = {}
    c1 = ssd_inputs.resolve(1)
    out[c1["name"]] = time_scan(c1, dev, 2101, torch.float32, steps, warmup, hbm)
    c3 = ssd_inputs.resolve(3)
    out[c3["name"]] = time_scan(c3, dev, 2103, torch.float32, steps, warmup, hbm)
    c2 = ssd_inputs.resolve(SCAN_CFG)
    out[c2["name"] + "_bf16y"] = time_scan(c2, dev, 2102, torch.bfloat16, steps, warmup, hbm)
    out[c1["name"] + "_backward"] = time_backward(c1, dev, 2111, steps, warmup, hbm)
    sweep = []
    for L in (4096, 32768, 131072, 524288):
        c = dict(c2, batch=1, seqlen=L, init="zeros", name=f"sweep_{L}")
        r = time_scan(c, dev, 2200 + L % 997, torch.float32, steps, warmup, hbm)
        r["seqlen"] = L
        sweep.append(r)
    return out, sweep


def run_ours(args):
    import torch
    import mamba_ssd_scan_03_b200 as ssd

    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", torch.cuda.current_device())
    hbm, tflops, peak_src = peaks()

    # ---------------- chunked scan (the headline) ----------------
    inp = ssd_inputs.make_scan_inputs(SCAN_CFG)
    c = inp["cfg"]
    names = ("x", "dt", "A", "B", "C", "D", "init")
    t = {k: to_dev(inp[k], k in ("x", "B", "C"), dev) for k in names}
    y = torch.empty(t["x"].shape, dtype=torch.float32, device=dev)  # y in float32
    fin = torch.empty_like(t["init"])
    ws = torch.empty(ssd.workspace_size(c["batch"], c["seqlen"], c["nheads"], c["headdim"],
                                        c["dstate"], c["ngroups"], c["chunk"]),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def scan_once():
        ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], c["chunk"],
                           init_state=t["init"], workspace=ws, out=y, final_out=fin)

    for _ in range(args.warmup):
        scan_once()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    barrier(world)
    torch.cuda.synchronize()
    with Clocks(local) as clk:
        ev[0].record(stream)
        for i in range(args.steps):
            scan_once()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), world)
    status = ssd.device_status()
    ms_per_step = total_ms / args.steps
    tokens = c["batch"] * c["seqlen"]
    value = world * tokens * args.steps / (total_ms / 1e3)
    nbytes = scan_bytes(c)
    achieved = nbytes / (statistics.mean(per) / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4),
            "traffic": args.traffic if args.traffic is not None else measured_traffic("scan"),
            "kernel": "ssd_chunk_scan_fwd (one call)",
            "algorithmic_bytes": nbytes, "flops": scan_flops(c),
            "peak_source": peak_src, "frac_spec": round(achieved / SPEC_HBM_GBS, 4),
            "spec_gbs": SPEC_HBM_GBS,
            "flop_frac": round(scan_flops(c) / (statistics.mean(per) / 1e3) / 1e12 / tflops, 4)}
    plan = ssd.plan_info(c["batch"], c["seqlen"], c["nheads"], c["headdim"], c["dstate"],
                         c["ngroups"], c["chunk"])

    # ---------------- e2e through the public API with host buffers ----------------
    pinned = {k: t[k].cpu().pin_memory() for k in names}
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    f_host = torch.empty(fin.shape, dtype=fin.dtype).pin_memory()
    dbuf = {k: torch.empty_like(t[k]) for k in names}
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = y_host.numel() * y_host.element_size() + f_host.numel() * f_host.element_size()

    # Pipelined over batch rows on three streams: row r's inputs go up while row r - 1 is
    # scanned and row r - 2's y and final state come down (every row's copies and scan are
    # inside the step; a buffer is reused only after its previous reader is done).
    s_up, s_run, s_down = (torch.cuda.Stream(device=dev) for _ in range(3))
    rows = c["batch"]
    row_names = [k for k in names if k not in ("A", "D")]
    ev_up = [torch.cuda.Event() for _ in range(rows)]
    ev_run = [torch.cuda.Event() for _ in range(rows)]
    ev_down = [torch.cuda.Event() for _ in range(rows)]
    ev_shared = torch.cuda.Event()
    started = [False]
    ws_row = torch.empty(max(1, ssd.workspace_size(1, c["seqlen"], c["nheads"], c["headdim"],
                                                   c["dstate"], c["ngroups"], c["chunk"])),
                         dtype=torch.uint8, device=dev)

    def e2e_once():
        with torch.cuda.stream(s_up):
            if started[0]:
                s_up.wait_event(ev_run[rows - 1])  # the previous step's scans have read A and D
            for k in ("A", "D"):
                dbuf[k].copy_(pinned[k], non_blocking=True)
            ev_shared.record(s_up)
        for r in range(rows):
            with torch.cuda.stream(s_up):
                if started[0]:
                    s_up.wait_event(ev_run[r])  # the previous step's scan of row r has read it
                for k in row_names:
                    dbuf[k][r].copy_(pinned[k][r], non_blocking=True)
                ev_up[r].record(s_up)
            with torch.cuda.stream(s_run):
                s_run.wait_event(ev_up[r])
                s_run.wait_event(ev_shared)
                if started[0]:
                    s_run.wait_event(ev_down[r])  # the previous step's y of row r is down
                sl = slice(r, r + 1)
                ssd.chunk_scan_fwd(dbuf["x"][sl], dbuf["dt"][sl], dbuf["A"], dbuf["B"][sl],
                                   dbuf["C"][sl], dbuf["D"], c["chunk"],
                                   init_state=dbuf["init"][sl], workspace=ws_row, out=y[sl],
                                   final_out=fin[sl])
                ev_run[r].record(s_run)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_run[r])
                y_host[r].copy_(y[r], non_blocking=True)
                f_host[r].copy_(fin[r], non_blocking=True)
                ev_down[r].record(s_down)
        started[0] = True

    e2e_steps = max(1, min(args.steps, 5))
    for _ in range(2):
        e2e_once()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    for _ in range(e2e_steps):
        e2e_once()
    s_down.wait_event(ev_run[rows - 1])
    e1.record(s_down)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e = {"value": world * tokens * e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
           "pipeline": "per batch row: H2D, ssd_chunk_scan_fwd and D2H on three streams"}
    del pinned, dbuf

    # ---------------- decode workload: 1000 ssd_step calls ----------------
    dec = ssd_inputs.make_decode_inputs(DECODE_CFG)
    dc = dec["cfg"]
    st = to_dev(dec["state"], False, dev)
    A4, D4 = to_dev(dec["A"], False, dev), to_dev(dec["D"], False, dev)
    n_dec_inputs = 8
    steps_in = []
    for k in range(n_dec_inputs):  # distinct per-step inputs, cycled
        s = ssd_inputs.decode_step_inputs(dec, k)
        steps_in.append({n: to_dev(s[n], n != "dt", dev) for n in ("x", "dt", "B", "C")})
    ydec = torch.empty(steps_in[0]["x"].shape, dtype=torch.float32, device=dev)

    def dec_once(k):
        s = steps_in[k % n_dec_inputs]
        ssd.step(st, s["x"], s["dt"], A4, s["B"], s["C"], D4, out=ydec)

    for k in range(max(3, args.warmup)):
        dec_once(k)
    torch.cuda.synchronize()
    n_dec = dc["decode_steps"]
    barrier(world)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local) as clk_dec:
        d0.record(stream)
        for k in range(n_dec):
            dec_once(k)
        d1.record(stream)
        torch.cuda.synchronize()
    dec_ms = max_over_ranks(d0.elapsed_time(d1), world)
    sb = step_bytes(dc)
    dec_ach = sb / (dec_ms / n_dec / 1e3) / 1e9
    decode = {"metric": "decode steps/s", "value": world * n_dec / (dec_ms / 1e3),
              "unit": "steps/s", "tokens_per_s": world * dc["batch"] * n_dec / (dec_ms / 1e3),
              "steps": n_dec, "ms_per_step": dec_ms / n_dec,
              "config": {"workload": dc["name"], "batch": dc["batch"], "nheads": dc["nheads"],
                         "headdim": dc["headdim"], "dstate": dc["dstate"]},
              "roofline": {"bound": "hbm", "achieved": round(dec_ach, 1), "peak": hbm,
                           "unit": "GB/s", "frac": round(dec_ach / hbm, 4),
                           "frac_spec": round(dec_ach / SPEC_HBM_GBS, 4),
                           "traffic": (args.decode_traffic if args.decode_traffic is not None
                                       else measured_traffic("decode")),
                           "kernel": "step_n128_kernel",
                           "algorithmic_bytes": sb, "peak_source": peak_src},
              "clocks": clk_dec.summary(), "gpu_launches": n_dec}

    # ---------------- the other scan workloads (secondary keys) ----------------
    extras, sweep = (None, None) if args.no_extras else scan_extras(dev, hbm)

    # ---------------- CPU baseline: the float64 oracle on a bounded sample -----------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp, args.cpu_rows)

    out = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic",
           "config": {"workload": c["name"], "batch": c["batch"], "seqlen": c["seqlen"],
                      "nheads": c["nheads"], "headdim": c["headdim"], "dstate": c["dstate"],
                      "ngroups": c["ngroups"], "chunk": c["chunk"], "init_state": c["init"],
                      "parallelism": f"replicas{world}" if world > 1 else "single",
                      "y_dtype": "f32",
                      "l2": "inputs and outputs larger than L2 (1055 MB per step > 126 MB), "
                            "no flush"},
           "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk.summary(),
           "gpu_launches": plan["launches"] * args.steps, "plan": plan, "decode": decode,
           "scan_workloads": extras, "length_sweep": sweep, "device_status": status,
           "path": "tcgen05" if ssd.path(c["batch"], c["seqlen"], c["nheads"], c["headdim"],
                                        c["dstate"], c["ngroups"], c["chunk"]) == 1 else "simt"}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def cpu_baseline(inp, rows=1):
    """The oracle as it stands, all host cores, on batch rows [0, rows) of the workload."""
    import oracle
    c = inp["cfg"]
    H, P, L = c["nheads"], c["headdim"], c["seqlen"]
    b = np.repeat(np.arange(rows), H * P)
    h = np.tile(np.repeat(np.arange(H), P), rows)
    p = np.tile(np.arange(P), rows * H)
    ids = oracle.chain_ids(b, h, p, H, P)
    init = None if inp["init"] is None else inp["init"][b, h, p]
    cores = oracle.default_threads()
    t0 = time.perf_counter()
    oracle.scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], init=init,
                chains=ids, nthreads=cores)
    sec = time.perf_counter() - t0
    return {"value": rows * L / sec, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"batch rows 0..{rows - 1} of {c['batch']} (all {H} heads x {P} channels, "
                      f"{L} tokens), float64 sequential recurrence, {sec:.2f} s"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = ssd_inputs.make_scan_inputs(SCAN_CFG)
    c = inp["cfg"]
    for _ in range(args.warmup):
        cpu_baseline(inp, 1)
    runs = [cpu_baseline(inp, 1) for _ in range(args.steps)]
    tok_s = statistics.mean(r["value"] for r in runs)
    sec = c["seqlen"] / tok_s
    out = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": c["name"], "batch": c["batch"], "seqlen": c["seqlen"],
                      "nheads": c["nheads"], "headdim": c["headdim"], "dstate": c["dstate"],
                      "ngroups": c["ngroups"], "chunk": c["chunk"]},
           "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "kind": "oracle",
                            "cores": runs[0]["cores"], "sample": runs[0]["sample"]},
           "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_profile(args):
    """W + K calls of one workload and nothing else (for ncu launch lists and captures)."""
    import torch
    import mamba_ssd_scan_03_b200 as ssd
    dev = torch.device("cuda", 0)
    if args.profile == "scan":
        inp = ssd_inputs.make_scan_inputs(SCAN_CFG, seqlen=args.seqlen)
        c = inp["cfg"]
        t = {k: to_dev(inp[k], k in ("x", "B", "C"), dev)
             for k in ("x", "dt", "A", "B", "C", "D", "init")}
        for _ in range(args.warmup + args.steps):
            ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], c["chunk"],
                               init_state=t["init"])
    elif args.profile == "backward":
        c = ssd_inputs.resolve(1)  # the 130M-layer shape, float32 dy
        t = device_scan_inputs(c, dev, 1101)
        g = torch.Generator(device=dev).manual_seed(1108)
        dy = torch.randn(t["x"].shape, generator=g, device=dev)
        for _ in range(args.warmup + args.steps):
            ssd.chunk_scan_bwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], dy,
                               init_state=t["init"])
    else:
        dec = ssd_inputs.make_decode_inputs(DECODE_CFG)
        st = to_dev(dec["state"], False, dev)
        A4, D4 = to_dev(dec["A"], False, dev), to_dev(dec["D"], False, dev)
        s = ssd_inputs.decode_step_inputs(dec, 0)
        t = {n: to_dev(s[n], n != "dt", dev) for n in ("x", "dt", "B", "C")}
        for _ in range(args.warmup + args.steps):
            ssd.step(st, t["x"], t["dt"], A4, t["B"], t["C"], D4)
    torch.cuda.synchronize()
    assert ssd.device_status() == 0


def run_glue(args):
    """CUDA-event timing of the three block-step kernels (inputs seeded on the device)."""
    import torch
    import mamba_ssd_scan_03_b200 as ssd
    dev = torch.device("cuda", 0)
    c = ssd_inputs.resolve(SCAN_CFG)
    Bt, L, H, P, G, N = (c["batch"], c["seqlen"], c["nheads"], c["headdim"], c["ngroups"],
                         c["dstate"])
    cdim, K = H * P + 2 * G * N, 4
    gen = torch.Generator(device=dev).manual_seed(2002)
    rnd = lambda *shape, dtype=torch.float32: torch.randn(*shape, generator=gen, device=dev,
                                                          dtype=dtype)
    u = rnd(Bt, L, cdim, dtype=torch.bfloat16)
    w, cb = rnd(cdim, K) / 2, rnd(cdim) / 10
    conv_out = torch.empty_like(u)
    raw, dtb = rnd(Bt, L, H), rnd(H) - 4
    dt = torch.empty_like(raw)
    y, z = rnd(Bt, L, H, P), rnd(Bt, L, H, P, dtype=torch.bfloat16)
    gate_out = torch.empty_like(z)
    ntok = Bt * L
    cases = {
        "conv_silu": (lambda: ssd.conv_silu(u, w, cb, out=conv_out), ntok * cdim * 4 + cdim * 20,
                      f"[{Bt},{L},{cdim}] bf16, width {K}"),
        "dt_softplus": (lambda: ssd.dt_softplus(raw, dtb, out=dt), ntok * H * 8 + H * 4,
                        f"[{Bt},{L},{H}] f32"),
        "gate_silu": (lambda: ssd.gate_silu(y, z, out=gate_out), ntok * H * P * 8,
                      f"[{Bt},{L},{H},{P}] y f32, z and out bf16"),
    }
    hbm, _, src = peaks()
    res = {}
    for name, (fn, nbytes, shape) in cases.items():
        for _ in range(args.warmup):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(args.steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[name] = {"shape": shape, "bytes": nbytes, "ms": round(ms, 5),
                     "GB/s": round(gbs, 1), "frac": round(gbs / hbm, 4),
                     "frac_spec": round(gbs / SPEC_HBM_GBS, 4)}
    assert ssd.device_status() == 0
    print(json.dumps({"glue": res, "peak_hbm_gbs": hbm, "peak_src": src,
                      "steps": args.steps, "warmup": args.warmup}), flush=True)


# The selective scan needs one exp per (token, channel, state) and is bound by the SFU (MUFU)
# ex2 rate: 16 results per clock per SM (4 per SM sub-partition) x 148 SMs x the 1965 MHz
# maximum SM clock.
SFU_EX2_PER_CLK_SM = 16
N_SM = 148
SM_MAX_MHZ = 1965.0


def run_selective(args):
    import torch
    import mamba_ssd_scan_03_b200 as ssd
    dev = torch.device("cuda", 0)
    inp = ssd_inputs.make_selective_inputs(1)
    c = inp["cfg"]
    Bt, L, dim, N, G = c["batch"], c["seqlen"], c["dim"], c["dstate"], c["ngroups"]
    t = {k: to_dev(inp[k], k in ("x", "B", "C"), dev) for k in ("x", "dt", "A", "B", "C", "D")}
    y = torch.empty((Bt, L, dim), dtype=torch.float32, device=dev)
    fin = torch.empty((Bt, dim, N), dtype=torch.float32, device=dev)

    def once():
        ssd.selective_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], None, out=y,
                               final_out=fin)

    for _ in range(args.warmup):
        once()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(0) as clk:
        torch.cuda.synchronize()
        e0.record()
        for _ in range(args.steps):
            once()
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    assert ssd.device_status() == 0
    ntok = Bt * L
    exps = ntok * dim * N
    peak = SFU_EX2_PER_CLK_SM * N_SM * SM_MAX_MHZ * 1e6
    nbytes = ntok * dim * (2 + 4 + 4) + 2 * ntok * G * N * 2 + Bt * dim * N * 4 + dim * N * 4
    hbm, _, src = peaks()
    out = {"metric": "selective scan tokens/s (16 states per channel)",
           "value": round(ntok / (ms * 1e-3), 1), "unit": "tokens/s", "ms_per_call": round(ms, 4),
           "steps": args.steps, "warmup": args.warmup, "dtype": "f32", "data": "synthetic",
           "config": {"workload": c["name"], "batch": Bt, "seqlen": L, "dim": dim, "dstate": N,
                      "ngroups": G, "io": c["io"], "y_dtype": "f32",
                      "l2": "inputs larger than L2"},
           "roofline": {"bound": "alu", "achieved": round(exps / (ms * 1e-3) / 1e12, 4),
                        "peak": round(peak / 1e12, 4), "unit": "Tex2/s",
                        "frac": round(exps / (ms * 1e-3) / peak, 4),
                        "peak_src": "16 ex2/clk/SM x 148 SMs x 1965 MHz"},
           "hbm": {"bytes": nbytes, "GB/s": round(nbytes / (ms * 1e-3) / 1e9, 1),
                   "frac": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4), "peak_src": src},
           "gpu_launches": args.steps, "clocks": clk.summary()}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=1)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the secondary scan workloads and the length sweep")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per scan call (null when not measured)")
    ap.add_argument("--decode-traffic", type=float, default=None)
    ap.add_argument("--profile", choices=["scan", "decode", "backward"], default=None)
    ap.add_argument("--glue", action="store_true")
    ap.add_argument("--selective", action="store_true")
    ap.add_argument("--seqlen", type=int, default=None,
                    help="with --profile scan: a shorter sequence (smaller capture)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.glue:
        run_glue(args)
    elif args.selective:
        run_selective(args)
    elif args.profile:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
