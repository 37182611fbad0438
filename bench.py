"""Benchmark of the quantized-state decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: GDN serving scale -- batch 512 requests x 32 value heads (16 key
heads), d = 128, 6-bit nominal budget with per-head widths {4, 6, 8} and 5 %
FP16 pivot heads, state warmed up by 64 unquantized steps with 2 % outlier
columns x20 (synthetic, seeded). One step = one decode step of every
(request, head) state tile = one launch of the fused kernel.

Prints one JSON line (rank 0). ``value`` is (request*head)-steps/s over all
ranks with inputs resident in HBM; ``e2e`` is the same through the C ABI's
host-buffer step (sq_decode_step_host): the step's activations are copied
from pinned host memory inside the call, overlapping the previous step, and
o is written into pinned host memory, all inside the timed region; ``roofline`` compares the kernel's algorithmic
state bytes (codes + row scales + pivots, read and written once) per launch
with the measured HBM copy bandwidth; ``cpu_baseline`` times the CPU oracle
on a bounded sample of the same workload.

Multi-GPU: each rank owns its own 512 requests (requests are independent;
no collective on the data path) -> weak scaling; timing is the max over
ranks. ``--impl reference`` times the CPU oracle as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-state decode (request·head)-steps/s; achieved HBM GB/s vs B200 peak"
UNIT = "(request*head)-steps/s"
CONFIG_ID = 3
# single-layer step workloads: the serving scale (the headline) and the
# three smaller configurations, whose pools fit the 126 MB L2
STEP_WORKLOADS = {"serving": 3, "plumbing": 0, "gdn_layer": 1, "kda_layer": 2}
FALLBACK_HBM_GBS = 6650.0
DATASHEET_HBM_GBS = 8000.0
L2_BYTES = 126 * 1024 * 1024


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def workload_config(w, pool_bytes=None):
    c = w.cfg
    if c.gate_kind == 0:
        gate = "GDN (one gate per head)"
        units = "per-head"
    else:
        gate = "KDA (one gate per key channel)"
        units = "per-key-row"
    widths = f"{units} {{{','.join(str(b) for b in c.widths)}}}, {c.nominal_bits}-bit nominal"
    if c.pivot_frac:
        widths += f", {round(100 * c.pivot_frac)}% FP16 pivot {'heads' if c.gate_kind == 0 else 'rows'}"
    cfg = {"workload": c.name, "batch_per_gpu": w.B, "h_v": c.h_v, "h_k": c.h_k, "d": c.d, "gate": gate,
           "widths": widths}
    if c.warmup_steps:
        cfg["warmup"] = f"{c.warmup_steps} unquantized steps, {round(100 * c.outlier_frac)}% outlier columns x20"
    if pool_bytes is not None:
        mb = pool_bytes / 1e6
        if pool_bytes > L2_BYTES:
            cfg["l2"] = f"state {mb:.0f} MB > 126 MB L2 (no flush); 8 rotating input sets"
        else:
            cfg["l2"] = (f"L2-resident: state {mb:.1f} MB < 126 MB L2, so the step runs from L2 "
                         f"(no HBM roofline claim; GB/s below are algorithmic bytes over time)")
    return cfg


# ------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9 and f[1].replace(".", "").isdigit():
                    rows.append(f)
        finally:
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm = [float(r[1]) for r in rows]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "samples": len(rows),
                "reasons": sorted(reasons)}


# --------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank, cid=CONFIG_ID):
    import torch
    from quantized_linear_attention_sq_b200 import _abi, build, shards, synth
    from quantized_linear_attention_sq_b200.state import StatePool

    torch.cuda.set_device(local_rank)
    build.build()
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    w = synth.workload(cid, seed=shards.rank_seed(args.seed, rank))   # each rank: its own requests
    c = w.cfg
    cal = w.calib()
    B = c.batch
    dev = torch.device("cuda", local_rank)

    def make(fmt):
        return StatePool(B, c.h_v, c.h_k, c.d, c.gate_kind, fmt, cal.unit_bits, cal.pivot, cal.col_scale,
                         cal.row_impact)

    # initial state: S0, 64 unquantized warm-up steps on the GPU (FP32 kernel), outliers, quantize
    S = torch.from_numpy(w.initial_state()).to(dev)
    fp = make(_abi.SQ_FMT_FP32)
    o = torch.empty((B, c.h_v, c.d), device=dev)
    for t in range(-c.warmup_steps, 0):
        q, k, v, beta, g = (torch.from_numpy(x).to(dev) for x in w.step_inputs(t))
        fp.decode_step(S, q, k, v, beta, g, o)
    if c.outlier_frac:
        S *= torch.from_numpy(w.outlier_mask()).to(dev)[None, :, None, :]
    sp = make(_abi.SQ_FMT_PACKED)
    pool = sp.new_pool()
    clip = clip_fraction(S, cal, c)
    sp.quantize_state(pool, S)
    torch.cuda.synchronize()
    setup_status = sp.get_status()
    sp.exact_count(clear=True)
    NI = 8
    host_inputs = [w.step_inputs(t) for t in range(NI)]
    dev_inputs = [[torch.from_numpy(x).to(dev) for x in xs] for xs in host_inputs]
    stream = torch.cuda.current_stream()
    if args.profile:
        # profiling mode: the same prepared state, N packed steps, no timing
        for i in range(args.profile):
            sp.decode_step(pool, *dev_inputs[i % NI], o)
        torch.cuda.synchronize()
        print(json.dumps({"profile_steps": args.profile, "status_after_setup": setup_status,
                          "status_bits": sp.get_status(), "launch": sp.launch_plan(),
                          "exact_sum_columns": sp.exact_count()}), flush=True)
        sp.close()
        fp.close()
        return

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(x):
        return shards.max_over_ranks(x, dist, dev)

    # ---- device-resident timing (per-launch events on the launching stream)
    def timed_device(spool, pl, K, W):
        for i in range(W):
            spool.decode_step(pl, *dev_inputs[i % NI], o)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        n0 = spool.launches()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(K):
            ev[i][0].record(stream)
            spool.decode_step(pl, *dev_inputs[i % NI], o)
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        launches = spool.launches() - n0
        per = [a.elapsed_time(b) for a, b in ev]
        return t0.elapsed_time(t1), per, launches

    props = torch.cuda.get_device_properties(local_rank)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local_rank)
    with ClockSampler(gpu_id) as clk:
        total_ms, per_ms, launches = timed_device(sp, pool, args.steps, args.warmup)
    clocks = clk.summary()
    total_ms = max_over_ranks(total_ms)
    kern_ms = statistics.mean(per_ms)
    # ---- end to end through the public API: pinned host activations in, o out
    # (sq_decode_step_host: the step's inputs are copied from page-locked host
    # memory inside the call, overlapping the previous step; o is written
    # into page-locked host memory by the kernel)
    pinned = [[torch.from_numpy(x).pin_memory() for x in xs] for xs in host_inputs]
    o_host = torch.empty((B, c.h_v, c.d), dtype=torch.float32).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in pinned[0])
    d2h = o_host.numel() * o_host.element_size()
    for i in range(args.warmup):
        sp.decode_step_host(pool, *pinned[i % NI], o_host)
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        sp.decode_step_host(pool, *pinned[i % NI], o_host)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    st_bits = sp.get_status()
    exact_cols = sp.exact_count() / (2 * (args.steps + args.warmup))
    # ---- FP32-state step on the same workload (unquantized comparison)
    fp_pool = S  # warmed-up fp32 state, same requests
    fp_total, fp_per, _ = timed_device(fp, fp_pool, max(4, args.steps // 4), args.warmup)
    fp_total = max_over_ranks(fp_total)
    rep = sp.report
    frep = fp.report
    units = B * c.h_v
    value = shards.job_rate(units, args.steps, total_ms, world)
    bytes_launch = B * rep["state_bytes_per_step"]
    peak, peak_kind = peaks()
    achieved = bytes_launch / (kern_ms / 1e3) / 1e9
    fp_bytes = B * frep["state_bytes_per_step"]
    fp_kern = statistics.mean(fp_per)
    l2_resident = B * rep["slot_bytes"] <= L2_BYTES
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded, no dataset)",
        "config": workload_config(w, B * rep["slot_bytes"]),
        "e2e": {"value": shards.job_rate(units, args.steps, e2e_ms, world), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "roofline": {"bound": "l2" if l2_resident else "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "frac_of_datasheet_8tbs": achieved / DATASHEET_HBM_GBS,
                     "traffic": profiled_traffic() if cid == CONFIG_ID else None,
                     "kernel": f"k_decode_step_packed<{c.d}>", "algorithmic_bytes_per_launch": bytes_launch,
                     "kernel_ms": kern_ms, "kernel_ms_median": statistics.median(per_ms),
                     "peak_kind": f"{peak_kind} hbm_gbs (copy)"},
        "state": {"bits_per_value": rep["bits_per_value"], "slot_bytes": rep["slot_bytes"],
                  "clip_fraction": clip,
                  "compression_vs_fp32": 32.0 / rep["bits_per_value"], "status_after_setup": setup_status,
                  "status_bits": st_bits, "exact_sum_columns_per_step": exact_cols},
        "launch": sp.launch_plan(),
        "fp32_state": {"value": shards.job_rate(units, max(4, args.steps // 4), fp_total, world),
                       "kernel_ms": fp_kern, "achieved_gbs": fp_bytes / (fp_kern / 1e3) / 1e9,
                       "frac": fp_bytes / (fp_kern / 1e3) / 1e9 / peak,
                       "speedup_quantized_vs_fp32": fp_kern / kern_ms},
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args, target_s=args.cpu_seconds, cid=cid)
        one = cpu_baseline(args, target_s=max(2.0, args.cpu_seconds / 4), cid=cid, cores=1)
        out["cpu_baseline"]["single_core"] = {"value": one["value"], "unit": UNIT, "sample": one["sample"]}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    sp.close()
    fp.close()
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_window(args, rank, world, local_rank, cid=CONFIG_ID):
    """The per-window variant (sq_window_step) on the serving workload:
    W-token windows, timed over whole windows so that the share of
    window-end requantizations is the variant's own (one token in W)."""
    import torch
    from quantized_linear_attention_sq_b200 import _abi, build, shards, synth
    from quantized_linear_attention_sq_b200.state import StatePool

    torch.cuda.set_device(local_rank)
    build.build()
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    W = args.window
    w = synth.workload(cid, seed=shards.rank_seed(args.seed, rank))
    c = w.cfg
    cal = w.calib()
    B = c.batch
    dev = torch.device("cuda", local_rank)

    def make(fmt):
        return StatePool(B, c.h_v, c.h_k, c.d, c.gate_kind, fmt, cal.unit_bits, cal.pivot, cal.col_scale,
                         cal.row_impact)

    S = torch.from_numpy(w.initial_state()).to(dev)
    fp = make(_abi.SQ_FMT_FP32)
    o = torch.empty((B, c.h_v, c.d), device=dev)
    for t in range(-c.warmup_steps, 0):
        q, k, v, beta, g = (torch.from_numpy(x).to(dev) for x in w.step_inputs(t))
        fp.decode_step(S, q, k, v, beta, g, o)
    if c.outlier_frac:
        S *= torch.from_numpy(w.outlier_mask()).to(dev)[None, :, None, :]
    fp.close()
    sp = make(_abi.SQ_FMT_PACKED)
    pool = sp.new_pool()
    sp.quantize_state(pool, S)
    del S
    wbuf = sp.new_window_buffer(W)
    rec_w, buf_bytes = sp.window_buffer_bytes(W)
    torch.cuda.synchronize()
    setup_status = sp.get_status()
    NI = 8
    host_inputs = [w.step_inputs(t) for t in range(NI)]
    dev_inputs = [[torch.from_numpy(x).to(dev) for x in xs] for xs in host_inputs]
    stream = torch.cuda.current_stream()
    if args.profile:
        for i in range(args.profile):
            sp.window_step(pool, wbuf, W, *dev_inputs[i % NI], o)
        torch.cuda.synchronize()
        print(json.dumps({"profile_steps": args.profile, "window": W, "status_after_setup": setup_status,
                          "status_bits": sp.get_status()}), flush=True)
        sp.close()
        return
    K = max(W, args.steps // W * W)
    Wm = max(W, (args.warmup + W - 1) // W * W)   # the timed region starts at a window's first token

    def barrier():
        if dist is not None:
            dist.barrier()

    for i in range(Wm):
        sp.window_step(pool, wbuf, W, *dev_inputs[i % NI], o)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    n0 = sp.launches()
    props = torch.cuda.get_device_properties(local_rank)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local_rank)
    with ClockSampler(gpu_id) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(K):
            ev[i][0].record(stream)
            sp.window_step(pool, wbuf, W, *dev_inputs[i % NI], o)
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
    clocks = clk.summary()
    launches = sp.launches() - n0
    total_ms = shards.max_over_ranks(t0.elapsed_time(t1), dist, dev)
    per = [a.elapsed_time(b) for a, b in ev]
    kern_ms = statistics.mean(per)
    end_ms = statistics.mean(per[W - 1::W])                       # window-end tokens
    mid = [x for i, x in enumerate(per) if i % W != W - 1]
    mid_ms = statistics.mean(mid) if mid else end_ms
    # ---- end to end: pinned host inputs copied in, o copied out, every token
    pinned = [[torch.from_numpy(x).pin_memory() for x in xs] for xs in host_inputs]
    o_host = torch.empty((B, c.h_v, c.d), dtype=torch.float32).pin_memory()
    stage = [torch.empty_like(x) for x in dev_inputs[0]]
    h2d = sum(x.numel() * x.element_size() for x in pinned[0])
    d2h = o_host.numel() * o_host.element_size()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier()
    e0.record(stream)
    for i in range(K):
        for dst, src in zip(stage, pinned[i % NI]):
            dst.copy_(src, non_blocking=True)
        sp.window_step(pool, wbuf, W, *stage, o)
        o_host.copy_(o, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = shards.max_over_ranks(e0.elapsed_time(e1), dist, dev)
    st_bits = sp.get_status()
    rep = sp.report
    gd = c.d if c.gate_kind == _abi.SQ_GATE_KEY_CHANNEL else 1
    # algorithmic bytes of one token, averaged over a window: the packed
    # record read every token and written at the window's end, the buffered
    # rows read (on average (W - 1) / 2 of them) and the token's row written
    row = 4 * (2 * c.d + gd)
    per_tile = rep["slot_bytes"] / c.h_v * (1 + 1 / W) + row * ((W - 1) / 2 + 1)
    units = B * c.h_v
    bytes_launch = units * per_tile
    peak, peak_kind = peaks()
    achieved = bytes_launch / (kern_ms / 1e3) / 1e9
    cfg = workload_config(w, B * rep["slot_bytes"] + buf_bytes)
    cfg["window"] = W
    cfg["window_buffer_bytes"] = buf_bytes
    out = {
        "metric": METRIC, "value": shards.job_rate(units, K, total_ms, world), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": Wm, "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32/f64", "data": "synthetic (seeded, no dataset)", "config": cfg,
        "e2e": {"value": shards.job_rate(units, K, e2e_ms, world), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "kernel": f"k_window_step<{c.d}>",
                     "algorithmic_bytes_per_launch": bytes_launch, "kernel_ms": kern_ms,
                     "kernel_ms_inside_window": mid_ms, "kernel_ms_window_end": end_ms,
                     "peak_kind": f"{peak_kind} hbm_gbs (copy)"},
        "state": {"bits_per_value": rep["bits_per_value"], "status_after_setup": setup_status,
                  "status_bits": st_bits},
        "clocks": clocks,
    }
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    sp.close()
    if rank == 0:
        print(json.dumps(out), flush=True)


def profiled_traffic():
    """DRAM bytes (read + write) per launch of the packed step from the ncu
    capture recorded under profiles/, or None once the kernel source has
    changed since that capture."""
    import hashlib
    rec_path = os.path.join(ROOT, "profiles", "k_decode_step_packed_gdn_serving_b512.traffic.json")
    try:
        rec = json.load(open(rec_path))
        h = hashlib.sha256()
        for f in rec["sources"]:
            h.update(open(os.path.join(ROOT, f), "rb").read())
    except (OSError, ValueError, KeyError, TypeError):
        return None
    if h.hexdigest() != rec["kernel_source_sha256"]:
        return None
    return rec["dram_bytes_read"] + rec["dram_bytes_write"]


def clip_fraction(S, cal, c):
    """Share of the quantized rows' entries that the row scale clips when
    the state S [B, h_v, d, d] is quantized: |T_ij| / r_i rounds beyond qmax,
    with T = S / c and r_i the fp16 round-up of min(phi_i, 1) max_j |T_ij| /
    qmax_i (rows with phi_i < 1 clip their largest entries). Widths per head
    (GDN) or per key row (KDA); pivot units are not counted."""
    import torch

    dev = S.device
    h_v, d = c.h_v, c.d
    bits = np.broadcast_to(cal.unit_bits.reshape(h_v, -1), (h_v, d)).astype("float64")
    piv = np.broadcast_to(cal.pivot.reshape(h_v, -1), (h_v, d))
    keep = torch.from_numpy(np.ascontiguousarray(piv == 0)).to(dev)                   # [h_v, d] rows
    qmax = torch.from_numpy((2.0 ** (bits - 1) - 1).astype("float32")).to(dev)       # [h_v, d]
    ic = 1.0 / torch.from_numpy(cal.col_scale).to(dev)                               # [h_v, d] columns
    phi = torch.from_numpy(np.minimum(cal.row_impact, 1.0).astype("float32")).to(dev)  # [h_v, d] rows
    clipped = 0
    total = 0
    for b0 in range(0, S.shape[0], 64):                                              # bounded temporaries
        T = S[b0:b0 + 64] * ic[None, :, None, :]
        m = T.abs().amax(dim=3)                                                      # [b, h_v, d]
        s = phi[None] * m / qmax[None]
        h = s.to(torch.float16)
        up = (h.float() < s) & (h.float() < 65504)
        h = torch.where(up, (h.view(torch.int16) + 1).view(torch.float16), h)         # round toward +inf
        r = h.float()
        lim = qmax[None, :, :, None] + 0.5
        over = (T.abs() * (1.0 / r).unsqueeze(3)) > lim
        over = over & keep[None, :, :, None] & (r > 0).unsqueeze(3)
        clipped += int(over.sum())
        total += int(keep.sum()) * T.shape[0] * d
    return clipped / max(total, 1)


# ------------------------------------------------------- the CPU oracle
def cpu_baseline(args, target_s=15.0, steps=None, cid=CONFIG_ID, cores=None):
    """Time the CPU oracle (as it stands) on a bounded sample of the
    workload, tiles split over all host cores: a short probe measures the
    oracle's rate on this host, then `steps` decode steps (default: as many
    as fit) on as many of the batch's requests as make the timed part last
    about `target_s` seconds."""
    import oracle
    from quantized_linear_attention_sq_b200 import synth

    w = synth.workload(cid, seed=args.seed)
    c = w.cfg
    cal = w.calib()
    cores = cores or oracle.cores_available()

    def setup(reqs):
        o_ = oracle.Oracle(len(reqs), c.h_v, c.h_k, c.d, c.gate_kind, cal.unit_bits, cal.pivot, cal.col_scale,
                           cal.row_impact)
        pool = o_.new_pool()
        S = w.initial_state(reqs)
        if c.outlier_frac:
            S *= w.outlier_mask()[None, :, None, :]
        o_.quantize(pool, S)
        return o_, pool

    # probe: one step on a few requests gives the tile-steps per second
    probe = list(range(min(c.batch, 2 * cores)))
    o_, pool = setup(probe)
    x = w.step_inputs(0, probe)
    t0 = time.perf_counter()
    o_.step(pool, *x, threads=cores)
    rate = len(probe) * c.h_v / max(time.perf_counter() - t0, 1e-6)
    budget = rate * target_s  # tile-steps
    if steps is None:
        steps = max(1, min(64, int(budget // (c.batch * c.h_v))))
    n_req = max(1, min(c.batch, int(budget // (steps * c.h_v))))
    reqs = list(range(n_req))
    o_, pool = setup(reqs)
    inputs = [w.step_inputs(t, reqs) for t in range(min(steps, 8))]
    t0 = time.perf_counter()
    for t in range(steps):
        o_.step(pool, *inputs[t % len(inputs)], threads=cores)
    dt = time.perf_counter() - t0
    units = len(reqs) * c.h_v * steps
    return {"value": units / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{len(reqs)} of {c.batch} requests x {c.h_v} heads x {steps} steps "
                      f"({units} tile-steps, {dt:.1f} s wall on {cores} threads)"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    # each of the --steps steps is a bounded sample of the workload; the whole
    # run is sized to 4 x --cpu-seconds of CPU time (a minute by default)
    cb = cpu_baseline(args, target_s=4.0 * args.cpu_seconds, steps=max(1, args.steps))
    import oracle
    from quantized_linear_attention_sq_b200 import synth
    w = synth.workload(CONFIG_ID, seed=args.seed)
    cal = w.calib()
    c = w.cfg
    slot_bytes = oracle.Oracle(1, c.h_v, c.h_k, c.d, c.gate_kind, cal.unit_bits, cal.pivot, cal.col_scale,
                               cal.row_impact).layout.slot_bytes
    full_step_ms = 1e3 * w.cfg.batch * w.cfg.h_v / cb["value"]  # one whole-batch step at the sample's rate
    out = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": full_step_ms,
           "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded, no dataset)",
           "config": workload_config(w, w.B * slot_bytes), "cpu_baseline": cb,
           "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
           "note": "reference arm = the plain CPU oracle of the same step (no upstream code exists to install)"}
    print(json.dumps(out), flush=True)


# ------------------------------------------- 8-layer KDA rollout
def run_rollout(args, rank, world, local_rank):
    """The long-rollout workload (8 KDA layers, 256 requests x 32 heads per
    GPU, per-row widths {2,4,6} at 4-bit nominal, 3 % FP16 pivot rows): one
    token = one step of every layer. Two parts, one JSON line:
      - the full rollout: 2048 tokens with inputs drawn on the device for
        every layer and token; the quantized step of each token is timed
        with CUDA events (input drawing excluded); the same inputs drive the
        FP32-state step of every layer, and every 256 tokens the dequantized
        quantized state is compared with the FP32 state (relative
        Frobenius, per layer and over all layers: the drift of the
        quantized rollout);
      - launch overhead: per-layer launches vs one CUDA graph holding 4
        tokens x 8 layers of launches, on 4 recycled input sets."""
    import torch
    from quantized_linear_attention_sq_b200 import _abi, build, shards, synth
    from quantized_linear_attention_sq_b200.rollout import LayerStack
    from quantized_linear_attention_sq_b200.state import StatePool

    torch.cuda.set_device(local_rank)
    build.build()
    dev = torch.device("cuda", local_rank)
    cid = 4
    nl = synth.CONFIGS[cid].layers
    works = [synth.workload(cid, seed=shards.rank_seed(args.seed, rank), layer=l) for l in range(nl)]
    c = works[0].cfg
    B = c.batch
    layers, pools, fps, fstates = [], [], [], []
    for w in works:
        cal = w.calib()
        fp = StatePool(B, c.h_v, c.h_k, c.d, c.gate_kind, _abi.SQ_FMT_FP32)
        S = torch.from_numpy(w.initial_state()).to(dev)
        o = torch.empty((B, c.h_v, c.d), device=dev)
        for t in range(-c.warmup_steps, 0):
            fp.decode_step(S, *w.step_inputs_device(t), o)
        S *= torch.from_numpy(w.outlier_mask()).to(dev)[None, :, None, :]
        sp = StatePool(B, c.h_v, c.h_k, c.d, c.gate_kind, _abi.SQ_FMT_PACKED, cal.unit_bits, cal.pivot,
                       cal.col_scale, cal.row_impact)
        pool = sp.new_pool()
        sp.quantize_state(pool, S)
        torch.cuda.synchronize()
        layers.append(sp)
        pools.append(pool)
        fps.append(fp)
        fstates.append(S)   # the FP32-state rollout starts from the same state
    stream = torch.cuda.current_stream()
    units = B * c.h_v * nl
    bytes_token = sum(B * sp.report["state_bytes_per_step"] for sp in layers)
    peak, peak_kind = peaks()

    # ---- the full rollout with its drift
    n_tok = c.steps
    outs = [torch.empty((B, c.h_v, c.d), device=dev) for _ in works]
    ofp = torch.empty((B, c.h_v, c.d), device=dev)
    deq = torch.empty((B, c.h_v, c.d, c.d), device=dev)

    def drift():
        num = den = 0.0
        per = []
        for sp, pool, S in zip(layers, pools, fstates):
            sp.dequantize_state(pool, deq)
            dn = float(torch.linalg.vector_norm(deq - S)) ** 2
            dd = float(torch.linalg.vector_norm(S)) ** 2
            per.append((dn / dd) ** 0.5)
            num += dn
            den += dd
        return (num / den) ** 0.5, per

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_tok)]
    curve = []
    with ClockSampler(local_rank) as clk:
        for t in range(n_tok):
            xs = [w.step_inputs_device(t) for w in works]
            ev[t][0].record(stream)
            for sp, pool, x, o in zip(layers, pools, xs, outs):
                sp.decode_step(pool, *x, o)
            ev[t][1].record(stream)
            for fp, S, x in zip(fps, fstates, xs):
                fp.decode_step(S, *x, ofp)
            if (t + 1) % 256 == 0:
                tot, per = drift()
                curve.append({"step": t + 1, "rel_frobenius": tot, "per_layer": per})
    clocks = clk.summary()
    torch.cuda.synchronize()
    roll_ms = sum(a.elapsed_time(b) for a, b in ev)
    status = [sp.get_status() for sp in layers]
    for fp in fps:
        fp.close()
    del fstates

    # ---- launch overhead: eager per-layer launches vs one CUDA graph
    stack = LayerStack(layers)
    NI = 4
    inputs = [[list(w.step_inputs_device(10_000 + t)) for w in works] for t in range(NI)]
    outs4 = [[torch.empty((B, c.h_v, c.d), device=dev) for _ in works] for _ in range(NI)]
    K = max(NI, args.steps // NI * NI)

    def timed(fn, reps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    def eager_block():
        for t in range(NI):
            stack.step(pools, inputs[t], outs4[t])

    eager_ms = timed(eager_block, K // NI)
    graph = stack.capture(pools, inputs, outs4)
    graph_ms = timed(graph.replay, K // NI)
    out = {"metric": "8-layer KDA rollout (request*head*layer)-steps/s", "unit": "(request*head*layer)-steps/s",
           "value": units * n_tok / (roll_ms / 1e3), "n_gpus": world, "higher_is_better": True,
           "config": {"workload": c.name, "batch_per_gpu": B, "h_v": c.h_v, "d": c.d, "layers": nl,
                      "gate": "KDA (one gate per key channel)",
                      "widths": "per-row {2,4,6}, 4-bit nominal, 3% FP16 pivot rows",
                      "inputs": "drawn on the device per layer and token (Philox, seeded)"},
           "rollout": {"tokens": n_tok, "ms_per_token": roll_ms / n_tok,
                       "achieved_gbs": bytes_token / (roll_ms / n_tok / 1e3) / 1e9,
                       "frac": bytes_token / (roll_ms / n_tok / 1e3) / 1e9 / peak,
                       "drift_vs_fp32_state": curve, "clocks": clocks, "status_bits": status},
           "launch_overhead": {
               "eager": {"ms_per_token": eager_ms / K, "launches_per_token": nl},
               "graph": {"ms_per_token": graph_ms / K, "tokens_per_replay": NI, "launches_per_replay": NI * nl},
               "graph_speedup": eager_ms / graph_ms},
           "peak_kind": f"{peak_kind} hbm_gbs (copy)"}
    del graph
    stack.close()
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_calibration(args, rank, world, local_rank):
    """The calibration workload on the serving layer's shape (32 value heads,
    16 key heads, d = 128, GDN): a 512-sample fp32 state trace (1 GiB, beyond
    L2) and 4096 tokens of queries and gates (synthetic, seeded). The timed
    kernel is the trace pass (fp64 running sums of S^2, one launch per pass
    over the whole trace); the whole calibration (accumulators, trace pass,
    token pass, tables, allocation) is timed on the host clock around a
    synchronised run. Prints its own JSON line."""
    import torch
    from quantized_linear_attention_sq_b200 import build, shards, synth
    from quantized_linear_attention_sq_b200.calibrate import TraceCalibrator

    torch.cuda.set_device(local_rank)
    build.build()
    dev = torch.device("cuda", local_rank)
    c = synth.CONFIGS[CONFIG_ID]
    n_states, n_tok = args.trace_samples, 4096
    states, q, g = synth.calibration_trace(c.h_v, c.h_k, c.d, c.gate_kind, n_states, n_tok,
                                           seed=shards.rank_seed(args.seed, rank))
    S = torch.from_numpy(states).to(dev)
    qd, gd = torch.from_numpy(q).to(dev), torch.from_numpy(g).to(dev)
    del states
    stream = torch.cuda.current_stream()
    cal = TraceCalibrator(c.h_v, c.h_k, c.d, c.gate_kind)
    for _ in range(args.warmup):
        cal.add_states(S)
    torch.cuda.synchronize()
    K = max(1, min(args.steps, 200))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        e0.record(stream)
        for _ in range(K):
            cal.add_states(S)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / K
    cal.close()
    # the whole calibration, once more from empty accumulators
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    cal = TraceCalibrator(c.h_v, c.h_k, c.d, c.gate_kind)
    cal.add_states(S)
    cal.add_tokens(qd, gd)
    tabs = cal.finish(c.widths, c.nominal_bits, c.pivot_frac)
    whole_ms = (time.perf_counter() - t0) * 1e3
    cal.close()
    E = c.h_v * c.d * c.d
    alg_bytes = n_states * E * 4 + 2 * E * 8
    peak, peak_kind = peaks()
    achieved = alg_bytes / (ms / 1e3) / 1e9
    out = {"metric": "calibration trace pass, state samples/s", "unit": "state-samples/s", "n_gpus": world,
           "steps": K, "warmup": args.warmup, "ms_per_step": ms, "value": n_states * c.h_v / (ms / 1e3),
           "higher_is_better": True, "dtype": "f64 sums of f32", "data": "synthetic",
           "config": {"workload": "calib_trace_gdn_hv32_hk16_d128", "trace_samples": n_states,
                      "tokens": n_tok, "trace_bytes": n_states * E * 4, "l2": f"{n_states * E * 4 / 2**20:.0f} MiB trace > 126 MB L2"},
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                        "frac": achieved / peak, "kernel": "k_trace_sum<4,true>",
                        "peak_kind": f"{peak_kind} hbm_gbs (copy)"},
           "whole_calibration_ms": whole_ms,
           "tables": {"pivot_heads": int(tabs.pivot.sum()),
                      "widths": {str(b): int((tabs.unit_bits[tabs.pivot == 0] == b).sum()) for b in c.widths}},
           "clocks": clk.summary()}
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_prefill(args, rank, world, local_rank):
    """The prefill handoff on the serving shape (512 requests x 32 value
    heads, 16 key heads, d = 128, GDN, the serving calibration): a prompt of
    --prompt-len tokens per request from a zero state, every (request, head)
    state kept on chip over the prompt and quantized once into its pool slot.
    One launch per step. Bound by fp32 arithmetic: 7 d^2 flops per (request,
    head, token) (gate d^2, S^T k 2d^2, update 2d^2, S^T q 2d^2). Prints its
    own JSON line."""
    import torch
    from quantized_linear_attention_sq_b200 import _abi, build, shards, synth
    from quantized_linear_attention_sq_b200.state import StatePool

    torch.cuda.set_device(local_rank)
    build.build()
    dev = torch.device("cuda", local_rank)
    w = synth.workload(CONFIG_ID, seed=shards.rank_seed(args.seed, rank))
    c = w.cfg
    B, L = c.batch, args.prompt_len
    cal = w.calib()
    sp = StatePool(B, c.h_v, c.h_k, c.d, c.gate_kind, _abi.SQ_FMT_PACKED, cal.unit_bits, cal.pivot,
                   cal.col_scale, cal.row_impact)
    pool = sp.new_pool()
    prompt = [torch.from_numpy(x).to(dev) for x in w.prompt_inputs(L)]
    o = torch.empty((B, L, c.h_v, c.d), device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        sp.prefill(pool, *prompt, o)
    torch.cuda.synchronize()
    K = max(1, min(args.steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        e0.record(stream)
        for _ in range(K):
            sp.prefill(pool, *prompt, o)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / K
    status = sp.get_status()
    sp.close()
    clocks = clk.summary()
    flops = 7.0 * c.d * c.d * B * c.h_v * L
    sm_mhz = clocks.get("sm_max_mhz") or 1965.0
    peak_tflops = 148 * 128 * 2 * sm_mhz * 1e6 / 1e12
    achieved = flops / (ms / 1e3) / 1e12
    out = {"metric": "prefill handoff, prompt tokens/s", "unit": "request-tokens/s", "n_gpus": world,
           "steps": K, "warmup": args.warmup, "ms_per_step": ms, "value": B * L * world / (ms / 1e3),
           "higher_is_better": True, "scaling": "weak", "dtype": "f32", "data": "synthetic",
           "config": {"workload": f"prefill_gdn_b{B}_hv{c.h_v}_hk{c.h_k}_d{c.d}_L{L}", "batch_per_gpu": B,
                      "prompt_len": L, "handoff": "quantized once into the packed pool (6-bit nominal)"},
           "roofline": {"bound": "alu", "achieved": achieved, "peak": peak_tflops, "unit": "TFLOP/s",
                        "frac": achieved / peak_tflops, "kernel": "k_prefill<128>",
                        "peak_kind": "derived: 148 SMs x 128 fp32 lanes x 2 flops x max SM clock"},
           "status_bits": status, "clocks": clocks}
    if rank == 0:
        print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(STEP_WORKLOADS) + ["kda_rollout_8layers", "calibration", "prefill",
                                                                   "window_serving"],
                    default="serving",
                    help="serving: the headline GDN workload (batch 512); plumbing, gdn_layer, kda_layer: "
                         "the smaller L2-resident configurations; kda_rollout_8layers: 8 KDA layers, "
                         "2048 steps with the drift against the FP32-state path, plus per-layer launches "
                         "vs one CUDA graph; calibration: the trace pass of the calibration library on "
                         "the serving layer's shape; prefill: the prefill handoff on the serving shape; "
                         "window_serving: the per-window variant (--window tokens per window) on the "
                         "serving workload")
    ap.add_argument("--window", type=int, default=16, help="window_serving: tokens per window")
    ap.add_argument("--trace-samples", type=int, default=512,
                    help="calibration workload: state samples in the trace (512 = 1 GiB)")
    ap.add_argument("--prompt-len", type=int, default=128, help="prefill workload: tokens per prompt")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="approximate CPU time of the oracle baseline sample")
    ap.add_argument("--profile", type=int, default=0,
                    help="prepare the workload, run this many packed steps untimed, exit (for ncu)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
    elif args.workload == "kda_rollout_8layers":
        run_rollout(args, rank, world, local_rank)
    elif args.workload == "calibration":
        run_calibration(args, rank, world, local_rank)
    elif args.workload == "prefill":
        run_prefill(args, rank, world, local_rank)
    elif args.workload == "window_serving":
        run_window(args, rank, world, local_rank)
    else:
        run_ours(args, rank, world, local_rank, cid=STEP_WORKLOADS[args.workload])


if __name__ == "__main__":
    main()
