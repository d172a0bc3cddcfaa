#!/usr/bin/env python
"""Benchmark of the DiG GLA token mixer on B200.

One step = the whole hot path over one batch of the DiG-S/2 1792x1792 workload
(B=2, 112x112 token grid, L=12544, 6 heads, d_k=32, d_v=64, bf16 inputs):
GLA forward with the fused Swish(r)*RMSNorm(o) epilogue, GLA backward
(dq, dk, dv, dlog alpha) and the SREM reorient + 3x3 depthwise conv (C=384).
Step i runs scan mode i % 4, as layer i of DiG would.  Inputs are resident in
HBM; L2 is flushed (512 MiB write) before every step, outside the timed events.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 the script runs under torchrun, one rank per GPU, each rank an
independent replica (the path has no data-path collective); time is the max over
ranks.  Prints one JSON line on rank 0.
"""
import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_linear_attention_fwd_b200 import inputs  # noqa: E402

METRIC = "GLA fwd+bwd tokens/s at L=4096/12544/16384; % of roofline (tensor/HBM)"
WORKLOAD_INDEX = 3  # DiG-S/2 at 1792^2: the configuration that carries every hot-path step
L2_FLUSH_BYTES = 512 << 20


def max_over_ranks(value, world, device):
    """The largest of `value` over the ranks: the time of the slowest replica."""
    if world <= 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def algorithmic_bytes(w):
    """Bytes each kernel must move once (inputs read once, outputs written once)."""
    BL, H, dk, dv = w.B * w.L, w.H, w.dk, w.dv
    e = 2  # bf16 storage
    qk = BL * H * dk * e
    vv = BL * H * dv * e
    z = BL * dk * 4  # one gate shared by the heads, fp32
    fwd = 2 * qk + vv + z + vv + 2 * vv        # q k v z r in; o y out
    bwd = 2 * qk + vv + z + vv + 2 * qk + vv + z  # q k v z dO in; dq dk dv dlogalpha out
    conv = 2 * BL * w.conv_C * e
    # the backward ops outside the step: the epilogue's (o r dY in; d_o d_r out) and the
    # conv's (x dY in; dx out); the fp32 parameter vectors are a few KB
    epi_bwd = 5 * vv
    conv_bwd = 3 * BL * w.conv_C * e
    # the gate projection (D -> rank -> d_k): x in, z and u out; backward x u z dla in, dx out
    gate_fwd = BL * (w.D * e + w.dk * 4 + w.rank * 4)
    gate_bwd = BL * (2 * w.D * e + w.rank * 4 + 2 * w.dk * 4)
    return {"fwd": fwd, "bwd": bwd, "conv": conv, "epi_bwd": epi_bwd, "conv_bwd": conv_bwd,
            "gate_fwd": gate_fwd, "gate_bwd": gate_bwd}


def metric_bytes(w):
    """Bytes of the metric's GLA fwd and bwd with d log(alpha) counted once per head
    (the per-token-head convention of the metric's roofline): fwd reads q k v z and
    writes o; bwd reads q k v z dO and writes dq dk dv and a per-head d log(alpha)."""
    BL, H, dk, dv = w.B * w.L, w.H, w.dk, w.dv
    e = 2
    fwd = BL * (H * (2 * dk + 2 * dv) * e + dk * 4)
    bwd = BL * (H * (2 * dk + 2 * dv) * e + dk * 4 + H * (2 * dk + dv) * e + H * dk * 4)
    return fwd, bwd


# This library's kernels per op, in launch order, and the sources they are built from.
OP_KERNELS = {  # this library's kernels per op on the bench workload (bf16, d_k = 32, d_v = 64)
    # row scan orders: tile-copy dS and output kernels; column orders: the row-piece ones
    "fwd": ["gla_gate_kernel", "gla_reduce_tma_kernel | gla_chunk_state_kernel", "gla_state_scan_kernel",
            "gla_out_tma_kernel | gla_chunk_out_kernel"],
    # the exact gradient kernel is launched on the list of units the fp16 kernel hands back (empty here)
    "bwd": ["gla_reduce_tma_kernel | gla_chunk_dh_kernel", "gla_state_scan_kernel", "gla_grad_tma_kernel",
            "gla_chunk_grad_kernel"],
    "conv": ["srem_dwconv_kernel"],
    "epi_bwd": ["epilogue_bwd_kernel"],
    "conv_bwd": ["srem_dwconv_bwd_kernel"],
    "gate_fwd": ["gate_proj_tc_kernel"],
    "gate_bwd": ["gate_proj_bwd_tc_kernel"],
}
STEP_OPS = ("fwd", "bwd", "conv")  # the ops of one timed step
_CHUNK_SRC = ["gla_chunk.cuh", "gla_common.cuh", "sm100.cuh", "dig_common.cuh", "gla.h"]
_TMA_SRC = ["tma.cuh", "tma_tiles.cuh", "tmap.cu", "tmap.h"]
OP_SOURCES = {
    "fwd": ["gla_fwd.cu", "gla_state_tma.cu", "gla_fwd_tma.cu", "gla_strong.cuh"] + _TMA_SRC + _CHUNK_SRC,
    "bwd": ["gla_bwd.cu", "gla_bwd_tma.cu", "gla_state_tma.cu", "gla_fwd.cu", "gla_strong.cuh"] + _TMA_SRC +
           _CHUNK_SRC,
    "conv": ["srem.cu", "srem.cuh", "dig_common.cuh", "gla.h"],
    "epi_bwd": ["epilogue_bwd.cu", "gla_common.cuh", "sm100.cuh", "dig_common.cuh", "bwd_ops.h"],
    "conv_bwd": ["srem_bwd.cu", "srem.cuh", "gla_common.cuh", "sm100.cuh", "dig_common.cuh", "bwd_ops.h"],
    "gate_fwd": ["gate_proj_tc.cu", "gate_proj.cu", "gate_proj.h", "tma.cuh", "tma_tiles.cuh", "tmap.cu",
                 "gla_common.cuh", "sm100.cuh", "dig_common.cuh"],
    "gate_bwd": ["gate_proj_bwd_tc.cu", "gate_proj.cu", "gate_proj.h", "tma.cuh", "tma_tiles.cuh", "tmap.cu",
                 "gla_common.cuh", "sm100.cuh", "dig_common.cuh"],
}
OP_NAMES = {"fwd": "dig_gla_fwd", "bwd": "dig_gla_bwd_saved", "conv": "dig_srem_reorient_dwconv",
            "epi_bwd": "dig_epilogue_bwd", "conv_bwd": "dig_srem_reorient_dwconv_bwd",
            "gate_fwd": "dig_gate_proj_fwd", "gate_bwd": "dig_gate_proj_bwd"}


def _src_hash(names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "gated_linear_attention_fwd_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(kernel, srcs, scale):
    """DRAM bytes per call of an op (summed over its kernels) from the committed
    ncu capture, if the op's sources are unchanged since."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel)
    if not d or d.get("source_sha") != _src_hash(srcs):
        return None
    return float(d["dram_bytes_per_call"]) * scale


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        finally:
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows]
        mx = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        loaded = [s for s in sm if s > 0.5 * mx] or sm
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


def cpu_sample(w, x, steps=1, min_seconds=0.0):
    """The fp64 oracle on batch element 0 (all heads): forward + epilogue + backward + conv.
    Runs `steps` steps, or more until at least `min_seconds` have passed."""
    import oracle
    sl = lambda a: a[:1]
    t0 = time.perf_counter()
    i = 0
    while i < steps or time.perf_counter() - t0 < min_seconds:
        mode = i % 4
        i += 1
        o = oracle.gla_fwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["z"]), w.inv_tau, w.grid_h, w.grid_w, mode)
        oracle.epilogue(o, sl(x["r"]))
        oracle.gla_bwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["z"]), w.inv_tau, sl(x["dO"]), w.grid_h, w.grid_w,
                       mode)
        oracle.srem_dwconv(sl(x["x_conv"]), x["w_conv"], None, mode)
    dt = time.perf_counter() - t0
    return w.L * i / dt, dt, min(w.H, oracle.num_threads()), i


def run_reference(args, rank, world):
    """The oracle, timed on the host cores, as the reference arm."""
    w = inputs.WORKLOADS[WORKLOAD_INDEX]
    if rank != 0:
        return None
    x = inputs.make_inputs(w)
    cpu_sample(w, x, steps=args.warmup)
    tps, dt, cores, _ = cpu_sample(w, x, steps=args.steps)
    sample = "oracle (fp64 C, OpenMP over heads) on batch element 0 of %s: fwd+epilogue+bwd+conv, %d tokens/step" % (
        w.name, w.L)
    line = {"impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(w, world),
            "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return line


def _config(w, world):
    return {"workload": "%s: B=%d, %dx%d token grid (L=%d), H=%d, d_k=%d, d_v=%d, bf16 inputs; fwd + Swish*RMSNorm "
                        "epilogue + bwd + SREM 3x3 dwconv (C=%d); scan mode cycles over the 4 DiG directions"
                        % (w.name, w.B, w.grid_h, w.grid_w, w.L, w.H, w.dk, w.dv, w.conv_C),
            "global_batch": w.B * world, "seq_len": w.L, "parallelism": "replicas x%d" % world,
            "l2": "flushed (512 MiB write) before every step, outside the timed events",
            "e2e": "all inputs copied in and all outputs copied out every step (pinned host buffers); copies on "
                   "their own streams overlap the neighbouring steps' compute, two device buffer sets alternate"}


def time_next_ops(dig, w, dev, stream, o, r, dY, xc, wc, dla, flush, warmup, iters):
    """Mean event-timed seconds of one call of each op outside the step: the
    epilogue backward (with d_gamma), the conv backward (with dw, dbias), and the
    gate projection forward and backward (with u, dW1, dW2, db), on the step's
    workload with synthetic tensors of its shapes."""
    g = torch.Generator(device=dev).manual_seed(1)
    xg = torch.randn(w.B * w.L, w.D, device=dev, generator=g).to(xc.dtype)
    W1 = 0.02 * torch.randn(w.D, w.rank, device=dev, generator=g)
    W2 = 0.02 * torch.randn(w.rank, w.dk, device=dev, generator=g)
    zg, ug = torch.empty(w.B * w.L, w.dk, device=dev), torch.empty(w.B * w.L, w.rank, device=dev)
    dxg, dW1, dW2, dbg = torch.empty_like(xg), torch.empty_like(W1), torch.empty_like(W2), torch.empty(w.dk, device=dev)
    d_o, d_r = torch.empty_like(o), torch.empty_like(o)
    d_gamma = torch.empty(w.dv, device=dev)
    dyc = torch.randn(w.B, w.L, w.conv_C, device=dev, generator=g).to(xc.dtype)
    dx = torch.empty_like(xc)
    dw, db = torch.empty(w.conv_C, 3, 3, device=dev), torch.empty(w.conv_C, device=dev)
    calls = {
        "epi_bwd": lambda i: dig.dig_epilogue_bwd(o, r, dY, d_o, d_r, None, 1e-5, d_gamma, stream=stream),
        "conv_bwd": lambda i: dig.dig_srem_reorient_dwconv_bwd(xc, wc, dyc, dx, i % 4, dw, db, stream=stream),
        "gate_fwd": lambda i: dig.dig_gate_proj_fwd(xg, W1, W2, zg, None, ug, stream=stream),
        "gate_bwd": lambda i: dig.dig_gate_proj_bwd(xg, W1, W2, ug, zg, dla.view(-1, w.dk), w.inv_tau, dxg, dW1, dW2,
                                                    dbg, stream=stream),
    }
    out = {}
    for op, call in calls.items():
        for i in range(warmup):
            call(i)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
        for i in range(iters):
            flush.fill_(float(i))
            evs[i][0].record(stream)
            call(i)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        out[op] = float(np.mean([a.elapsed_time(b) for a, b in evs])) * 1e-3
    return out


# The metric's three shapes: L = 4096 (DiG-S/2 1024^2), 12544 (DiG-S/2 1792^2, the step
# above) and 16384 (DiG-XL/2 2048^2).
PER_CONFIG = (2, 3, 4)


def time_gla_config(dig, index, dev, stream, flush, warmup, iters, seed_offset=0):
    """Event-timed mean seconds of dig_gla_fwd (bf16 o; with the Swish*RMSNorm epilogue
    where the workload has it) and of dig_gla_bwd_saved (bf16 dq dk dv) on one workload,
    L2 flushed before every call pair, scan mode cycling."""
    w = inputs.WORKLOADS[index]
    x = inputs.make_inputs(w, seed=inputs.SEED_BASE + index + seed_offset, with_conv=False)
    t = lambda a, dt=torch.bfloat16: torch.from_numpy(a).to(dev).to(dt).contiguous()
    q, k, v, dO = t(x["q"]), t(x["k"]), t(x["v"]), t(x["dO"])
    z = t(x["z"], torch.float32)
    r = t(x["r"]) if w.epilogue else None
    B, L, H = w.B, w.L, w.H
    o = torch.empty(B, L, H, w.dv, device=dev, dtype=torch.bfloat16)
    y = torch.empty_like(o) if w.epilogue else None
    dq, dk_, dv_, dla = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(z)
    ws_f = dig.new_workspace(B, H, L, w.dk, w.dv, device=dev)
    ws_b = dig.new_workspace(B, H, L, w.dk, w.dv, backward=True, device=dev)

    def call(i, ev=None):
        mode = i % 4
        if ev:
            ev[0].record(stream)
        dig.dig_gla_fwd(q, k, v, z, w.inv_tau, o, w.grid_h, w.grid_w, mode, ws_f, r=r, y=y, stream=stream)
        if ev:
            ev[1].record(stream)
        dig.dig_gla_bwd_saved(q, k, v, z, w.inv_tau, dO, dq, dk_, dv_, dla, w.grid_h, w.grid_w, mode, ws_f, ws_b,
                              stream=stream)
        if ev:
            ev[2].record(stream)

    for i in range(warmup):
        flush.fill_(float(i))
        call(i)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(iters)]
    for i in range(iters):
        flush.fill_(float(i))
        call(i, evs[i])
    torch.cuda.synchronize()
    for ws in (ws_f, ws_b):
        st = dig.dig_read_status(ws)
        if st != dig.DIG_OK:
            raise RuntimeError("device status on %s: %s" % (w.name, dig.lib.dig_status_string(st).decode()))
    t_f = float(np.mean([e[0].elapsed_time(e[1]) for e in evs])) * 1e-3
    t_b = float(np.mean([e[1].elapsed_time(e[2]) for e in evs])) * 1e-3
    return t_f, t_b


def time_dig_block(dev, flush, warmup, iters):
    """Event-timed mean microseconds of one synthetic DiG-S/2 block forward at the
    bench workload's shape (dense projections by cuBLAS, the rest by libdig.so) and
    of the GLA mixer call inside it, averaged over the four layers' scan orders,
    L2 flushed before every block."""
    from gated_linear_attention_fwd_b200 import dig_block
    w = inputs.WORKLOADS[WORKLOAD_INDEX]
    B, L = w.B, w.L
    blk_us, mix_us = [], []
    for layer in range(4):
        blk = dig_block.dig_s2(w.grid_h, w.grid_w, layer=layer, seed=layer, device=dev)
        g = torch.Generator(device="cpu").manual_seed(100 + layer)
        x0 = torch.randn(B, L, blk.D, generator=g).to(dev, torch.bfloat16)
        cond = torch.randn(B, blk.D, generator=g).to(dev, torch.bfloat16)
        buf = blk.buffers(B, L, dev)
        x = x0.clone()
        for i in range(warmup):
            blk.forward(x, cond, buf)
        timing, evs = {}, []
        for i in range(iters):
            x.copy_(x0)
            flush.fill_(float(i))
            e = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            e[0].record()
            blk.forward(x, cond, buf, timing=timing)
            e[1].record()
            evs.append(e)
        torch.cuda.synchronize()
        blk_us.append(float(np.mean([a.elapsed_time(b) for a, b in evs])) * 1e3)
        mix_us.append(float(np.mean([a.elapsed_time(b) for a, b in timing["mixer_events"]])) * 1e3)
    return float(np.mean(blk_us)), float(np.mean(mix_us))


def per_config_record(index, t_f, t_b, world, hbm, tflops):
    """tokens/s of fwd+bwd and the fraction of roofline of each, with the metric's bytes."""
    w = inputs.WORKLOADS[index]
    fb, bb = metric_bytes(w)
    epi = 2 * w.B * w.L * w.H * w.dv * 2 if w.epilogue else 0  # r in, y out (o is counted above)
    roof_f = (fb + epi) / (hbm * 1e9)
    roof_b = bb / (hbm * 1e9)
    return {"workload": "%s: B=%d, %dx%d grid (L=%d), H=%d, d_k=%d, d_v=%d, bf16%s"
                        % (w.name, w.B, w.grid_h, w.grid_w, w.L, w.H, w.dk, w.dv,
                           ", fwd with Swish*RMSNorm epilogue" if w.epilogue else ""),
            "seq_len": w.L, "tokens_per_s": w.B * w.L * world / (t_f + t_b),
            "fwd_us": t_f * 1e6, "bwd_us": t_b * 1e6,
            "fwd_bytes": fb + epi, "bwd_bytes": bb,
            "fwd_frac": roof_f / t_f, "bwd_frac": roof_b / t_b,
            "roofline_tokens_per_s": w.B * w.L * world / (roof_f + roof_b),
            "frac": (roof_f + roof_b) / (t_f + t_b), "bound": "hbm", "peak_gbs": hbm}


def run_guarded(fn, world, device):
    """Runs fn() on every rank; returns (result, None) when it succeeded on all ranks and
    ({}, message) otherwise, with every rank taking the same branch (one all-reduce of an
    error flag) so that the collectives that follow stay paired.  A CUDA error leaves the
    context unusable, so it is raised instead of being reported."""
    result, err = {}, None
    try:
        result = fn()
    except Exception as e:  # noqa: BLE001
        torch.cuda.synchronize()  # raises if the error was a device fault
        err = "%s: %s" % (type(e).__name__, str(e).splitlines()[0] if str(e) else "")
    if world > 1:
        flag = torch.tensor([1.0 if err else 0.0], dtype=torch.float64, device=device)
        torch.distributed.all_reduce(flag, op=torch.distributed.ReduceOp.MAX)
        if flag.item() and err is None:
            err = "failed on another rank"
    return (result, None) if err is None else ({}, err)


def run_ours(args, rank, world, local_rank):
    from gated_linear_attention_fwd_b200 import dig
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = inputs.WORKLOADS[WORKLOAD_INDEX]
    x = inputs.make_inputs(w, seed=inputs.SEED_BASE + WORKLOAD_INDEX + rank)
    bf = torch.bfloat16
    t = lambda a, dt=bf: torch.from_numpy(a).to(dev).to(dt).contiguous()
    B, L, H, dk, dv = w.B, w.L, w.H, w.dk, w.dv
    q, k, v, r, dO, xc = t(x["q"]), t(x["k"]), t(x["v"]), t(x["r"]), t(x["dO"]), t(x["x_conv"])
    z, wc = t(x["z"], torch.float32), t(x["w_conv"], torch.float32)
    o = torch.empty(B, L, H, dv, device=dev, dtype=bf)
    y = torch.empty_like(o)
    dq, dk_, dv_ = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dla = torch.empty_like(z)
    yc = torch.empty(B, L, w.conv_C, device=dev, dtype=bf)
    ws_f = dig.new_workspace(B, H, L, dk, dv, device=dev)
    ws_b = dig.new_workspace(B, H, L, dk, dv, backward=True, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i, ev=None, t=None, strm=None):
        """One step: forward + epilogue, backward from the forward's records, SREM conv."""
        t = t or {"q": q, "k": k, "v": v, "z": z, "r": r, "dO": dO, "x": xc, "w": wc,
                  "o": o, "y": y, "dq": dq, "dk": dk_, "dv": dv_, "dla": dla, "yc": yc}
        strm = strm or stream
        mode = i % 4
        if ev:
            ev[0].record(strm)
        dig.dig_gla_fwd(t["q"], t["k"], t["v"], t["z"], w.inv_tau, t["o"], w.grid_h, w.grid_w, mode, ws_f,
                        r=t["r"], y=t["y"], stream=strm)
        if ev:
            ev[1].record(strm)
        # the backward of a training step reuses the forward's gate factors and chunk states
        dig.dig_gla_bwd_saved(t["q"], t["k"], t["v"], t["z"], w.inv_tau, t["dO"], t["dq"], t["dk"], t["dv"], t["dla"],
                              w.grid_h, w.grid_w, mode, ws_f, ws_b, stream=strm)
        if ev:
            ev[2].record(strm)
        dig.dig_srem_reorient_dwconv(t["x"], t["w"], None, t["yc"], mode, stream=strm)
        if ev:
            ev[3].record(strm)

    for i in range(args.warmup):
        flush.fill_(float(i))
        step(i)
    torch.cuda.synchronize()
    for ws in (ws_f, ws_b):
        st = dig.dig_read_status(ws)
        if st != dig.DIG_OK:
            raise RuntimeError("device status after warm-up: %s" % dig.lib.dig_status_string(st).decode())

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))       # evict L2 (outside the events)
            step(i, evs[i])
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    per = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(3)] for i in range(args.steps)])  # ms
    step_ms = max_over_ranks(float(per.sum(axis=1).mean()), world, dev)
    for ws in (ws_f, ws_b):
        st = dig.dig_read_status(ws)
        if st != dig.DIG_OK:
            raise RuntimeError("device status after timing: %s" % dig.lib.dig_status_string(st).decode())

    # end to end: steps through the C ABI with pinned host buffers.  Every step
    # copies all its inputs in (H2D stream), runs on the compute stream and copies
    # all its outputs back (D2H stream).  Two device buffer sets alternate, so a
    # step's copies overlap its neighbours' compute, as a training loop's input
    # feed does; the time is that of the whole run from the first copy in to the
    # last copy out, divided by the steps.
    names_in = ("q", "k", "v", "z", "r", "dO", "x", "w")
    cur = {"q": q, "k": k, "v": v, "z": z, "r": r, "dO": dO, "x": xc, "w": wc,
           "o": o, "y": y, "dq": dq, "dk": dk_, "dv": dv_, "dla": dla, "yc": yc}
    names_out = ("o", "y", "dq", "dk", "dv", "dla", "yc")
    host_in = {n: cur[n].cpu().pin_memory() for n in names_in}
    host_out = {n: cur[n].cpu().pin_memory() for n in names_out}
    sets = [cur, {n: torch.empty_like(a) for n, a in cur.items()}]
    h2d = sum(a.numel() * a.element_size() for a in host_in.values())
    d2h = sum(a.numel() * a.element_size() for a in host_out.values())
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    done = {kind: [torch.cuda.Event(), torch.cuda.Event()] for kind in ("h2d", "cmp", "d2h")}

    def e2e_run(n, first):
        for i in range(first, first + n):
            b, t = i % 2, sets[i % 2]
            if i - first >= 2:
                s_h2d.wait_event(done["cmp"][b])  # step i-2 has consumed this set's inputs
            with torch.cuda.stream(s_h2d):
                for n_ in names_in:
                    t[n_].copy_(host_in[n_], non_blocking=True)
            done["h2d"][b].record(s_h2d)
            stream.wait_event(done["h2d"][b])
            if i - first >= 2:
                stream.wait_event(done["d2h"][b])  # step i-2's outputs are back on the host
            step(i, t=t, strm=stream)
            done["cmp"][b].record(stream)
            s_d2h.wait_event(done["cmp"][b])
            with torch.cuda.stream(s_d2h):
                for n_ in names_out:
                    host_out[n_].copy_(t[n_], non_blocking=True)
            done["d2h"][b].record(s_d2h)

    e2e_steps = max(4, min(args.steps, 12))
    e2e_run(2, 0)  # warm-up
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_h2d)
    e2e_run(e2e_steps, 2)
    e1.record(s_d2h)
    e1.synchronize()
    e2e_step_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)

    # the ops outside the step (backward of the epilogue and the conv, the gate
    # projection and its backward): each timed alone with CUDA events, L2 flushed
    # before every call, on the bench's workload
    # (an error there is reported in the line instead of costing the step's numbers)
    aux_t, aux_err = run_guarded(lambda: time_next_ops(dig, w, dev, stream, o, r, dO, xc, wc, dla, flush,
                                                       args.warmup, max(args.steps, 10)), world, dev)
    aux_t = {op: max_over_ranks(tv, world, dev) for op, tv in aux_t.items()} if aux_err is None else {}

    # the metric's three shapes, each timed the same way (fwd + bwd from the forward's records)
    cfg_t, cfg_err = {}, None
    if not args.no_per_config:
        def _cfgs():
            out = {}
            for idx in PER_CONFIG:
                if idx == WORKLOAD_INDEX:
                    continue
                out[idx] = time_gla_config(dig, idx, dev, stream, flush, args.warmup, max(args.steps, 10), rank)
            return out
        cfg_t, cfg_err = run_guarded(_cfgs, world, dev)
        if cfg_err is None:
            cfg_t = {i: (max_over_ranks(a, world, dev), max_over_ranks(b, world, dev)) for i, (a, b) in cfg_t.items()}

    # the mixer in its block: a synthetic DiG-S/2 block forward at the same shape
    blk_t, blk_err = run_guarded(lambda: time_dig_block(dev, flush, args.warmup, max(args.steps, 10)), world, dev)
    if blk_err is None:
        blk_t = tuple(max_over_ranks(tv, world, dev) for tv in blk_t)

    if rank != 0:
        return None
    hbm, tflops, peak_kind = _peaks()
    algo = algorithmic_bytes(w)
    step_algo = sum(algo[op] for op in STEP_OPS)
    t_f, t_b, t_c = [float(per[:, j].mean()) * 1e-3 for j in range(3)]
    # Each op is a short sequence of this library's kernels launched by one C-ABI
    # call; its roofline is taken over the whole sequence (algorithmic bytes of
    # the op / event-timed duration of the call), the per-kernel shares are in
    # the ncu launch list under profiles/.
    names = {"fwd": ("dig_gla_fwd", OP_SOURCES["fwd"], t_f),
             "bwd": ("dig_gla_bwd_saved", OP_SOURCES["bwd"], t_b),
             "conv": ("dig_srem_reorient_dwconv", OP_SOURCES["conv"], t_c)}
    dom = max(names, key=lambda n: names[n][2])
    kname, srcs, tdom = names[dom]
    achieved = algo[dom] / tdom / 1e9
    tokens = B * L * world
    line = {
        "metric": METRIC, "value": tokens / (step_ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config(w, world),
        "roofline": {"bound": "hbm", "kernel": kname, "kernels": OP_KERNELS[dom], "achieved": achieved, "peak": hbm,
                     "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": _traffic(kname, srcs, 1.0),
                     "algorithmic_bytes": algo[dom], "peak_source": peak_kind,
                     "step_frac": (step_algo / hbm / 1e9) / (step_ms * 1e-3)},
        "ops_us": {"dig_gla_fwd": t_f * 1e6, "dig_gla_bwd_saved": t_b * 1e6, "dig_srem_reorient_dwconv": t_c * 1e6},
        "e2e": {"value": tokens / (e2e_step_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": sum(len(OP_KERNELS[op]) for op in STEP_OPS) * args.steps,
        "clocks": clk.summary(),
        "next_ops": {OP_NAMES[op]: {"us": t * 1e6, "achieved": algo[op] / t / 1e9, "unit": "GB/s",
                                        "frac": algo[op] / t / 1e9 / hbm, "algorithmic_bytes": algo[op],
                                        "traffic": _traffic(OP_NAMES[op], OP_SOURCES[op], 1.0),
                                        "kernels": OP_KERNELS[op]}
                         for op, t in aux_t.items()} if aux_err is None else {"error": aux_err},
    }
    if not args.no_per_config:
        t_step_fb = (t_f, t_b)
        recs = {}
        for idx in PER_CONFIG:
            tf_, tb_ = t_step_fb if idx == WORKLOAD_INDEX else cfg_t.get(idx, (None, None))
            if tf_ is not None:
                recs[inputs.WORKLOADS[idx].name] = per_config_record(idx, tf_, tb_, world, hbm, tflops)
        line["per_config"] = recs if cfg_err is None else dict(recs, error=cfg_err)
        line["per_config_note"] = ("fwd+bwd (dig_gla_fwd + dig_gla_bwd_saved, bf16 outputs) per metric shape; "
                                   "bytes count d log(alpha) once per head; fractions of the measured HBM copy "
                                   "bandwidth")
    if blk_err is None:
        b_us, m_us = blk_t
        line["dig_block"] = {"block_us": b_us, "mixer_us": m_us, "mixer_share": m_us / b_us,
                             "config": "DiG-S/2 block forward at %s (B=%d, L=%d, D=384), scan orders cycling"
                                       % (w.name, B, L),
                             "note": "adaLN + GLA layer (q/k/v/r/out projections by cuBLAS, gate projection, "
                                     "dig_gla_fwd with the Swish*RMSNorm epilogue) + FFN + SREM conv; mixer = the "
                                     "dig_gla_fwd call; random weights, synthetic tokens and conditioning"}
    else:
        line["dig_block"] = {"error": blk_err}
    if world == 1 and not args.no_cpu_baseline:
        tps, dt, cores, n = cpu_sample(w, x, steps=1, min_seconds=10.0)
        import oracle
        nthreads = oracle.num_threads()
        oracle.set_num_threads(1)
        try:
            tps1, dt1, _, n1 = cpu_sample(w, x, steps=1, min_seconds=5.0)
        finally:
            oracle.set_num_threads(nthreads)
        line["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "nproc": os.cpu_count(),
                                "sample": "oracle (fp64 C, OpenMP over heads) on batch element 0 of %s, all heads: "
                                          "%d steps (fwd+epilogue+bwd+conv, %d tokens each, scan modes cycling), "
                                          "%.1f s" % (w.name, n, w.L, dt),
                                "single_thread": {"value": tps1, "unit": "tokens/s", "cores": 1,
                                                  "sample": "the same steps on one thread: %d steps, %.1f s"
                                                            % (n1, dt1)}}
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="skip the L=4096 and L=16384 shapes")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        ap.error("--gpus %d but WORLD_SIZE=%d (launch N>1 with torchrun)" % (args.gpus, world))
    if world > 1 and args.impl == "ours":
        import datetime
        torch.distributed.init_process_group(backend="nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        else:
            line = run_ours(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1 and args.impl == "ours":
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
