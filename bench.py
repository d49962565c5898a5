#!/usr/bin/env python
"""Benchmark of the KDA hot path on B200 — prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline (`value`): chunked-prefill throughput, tokens/s over all N GPUs, on the
H = 96, d = 128 prefill workload (B=4, T=8192, chunk 64, bf16 I/O, fp32 state).
A step is one kda_forward_chunked call over that batch.  The same line carries the
decode workload (B=256, H=96, 20 chained in-place steps; GB/s of state traffic), the
layer decode step with its conv cache on the same shape, and the full layer workload
(B=2, T=16384; tokens/s), each with its roofline.

Multi-GPU: one process per GPU (torchrun); every rank runs its own replica of the
workload (heads and sequences are independent — no data-path collective), a barrier
brackets the timed region and the time is the max over ranks.  `value` is the
aggregate (N x per-rank tokens) / max time: weak scaling.

`--impl reference` times the fp64 CPU oracle (the only other place this file runs
`oracle/`) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA tokens/s (prefill, H=96 d=128) and decode GB/s; fraction of roofline"
PREFILL = "prefill_bf16_B4_T8192_H96_d128"
DECODE = "decode_bf16_B256_H96_d128_x20"
LAYER = "layer_bf16_B2_T16384_H96_d128"
VARLEN = "varlen_bf16_T32768_H96_d128"
L2_BYTES = 126 * 1024 * 1024

# Algorithmic work (per token-head, d = 128, C = 64):
#   prefill reads q, k, v, g (4 x 256 B) and beta (2 B) and writes o (256 B): 1282 B,
#   plus the fp32 state (64 KiB per head) read if given and written at the end.
#   layer reads q/k/v raw (768 B), g raw (256 B), b raw (2 B), gate raw (256 B) and writes
#   out (256 B): 1538 B, plus the final state.
#   decode reads and writes the fp32 state (2 x 64 KiB per head) and moves 1282 B of I/O.
#   chunked FLOPs as issued on full 64-row tiles: 10*C*d + 6*d^2 = 180224 per token-head.
PREFILL_BYTES_PER_TOKEN_HEAD = 1282
LAYER_BYTES_PER_TOKEN_HEAD = 1538
# backward, per token-head at d = 128 (16-token chunks): the state products issued by the
# forward sweep and the reverse sweep (9 d^2 multiply-adds) and the chunk-local ones
# (12 * 16 * d), counted as 2 FLOP per multiply-add
BWD_FLOPS_PER_TOKEN_HEAD = 2 * (9 * 128 * 128 + 12 * 16 * 128)
FLOPS_PER_TOKEN_HEAD = 180224


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--skip", default="", help="comma list of: varlen,backward,decode,layer_decode,layer,e2e,cpu")
    return ap.parse_args()


# ----------------------------------------------------------------------------- infra


def dist_env():
    from gated_delta_rule_155_b200.dist_util import env

    return env()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed regions run."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        sm, smax, reasons, n = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.file.read().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            n += 1
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.file.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": n}


# The source files each profiled kernel is compiled from; a capture stays valid while these
# are unchanged (a change elsewhere in csrc/ does not void it).
KERNEL_SOURCES = {
    "kda_chunk_tc": ("chunk_tc.cu", "tc_common.cuh", "common.cuh", "internal.h"),
    "kda_chunk_tc_packed": ("chunk_tc.cu", "tc_common.cuh", "common.cuh", "internal.h"),
    "kda_layer_tc": ("layer_tc.cu", "tc_common.cuh", "common.cuh", "internal.h"),
    "kda_backward": ("backward.cu", "common.cuh", "internal.h"),
    "kda_decode": ("decode.cu", "common.cuh", "internal.h"),
    "kda_layer_decode": ("layer_decode.cu", "common.cuh", "internal.h"),
}


def kernel_source_sha(kernel=None):
    """16 hex digits of the SHA-256 of `kernel`'s source files (all of csrc/ if None or unknown)."""
    import glob
    csrc = os.path.join(ROOT, "gated_delta_rule_155_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel)
    paths = ([os.path.join(csrc, f) for f in names] if names
             else sorted(glob.glob(os.path.join(csrc, "*"))))
    h = hashlib.sha256()
    for p in paths:
        h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def traffic_for(kernel):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, if the kernel's sources
    have not changed since it was captured; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(kernel)
    if not e or e.get("source_sha") != kernel_source_sha(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- timing


def timed(torch, fn, steps, warmup, stream, barrier, per_launch=True):
    """Run fn() warmup times untimed, then `steps` times bracketed by barrier + sync.
    Returns (total_ms, [per-launch ms]) measured with CUDA events on `stream`."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for a, b in ev:
            if per_launch:
                a.record(stream)
            fn()
            if per_launch:
                b.record(stream)
        t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    total = t0.elapsed_time(t1)
    launches = [a.elapsed_time(b) for a, b in ev] if per_launch else []
    return total, launches


# ----------------------------------------------------------------------------- our arm


def run_ours(args):
    import torch

    ws, rank, local = dist_env()
    skip = set(filter(None, args.skip.split(",")))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if ws > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))

    def barrier():
        if dist is not None:
            dist.barrier()

    from gated_delta_rule_155_b200.dist_util import aggregate_rate
    from gated_delta_rule_155_b200.dist_util import max_over_ranks as _mor

    def max_over_ranks(x):
        return _mor(x, dist, dev)

    from gated_delta_rule_155_b200 import build, inputs
    if rank == 0:
        build.build()
    barrier()
    from gated_delta_rule_155_b200 import kda

    pk = peaks()
    stream = torch.cuda.Stream(device=dev)
    launches_per = {}
    res = {}

    # ------------------------------------------------------------------ prefill (headline)
    w = inputs.WORKLOADS[PREFILL]
    B, T, H, dk, dv = w["B"], w["T"], w["H"], w["dk"], w["dv"]
    d = inputs.prefill_inputs(B, T, H, dk, dv, io=w["io"], seed=w["seed"])
    host = {n: d[n].pin_memory() for n in ("q", "k", "v", "g", "beta")}
    dv_in = {n: host[n].to(dev) for n in host}
    out = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    sT = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)

    def prefill_step():
        kda.kda_forward_chunked(dv_in["q"], dv_in["k"], dv_in["v"], dv_in["g"], dv_in["beta"],
                                None, out, sT, stream=stream)

    clocks = Clocks(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                    else os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])
    clocks.start()
    total, per = timed(torch, prefill_step, args.steps, args.warmup, stream, barrier)
    kda.kda_check_device_error(stream)
    ms = max_over_ranks(total / args.steps)
    launch_ms = max_over_ranks(statistics.mean(per))
    ntok = B * T
    value = aggregate_rate(ntok, ms, ws)
    kname = "kda_chunk_tc" if (w["io"] == "bf16" and dk == 128 and dv == 128) else "kda_chunk_simt"
    bytes_launch = B * T * H * PREFILL_BYTES_PER_TOKEN_HEAD + B * H * dk * dv * 4
    flops_launch = B * T * H * FLOPS_PER_TOKEN_HEAD
    achieved = bytes_launch / (launch_ms / 1e3) / 1e9
    traffic = traffic_for(kname)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": traffic,
                "peak_source": f"{pk['source']} HBM copy (MEASURED_PEAKS.json hbm_gbs)"
                if pk["source"] == "measured" else "fallback 6.65 TB/s",
                "kernel": kname, "launch_ms": round(launch_ms, 4),
                "bytes_per_launch": bytes_launch,
                "tensor": {"flops_per_launch": flops_launch,
                           "achieved_tflops": round(flops_launch / (launch_ms / 1e3) / 1e12, 1),
                           "peak_tflops": pk["bf16_tflops"],
                           "frac": round(flops_launch / (launch_ms / 1e3) / 1e12 / pk["bf16_tflops"], 4)}}
    launches_per["prefill"] = 1

    # e2e through the C ABI from pinned host buffers: every step copies all inputs host -> device,
    # runs the prefill and copies the whole output back.  Sequence by sequence on three streams,
    # so that the copy of sequence b + 1 in, the prefill of sequence b and the copy of sequence
    # b - 1 out overlap (host->device and device->host use separate copy engines).
    e2e = None
    if "e2e" not in skip:
        out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(B)]
        ev_done = [torch.cuda.Event() for _ in range(B)]

        def e2e_step():
            s_in.wait_stream(stream)       # after the step's start event
            for b in range(B):
                with torch.cuda.stream(s_in):
                    for n in host:
                        dv_in[n][b].copy_(host[n][b], non_blocking=True)
                    ev_in[b].record(s_in)
                stream.wait_event(ev_in[b])
                kda.kda_forward_chunked(dv_in["q"][b:b + 1], dv_in["k"][b:b + 1], dv_in["v"][b:b + 1],
                                        dv_in["g"][b:b + 1], dv_in["beta"][b:b + 1], None, out[b:b + 1],
                                        sT[b:b + 1], stream=stream)
                ev_done[b].record(stream)
                s_out.wait_event(ev_done[b])
                with torch.cuda.stream(s_out):
                    out_host[b].copy_(out[b], non_blocking=True)
            stream.wait_stream(s_out)      # before the step's end event

        ne = max(1, args.e2e_steps)
        tot_e, _ = timed(torch, e2e_step, ne, 1, stream, barrier, per_launch=False)
        launches_per["e2e"] = ne * B
        ms_e = max_over_ranks(tot_e / ne)
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        e2e = {"value": round(ws * ntok / (ms_e / 1e3), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": out.numel() * out.element_size(),
               "ms_per_step": round(ms_e, 3)}
    del dv_in, out, sT, d
    torch.cuda.empty_cache()

    # ------------------------------------------------------------------ packed variable length
    if "varlen" not in skip:
        wv = inputs.WORKLOADS[VARLEN]
        lens = inputs.packed_lengths(wv["total"], wv["max_len"], wv["seed"])
        dl = inputs.varlen_inputs(lens, wv["H"], wv["dk"], wv["dv"], io=wv["io"], seed=wv["seed"])
        xv = {n: dl[n].to(dev) for n in ("q", "k", "v", "g", "beta", "cu_seqlens")}
        Tt, Hv, Nv = wv["total"], wv["H"], len(lens)
        ov = torch.empty((Tt, Hv, wv["dv"]), dtype=torch.bfloat16, device=dev)
        sv = torch.empty((Nv, Hv, wv["dk"], wv["dv"]), dtype=torch.float32, device=dev)

        def varlen_step():
            kda.kda_forward_chunked_varlen(xv["q"], xv["k"], xv["v"], xv["g"], xv["beta"], xv["cu_seqlens"],
                                           None, ov, sv, stream=stream)

        total_v, per_v = timed(torch, varlen_step, args.steps, args.warmup, stream, barrier)
        kda.kda_check_device_error(stream)
        ms_v = max_over_ranks(total_v / args.steps)
        lms_v = max_over_ranks(statistics.mean(per_v))
        bytes_v = Tt * Hv * PREFILL_BYTES_PER_TOKEN_HEAD + Nv * Hv * wv["dk"] * wv["dv"] * 4
        ach_v = bytes_v / (lms_v / 1e3) / 1e9
        res["varlen"] = {
            "workload": f"kda_forward_chunked_varlen, {Tt} tokens packed as {Nv} sequences of "
                        f"{min(lens)}..{max(lens)} tokens (uniform 1..{wv['max_len']}, seed {wv['seed']}), "
                        f"H={Hv} dk=dv=128 bf16, zero initial state",
            "value": round(aggregate_rate(Tt, ms_v, ws), 1), "unit": "tokens/s", "ms_per_step": round(ms_v, 4),
            "roofline": {"bound": "hbm", "achieved": round(ach_v, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(ach_v / pk["hbm_gbs"], 4), "traffic": traffic_for("kda_chunk_tc_packed"),
                         "kernel": "kda_chunk_tc (packed)", "launch_ms": round(lms_v, 4), "bytes_per_launch": bytes_v}}
        launches_per["varlen"] = 1
        del xv, ov, sv, dl
        torch.cuda.empty_cache()

    # ------------------------------------------------------------------ backward (gradients)
    if "backward" not in skip:
        wb = inputs.WORKLOADS[PREFILL]
        Bb, Tb, Hb, db_ = wb["B"], wb["T"], wb["H"], wb["dk"]
        dbk = inputs.prefill_inputs(Bb, Tb, Hb, db_, db_, io=wb["io"], seed=wb["seed"])
        xb = {n: dbk[n].to(dev) for n in ("q", "k", "v", "g", "beta")}
        gen = torch.Generator().manual_seed(7)
        dO_b = torch.randn((Bb, Tb, Hb, db_), generator=gen).to(torch.bfloat16).to(dev)
        grads = {n: torch.empty_like(xb[m]) for n, m in (("dq", "q"), ("dk", "k"), ("dv", "v"), ("dg", "g"),
                                                          ("dbeta", "beta"))}
        ds0 = torch.empty((Bb, Hb, db_, db_), dtype=torch.float32, device=dev)
        ws_b = torch.empty(kda.kda_backward_workspace_size(Bb, Tb, Hb, db_, db_, torch.bfloat16),
                           dtype=torch.uint8, device=dev)

        def backward_step():
            kda.kda_backward_chunked(xb["q"], xb["k"], xb["v"], xb["g"], xb["beta"], dO_b, None, None,
                                     grads=grads, d_initial_state=ds0, workspace=ws_b, stream=stream)

        nb = max(1, args.steps // 4)
        total_b, per_b = timed(torch, backward_step, nb, max(1, args.warmup // 3), stream, barrier)
        kda.kda_check_device_error(stream)
        ms_b = max_over_ranks(total_b / nb)
        lms_b = max_over_ranks(statistics.mean(per_b))
        flops_b = Bb * Tb * Hb * BWD_FLOPS_PER_TOKEN_HEAD
        alu_peak = 148 * 128 * 2 * 1.965e9 / 1e12
        ach_b = flops_b / (lms_b / 1e3) / 1e12
        res["backward"] = {
            "workload": "kda_backward_chunked B=4 T=8192 H=96 dk=dv=128 bf16 (the prefill workload, "
                        "dO ~ N(0,1) bf16, zero initial state), fp32 arithmetic on CUDA cores",
            "value": round(aggregate_rate(Bb * Tb, ms_b, ws), 1), "unit": "tokens/s", "ms_per_step": round(ms_b, 3),
            "roofline": {"bound": "alu", "achieved": round(ach_b, 2), "peak": round(alu_peak, 1), "unit": "TFLOP/s",
                         "frac": round(ach_b / alu_peak, 4), "traffic": traffic_for("kda_backward"),
                         "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x 1965 MHz",
                         "kernel": "kda_backward", "launch_ms": round(lms_b, 3), "flops_per_launch": flops_b,
                         "workspace_bytes": ws_b.numel()}}
        launches_per["backward"] = nb
        del xb, dO_b, grads, ds0, ws_b, dbk
        torch.cuda.empty_cache()

    # ------------------------------------------------------------------ decode
    if "decode" not in skip:
        wd = inputs.WORKLOADS[DECODE]
        Bd, Hd = wd["B"], wd["H"]
        dd = inputs.decode_inputs(Bd, Hd, wd["dk"], wd["dv"], steps=wd["steps"], io=wd["io"],
                                  seed=wd["seed"], s0_std=wd["s0_std"])
        state = dd["state"].to(dev)
        steps_in = [{n: x[n].to(dev) for n in x} for x in dd["steps"]]
        od = torch.empty((Bd, Hd, wd["dv"]), dtype=torch.bfloat16, device=dev)

        def decode_run():
            for x in steps_in:
                kda.kda_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], state, od, stream=stream)

        reps = max(1, args.steps // 10)
        total_d, per_d = timed(torch, decode_run, reps, max(1, args.warmup // 3), stream, barrier,
                               per_launch=False)
        kda.kda_check_device_error(stream)
        ms_d = max_over_ranks(total_d / (reps * wd["steps"]))
        state_bytes = 2 * Bd * Hd * wd["dk"] * wd["dv"] * 4
        io_bytes = Bd * Hd * (3 * wd["dk"] * 2 + wd["dv"] * 2 * 2 + 2)
        gbs = (state_bytes + io_bytes) / (ms_d / 1e3) / 1e9
        res["decode"] = {
            "workload": "kda_decode_step B=256 H=96 dk=dv=128 bf16 I/O, fp32 state in place, 20 chained steps",
            "value": round(ws * gbs, 1), "unit": "GB/s", "ms_per_step": round(ms_d, 4),
            "tokens_per_s": round(ws * Bd / (ms_d / 1e3), 1),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                         "frac_of_8TBs": round(gbs / 8000.0, 4), "traffic": traffic_for("kda_decode"),
                         "kernel": "kda_decode", "bytes_per_launch": state_bytes + io_bytes,
                         "note": "the state is read and written in place (same lines), which a plain "
                                 "copy's read-A/write-B peak does not model; frac can exceed 1"}}
        launches_per["decode"] = wd["steps"] * reps
        del state, steps_in, od, dd
        torch.cuda.empty_cache()

    # ------------------------------------------------------------------ layer decode (conv cache)
    if "layer_decode" not in skip:
        wd = inputs.WORKLOADS[DECODE]
        Bd, Hd, dd_ = wd["B"], wd["H"], wd["dk"]
        Ld = inputs.layer_inputs(Bd, wd["steps"], Hd, dd_, dd_, io=wd["io"], seed=wd["seed"], conv_std=0.5,
                                 s0_std=wd["s0_std"])
        to = lambda x: None if x is None else x.contiguous().to(dev)
        state = to(Ld["s0"])
        caches = [torch.zeros((Bd, 3, Hd * dd_), dtype=torch.bfloat16, device=dev) for _ in range(3)]
        fixed = {n: to(Ld[n]) for n in ("conv_q", "conv_k", "conv_v", "A_log", "dt_bias", "o_norm_w")}
        steps_in = [{n: to(Ld[n][:, t]) for n in ("q_raw", "k_raw", "v_raw", "g_raw", "b_raw", "o_gate_raw")}
                    for t in range(wd["steps"])]
        od = torch.empty((Bd, Hd, dd_), dtype=torch.bfloat16, device=dev)

        def layer_decode_run():
            for x in steps_in:
                kda.kda_layer_decode_step(x["q_raw"], x["k_raw"], x["v_raw"], fixed["conv_q"], fixed["conv_k"],
                                          fixed["conv_v"], *caches, x["g_raw"], fixed["A_log"], fixed["dt_bias"],
                                          x["b_raw"], x["o_gate_raw"], state, fixed["o_norm_w"], out=od,
                                          stream=stream)

        reps = max(1, args.steps // 10)
        total_ld, _ = timed(torch, layer_decode_run, reps, max(1, args.warmup // 3), stream, barrier,
                            per_launch=False)
        kda.kda_check_device_error(stream)
        ms_ld = max_over_ranks(total_ld / (reps * wd["steps"]))
        state_bytes = 2 * Bd * Hd * dd_ * dd_ * 4
        # raw q, k, v, g, gate and out (bf16), beta, the three caches read and written
        io_bytes = Bd * Hd * (6 * dd_ * 2 + 2 + 2 * 3 * 3 * dd_ * 2)
        gbs = (state_bytes + io_bytes) / (ms_ld / 1e3) / 1e9
        res["layer_decode"] = {
            "workload": "kda_layer_decode_step B=256 H=96 dk=dv=128 bf16 (conv cache + prologue + recurrence + "
                        "epilogue), fp32 state in place, 20 chained steps",
            "value": round(ws * gbs, 1), "unit": "GB/s", "ms_per_step": round(ms_ld, 4),
            "tokens_per_s": round(ws * Bd / (ms_ld / 1e3), 1),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                         "frac_of_8TBs": round(gbs / 8000.0, 4), "traffic": traffic_for("kda_layer_decode"),
                         "kernel": "kda_layer_decode", "bytes_per_launch": state_bytes + io_bytes,
                         "note": "the state is read and written in place (same lines), which a plain "
                                 "copy's read-A/write-B peak does not model; frac can exceed 1"}}
        launches_per["layer_decode"] = wd["steps"] * reps
        del state, caches, steps_in, od, Ld, fixed
        torch.cuda.empty_cache()

    # ------------------------------------------------------------------ layer
    if "layer" not in skip:
        wl = inputs.WORKLOADS[LAYER]
        Bl, Tl, Hl = wl["B"], wl["T"], wl["H"]
        L = inputs.layer_inputs(Bl, Tl, Hl, wl["dk"], wl["dv"], io=wl["io"], seed=wl["seed"],
                                conv_std=wl["conv_std"])
        Ld = {n: (None if L[n] is None else L[n].to(dev)) for n in L}
        ol = torch.empty((Bl, Tl, Hl, wl["dv"]), dtype=torch.bfloat16, device=dev)
        sl = torch.empty((Bl, Hl, wl["dk"], wl["dv"]), dtype=torch.float32, device=dev)
        need = kda.kda_layer_workspace_size(Bl, Tl, Hl, wl["dk"], wl["dv"], torch.bfloat16)
        wsp = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)

        def layer_step():
            kda.kda_layer_forward(Ld["q_raw"], Ld["k_raw"], Ld["v_raw"], Ld["conv_q"], Ld["conv_k"],
                                  Ld["conv_v"], Ld["g_raw"], Ld["A_log"], Ld["dt_bias"], Ld["b_raw"],
                                  Ld["o_gate_raw"], Ld["o_norm_w"], out=ol, final_state=sl,
                                  workspace=wsp if need else None, stream=stream)

        nl = max(1, args.steps // 4)
        total_l, per_l = timed(torch, layer_step, nl, max(1, args.warmup // 2), stream, barrier)
        kda.kda_check_device_error(stream)
        ms_l = max_over_ranks(total_l / nl)
        bytes_l = Bl * Tl * Hl * LAYER_BYTES_PER_TOKEN_HEAD + Bl * Hl * wl["dk"] * wl["dv"] * 4
        gbs_l = bytes_l / (ms_l / 1e3) / 1e9
        res["layer"] = {
            "workload": "kda_layer_forward B=2 T=16384 H=96 dk=dv=128 bf16 (conv4+SiLU, l2norm, gate, "
                        "beta, chunked delta rule, RMSNorm x sigmoid gate)",
            "value": round(ws * Bl * Tl / (ms_l / 1e3), 1), "unit": "tokens/s",
            "ms_per_step": round(ms_l, 3), "workspace_bytes": need,
            "roofline": {"bound": "hbm", "achieved": round(gbs_l, 1), "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs_l / pk["hbm_gbs"], 4),
                         "traffic": traffic_for("kda_layer_tc") if need == 0 else None,
                         "bytes_per_step": bytes_l}}
        launches_per["layer"] = (3 if need else 1) * nl
        del Ld, ol, sl, wsp, L
        torch.cuda.empty_cache()

    clk = clocks.stop()

    cpu = None
    if rank == 0 and ws == 1 and "cpu" not in skip:
        cpu = cpu_baseline_prefill()
        if "decode" in res:
            res["decode"]["cpu_baseline"] = cpu_baseline_decode()
        if "layer" in res:
            res["layer"]["cpu_baseline"] = cpu_baseline_layer()

    gpu_launches = args.steps * (launches_per["prefill"] + launches_per.get("varlen", 0)) + \
        launches_per.get("backward", 0) + launches_per.get("decode", 0) + launches_per.get("layer_decode", 0) + \
        launches_per.get("layer", 0) + launches_per.get("e2e", 0)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if kname == "kda_chunk_tc" else "f32", "data": "synthetic",
        "config": {"workload": "kda_forward_chunked B=4 T=8192 H=96 dk=dv=128 chunk=64, bf16 q/k/v/g/beta, "
                               "fp32 state", "B": B, "T": T, "H": H, "dk": dk, "dv": dv, "chunk": 64,
                   "l2": "inputs (4.03 GB per step) are larger than L2 (126 MB); no flush",
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": gpu_launches,
        "clocks": clk, **res,
    }
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- oracle (CPU)


def cpu_baseline_prefill(min_seconds=10.0, max_reps=40):
    """The fp64 oracle, as it stands, on a bounded sample of the prefill workload: n heads of
    the T = 8192 sequences (heads are independent), all host threads, run repeatedly until
    about `min_seconds` of CPU work have been timed.  Returns the cpu_baseline object; value
    in tokens/s of the full 96-head workload."""
    import oracle
    from gated_delta_rule_155_b200 import inputs

    w = inputs.WORKLOADS[PREFILL]
    cores = oracle.max_threads()
    nh = int(min(96, max(8, 2 * cores)))
    d = inputs.prefill_inputs(1, w["T"], nh, w["dk"], w["dv"], io=w["io"], seed=w["seed"])
    arrs = [d[n].double().numpy() for n in ("q", "k", "v", "g", "beta")]
    reps, total = 0, 0.0
    while reps < max_reps and (total < min_seconds or reps == 0):
        t0 = time.perf_counter()
        oracle.recurrent(*arrs, None, nthreads=cores)
        total += time.perf_counter() - t0
        reps += 1
    token_heads = nh * w["T"] * reps
    return {"value": round(token_heads / total / w["H"], 2), "unit": "tokens/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{reps} runs of {nh} heads x T={w['T']} of the prefill workload (fp64 token "
                      f"recurrence, {token_heads} token-heads, {total:.1f} s); tokens/s = token-heads/s / 96"}


def cpu_baseline_decode(min_seconds=3.0, max_reps=20):
    """The fp64 oracle's decode step on a sample of the decode workload: 4 of the 256
    sequences, all 96 heads, the 20 chained steps; repeated until about `min_seconds`.
    Returns the cpu_baseline object in GB/s of the same algorithmic bytes per (b, h) step
    (state read and written, and the I/O) and in tokens/s."""
    import oracle
    from gated_delta_rule_155_b200 import inputs

    w = inputs.WORKLOADS[DECODE]
    nb = 4
    dd = inputs.decode_inputs(nb, w["H"], w["dk"], w["dv"], steps=w["steps"], io=w["io"], seed=w["seed"],
                              s0_std=w["s0_std"])
    steps = [[x[n].double().numpy() for n in ("q", "k", "v", "g", "beta")] for x in dd["steps"]]
    cores = oracle.max_threads()
    reps, total = 0, 0.0
    while reps < max_reps and (total < min_seconds or reps == 0):
        st = dd["state"].double().numpy()
        t0 = time.perf_counter()
        for x in steps:
            _, st = oracle.decode(*x, st, nthreads=cores)
        total += time.perf_counter() - t0
        reps += 1
    head_steps = nb * w["H"] * w["steps"] * reps
    per = 2 * w["dk"] * w["dv"] * 4 + (3 * w["dk"] * 2 + w["dv"] * 2 * 2 + 2)
    return {"value": round(head_steps * per / total / 1e9, 3), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "tokens_per_s": round(head_steps / total / w["H"], 1),
            "sample": f"{reps} runs of {nb} sequences x {w['H']} heads x {w['steps']} chained steps of the decode "
                      f"workload (fp64 decode step, {total:.1f} s); GB/s of the kernel's algorithmic bytes"}


def cpu_baseline_layer(min_seconds=5.0, max_reps=20):
    """The fp64 layer oracle (conv + SiLU, L2-norm, gate, beta, token recurrence, RMSNorm x
    sigmoid gate) on the first 8 heads of one T = 16384 sequence of the layer workload;
    repeated until about `min_seconds`.  tokens/s = token-heads/s / 96."""
    import oracle
    from gated_delta_rule_155_b200 import inputs

    w = inputs.WORKLOADS[LAYER]
    nh, d = 8, w["dk"]
    L = inputs.layer_inputs(1, w["T"], nh, d, w["dv"], io=w["io"], seed=w["seed"], conv_std=w["conv_std"])
    arrs = [None if L[n] is None else L[n].double().numpy()
            for n in ("q_raw", "k_raw", "v_raw", "conv_q", "conv_k", "conv_v", "g_raw", "A_log", "dt_bias",
                      "b_raw", "o_gate_raw", "o_norm_w")]
    cores = oracle.max_threads()
    reps, total = 0, 0.0
    while reps < max_reps and (total < min_seconds or reps == 0):
        t0 = time.perf_counter()
        oracle.layer(*arrs, nthreads=cores)
        total += time.perf_counter() - t0
        reps += 1
    token_heads = nh * w["T"] * reps
    return {"value": round(token_heads / total / w["H"], 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} runs of {nh} heads x T={w['T']} of the layer workload (fp64 layer core, "
                      f"{token_heads} token-heads, {total:.1f} s); tokens/s = token-heads/s / {w['H']}"}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    from gated_delta_rule_155_b200 import inputs

    w = inputs.WORKLOADS[PREFILL]
    cores = oracle.max_threads()
    nh = int(min(96, max(4, cores)))
    d = inputs.prefill_inputs(1, w["T"], nh, w["dk"], w["dv"], io=w["io"], seed=w["seed"])
    arrs = [d[n].double().numpy() for n in ("q", "k", "v", "g", "beta")]
    for _ in range(args.warmup):
        oracle.recurrent(*arrs, None, nthreads=cores)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.recurrent(*arrs, None, nthreads=cores)
        times.append(time.perf_counter() - t0)
    mean = statistics.mean(times)
    token_heads = nh * w["T"]
    value = token_heads / mean / w["H"]
    sample = (f"{nh} heads x T={w['T']} of the prefill workload per step (fp64 token recurrence); "
              "tokens/s = token-heads/s / 96")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(mean * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "kda_forward_chunked B=4 T=8192 H=96 dk=dv=128 chunk=64, bf16 q/k/v/g/beta, "
                               "fp32 state", "B": w["B"], "T": w["T"], "H": w["H"], "dk": 128, "dv": 128,
                   "chunk": 64, "sample": sample},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
