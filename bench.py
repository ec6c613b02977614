#!/usr/bin/env python
"""Benchmark of the HiF4 W4A4 hot path on B200 — one JSON line on rank 0.

Headline workload: the Wan2.2-14B-shaped FFN, per GPU 57600 tokens x 5120 ->
13824 (tanh-GELU) -> 5120, both linears W4A4 HiF4 fake-quantized with a
1 %-of-K protected-channel mask from the tail-percentile rule.  One step =
fake quantization of X (hif4_fake_quantize), W1 decode (hif4_weight_decode),
the first tcgen05 GEMM with bias, GELU and the fake quantization of the
hidden activation in its epilogue (hif4_gemm_bf16_fq), W2 decode, the second
GEMM (hif4_gemm_bf16) — the kernels, in the order, that hif4_ffn_w4a4
launches.  value = FLOPs of both GEMMs (2 M N K each) over all ranks /
max-over-ranks step time.

The same JSON line carries the other rows of the path, each timed the same
way: the quantizer sweep (quantize, dequantize at 2^20 ... 2^30 BF16 values,
powers of 4; the 2^30 entry repeated as "quantize" / "dequantize") and the
calibration workload (16 x 14400 tokens x 5120 channels),
as GB/s of algorithmic bytes and a fraction of HBM roofline; and HiGPTQ
scheme one on W1 (13824 x 5120, Hessian of the step's activations), as
TFLOP/s against a composite roofline of its split-TF32 error-feedback
updates and its FP64 factor.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hif4|reference]

Multi-GPU (torchrun, one process per GPU): tokens are sharded (each rank its
own 57600-token batch, weights replicated), no data-path collective; weak
scaling.  ``--impl reference`` times the CPU oracle (the only reference this
method has) on a bounded token sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4 HiF4 linear TFLOP/s & quantizer GB/s at Wan2.2 shapes, % of roofline"
TOKENS, D_MODEL, D_FFN = 57600, 5120, 13824
CALIB_T, CALIB_C = 16 * 14400, 5120
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
DATASHEET = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}                # B200 datasheet figures, for context

# DRAM traffic per launch from an ncu capture, keyed by the SHA-256 (first 16
# hex digits) of the kernel source it was taken on; stale entries read as null.
NCU_TRAFFIC = {
    # the FFN's two GEMMs on 8192 of the 57600 tokens (one ncu pass, dram__bytes_read/write.sum):
    # GEMM 1 (fused fake-quant epilogue) read 660 MB + wrote 207 MB, GEMM 2 read 1284 MB + wrote 81 MB;
    # every term grows with the rows (A and C once, the weight once per 2048 rows), so x 57600 / 8192:
    # 6.10 and 9.60 GB, mean per launch
    ("gemm", "959d655b55f5bfa5"): 7.847e+09,
}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=40)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["hif4", "reference"], default="hif4")
    p.add_argument("--no-components", action="store_true", help="skip the quantizer / calibration lines")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-sample-rows", type=int, default=8)
    p.add_argument("--tokens", type=int, default=TOKENS, help="tokens per GPU (default: Wan2.2 57600)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0)), "source": "measured"}
    except Exception:
        return dict(FALLBACK, source="fallback")


def src_hash(*names):
    h = hashlib.sha256()
    for n in names:
        h.update(open(os.path.join(ROOT, "block_floating_point_hif4_b200", "csrc", n), "rb").read())
    return h.hexdigest()[:16]


# --------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples every 50 ms; started before the warm-up (the tool
    takes a moment to start) and filtered to the timed region by timestamp."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.t0 = self.t1 = None

    def mark_start(self):
        import datetime
        self.t0 = datetime.datetime.now()

    def mark_end(self):
        import datetime
        self.t1 = datetime.datetime.now()

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.uuid, "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        import datetime
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f")
                if self.t0 and self.t1 and not (self.t0 <= ts <= self.t1):
                    continue
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ CPU oracle

def oracle_ffn_sample(rows: int, seed: int = 3, threads: int | None = None, steps: int = 1, prep=None):
    """Time the CPU oracle on `rows` tokens of the FFN workload (numpy-seeded
    inputs of the same recipe).  Per step: activation fake quantization, the
    full weight decode of W1 and W2, both FP64 products, the GELU, the BF16
    rounding and fake quantization of the hidden activation.
    Returns (flop per step, seconds per step list, threads)."""
    import numpy as np

    import oracle
    from block_floating_point_hif4_b200 import workloads as wl
    threads = threads or max(1, len(os.sched_getaffinity(0)))
    if prep is None:
        d = wl.ffn(M=max(rows, 2048), seed=seed)
        x = d["x"]
        p1 = oracle.percentile(x, threads=threads)
        _, m1, _ = oracle.channel_mask(p1)
        idx1 = np.nonzero(m1)[0].astype(np.int32)
        h = wl.ffn_hidden(2048)
        p2 = oracle.percentile(h, threads=threads)
        _, m2, _ = oracle.channel_mask(p2)
        idx2 = np.nonzero(m2)[0].astype(np.int32)
        c1, mt1, _ = oracle.quantize(d["w1"], m1)
        c2, mt2, _ = oracle.quantize(d["w2"], m2)
        prep = dict(x=x[:rows].copy(), idx1=idx1, idx2=idx2, c1=c1, mt1=mt1, c2=c2, mt2=mt2,
                    wm1=np.ascontiguousarray(d["w1"][:, idx1]), wm2=np.ascontiguousarray(d["w2"][:, idx2]))
    P = prep
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        w1 = _threaded_weight_hat(P["c1"], P["mt1"], D_FFN, D_MODEL, P["idx1"], P["wm1"], threads)
        w2 = _threaded_weight_hat(P["c2"], P["mt2"], D_MODEL, D_FFN, P["idx2"], P["wm2"], threads)
        xh = oracle.fake_quantize(P["x"], P["idx1"])
        hid = oracle.linear(xh, w1, None, gelu=True, threads=threads)
        hh = oracle.fake_quantize(oracle.round_bf16(hid), P["idx2"])
        oracle.linear(hh, w2, None, threads=threads)
        times.append(time.perf_counter() - t0)
    flop = 2 * 2.0 * rows * D_MODEL * D_FFN
    return flop, times, threads, prep


def _threaded_weight_hat(codes, meta, N, K, idx, wm, threads):
    import numpy as np

    import oracle
    out = np.empty((N, K), np.float64)
    bounds = np.linspace(0, N, threads + 1).astype(int)

    def run(i):
        a, b = bounds[i], bounds[i + 1]
        if b > a:
            out[a:b] = oracle.weight_hat(codes[a:b], meta[a:b], b - a, K, idx, wm[a:b])
    ts = [threading.Thread(target=run, args=(i,)) for i in range(threads)]
    [t.start() for t in ts]
    [t.join() for t in ts]
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    rows = args.cpu_sample_rows
    flop, times, threads, prep = oracle_ffn_sample(rows, steps=1)           # setup + first step
    _, warm, _, _ = oracle_ffn_sample(rows, steps=max(0, args.warmup - 1), prep=prep)
    _, timed, _, _ = oracle_ffn_sample(rows, steps=args.steps, prep=prep)
    sec = sum(timed) / len(timed)
    value = flop / sec / 1e12
    sample = ("%d of %d tokens per step of the FFN workload (weight decode of W1, W2 in full each step), "
              "FP64 oracle" % (rows, args.tokens))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(args):
    return {"workload": "wan22_ffn_%dx%dx%d" % (args.tokens, D_MODEL, D_FFN), "tokens_per_gpu": args.tokens,
            "d_model": D_MODEL, "d_ffn": D_FFN, "activation": "tanh-GELU",
            "protected_channels": "1%% of K per linear (%d, %d) from the tail-percentile rule"
                                  % (D_MODEL // 100, D_FFN // 100),
            "l2": "inputs larger than L2 (X %.0f MB, H %.0f MB per GPU)" % (args.tokens * D_MODEL * 2 / 1e6,
                                                                          args.tokens * D_FFN * 2 / 1e6),
            "parallelism": "dp%d (tokens sharded, weights replicated, no collective)" % args.gpus}


# ---------------------------------------------------------------- GPU arm

def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE %d" % (args.gpus, world))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    from block_floating_point_hif4_b200 import binding as H
    from block_floating_point_hif4_b200 import workloads as wl
    H.lib()
    P = peaks()
    M, D, F = args.tokens, D_MODEL, D_FFN
    stream = torch.cuda.current_stream()

    from block_floating_point_hif4_b200 import sharding

    def barrier():
        sharding.barrier(dev)

    def max_over_ranks(v: float) -> float:
        return sharding.max_over_ranks(v, dev)

    # ---- setup (untimed): inputs, calibration, weight quantization
    x, _ = wl.device_rows(M, D, seed=sharding.rank_seed(3, rank), device=dev)
    w1 = wl.device_weight(F, D, 0.015, seed=31, device=dev)
    w2 = wl.device_weight(D, F, 0.015, seed=32, device=dev)
    _, _, mask1, idx1 = H.calib_percentile_mask(x)
    w1c, w1m = H.quantize(w1, mask1)
    w1k = w1[:, idx1.long()].contiguous()
    hbuf = torch.empty(M, F, dtype=torch.bfloat16, device=dev)
    ybuf = torch.empty(M, D, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(H.linear_w4a4_workspace(M, max(D, F), max(D, F)), dtype=torch.uint8, device=dev)
    H.linear_w4a4(x, w1c, w1m, F, idx1, w1k, None, gelu=True, out=hbuf, workspace=ws)
    _, _, mask2, idx2 = H.calib_percentile_mask(hbuf)
    del hbuf, ws
    w2c, w2m = H.quantize(w2, mask2)
    w2k = w2[:, idx2.long()].contiguous()
    del w1, w2
    xhat1 = torch.empty(M, D, dtype=torch.bfloat16, device=dev)
    xhat2 = torch.empty(M, F, dtype=torch.bfloat16, device=dev)
    what1 = torch.empty(F, D, dtype=torch.bfloat16, device=dev)
    what2 = torch.empty(D, F, dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()

    stages = ["fake_quant_1", "weight_decode_1", "gemm_1_gelu_fq", "weight_decode_2", "gemm_2"]

    def step(evs=None):
        def mark(i):
            if evs is not None:
                evs[i].record(stream)
        mark(0)
        H.fake_quantize(x, mask1, out=xhat1, status=status)
        mark(1)
        H.weight_decode(w1c, w1m, F, D, idx1, w1k, out=what1, status=status)
        mark(2)
        H.gemm_bf16_fq(xhat1, what1, None, gelu=True, out_chan_mask=mask2, out=xhat2, status=status)
        mark(3)
        H.weight_decode(w2c, w2m, D, F, idx2, w2k, out=what2, status=status)
        mark(4)
        H.gemm_bf16(xhat2, what2, None, gelu=False, out=ybuf, status=status)
        mark(5)

    # fake-quant, 2 x (dequant + column scatter), 2 x GEMM
    launches_per_step = 1 + 2 * 2 + 2

    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(uuid) as clk:
        for _ in range(args.warmup):
            step()
        barrier()
        clk.mark_start()
        t_start.record(stream)
        for k in range(args.steps):
            step(evs[k])
        t_end.record(stream)
        barrier()
        clk.mark_end()
    ms_total = t_start.elapsed_time(t_end)
    ms_step = max_over_ranks(ms_total / args.steps)
    per_stage = {s: [] for s in stages}
    for k in range(args.steps):
        for i, s in enumerate(stages):
            per_stage[s].append(evs[k][i].elapsed_time(evs[k][i + 1]))
    stage_ms = {s: statistics.mean(v) for s, v in per_stage.items()}
    if H.get_status(status) not in (0, H.ERR_NONFINITE):
        raise SystemExit("device status word reports an error: %d" % H.get_status(status))

    flop_gemm = 2.0 * M * D * F                      # each of the two GEMMs
    flop_step = 2 * flop_gemm
    value = sharding.aggregate_throughput(flop_step, world, ms_step * 1e-3) / 1e12
    gemm_ms = max_over_ranks((stage_ms["gemm_1_gelu_fq"] + stage_ms["gemm_2"]) / 2)
    achieved = flop_gemm / (gemm_ms * 1e-3) / 1e12
    # The timed region is a burst (steps x step time, well under the seconds-long
    # loop the sustained figure was taken over): the burst peak is the denominator.
    peak = P["bf16_tflops"]
    gh = src_hash("hif4_gemm.cuh", "hif4_sm100.cuh", "hif4_encode.cuh", "hif4_internal.cuh")
    traffic = NCU_TRAFFIC.get(("gemm", gh))
    timed_s = ms_step * args.steps * 1e-3
    roofline = {"kernel": "k_gemm (hif4_gemm_bf16_fq, hif4_gemm_bf16)", "bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                "peak_source": "%s bf16 burst (timed region %.2f s)" % (P["source"], timed_s),
                "peak_sustained": P["bf16_tflops_sustained"],
                "frac_sustained": achieved / P["bf16_tflops_sustained"],
                "algorithmic_per_launch": "2*M*N*K = %.4g FLOP" % flop_gemm,
                "avg_launch_ms": gemm_ms, "frac_datasheet": achieved / DATASHEET["bf16_tflops"]}

    share = {s: v / sum(stage_ms.values()) for s, v in stage_ms.items()}
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(args),
            "roofline": roofline, "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(),
            "stages_ms": {s: round(v, 4) for s, v in stage_ms.items()},
            "stage_share": {s: round(v, 4) for s, v in share.items()}}

    # ---- e2e: the public FFN call on pinned host buffers (hif4_ffn_w4a4_host):
    # every step copies X in and Y out; the library overlaps those copies with
    # the compute chunk by chunk.  Timed on the caller's stream, which the call
    # completes only after the last row of Y is on the host.
    if not args.no_e2e:
        xh = torch.empty(M, D, dtype=torch.bfloat16, pin_memory=True)
        xh.copy_(x)
        yh = torch.empty(M, D, dtype=torch.bfloat16, pin_memory=True)
        ws = torch.empty(H.ffn_w4a4_host_workspace(M, D, F), dtype=torch.uint8, device=dev)

        def e2e_step():
            H.ffn_w4a4_host(xh, w1c, w1m, F, w2c, w2m, idx1, w1k, None, idx2, w2k, None, out=yh, workspace=ws,
                            status=status)
        for _ in range(args.warmup):
            e2e_step()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
        # the copies alone (same bytes, both directions at once, no compute):
        # the end-to-end bound when they take longer than the compute
        yd = torch.empty(M, D, dtype=torch.bfloat16, device=dev)
        xd = torch.empty(M, D, dtype=torch.bfloat16, device=dev)
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(args.steps):
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)
            with torch.cuda.stream(s_in):
                xd.copy_(xh, non_blocking=True)
            with torch.cuda.stream(s_out):
                yh.copy_(yd, non_blocking=True)
            stream.wait_stream(s_in)
            stream.wait_stream(s_out)
        c1.record(stream)
        barrier()
        copy_ms = max_over_ranks(c0.elapsed_time(c1) / args.steps)
        line["e2e"] = {"value": world * flop_step / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                       "h2d_bytes_per_step": M * D * 2, "d2h_bytes_per_step": M * D * 2,
                       "ms_per_step": e2e_ms,
                       "copies_alone_ms_per_step": copy_ms,
                       "bound": "host copies" if copy_ms > ms_step else "compute",
                       "api": "hif4_ffn_w4a4_host: pinned host X in, Y out, copies overlapped with compute"}
        del xh, yh, ws, xd, yd

    del xhat1, xhat2, what1, what2, ybuf, x
    torch.cuda.empty_cache()

    # ---- the other rows of the path: quantizer sweep and calibration
    if not args.no_components:
        comps = {}
        sweep = quant_sweep(H, wl, dev, stream, args, barrier, max_over_ranks, world, P)
        comps["quantize"] = dict(sweep["quantize"][-1])
        comps["dequantize"] = dict(sweep["dequantize"][-1])
        comps["quant_sweep"] = sweep
        torch.cuda.empty_cache()
        acts = wl.calib_torch(CALIB_T, CALIB_C, dev)
        cws = torch.empty(H.calib_workspace(CALIB_T, CALIB_C), dtype=torch.uint8, device=dev)
        outs = (torch.empty(CALIB_C, dtype=torch.bfloat16, device=dev),
                torch.empty(CALIB_C, dtype=torch.float32, device=dev),
                torch.empty(CALIB_C, dtype=torch.uint8, device=dev),
                torch.empty(CALIB_C // 100, dtype=torch.int32, device=dev))
        comps["calib_percentile_mask"] = time_op(
            lambda: H.calib_percentile_mask(acts, workspace=cws, out=outs), args, stream, barrier, max_over_ranks,
            world, CALIB_T * CALIB_C * 2.0, P)
        comps["calib_percentile_mask"]["workload"] = \
            "calib 230400 x 5120 BF16, 2 B/elem read once (algorithmic); two radix passes read it twice"
        del acts
        torch.cuda.empty_cache()
        # HiGPTQ scheme one on the FFN's W1 with the Hessian of the layer input
        xg, _ = wl.device_rows(M, D, seed=sharding.rank_seed(3, rank), device=dev)
        w1g = wl.device_weight(F, D, 0.015, seed=31, device=dev)
        Hg = H.hessian(xg)
        del xg
        gws = torch.empty(H.lib().hif4_higptq1_workspace(F, D, 128), dtype=torch.uint8, device=dev)
        r = time_op(lambda: H.higptq1(w1g, Hg, idx1, 0.01, 128, workspace=gws), args, stream, barrier,
                    max_over_ranks, world, 0.0, P)
        # Composite roofline of the call: the FP32 error-feedback updates
        # (N K^2 FLOP) at the split-TF32 tensor rate (three TF32 products per
        # FP32 product) plus the FP64 factor (2 K^3 / 3 FLOP) at the FP64
        # peak.  TF32 peak = the bf16 peak x the nominal 1.1 / 2.25 ratio.
        fp64_peak = 148 * 64 * 2 * P["sm_max_mhz"] * 1e6 / 1e12
        tf32x3_peak = P["bf16_tflops"] * (1.1 / 2.25) / 3.0
        upd_flop, fac_flop = float(F) * D * D, 2.0 * float(D) ** 3 / 3.0
        # the updates also read and write W's remaining columns once per block
        upd_bytes = 8.0 * F * sum(D - b1 for b1 in range(128, D, 128))
        t_upd_ms = max(upd_flop / (tf32x3_peak * 1e12), upd_bytes / (P["hbm_gbs"] * 1e9)) * 1e3
        t_min_ms = t_upd_ms + fac_flop / (fp64_peak * 1e12) * 1e3
        flop = upd_flop + fac_flop
        tf = world * flop / (r["ms"] * 1e-3) / 1e12
        comp_peak = flop / (t_min_ms * 1e-3) / 1e12
        comps["higptq1"] = {"value": tf, "unit": "TFLOP/s", "ms": r["ms"], "bound": "tensor (FP64 + split TF32)",
                            "peak": comp_peak, "frac": tf / world / comp_peak, "roofline_ms": t_min_ms,
                            "peak_source": "composite: the updates at max(N K^2 at %.0f TFLOP/s (TF32 = %s bf16 "
                                           "burst x 1.1/2.25, /3 for the split products), %.2f GB of W read and "
                                           "written at %.0f GB/s) + 2 K^3/3 at %.1f TFLOP/s FP64 (derived: 148 SMs "
                                           "x 64 FP64 lanes x 2 x %.0f MHz)"
                                           % (tf32x3_peak, P["source"], upd_bytes / 1e9, P["hbm_gbs"], fp64_peak,
                                              P["sm_max_mhz"]),
                            "workload": "HiGPTQ scheme one, W1 %d x %d (Wan2.2 FFN), Hessian of %d x %d "
                                        "activations, block 128, 1%% protected; FLOPs counted: the FP32 "
                                        "error-feedback updates (N K^2) plus the FP64 factor (2 K^3 / 3)"
                                        % (F, D, M, D)}
        del w1g, Hg, gws
        torch.cuda.empty_cache()
        # the attention projection (57600 x 5120 -> 5120, bias, 51 protected
        # channels) through the public linear call, device buffers
        xa, _ = wl.device_rows(M, D, seed=sharding.rank_seed(2, rank), device=dev)
        wa = wl.device_weight(D, D, 0.015, seed=21, device=dev)
        _, _, ma, ia = H.calib_percentile_mask(xa)
        wac, wam = H.quantize(wa, ma)
        wak = wa[:, ia.long()].contiguous()
        ba = wl.device_weight(1, D, 0.01, seed=22, device=dev).view(D).contiguous()
        ya = torch.empty(M, D, dtype=torch.bfloat16, device=dev)
        aws = torch.empty(H.linear_w4a4_workspace(M, D, D), dtype=torch.uint8, device=dev)
        r = time_op(lambda: H.linear_w4a4(xa, wac, wam, D, ia, wak, ba, out=ya, workspace=aws), args, stream,
                    barrier, max_over_ranks, world, 0.0, P)
        aflop = 2.0 * M * D * D
        atf = world * aflop / (r["ms"] * 1e-3) / 1e12
        comps["linear_attn_proj"] = {"value": atf, "unit": "TFLOP/s", "ms": r["ms"], "bound": "tensor",
                                     "peak": P["bf16_tflops"], "frac": atf / world / P["bf16_tflops"],
                                     "frac_datasheet": atf / world / DATASHEET["bf16_tflops"],
                                     "peak_source": "%s bf16 burst" % P["source"],
                                     "workload": "hif4_linear_w4a4 57600 x 5120 -> 5120, bias, 51 protected "
                                                 "channels; activation fake-quant, weight decode and GEMM all "
                                                 "timed"}
        del xa, wa, wac, wam, wak, ba, ya, aws
        torch.cuda.empty_cache()
        comps["fp8_remap_gemm"] = fp8_remap_vs_bf16(H, wl, dev, rank, args, stream, barrier, max_over_ranks,
                                                     world, P)
        line["components"] = comps
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            add_cpu_component_rates(comps)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            flop, times, thr, _ = oracle_ffn_sample(args.cpu_sample_rows, steps=2)
            sec = min(times)
            line["cpu_baseline"] = {"value": flop / sec / 1e12, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                                    "sample": "%d of %d tokens of the FFN workload per step (full W1/W2 decode "
                                              "each step), FP64 oracle, best of 2" % (args.cpu_sample_rows, M)}
        except Exception as e:  # pragma: no cover
            line["cpu_baseline"] = {"value": None, "unit": "TFLOP/s", "cores": None, "kind": "oracle",
                                    "sample": "failed: %s" % e}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def add_cpu_component_rates(comps):
    """The CPU oracle's rate on a bounded sample of each component workload,
    beside the GPU line (kind "oracle"; not a target)."""
    import numpy as np

    import oracle
    from block_floating_point_hif4_b200 import workloads as wl
    thr = max(1, len(os.sched_getaffinity(0)))
    n = 1 << 24
    xb = wl.quant_sweep(n, seed=1)
    rows = np.ascontiguousarray(xb[: n // 1024 * 1024].reshape(-1, 1024))
    codes, meta, _ = oracle.quantize(rows)
    q = cpu_rate(lambda: _threaded_row_chunks(lambda a, b: oracle.quantize(rows[a:b]), rows.shape[0], thr),
                 n * 2.5625) / 1e9
    d = cpu_rate(lambda: _threaded_row_chunks(lambda a, b: oracle.dequantize(codes[a:b], meta[a:b], 1024),
                                              rows.shape[0], thr), n * 2.5625) / 1e9
    acts, _ = wl.calib(T=14400, C=512, seed=4)
    c = cpu_rate(lambda: oracle.percentile(acts, threads=thr), acts.size * 2.0) / 1e9
    sample = "2^24 elements of the quantizer sweep, rows split over %d threads" % thr
    comps["quantize"]["cpu_baseline"] = {"value": q, "unit": "GB/s", "cores": thr, "kind": "oracle",
                                         "sample": sample}
    comps["dequantize"]["cpu_baseline"] = {"value": d, "unit": "GB/s", "cores": thr, "kind": "oracle",
                                           "sample": sample}
    comps["calib_percentile_mask"]["cpu_baseline"] = {"value": c, "unit": "GB/s", "cores": thr, "kind": "oracle",
                                                      "sample": "14400 tokens x 512 channels of the calibration "
                                                                "recipe, percentiles (sort per channel)"}


def fp8_remap_vs_bf16(H, wl, dev, rank, args, stream, barrier, max_over_ranks, world, P):
    """The first FFN GEMM's product (57600 x 13824 x 5120, no protected
    channels) on the FP8 tensor cores with the exact E4M3 remap and per-unit
    FP32 promotion (hif4_gemm_f8), timed beside the BF16 tcgen05 GEMM on the
    same dequantized operands (hif4_gemm_bf16); both write BF16."""
    import torch

    from block_floating_point_hif4_b200 import sharding
    M, D, F = args.tokens, D_MODEL, D_FFN
    x, _ = wl.device_rows(M, D, seed=sharding.rank_seed(3, rank), device=dev)
    w = wl.device_weight(F, D, 0.015, seed=31, device=dev)
    ca, ma = H.quantize(x)
    cb, mb = H.quantize(w)
    del x, w
    qa, sa = H.to_e4m3(ca, ma, D, pad_rows=128)
    qb, sb = H.to_e4m3(cb, mb, D, pad_rows=256)
    ah, bh = H.dequantize(ca, ma, D), H.dequantize(cb, mb, D)
    y = torch.empty(M, F, dtype=torch.bfloat16, device=dev)
    flop = 2.0 * M * F * D
    r8 = time_op(lambda: H.gemm_f8(qa, sa, qb, sb, out=y), args, stream, barrier, max_over_ranks, world, 0.0, P)
    r16 = time_op(lambda: H.gemm_bf16(ah, bh, out=y), args, stream, barrier, max_over_ranks, world, 0.0, P)
    del ca, ma, cb, mb, qa, sa, qb, sb, ah, bh, y
    torch.cuda.empty_cache()
    tf8, tf16 = world * flop / (r8["ms"] * 1e-3) / 1e12, world * flop / (r16["ms"] * 1e-3) / 1e12
    return {"value": tf8, "unit": "TFLOP/s", "ms": r8["ms"], "bound": "alu (per-unit FP32 promotion)",
            "bf16_ms": r16["ms"], "bf16_value": tf16, "speedup_vs_bf16": r16["ms"] / r8["ms"],
            "workload": "hif4_gemm_f8 57600 x 13824 x 5120 (E4M3 remap, per-unit FP32 scales, BF16 out) "
                        "beside hif4_gemm_bf16 on the dequantized operands"}


def quant_sweep(H, wl, dev, stream, args, barrier, max_over_ranks, world, P):
    """The quantizer bandwidth sweep: hif4_quantize and hif4_dequantize at
    2^20 ... 2^30 BF16 values (powers of 4), each size as a contiguous
    (n / 1024) x 1024 view.  Sizes whose bytes per call are below three times
    the L2 capacity rotate over enough copies of the input and output buffers
    that consecutive calls never find their data in L2.  Each timed step
    replays a CUDA graph of `reps` calls (launch overhead off the host), so
    the small sizes show the kernels' own launch and tail cost."""
    import math

    import torch
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    out = {"quantize": [], "dequantize": []}
    for e in (20, 22, 24, 26, 28, 30):
        n = 1 << e
        per_call = n * 2.5625
        sets = max(1, math.ceil(3 * l2 / per_call))
        reps = sets * max(1, math.ceil(8 / sets))
        base = wl.quant_sweep_torch(n, dev).view(-1, 1024)
        xs = [base] + [base.clone() for _ in range(sets - 1)]
        codes = [torch.empty(n // 1024, 512, dtype=torch.uint8, device=dev) for _ in range(sets)]
        meta = [torch.empty(n // 1024, 16, dtype=torch.int32, device=dev) for _ in range(sets)]
        ys = [torch.empty_like(base) for _ in range(sets)]
        ops = {"quantize": lambda i: H.quantize(xs[i], codes=codes[i], meta=meta[i]),
               "dequantize": lambda i: H.dequantize(codes[i], meta[i], 1024, out=ys[i])}
        for name in ("quantize", "dequantize"):
            fn = ops[name]
            for i in range(sets):                          # eager first calls (per-device set-up)
                fn(i)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for r in range(reps):
                    fn(r % sets)
            r = time_op(g.replay, args, stream, barrier, max_over_ranks, world, per_call * reps, P)
            r["ms"] /= reps
            r.update({"n": n, "log2_n": e, "buffer_sets": sets, "calls_per_graph": reps,
                      "l2": "rotating over %d buffer sets (%.0f MB per call; L2 %.0f MB)"
                            % (sets, per_call / 1e6, l2 / 1e6) if sets > 1 else "inputs larger than L2",
                      "workload": "quant_sweep 2^%d BF16 (rows of 5120, t3 x 0.05 x row lognormal), "
                                  "2.5625 B/elem" % e})
            out[name].append(r)
            del g
        del base, xs, codes, meta, ys
        torch.cuda.empty_cache()
    return out


def time_op(fn, args, stream, barrier, max_over_ranks, world, bytes_per_call, P):
    import torch
    for _ in range(args.warmup):
        fn()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        fn()
    e1.record(stream)
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
    gbs = world * bytes_per_call / (ms * 1e-3) / 1e9
    return {"value": gbs, "unit": "GB/s", "ms": ms, "bound": "hbm", "peak": P["hbm_gbs"],
            "frac": gbs / world / P["hbm_gbs"], "frac_datasheet": gbs / world / DATASHEET["hbm_gbs"],
            "peak_source": P["source"], "l2": "inputs larger than L2"}


def _threaded_row_chunks(fn, rows, threads):
    """fn(r0, r1) over `threads` equal row ranges at once (the oracle's C
    calls release the interpreter lock)."""
    import numpy as np
    bounds = np.linspace(0, rows, threads + 1).astype(int)
    ts = [threading.Thread(target=fn, args=(bounds[i], bounds[i + 1])) for i in range(threads)
          if bounds[i + 1] > bounds[i]]
    [t.start() for t in ts]
    [t.join() for t in ts]


def cpu_rate(fn, units, reps=2):
    """Best-of-`reps` wall-clock rate (units per second) of a CPU oracle call."""
    best = None
    for _ in range(reps):
        t0 = time.perf_counter()
        fn()
        dt = time.perf_counter() - t0
        best = dt if best is None else min(best, dt)
    return units / best


if __name__ == "__main__":
    sys.exit(main())
