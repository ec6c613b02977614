"""Run one libhif4 operation a few times on seeded device inputs — the
command to put under a profiler (ncu) or to time one kernel in isolation.

    python -m block_floating_point_hif4_b200.profile OP [--log2n N] [--tokens T] [--reps R]

OP: quantize | dequantize | fake_quantize | gemm | gemm_gelu | gemm_fq | calib |
linear | ffn | higptq.  gemm_fq is the FFN's first GEMM: bias-free, tanh-GELU and the
HiF4 fake quantization of its output (1 % protected columns) in the epilogue;
ffn is the whole W4A4 FFN block (hif4_ffn_w4a4, --n = hidden width);
higptq times HiGPTQ scheme one on an --n x --channels weight with the
Hessian of --tokens activation rows (the Hessian itself untimed);
fake_quantize_x is the FFN step's first call: --tokens x --channels
activations with 1 % protected channels.
Sizes default to small cases that still exceed the 126 MB L2 (a few hundred
MB on the device).  Prints the mean CUDA-event time per call.
"""
from __future__ import annotations

import argparse
import sys


def main(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("op", choices=["quantize", "dequantize", "fake_quantize", "fake_quantize_x", "gemm", "gemm_gelu",
                                  "gemm_fq", "calib", "linear", "ffn", "higptq"])
    p.add_argument("--log2n", type=int, default=28, help="elements for quantize/dequantize/fake_quantize")
    p.add_argument("--protect", type=float, default=0.01,
                   help="fake_quantize_x: fraction of protected channels (0 = no mask)")
    p.add_argument("--tokens", type=int, default=57600)
    p.add_argument("--channels", type=int, default=5120)
    p.add_argument("--n", type=int, default=5120, help="output features for gemm/linear")
    p.add_argument("--reps", type=int, default=3)
    p.add_argument("--blocksize", type=int, default=128, help="HiGPTQ block (64, 128, 192, 256)")
    a = p.parse_args(argv)

    import torch

    from . import binding as H
    from . import workloads as wl
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    H.lib()
    if a.op in ("quantize", "dequantize", "fake_quantize"):
        n = 1 << a.log2n
        x = wl.quant_sweep_torch(n, dev).view(-1, 1024)
        codes, meta = H.quantize(x)
        y = torch.empty_like(x)
        fn = {"quantize": lambda: H.quantize(x, codes=codes, meta=meta),
              "dequantize": lambda: H.dequantize(codes, meta, 1024, out=y),
              "fake_quantize": lambda: H.fake_quantize(x, out=y)}[a.op]
        nbytes = n * (4.0 if a.op == "fake_quantize" else 2.5625)
    elif a.op == "fake_quantize_x":
        x, _ = wl.device_rows(a.tokens, a.channels, seed=3, device=dev)
        g = torch.Generator(device=dev)
        g.manual_seed(5)
        cm = (torch.rand(a.channels, device=dev, generator=g) < a.protect).to(torch.uint8) if a.protect > 0 else None
        y = torch.empty_like(x)
        fn = lambda: H.fake_quantize(x, cm, out=y)  # noqa: E731
        nbytes = 4.0 * a.tokens * a.channels
    elif a.op == "higptq":
        x, _ = wl.device_rows(a.tokens, a.channels, seed=3, device=dev)
        w = wl.device_weight(a.n, a.channels, 0.015, seed=31, device=dev)
        Hm = H.hessian(x)
        del x
        ws = torch.empty(H.lib().hif4_higptq1_workspace(a.n, a.channels, a.blocksize), dtype=torch.uint8,
                         device=dev)
        fn = lambda: H.higptq1(w, Hm, None, 0.01, a.blocksize, workspace=ws)  # noqa: E731
        nbytes = 2.0 * a.n * a.channels * a.channels / 2        # FLOPs of the lazy updates (N K^2 / 2 FMA)
    elif a.op == "calib":
        x = wl.calib_torch(a.tokens, a.channels, dev)
        ws = torch.empty(H.calib_workspace(a.tokens, a.channels), dtype=torch.uint8, device=dev)
        fn = lambda: H.calib_percentile_mask(x, workspace=ws)  # noqa: E731
        nbytes = 2.0 * a.tokens * a.channels
    else:
        x, _ = wl.device_rows(a.tokens, a.channels, seed=3, device=dev)
        w = wl.device_weight(a.n, a.channels, 0.015, seed=31, device=dev)
        y = torch.empty(a.tokens, a.n, dtype=torch.bfloat16, device=dev)
        if a.op == "gemm":
            fn = lambda: H.gemm_bf16(x, w, out=y)  # noqa: E731
        elif a.op == "gemm_gelu":
            fn = lambda: H.gemm_bf16(x, w, gelu=True, out=y)  # noqa: E731
        elif a.op == "gemm_fq":
            g = torch.Generator(device=dev)
            g.manual_seed(5)
            cm = (torch.rand(a.n, device=dev, generator=g) < 0.01).to(torch.uint8)
            fn = lambda: H.gemm_bf16_fq(x, w, gelu=True, out_chan_mask=cm, out=y)  # noqa: E731
        elif a.op == "ffn":
            w2 = wl.device_weight(a.channels, a.n, 0.015, seed=32, device=dev)
            w1c, w1m = H.quantize(w)
            w2c, w2m = H.quantize(w2)
            y = torch.empty(a.tokens, a.channels, dtype=torch.bfloat16, device=dev)
            ws = torch.empty(H.ffn_w4a4_workspace(a.tokens, a.channels, a.n), dtype=torch.uint8, device=dev)
            fn = lambda: H.ffn_w4a4(x, w1c, w1m, a.n, w2c, w2m, out=y, workspace=ws)  # noqa: E731
        else:
            wc, wm = H.quantize(w)
            ws = torch.empty(H.linear_w4a4_workspace(a.tokens, a.n, a.channels), dtype=torch.uint8, device=dev)
            fn = lambda: H.linear_w4a4(x, wc, wm, a.n, out=y, workspace=ws)  # noqa: E731
        nbytes = 2.0 * a.tokens * a.n * a.channels * (2 if a.op == "ffn" else 1)   # FLOPs
    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.reps
    unit = "TFLOP/s" if a.op in ("gemm", "gemm_gelu", "gemm_fq", "linear", "ffn", "higptq") else "GB/s"
    rate = nbytes / (ms * 1e-3) / (1e12 if unit == "TFLOP/s" else 1e9)
    print("%s: %.4f ms per call, %.1f %s" % (a.op, ms, rate, unit))
    return 0


if __name__ == "__main__":
    sys.exit(main())
