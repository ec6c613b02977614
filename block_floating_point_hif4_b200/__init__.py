"""libhif4 — HiFloat4 (HiF4) W4A4 fake-quantized linear hot path on B200.

The compute lives in ``libhif4.so`` (hand-written sm_100a CUDA kernels behind
the C ABI in ``include/hif4.h``); :mod:`.binding` marshals torch tensors into
it.  :mod:`.workloads` holds the seeded synthetic inputs.
"""
from .binding import (  # noqa: F401
    Hif4Error, calib_percentile_mask, calib_workspace, dequantize, fake_quantize, ffn_w4a4, ffn_w4a4_host,
    ffn_w4a4_host_workspace, ffn_w4a4_workspace, gemm_bf16, gemm_bf16_fq, gemm_f8, get_status, hessian, higptq1,
    higptq1_group_inputs, lib, linear_w4a4, linear_w4a4_workspace, ptq_state_pack, ptq_state_unpack, quantize,
    reset_status, to_e4m3, version, weight_decode,
)

__all__ = ["Hif4Error", "calib_percentile_mask", "calib_workspace", "dequantize", "fake_quantize", "ffn_w4a4",
           "ffn_w4a4_host", "ffn_w4a4_host_workspace", "ffn_w4a4_workspace", "gemm_bf16", "gemm_bf16_fq",
           "gemm_f8", "get_status", "hessian", "higptq1", "higptq1_group_inputs", "lib", "linear_w4a4",
           "linear_w4a4_workspace", "ptq_state_pack", "ptq_state_unpack", "quantize", "reset_status", "to_e4m3",
           "version", "weight_decode"]
