"""ctypes binding of libhif4.so — argument marshalling only.

Every function here forwards to the C ABI declared in ``include/hif4.h`` with
the same name (minus the ``hif4_`` prefix).  torch is used for device memory
and the current CUDA stream; all HiF4 arithmetic runs in the library's CUDA
kernels.  There is no CPU fallback: if ``libhif4.so`` is missing or fails to
load, :func:`lib` raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhif4.so")

OK = 0
ERR_INVALID_ARG, ERR_ALIGNMENT, ERR_SHAPE, ERR_WORKSPACE = 1, 2, 3, 4
ERR_CUDA, ERR_NONFINITE, ERR_TIMEOUT, ERR_UNSUPPORTED, ERR_FORMAT = 5, 6, 7, 8, 9
F32, BF16 = 0, 1
FLAG_NONFINITE, FLAG_TIMEOUT, FLAG_BAD_INDEX = 1, 2, 4
LINEAR_GELU_TANH = 1
LINEAR_OUT_F32 = 2
LINEAR_FAKE_QUANT_OUT = 4

# (name, restype, argtypes) of every exported entry point
_P, _I64, _U32, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint32, ctypes.c_int32, ctypes.c_size_t
SIGNATURES = {
    "hif4_quantize": (ctypes.c_int, [_P, ctypes.c_int, _I64, _I64, _I64, _P, _P, _P, _P, _P]),
    "hif4_dequantize": (ctypes.c_int, [_P, _P, _I64, _I64, ctypes.c_int, _P, _I64, _P]),
    "hif4_fake_quantize": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _I64, _P, _P]),
    "hif4_linear_w4a4_workspace": (_SZ, [_I64, _I64, _I64]),
    "hif4_linear_w4a4": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _I64, _P, _I32, _P, _P, _P, _I64,
                                        _U32, _P, _SZ, _P, _P]),
    "hif4_weight_decode": (ctypes.c_int, [_P, _P, _I64, _I64, _P, _I32, _P, _P, _I64, _P, _P]),
    "hif4_gemm_bf16": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _I64, _I64, _P, _P, _I64, _U32, _P, _P]),
    "hif4_gemm_bf16_fq": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _I64, _I64, _P, _P, _P, _I64, _U32, _P, _P]),
    "hif4_ffn_w4a4_workspace": (_SZ, [_I64, _I64, _I64]),
    "hif4_ffn_w4a4_host_workspace": (_SZ, [_I64, _I64, _I64, _I64, _U32]),
    "hif4_ffn_w4a4_host": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _I64, _P, _I32, _P, _P, _P, _P, _P, _I32,
                                          _P, _P, _P, _I64, _I64, _U32, _P, _SZ, _P, _P]),
    "hif4_ffn_w4a4": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _I64, _P, _I32, _P, _P, _P, _P, _P, _I32, _P,
                                     _P, _P, _I64, _U32, _P, _SZ, _P, _P]),
    "hif4_calib_workspace": (_SZ, [_I64, _I64]),
    "hif4_calib_percentile_mask": (ctypes.c_int, [_P, _I64, _I64, _I64, _U32, _U32, _U32, _U32, _P, _P, _P,
                                                  _P, _P, _SZ, _P]),
    "hif4_calib_noalloc_scratch_bytes": (_SZ, []),
    "hif4_calib_percentile_mask_noalloc": (ctypes.c_int, [_P, _I64, _I64, _I64, _U32, _U32, _U32, _U32, _P, _P,
                                                          _P, _P, _P]),
    "hif4_hessian_workspace": (_SZ, [_I64, _I64]),
    "hif4_hessian": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _SZ, _P, _P]),
    "hif4_higptq1_workspace": (_SZ, [_I64, _I64, _I64]),
    "hif4_higptq1_group_inputs_offset": (_SZ, [_I64, _I64, _I64]),
    "hif4_higptq1": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _I32, ctypes.c_double, _I64, _P, _P, _P, _P,
                                    _SZ, _P, _P]),
    "hif4_ptq_state_bytes": (_SZ, [_I64, _I64, _I32]),
    "hif4_ptq_state_pack": (ctypes.c_int, [_I64, _I64, _P, _P, _P, _I32, _P, _P, _SZ]),
    "hif4_ptq_state_info": (ctypes.c_int, [_P, _SZ, _P, _P, _P]),
    "hif4_ptq_state_unpack": (ctypes.c_int, [_P, _SZ, _P, _P, _P, _P]),
    "hif4_to_e4m3": (ctypes.c_int, [_P, _P, _I64, _I64, _P, _I64, _P, _I64, _P]),
    "hif4_gemm_f8": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _I64, _P, _I64, _I64, _P, _I64, _P, _I64, _U32, _P,
                                    _P]),
    "hif4_debug_wait_test": (None, [ctypes.c_uint32, ctypes.c_uint64]),
    "hif4_get_status": (ctypes.c_int, [_P, _P]),
    "hif4_reset_status": (ctypes.c_int, [_P, _P]),
    "hif4_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "hif4_last_cuda_error": (ctypes.c_char_p, []),
    "hif4_version": (ctypes.c_int, []),
}

_lock = threading.Lock()
_lib = None


class Hif4Error(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        msg = lib().hif4_status_string(code).decode()
        if code == ERR_CUDA:
            msg += ": " + lib().hif4_last_cuda_error().decode()
        super().__init__("%s failed: status %d (%s)" % (fn, code, msg))


def lib() -> ctypes.CDLL:
    """Load libhif4.so (built in-tree by ``build.py``); raises if absent."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError("libhif4.so is not built (run python -m block_floating_point_hif4_b200.build); "
                                   "there is no CPU fallback")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, code):
    if code != OK:
        raise Hif4Error(fn, code)


def _dev(t, name):
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    return t


# ------------------------------------------------------------------ calls

def quantize(x: torch.Tensor, chan_mask: torch.Tensor | None = None, *, codes=None, meta=None,
             status=None, stream=None):
    """HiF4 codes (uint8 [rows, cols/2]) and meta (int32 bit patterns [rows, cols/64])."""
    _dev(x, "x")
    assert x.dim() == 2 and x.stride(1) == 1
    dt = {torch.bfloat16: BF16, torch.float32: F32}[x.dtype]
    rows, cols = x.shape
    if codes is None:
        codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=x.device)
    if meta is None:
        meta = torch.empty(rows, cols // 64, dtype=torch.int32, device=x.device)
    _check("hif4_quantize", lib().hif4_quantize(_ptr(x), dt, rows, cols, x.stride(0), _ptr(chan_mask),
                                                _ptr(codes), _ptr(meta), _ptr(status), _stream(stream)))
    return codes, meta


def dequantize(codes: torch.Tensor, meta: torch.Tensor, cols: int, dtype=torch.bfloat16, *, out=None,
               stream=None):
    _dev(codes, "codes")
    rows = codes.shape[0]
    if out is None:
        out = torch.empty(rows, cols, dtype=dtype, device=codes.device)
    dt = {torch.bfloat16: BF16, torch.float32: F32}[out.dtype]
    _check("hif4_dequantize", lib().hif4_dequantize(_ptr(codes), _ptr(meta), rows, cols, dt, _ptr(out),
                                                    out.stride(0), _stream(stream)))
    return out


def fake_quantize(x: torch.Tensor, chan_mask: torch.Tensor | None = None, *, out=None, status=None,
                  stream=None):
    _dev(x, "x")
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    if out is None:
        out = torch.empty(rows, cols, dtype=torch.bfloat16, device=x.device)
    _check("hif4_fake_quantize", lib().hif4_fake_quantize(_ptr(x), rows, cols, x.stride(0), _ptr(chan_mask),
                                                          _ptr(out), out.stride(0), _ptr(status),
                                                          _stream(stream)))
    return out


def linear_w4a4_workspace(M: int, N: int, K: int) -> int:
    return int(lib().hif4_linear_w4a4_workspace(M, N, K))


def linear_w4a4(x: torch.Tensor, w_codes: torch.Tensor, w_meta: torch.Tensor, N: int,
                mask_idx: torch.Tensor | None = None, w_masked: torch.Tensor | None = None,
                bias: torch.Tensor | None = None, gelu: bool = False, *, out=None, workspace=None,
                status=None, stream=None):
    """y = fakequant(x) · deq(w)ᵀ + bias (BF16 out); protected columns in BF16."""
    _dev(x, "x")
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    M, K = x.shape
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    need = linear_w4a4_workspace(M, N, K)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    n_m = 0 if mask_idx is None else int(mask_idx.numel())
    flags = (LINEAR_GELU_TANH if gelu else 0) | (LINEAR_OUT_F32 if out.dtype == torch.float32 else 0)
    _check("hif4_linear_w4a4", lib().hif4_linear_w4a4(
        _ptr(x), M, K, x.stride(0), _ptr(w_codes), _ptr(w_meta), N, _ptr(mask_idx) if n_m else None, n_m,
        _ptr(w_masked) if n_m else None, _ptr(bias), _ptr(out), out.stride(0), flags, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream)))
    return out


def weight_decode(w_codes: torch.Tensor, w_meta: torch.Tensor, N: int, K: int,
                  mask_idx: torch.Tensor | None = None, w_masked: torch.Tensor | None = None, *, out=None,
                  status=None, stream=None):
    """BF16 N x K decoded weight with the protected columns restored."""
    _dev(w_codes, "w_codes")
    if out is None:
        out = torch.empty(N, K, dtype=torch.bfloat16, device=w_codes.device)
    n_m = 0 if mask_idx is None else int(mask_idx.numel())
    _check("hif4_weight_decode", lib().hif4_weight_decode(
        _ptr(w_codes), _ptr(w_meta), N, K, _ptr(mask_idx) if n_m else None, n_m, _ptr(w_masked) if n_m else None,
        _ptr(out), out.stride(0), _ptr(status), _stream(stream)))
    return out


def gemm_bf16(a: torch.Tensor, b: torch.Tensor, bias: torch.Tensor | None = None, gelu: bool = False, *,
              out=None, status=None, stream=None):
    """y = a · bᵀ + bias on BF16 operands (tcgen05, FP32 accumulate, BF16 out)."""
    _dev(a, "a")
    assert a.dtype == torch.bfloat16 and b.dtype == torch.bfloat16 and a.stride(1) == 1 and b.stride(1) == 1
    M, K = a.shape
    N = b.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=a.device)
    flags = (LINEAR_GELU_TANH if gelu else 0) | (LINEAR_OUT_F32 if out.dtype == torch.float32 else 0)
    _check("hif4_gemm_bf16", lib().hif4_gemm_bf16(
        _ptr(a), M, K, a.stride(0), _ptr(b), N, b.stride(0), _ptr(bias), _ptr(out), out.stride(0),
        flags, _ptr(status), _stream(stream)))
    return out


def to_e4m3(codes: torch.Tensor, meta: torch.Tensor, cols: int, *, pad_rows: int = 1, out=None, stream=None):
    """HiF4 codes -> (E4M3 bytes uint8 [rows, cols], unit scales FP32 [cols/64, lds]),
    lds = rows rounded up to `pad_rows` (128 for the FP8 GEMM's A, 256 for its B)."""
    _dev(codes, "codes")
    rows = codes.shape[0]
    lds = -(-rows // pad_rows) * pad_rows
    if out is None:
        out = (torch.empty(rows, cols, dtype=torch.uint8, device=codes.device),
               torch.zeros(cols // 64, lds, dtype=torch.float32, device=codes.device))
    q8, sc = out
    _check("hif4_to_e4m3", lib().hif4_to_e4m3(_ptr(codes), _ptr(meta), rows, cols, _ptr(q8), q8.stride(0),
                                              _ptr(sc), sc.stride(0), _stream(stream)))
    return q8, sc


def gemm_f8(a: torch.Tensor, sa: torch.Tensor, b: torch.Tensor, sb: torch.Tensor, *, out=None, out_f32=False,
            status=None, stream=None):
    """y = sum over units of sa sb (a_u · b_uᵀ) on the FP8 tensor cores (E4M3
    operands from to_e4m3, FP32 unit scales, FP32 promotion)."""
    _dev(a, "a")
    M, K = a.shape
    N = b.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.float32 if out_f32 else torch.bfloat16, device=a.device)
    flags = LINEAR_OUT_F32 if out.dtype == torch.float32 else 0
    _check("hif4_gemm_f8", lib().hif4_gemm_f8(_ptr(a), M, K, a.stride(0), _ptr(sa), sa.stride(0), _ptr(b), N,
                                              b.stride(0), _ptr(sb), sb.stride(0), _ptr(out), out.stride(0), flags,
                                              _ptr(status), _stream(stream)))
    return out


def gemm_bf16_fq(a: torch.Tensor, b: torch.Tensor, bias: torch.Tensor | None = None, gelu: bool = False,
                 out_chan_mask: torch.Tensor | None = None, *, out=None, status=None, stream=None):
    """hfq = fakequant(bf16(a · bᵀ + bias), optionally GELU'd) along N in the
    GEMM epilogue; out_chan_mask (u8 [N], nonzero = protected) columns kept."""
    _dev(a, "a")
    assert a.dtype == torch.bfloat16 and b.dtype == torch.bfloat16 and a.stride(1) == 1 and b.stride(1) == 1
    M, K = a.shape
    N = b.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=a.device)
    flags = LINEAR_GELU_TANH if gelu else 0
    _check("hif4_gemm_bf16_fq", lib().hif4_gemm_bf16_fq(
        _ptr(a), M, K, a.stride(0), _ptr(b), N, b.stride(0), _ptr(bias), _ptr(out_chan_mask), _ptr(out),
        out.stride(0), flags, _ptr(status), _stream(stream)))
    return out


def ffn_w4a4_workspace(M: int, D: int, F: int) -> int:
    return int(lib().hif4_ffn_w4a4_workspace(M, D, F))


def ffn_w4a4(x: torch.Tensor, w1_codes: torch.Tensor, w1_meta: torch.Tensor, F: int,
             w2_codes: torch.Tensor, w2_meta: torch.Tensor,
             mask1_idx: torch.Tensor | None = None, w1_masked: torch.Tensor | None = None,
             b1: torch.Tensor | None = None, mask2_idx: torch.Tensor | None = None,
             w2_masked: torch.Tensor | None = None, b2: torch.Tensor | None = None, *, out=None,
             workspace=None, status=None, stream=None):
    """y = fq(gelu(fq(x) · ŵ1ᵀ + b1)) · ŵ2ᵀ + b2, the W4A4 HiF4 FFN block (BF16 or FP32 out)."""
    _dev(x, "x")
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    M, D = x.shape
    if out is None:
        out = torch.empty(M, D, dtype=torch.bfloat16, device=x.device)
    need = ffn_w4a4_workspace(M, D, F)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    n1 = 0 if mask1_idx is None else int(mask1_idx.numel())
    n2 = 0 if mask2_idx is None else int(mask2_idx.numel())
    flags = LINEAR_OUT_F32 if out.dtype == torch.float32 else 0
    _check("hif4_ffn_w4a4", lib().hif4_ffn_w4a4(
        _ptr(x), M, D, x.stride(0), _ptr(w1_codes), _ptr(w1_meta), F, _ptr(mask1_idx) if n1 else None, n1,
        _ptr(w1_masked) if n1 else None, _ptr(b1), _ptr(w2_codes), _ptr(w2_meta),
        _ptr(mask2_idx) if n2 else None, n2, _ptr(w2_masked) if n2 else None, _ptr(b2), _ptr(out),
        out.stride(0), flags, _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)))
    return out


def ffn_w4a4_host_workspace(M: int, D: int, F: int, chunk_rows: int = 0, out_f32: bool = False) -> int:
    return int(lib().hif4_ffn_w4a4_host_workspace(M, D, F, chunk_rows, LINEAR_OUT_F32 if out_f32 else 0))


def ffn_w4a4_host(x_host: torch.Tensor, w1_codes: torch.Tensor, w1_meta: torch.Tensor, F: int,
                  w2_codes: torch.Tensor, w2_meta: torch.Tensor,
                  mask1_idx: torch.Tensor | None = None, w1_masked: torch.Tensor | None = None,
                  b1: torch.Tensor | None = None, mask2_idx: torch.Tensor | None = None,
                  w2_masked: torch.Tensor | None = None, b2: torch.Tensor | None = None, *, out=None,
                  chunk_rows: int = 0, workspace=None, status=None, stream=None):
    """The FFN block on HOST (ideally pinned) x; y returned in a host tensor.
    Copies overlap compute chunk by chunk.  Asynchronous on `stream`."""
    assert x_host.device.type == "cpu" and x_host.dtype == torch.bfloat16 and x_host.stride(1) == 1
    M, D = x_host.shape
    if out is None:
        out = torch.empty(M, D, dtype=torch.bfloat16, pin_memory=x_host.is_pinned())
    assert out.device.type == "cpu" and out.stride(1) == 1
    f32 = out.dtype == torch.float32
    dev = w1_codes.device
    if workspace is None:
        need = ffn_w4a4_host_workspace(M, D, F, chunk_rows, f32)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    n1 = 0 if mask1_idx is None else int(mask1_idx.numel())
    n2 = 0 if mask2_idx is None else int(mask2_idx.numel())
    _check("hif4_ffn_w4a4_host", lib().hif4_ffn_w4a4_host(
        ctypes.c_void_p(x_host.data_ptr()), M, D, x_host.stride(0), _ptr(w1_codes), _ptr(w1_meta), F,
        _ptr(mask1_idx) if n1 else None, n1, _ptr(w1_masked) if n1 else None, _ptr(b1), _ptr(w2_codes),
        _ptr(w2_meta), _ptr(mask2_idx) if n2 else None, n2, _ptr(w2_masked) if n2 else None, _ptr(b2),
        ctypes.c_void_p(out.data_ptr()), out.stride(0), chunk_rows, LINEAR_OUT_F32 if f32 else 0,
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream)))
    return out


def calib_workspace(T: int, C: int) -> int:
    return int(lib().hif4_calib_workspace(T, C))


def calib_percentile_mask(acts: torch.Tensor, q=(999, 1000), frac=(1, 100), *, workspace=None, out=None,
                          stream=None):
    """-> (pct bf16 [C], ratio f32 [C], mask uint8 [C], mask_idx int32 [n_top])."""
    _dev(acts, "acts")
    assert acts.dtype == torch.bfloat16 and acts.dim() == 2 and acts.stride(1) == 1
    T, C = acts.shape
    n_top = (C * frac[0]) // frac[1]
    dev = acts.device
    if out is None:
        out = (torch.empty(C, dtype=torch.bfloat16, device=dev), torch.empty(C, dtype=torch.float32, device=dev),
               torch.empty(C, dtype=torch.uint8, device=dev), torch.empty(max(n_top, 1), dtype=torch.int32,
                                                                            device=dev))
    pct, ratio, mask, midx = out
    need = calib_workspace(T, C)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check("hif4_calib_percentile_mask", lib().hif4_calib_percentile_mask(
        _ptr(acts), T, C, acts.stride(0), q[0], q[1], frac[0], frac[1], _ptr(pct), _ptr(ratio), _ptr(mask),
        _ptr(midx), _ptr(workspace), workspace.numel(), _stream(stream)))
    return pct, ratio, mask, midx[:n_top]


def hessian(x: torch.Tensor, *, out=None, workspace=None, status=None, stream=None):
    """H = XᵀX (FP32 K x K) of BF16 activations X (T x K)."""
    _dev(x, "x")
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    T, K = x.shape
    if out is None:
        out = torch.empty(K, K, dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.empty(max(1, int(lib().hif4_hessian_workspace(T, K))), dtype=torch.uint8, device=x.device)
    _check("hif4_hessian", lib().hif4_hessian(_ptr(x), T, K, x.stride(0), _ptr(out), _ptr(workspace),
                                              workspace.numel(), _ptr(status), _stream(stream)))
    return out


def higptq1(w: torch.Tensor, H: torch.Tensor, mask_idx: torch.Tensor | None = None, damp: float = 0.01,
            blocksize: int = 128, *, workspace=None, status=None, stream=None):
    """HiGPTQ scheme one -> (codes u8 [N, K/2], meta i32 [N, K/64], w_masked bf16 [N, n] or None)."""
    _dev(w, "w")
    assert w.dtype == torch.bfloat16 and w.dim() == 2 and w.stride(1) == 1
    assert H.dtype == torch.float32 and H.is_contiguous()
    N, K = w.shape
    n = 0 if mask_idx is None else int(mask_idx.numel())
    codes = torch.empty(N, K // 2, dtype=torch.uint8, device=w.device)
    meta = torch.empty(N, K // 64, dtype=torch.int32, device=w.device)
    wm = torch.empty(N, n, dtype=torch.bfloat16, device=w.device) if n else None
    if workspace is None:
        need = int(lib().hif4_higptq1_workspace(N, K, blocksize))
        workspace = torch.empty(max(1, need), dtype=torch.uint8, device=w.device)
    _check("hif4_higptq1", lib().hif4_higptq1(
        _ptr(w), N, K, w.stride(0), _ptr(H), _ptr(mask_idx) if n else None, n, float(damp), blocksize,
        _ptr(codes), _ptr(meta), _ptr(wm), _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)))
    return codes, meta, wm


def higptq1_group_inputs(workspace: torch.Tensor, N: int, K: int, blocksize: int = 128) -> torch.Tensor:
    """FP32 [N, K] view of a hif4_higptq1 workspace: after the call, the
    weights each 64-column group was quantized from (stream-ordered)."""
    off = int(lib().hif4_higptq1_group_inputs_offset(N, K, blocksize))
    if off == ctypes.c_size_t(-1).value:
        raise ValueError("invalid HiGPTQ shape")
    assert workspace.dtype == torch.uint8 and workspace.numel() >= off + N * K * 4
    return workspace[off:off + N * K * 4].view(torch.float32).view(N, K)


def ptq_state_pack(codes: torch.Tensor, meta: torch.Tensor, mask_idx: torch.Tensor | None = None,
                   w_masked: torch.Tensor | None = None) -> bytes:
    """Compact PTQ state record of one layer (see hif4.h) from its HiF4 codes
    [N, K/2] u8, meta [N, K/64] i32, protected indices [n] i32 and their BF16
    weight columns [N, n]; tensors on any device (copied to host memory)."""
    c = codes.detach().to("cpu").contiguous()
    m = meta.detach().to("cpu").contiguous()
    N, K = c.shape[0], c.shape[1] * 2
    n = 0 if mask_idx is None else int(mask_idx.numel())
    idx = None if n == 0 else mask_idx.detach().to("cpu", torch.int32).contiguous()
    wm = None if n == 0 else w_masked.detach().to("cpu").contiguous()
    size = int(lib().hif4_ptq_state_bytes(N, K, n))
    if size == 0:
        raise Hif4Error("hif4_ptq_state_bytes", ERR_INVALID_ARG)
    out = ctypes.create_string_buffer(size)
    _check("hif4_ptq_state_pack", lib().hif4_ptq_state_pack(
        N, K, _ptr(c), _ptr(m), _ptr(idx), n, _ptr(wm), ctypes.cast(out, ctypes.c_void_p), size))
    return out.raw


def ptq_state_unpack(record: bytes, device=None):
    """-> (codes u8 [N, K/2], meta i32 [N, K/64], mask_idx i32 [n] or None,
    w_masked bf16 [N, n] or None), on `device` (default: host)."""
    buf = ctypes.create_string_buffer(bytes(record), len(record))
    N, K, n = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int32()
    _check("hif4_ptq_state_info", lib().hif4_ptq_state_info(
        ctypes.cast(buf, ctypes.c_void_p), len(record), ctypes.byref(N), ctypes.byref(K), ctypes.byref(n)))
    N, K, n = N.value, K.value, n.value
    codes = torch.empty(N, K // 2, dtype=torch.uint8)
    meta = torch.empty(N, K // 64, dtype=torch.int32)
    idx = torch.empty(n, dtype=torch.int32) if n else None
    wm = torch.empty(N, n, dtype=torch.bfloat16) if n else None
    _check("hif4_ptq_state_unpack", lib().hif4_ptq_state_unpack(
        ctypes.cast(buf, ctypes.c_void_p), len(record), _ptr(codes), _ptr(meta), _ptr(idx), _ptr(wm)))
    if device is not None:
        codes, meta = codes.to(device), meta.to(device)
        idx = None if idx is None else idx.to(device)
        wm = None if wm is None else wm.to(device)
    return codes, meta, idx, wm


def get_status(status: torch.Tensor, stream=None) -> int:
    return int(lib().hif4_get_status(_ptr(status), _stream(stream)))


def reset_status(status: torch.Tensor, stream=None) -> None:
    _check("hif4_reset_status", lib().hif4_reset_status(_ptr(status), _stream(stream)))


def version() -> int:
    return int(lib().hif4_version())
