"""CPU oracle for the HiF4 W4A4 hot path — TEST INFRASTRUCTURE ONLY.

A plain, slow, double-precision C reference (``hif4_oracle.c``) plus numpy
marshalling.  It shares no code with the CUDA library.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference arm
may import this package; the product path never does.

Every function here is pinned by ``tests/test_oracle_*.py`` against facts the
source pages and mathematics fix (see the docstrings there).  Citations are
to page title and section:

* [HiF4 format] Huawei HiF4 calibration article (hwcomputing.csdn.net), §1.
* [TA abstract] "Tail-Aware HiFloat4: W4A4 Post-Training Quantization for
  Wan2.2", arXiv 2605.26628 record, abstract.
* [TA summary] agents-report.net summary of that report, "Method overview".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hif4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with plain gcc -O2 (no fast-math: IEEE order)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i64 = ctypes.c_long
            L.orc_e6m2_value.restype = ctypes.c_double
            L.orc_e6m2_value.argtypes = [ctypes.c_int]
            L.orc_select_scale_code.restype = ctypes.c_int
            L.orc_select_scale_code.argtypes = [ctypes.c_double]
            L.orc_round_magnitude.restype = ctypes.c_int
            L.orc_round_magnitude.argtypes = [ctypes.c_double, ctypes.c_double]
            L.orc_quantize_unit.restype = None
            L.orc_quantize_unit.argtypes = [P, P, P, P]
            L.orc_decode_element.restype = ctypes.c_double
            L.orc_decode_element.argtypes = [ctypes.c_uint, ctypes.c_uint32, ctypes.c_int]
            L.orc_quantize.restype = i64
            L.orc_quantize.argtypes = [P, ctypes.c_int, i64, i64, i64, P, P, P]
            L.orc_dequantize.restype = None
            L.orc_dequantize.argtypes = [P, P, i64, i64, P, i64]
            L.orc_fake_quantize.restype = i64
            L.orc_fake_quantize.argtypes = [P, i64, i64, i64, P, ctypes.c_int, P]
            L.orc_weight_hat.restype = None
            L.orc_weight_hat.argtypes = [P, P, i64, i64, P, ctypes.c_int, P, P]
            L.orc_gelu_tanh.restype = ctypes.c_double
            L.orc_gelu_tanh.argtypes = [ctypes.c_double]
            L.orc_gptq_factor.restype = ctypes.c_int
            L.orc_gptq_factor.argtypes = [P, i64, ctypes.c_double, P, P]
            L.orc_higptq1.restype = i64
            L.orc_higptq1.argtypes = [P, i64, i64, P, P, P, i64, P, P, P, P]
            L.orc_round_bf16.restype = ctypes.c_uint16
            L.orc_round_bf16.argtypes = [ctypes.c_double]
            L.orc_round_bf16_array.restype = None
            L.orc_round_bf16_array.argtypes = [P, i64, P]
            L.orc_linear.restype = None
            L.orc_linear.argtypes = [P, P, P, i64, i64, i64, ctypes.c_int, P]
            L.orc_percentile.restype = ctypes.c_int
            L.orc_percentile.argtypes = [P, i64, i64, i64, ctypes.c_uint, ctypes.c_uint, P]
            L.orc_channel_mask.restype = i64
            L.orc_channel_mask.argtypes = [P, i64, ctypes.c_uint, ctypes.c_uint, P, P]
            _lib = L
    return _lib


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


# ------------------------------------------------------------------ scalars

def e6m2_value(code: int) -> float:
    """Level-1 scale value 2^(E-31)(1+f/4) [HiF4 format; bias is a reading]."""
    return lib().orc_e6m2_value(int(code))


def select_scale_code(a: float) -> int:
    """Largest E6M2 code with 6.5·v < a (0 if none) [encode rule reading]."""
    return lib().orc_select_scale_code(float(a))


def round_magnitude(ax: float, step: float) -> int:
    """Nearest multiple m of ``step`` in 0..7, ties to even [encode rule]."""
    return lib().orc_round_magnitude(float(ax), float(step))


def quantize_unit(x, masked=None):
    """One 64-element unit → (64 nibble codes uint8, meta uint32)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64).reshape(64))
    m = None if masked is None else np.ascontiguousarray(np.asarray(masked, dtype=np.uint8).reshape(64))
    nib = np.zeros(64, np.uint8)
    meta = np.zeros(1, np.uint32)
    lib().orc_quantize_unit(_p(x), _p(m), _p(nib), _p(meta))
    return nib, int(meta[0])


def decode_element(nib: int, meta: int, i: int) -> float:
    return lib().orc_decode_element(int(nib), int(meta) & 0xFFFFFFFF, int(i))


# ------------------------------------------------------------------ tensors

def quantize(x: np.ndarray, chan_mask: np.ndarray | None = None):
    """Quantize a 2-D float32 or bf16-bit-pattern (uint16) array along rows.

    Returns (codes uint8 [rows, cols/2], meta uint32 [rows, cols/64], n_nonfinite).
    """
    assert x.ndim == 2
    if x.dtype == np.float32:
        dtype = 0
    elif x.dtype == np.uint16:
        dtype = 1
    else:
        raise TypeError("oracle.quantize takes float32 or bf16 bits (uint16)")
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    meta = np.zeros((rows, cols // 64), np.uint32)
    cm = None if chan_mask is None else np.ascontiguousarray(chan_mask.astype(np.uint8))
    n = lib().orc_quantize(_p(x), dtype, rows, cols, cols, _p(cm), _p(codes), _p(meta))
    if n < 0:
        raise ValueError("bad shape for HiF4 quantize (cols % 64 != 0?)")
    return codes, meta, int(n)


def dequantize(codes: np.ndarray, meta: np.ndarray, cols: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    rows = codes.shape[0]
    y = np.zeros((rows, cols), np.float64)
    lib().orc_dequantize(_p(codes), _p(meta), rows, cols, _p(y), cols)
    return y


def fake_quantize(x_bf16: np.ndarray, mask_idx=None) -> np.ndarray:
    """X̂ = deq(q(X with masked→0)), masked channels = X  (double, dense)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    mi = np.ascontiguousarray(np.asarray([] if mask_idx is None else mask_idx, dtype=np.int32))
    out = np.zeros((rows, cols), np.float64)
    n = lib().orc_fake_quantize(_p(x), rows, cols, cols, _p(mi) if mi.size else None,
                                int(mi.size), _p(out))
    if n < 0:
        raise ValueError("bad arguments for fake_quantize")
    return out


def weight_hat(codes, meta, N, K, mask_idx=None, w_masked_bf16=None) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    mi = np.ascontiguousarray(np.asarray([] if mask_idx is None else mask_idx, dtype=np.int32))
    wm = None
    if mi.size:
        wm = np.ascontiguousarray(w_masked_bf16, dtype=np.uint16)
        assert wm.shape == (N, mi.size)
    out = np.zeros((N, K), np.float64)
    lib().orc_weight_hat(_p(codes), _p(meta), N, K, _p(mi) if mi.size else None,
                         int(mi.size), _p(wm), _p(out))
    return out


def gelu_tanh(x: float) -> float:
    return lib().orc_gelu_tanh(float(x))


def gptq_factor(H: np.ndarray, damp: float = 0.01):
    """-> (U upper K x K with (H + damp mean(diag H) I)^{-1} = U^T U, dead flags K).

    Up to K = 1024 the C routine (textbook loops); beyond, the same three
    steps with numpy's Cholesky and inverse (library primitives), which the
    CPU tests pin against the C routine."""
    H = np.ascontiguousarray(H, dtype=np.float64)
    K = H.shape[0]
    if K > 1024:
        Hd = H.copy()
        dead = (np.diag(Hd) == 0).astype(np.uint8)
        Hd[np.diag_indices(K)] = np.where(dead == 1, 1.0, np.diag(Hd))
        Hd[np.diag_indices(K)] += damp * np.mean(np.diag(Hd))
        L = np.linalg.cholesky(Hd)
        Li = np.linalg.inv(L)
        U = np.linalg.cholesky(Li.T @ Li).T
        return np.ascontiguousarray(U), dead
    U = np.zeros((K, K), np.float64)
    dead = np.zeros(K, np.uint8)
    if lib().orc_gptq_factor(_p(H), K, float(damp), _p(U), _p(dead)) != 0:
        raise ValueError("Hessian is not positive definite after damping")
    return U, dead


def higptq1(w_bf16: np.ndarray, H: np.ndarray, chan_mask=None, damp: float = 0.01, blocksize: int = 128,
            threads: int = 1, factor=None):
    """HiGPTQ scheme one -> (codes N x K/2, meta N x K/64, wq N x K double,
    w_masked N x n_masked BF16 bits or None).  Rows are independent given the
    Hessian factor, so they are split over ``threads``."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    N, K = w.shape
    U, dead = gptq_factor(H, damp) if factor is None else factor
    cm = None if chan_mask is None else np.ascontiguousarray(chan_mask, dtype=np.uint8)
    nm = 0 if cm is None else int(np.count_nonzero(cm))
    codes = np.zeros((N, K // 2), np.uint8)
    meta = np.zeros((N, K // 64), np.uint32)
    wq = np.zeros((N, K), np.float64)
    wm = np.zeros((N, nm), np.uint16) if nm else None
    L = lib()

    def run(r0, r1):
        if r1 > r0:
            off = ctypes.c_void_p
            rc = L.orc_higptq1(off(w.ctypes.data + r0 * K * 2), r1 - r0, K, _p(U), _p(dead), _p(cm), blocksize,
                               off(codes.ctypes.data + r0 * (K // 2)), off(meta.ctypes.data + r0 * (K // 64) * 4),
                               off(wq.ctypes.data + r0 * K * 8),
                               off(wm.ctypes.data + r0 * nm * 2) if nm else None)
            if rc != 0:
                raise ValueError("bad arguments for higptq1")

    _split(N, threads, run)
    return codes, meta, wq, wm


def round_bf16(x) -> np.ndarray:
    """double array -> BF16 bit patterns (uint16), one round-to-nearest-even step."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.zeros(x.shape, np.uint16)
    lib().orc_round_bf16_array(_p(x), x.size, _p(out))
    return out


def linear(xhat: np.ndarray, what: np.ndarray, bias=None, gelu: bool = False,
           threads: int = 1) -> np.ndarray:
    """Y = X̂·Ŵᵀ + b in double (triple loop), optional GELU; rows split over
    ``threads`` Python threads (the C call releases the GIL)."""
    xhat = np.ascontiguousarray(xhat, dtype=np.float64)
    what = np.ascontiguousarray(what, dtype=np.float64)
    M, K = xhat.shape
    N = what.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    y = np.zeros((M, N), np.float64)
    L = lib()

    def run(r0, r1):
        if r1 > r0:
            L.orc_linear(ctypes.c_void_p(xhat.ctypes.data + r0 * K * 8), _p(what), _p(b),
                         r1 - r0, N, K, int(gelu), ctypes.c_void_p(y.ctypes.data + r0 * N * 8))

    _split(M, threads, run)
    return y


def percentile(acts_bf16: np.ndarray, q_num=999, q_den=1000, threads: int = 1) -> np.ndarray:
    """Per-channel order statistic of |x| keys → uint16 BF16 patterns."""
    a = acts_bf16
    assert a.dtype == np.uint16 and a.ndim == 2 and a.strides[1] == 2
    T, C = a.shape
    lda = a.strides[0] // 2
    out = np.zeros(C, np.uint16)
    L = lib()

    def run(c0, c1):
        if c1 > c0:
            r = L.orc_percentile(ctypes.c_void_p(a.ctypes.data + 2 * c0), T, c1 - c0, lda,
                                 q_num, q_den, ctypes.c_void_p(out.ctypes.data + 2 * c0))
            if r != 0:
                raise ValueError("bad arguments for percentile")

    _split(C, threads, run)
    return out


def channel_mask(pct_bf16: np.ndarray, mask_num=1, mask_den=100):
    """→ (ratio float32 [C], mask uint8 [C], n_masked)."""
    p = np.ascontiguousarray(pct_bf16, dtype=np.uint16)
    C = p.size
    ratio = np.zeros(C, np.float32)
    mask = np.zeros(C, np.uint8)
    n = lib().orc_channel_mask(_p(p), C, mask_num, mask_den, _p(ratio), _p(mask))
    if n < 0:
        raise ValueError("bad arguments for channel_mask")
    return ratio, mask, int(n)


def _split(n, threads, fn):
    threads = max(1, min(int(threads), n if n > 0 else 1))
    if threads == 1:
        fn(0, n)
        return
    bounds = [n * i // threads for i in range(threads + 1)]
    errs = []

    def wrap(a, b):
        try:
            fn(a, b)
        except Exception as e:  # pragma: no cover - surfaced below
            errs.append(e)

    ts = [threading.Thread(target=wrap, args=(bounds[i], bounds[i + 1])) for i in range(threads)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    if errs:
        raise errs[0]
