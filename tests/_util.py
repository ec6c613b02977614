"""Helpers shared by the GPU parity tests (host <-> device marshalling and
the tolerance the linear layer is held to)."""
import os

import numpy as np

THREADS = max(1, len(os.sched_getaffinity(0)))


def to_dev_bf16(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).cuda()


def to_host_bits(t) -> np.ndarray:
    import torch
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def meta_u32(t) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


def assert_linear_close(y_gpu: np.ndarray, y_ref: np.ndarray, rel_fro=5e-3, row_rel=2e-2):
    """Tolerance of the fake-quantized linear on its FP32 result: relative
    Frobenius error <= 5e-3 and every element within 2e-2 x the RMS of its
    row (FP64 reference).  Accepts FP32/FP64 values or BF16 bit patterns."""
    y = bf16_bits_to_f64(y_gpu) if y_gpu.dtype == np.uint16 else np.asarray(y_gpu, np.float64)
    assert y.shape == y_ref.shape
    assert np.all(np.isfinite(y))
    err = y - y_ref
    fro = np.linalg.norm(err) / max(np.linalg.norm(y_ref), 1e-300)
    assert fro <= rel_fro, "relative Frobenius error %.3e > %.1e" % (fro, rel_fro)
    rms = np.sqrt(np.mean(y_ref ** 2, axis=1, keepdims=True))
    worst = np.max(np.abs(err) / np.maximum(rms, 1e-300))
    assert worst <= row_rel, "max |dY| / row RMS = %.3e > %.1e" % (worst, row_rel)
    return fro, worst
