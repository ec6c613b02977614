"""The per-group validity check of a HiGPTQ scheme-one result [HiF4
article, section 3.1], shared by the GPU parity tests and the CPU test that
plants a wrong feedback in an oracle run to show that the check catches it.

A result is (codes, meta, w_masked BF16 bits or None, group inputs FP32
N x K), the group inputs being the values each 64-column group was
quantized from.  Each group is a correct HiGPTQ step when
  (a) its codes and metadata equal the oracle's plain HiF4 quantization of
      its inputs, bit for bit, and a protected column holds their BF16
      rounding; and
  (b) its inputs equal the FP64 GPTQ feedback W0_h - sum_{g<h} E_g U_{g,h},
      E_g = (W_g - Q_g) U_gg^-1 from the result's own W_g and Q_g, within
      2^-12 x (|W0| + (|D| |U_gg^-1|) |U_{g,h}|) (absolute values summed):
      about twice the worst case of FP32 arithmetic with split-TF32
      products (FP32 rounding of U, <= 1536-term FP32 accumulations per
      update launch: three products per element of a 512-deep super-block
      update, <= 64-term ones for E, one rounding of W per update: about
      2^-13.3 of that sum).
"""
import numpy as np

import oracle
from block_floating_point_hif4_b200 import workloads as wl


def check_group_steps(w_bits, idx, got, factor, rows=None):
    """Asserts (a) and (b) of the module docstring for every group of the
    given rows; returns the largest error / bound ratio of the feedback."""
    U, dead = factor
    K = w_bits.shape[1]
    rows = np.arange(w_bits.shape[0]) if rows is None else rows
    codes, meta, gin = got[0][rows], got[1][rows], got[3][rows]
    wm = None if got[2] is None else got[2][rows]
    mask = None
    if len(idx):
        mask = np.zeros(K, np.uint8)
        mask[idx] = 1
    # (a) each group = the plain HiF4 quantization of the values it was quantized from
    c_ref, m_ref, _ = oracle.quantize(np.ascontiguousarray(gin, np.float32), mask)
    assert np.array_equal(codes, c_ref), "codes differ from the plain quantization of the group inputs"
    assert np.array_equal(meta, m_ref), "metadata differ from the plain quantization of the group inputs"
    if len(idx):
        assert np.array_equal(wm, oracle.round_bf16(gin[:, idx].astype(np.float64)))
    # (b) the group inputs follow the FP64 error feedback from the GPU's own errors
    w0 = wl.bf16_bits_to_f32(w_bits[rows]).astype(np.float64)
    w0[:, dead == 1] = 0.0
    q = oracle.dequantize(codes, meta, K)
    if len(idx):
        q[:, idx] = wl.bf16_bits_to_f32(wm).astype(np.float64)
    d = gin.astype(np.float64) - q
    e = np.empty_like(d)
    dabs = np.empty_like(d)
    for g in range(K // 64):
        s = slice(64 * g, 64 * g + 64)
        ui = np.linalg.inv(U[s, s])
        e[:, s] = d[:, s] @ ui
        dabs[:, s] = np.abs(d[:, s]) @ np.abs(ui)
    grp = np.arange(K) // 64
    usb = np.where(grp[:, None] < grp[None, :], U, 0.0)           # U_{g,h}, g < h
    pred = w0 - e @ usb
    bound = 2.0 ** -12 * (np.abs(w0) + dabs @ np.abs(usb)) + 1e-30
    ratio = np.abs(pred - gin) / bound
    assert np.all(ratio <= 1.0), "group inputs off the FP64 feedback: max ratio %.3g at %s" % (
        ratio.max(), np.unravel_index(np.argmax(ratio), ratio.shape))
    return float(ratio.max())
