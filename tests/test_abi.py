"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point that include/hif4.h declares, and rejects bad arguments
before it touches a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hif4.h")


@pytest.fixture(scope="module")
def L():
    from block_floating_point_hif4_b200 import build
    build.build()
    from block_floating_point_hif4_b200 import binding
    return binding.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hif4_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_expected_calls():
    names = declared_functions()
    for want in ["hif4_quantize", "hif4_dequantize", "hif4_linear_w4a4", "hif4_calib_percentile_mask",
                 "hif4_fake_quantize", "hif4_get_status"]:
        assert want in names


def test_every_declared_symbol_is_exported(L):
    from block_floating_point_hif4_b200 import binding
    for name in declared_functions():
        assert hasattr(L, name), name
        assert name in binding.SIGNATURES, "binding lacks " + name


def test_status_strings_and_version(L):
    assert L.hif4_version() >= 100
    for code in range(10):
        assert L.hif4_status_string(code)


def test_workspace_sizes(L):
    M, N, K = 57600, 13824, 5120
    ws = L.hif4_linear_w4a4_workspace(M, N, K)
    assert ws >= 2 * (M * K + N * K) + K
    assert L.hif4_linear_w4a4_workspace(0, 1, 64) == 0
    assert L.hif4_calib_workspace(230400, 5120) >= 5120 * 384 * 4
    D, F = 5120, 13824
    assert L.hif4_ffn_w4a4_workspace(M, D, F) >= 2 * (M * D + F * D + M * F + D * F) + D + F
    assert L.hif4_ffn_w4a4_workspace(M, 0, F) == 0


def test_argument_errors_return_before_any_launch(L):
    P = ctypes.c_void_p
    fake = P(0x1000)          # never dereferenced: every call below fails validation first
    # cols not a multiple of 64
    assert L.hif4_quantize(fake, 1, 4, 100, 100, None, fake, fake, None, None) == 3
    # negative rows
    assert L.hif4_quantize(fake, 1, -1, 64, 64, None, fake, fake, None, None) == 1
    # ldx < cols
    assert L.hif4_quantize(fake, 1, 4, 128, 64, None, fake, fake, None, None) == 3
    # misaligned x
    assert L.hif4_quantize(P(0x1002), 1, 4, 64, 64, None, fake, fake, None, None) == 2
    # null output
    assert L.hif4_quantize(fake, 1, 4, 64, 64, None, None, fake, None, None) == 1
    # bad dtype
    assert L.hif4_quantize(fake, 7, 4, 64, 64, None, fake, fake, None, None) == 1
    # empty tensor is a no-op
    assert L.hif4_quantize(None, 1, 0, 64, 64, None, None, None, None, None) == 0
    assert L.hif4_dequantize(fake, fake, 4, 96, 1, fake, 96, None) == 3
    assert L.hif4_fake_quantize(fake, 4, 64, 64, None, P(0x1008), 64, None, None) == 2
    # linear: K % 64, workspace too small, mask without indices, misaligned y
    assert L.hif4_linear_w4a4(fake, 4, 100, 100, fake, fake, 8, None, 0, None, None, fake, 8, 0, fake, 1 << 30,
                              None, None) == 3
    assert L.hif4_linear_w4a4(fake, 4, 64, 64, fake, fake, 8, None, 0, None, None, fake, 8, 0, fake, 16,
                              None, None) == 4
    assert L.hif4_linear_w4a4(fake, 4, 64, 64, fake, fake, 8, None, 3, None, None, fake, 8, 0, fake, 1 << 30,
                              None, None) == 1
    assert L.hif4_linear_w4a4(fake, 4, 64, 64, fake, fake, 8, None, 0, None, None, P(0x1004), 8, 0, fake,
                              1 << 30, None, None) == 2
    assert L.hif4_linear_w4a4(fake, 4, 64, 64, fake, fake, 8, None, 0, None, None, fake, 8, 0x80, fake,
                              1 << 30, None, None) == 1
    # calibration: bad ratio, too small workspace
    assert L.hif4_calib_percentile_mask(fake, 10, 8, 8, 1001, 1000, 1, 100, fake, fake, fake, None, fake,
                                        1 << 30, None) == 1
    assert L.hif4_calib_percentile_mask(fake, 10, 8, 8, 999, 1000, 1, 100, fake, fake, fake, None, fake, 8,
                                        None) == 4
    # fused fake-quant GEMM: N % 64, FP32 output refused, misaligned mask
    assert L.hif4_gemm_bf16_fq(fake, 4, 64, 64, fake, 100, 64, None, None, fake, 100, 0, None, None) == 3
    assert L.hif4_gemm_bf16_fq(fake, 4, 64, 64, fake, 64, 64, None, None, fake, 64, 2, None, None) == 1
    assert L.hif4_gemm_bf16_fq(fake, 4, 64, 64, fake, 64, 64, None, P(0x1001), fake, 64, 0, None, None) == 2
    # the plain linear refuses the fused-output flag (it has no output mask)
    assert L.hif4_linear_w4a4(fake, 4, 64, 64, fake, fake, 64, None, 0, None, None, fake, 64, 4, fake,
                              1 << 30, None, None) == 1
    # FFN block: F % 64, unknown flag, workspace too small, mask2 count without indices
    ffn = L.hif4_ffn_w4a4
    assert ffn(fake, 4, 64, 64, fake, fake, 100, None, 0, None, None, fake, fake, None, 0, None, None, fake, 64,
               0, fake, 1 << 30, None, None) == 3
    assert ffn(fake, 4, 64, 64, fake, fake, 128, None, 0, None, None, fake, fake, None, 0, None, None, fake, 64,
               1, fake, 1 << 30, None, None) == 1
    assert ffn(fake, 4, 64, 64, fake, fake, 128, None, 0, None, None, fake, fake, None, 0, None, None, fake, 64,
               0, fake, 64, None, None) == 4
    assert ffn(fake, 4, 64, 64, fake, fake, 128, None, 0, None, None, fake, fake, None, 2, None, None, fake, 64,
               0, fake, 1 << 30, None, None) == 1
    assert L.hif4_get_status(None, None) == 1
