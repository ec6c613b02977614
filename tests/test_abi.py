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


def test_higptq_hessian_and_host_ffn_argument_errors(L):
    P = ctypes.c_void_p
    fake = P(0x1000)          # never dereferenced: every call below fails validation first
    # HiGPTQ workspace: K % 64 and unsupported block sizes give 0; it grows with N
    assert L.hif4_higptq1_workspace(16, 100, 128) == 0
    assert L.hif4_higptq1_workspace(16, 512, 100) == 0
    assert L.hif4_higptq1_workspace(16, 512, 320) == 0
    assert 0 < L.hif4_higptq1_workspace(16, 512, 0) == L.hif4_higptq1_workspace(16, 512, 128)
    assert L.hif4_higptq1_workspace(1024, 512, 128) > L.hif4_higptq1_workspace(16, 512, 128)
    ws = L.hif4_higptq1_workspace(16, 512, 128)
    # the group-inputs array lies inside the workspace, 256-byte aligned; refused shapes give (size_t)-1
    for N, K, bs in ((16, 512, 128), (3000, 1024, 64), (70, 320, 0), (13824, 5120, 128)):
        off = L.hif4_higptq1_group_inputs_offset(N, K, bs)
        assert off % 256 == 0 and off + N * K * 4 <= L.hif4_higptq1_workspace(N, K, bs)
    assert L.hif4_higptq1_group_inputs_offset(16, 100, 128) == ctypes.c_size_t(-1).value
    assert L.hif4_higptq1_group_inputs_offset(16, 512, 320) == ctypes.c_size_t(-1).value

    def gptq(w=fake, N=16, K=512, ldw=512, H=fake, idx=None, nm=0, damp=0.01, bs=128, codes=fake, meta=fake,
             wm=None, work=fake, wsb=ws):
        return L.hif4_higptq1(w, N, K, ldw, H, idx, nm, damp, bs, codes, meta, wm, work, wsb, None, None)

    assert gptq(K=100, ldw=100) == 3     # K not a multiple of 64
    assert gptq(ldw=256) == 3            # ldw < K
    assert gptq(bs=100) == 1             # block size not a multiple of 64
    assert gptq(bs=320) == 1             # block size above 256
    assert gptq(damp=-1.0) == 1          # negative damping
    assert gptq(N=0) == 1
    assert gptq(K=32832, ldw=32832) == 8  # K above the supported 32768
    assert gptq(nm=3) == 1               # protected count without indices
    assert gptq(H=None) == 1
    assert gptq(meta=P(0x1002)) == 2     # misaligned metadata
    assert gptq(wsb=ws - 1) == 4         # workspace too small
    assert gptq(work=P(0x1010)) == 2     # workspace not 256-byte aligned
    # Hessian
    assert L.hif4_hessian_workspace(3001, 256) > 0
    hs = L.hif4_hessian_workspace(3001, 256)
    assert L.hif4_hessian(fake, 3001, 100, 100, fake, fake, hs, None, None) == 3
    assert L.hif4_hessian(fake, 3001, 256, 128, fake, fake, hs, None, None) == 3
    assert L.hif4_hessian(None, 3001, 256, 256, fake, fake, hs, None, None) == 1
    assert L.hif4_hessian(fake, 3001, 256, 256, P(0x1004), fake, hs, None, None) == 2
    assert L.hif4_hessian(fake, 3001, 256, 256, fake, fake, hs - 1, None, None) == 4
    # FFN on host buffers: unknown flag, null host input, ldx < D, workspace too small
    fh = L.hif4_ffn_w4a4_host

    def ffn_host(x=fake, M=64, D=64, ldx=64, F=128, y=fake, ldy=64, flags=0, work=fake, wsb=1 << 30):
        return fh(x, M, D, ldx, fake, fake, F, None, 0, None, None, fake, fake, None, 0, None, None, y, ldy, 0,
                  flags, work, wsb, None, None)

    assert ffn_host(flags=0x10) == 1     # no such flag
    assert ffn_host(x=None) == 1
    assert ffn_host(ldx=32) == 3
    assert ffn_host(F=100) == 3
    assert ffn_host(wsb=64) == 4
    assert ffn_host(M=0) == 0            # nothing to do


def test_fp8_remap_and_gemm_argument_errors(L):
    P = ctypes.c_void_p
    fake = P(0x1000)          # never dereferenced: every call below fails validation first
    assert L.hif4_to_e4m3(fake, fake, 4, 100, fake, 128, fake, 4, None) == 3      # cols % 64
    assert L.hif4_to_e4m3(fake, fake, 4, 128, fake, 64, fake, 4, None) == 3       # ldq < cols
    assert L.hif4_to_e4m3(fake, fake, 4, 128, fake, 128, fake, 3, None) == 3      # lds < rows
    assert L.hif4_to_e4m3(P(0x1001), fake, 4, 128, fake, 128, fake, 4, None) == 2  # codes misaligned
    assert L.hif4_to_e4m3(fake, fake, 0, 128, fake, 128, fake, 0, None) == 0      # nothing to do

    def f8(M=200, K=256, lda=256, sa=fake, lds_a=256, N=300, ldb=256, sb=fake, lds_b=512, y=fake, ldy=300,
           flags=0):
        return L.hif4_gemm_f8(fake, M, K, lda, sa, lds_a, fake, N, ldb, sb, lds_b, y, ldy, flags, None, None)

    assert f8(K=100, lda=128, ldb=128) == 3      # K % 64
    assert f8(K=64, lda=64, ldb=64) == 3         # K below the 128-byte operand box
    assert f8(lds_a=200) == 3                    # row scales not padded to 128 rows
    assert f8(lds_b=300) == 3                    # column scales not padded to 256 columns
    assert f8(lda=200) == 3                      # lda < K
    assert f8(lda=264) == 2                      # lda not a multiple of 16 bytes
    assert f8(sa=P(0x1004)) == 2                 # scales not 16-byte aligned
    assert f8(flags=1) == 1                      # GELU is not an option of this product
    assert f8(y=None) == 1
    assert f8(M=0) == 0
