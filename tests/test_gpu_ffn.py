"""GPU checks of the fused FFN path.

1. hif4_gemm_bf16_fq (HiF4 fake quantization of the GEMM output inside its
   epilogue) is the same function as hif4_gemm_bf16 followed by
   hif4_fake_quantize: compared bit for bit on ragged shapes, protected
   output columns, bias, GELU and the generic path (huge and non-finite
   accumulators).  The standalone quantizer is itself pinned bit-exactly to
   the oracle by tests/test_gpu_quant.py.
2. hif4_ffn_w4a4 against the FP64 oracle composition
      Hhat = fq(bf16(gelu(fq(x) what1^T + b1)), mask2),  y = Hhat what2^T + b2
   with the linear layers' tolerance (relative Frobenius <= 5e-3, |dY| <=
   2e-2 x row RMS on the FP32 output).  The BF16 rounding of H can differ
   from the FP64 oracle's where FP32 accumulation lands next to a rounding
   boundary, so the fused Hhat is required to equal the oracle's on all but
   a small fraction of elements (<= 1e-3).
Method: Tail-Aware HiFloat4 arXiv abstract (W4A4 fake quantization of the
main linears, protected channels kept); the GELU between the two linears and
the BF16 hidden activation are the library's readings.
"""
import numpy as np
import pytest

import oracle
from block_floating_point_hif4_b200 import workloads as wl
from tests._util import THREADS, assert_linear_close, bf16_bits_to_f64, meta_u32, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import block_floating_point_hif4_b200 as h
    from block_floating_point_hif4_b200 import build
    build.build()
    return h


def _bf16(rng, shape, scale=1.0):
    return wl.f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def fused_vs_two_kernels(H, a_bits, b_bits, bias_bits=None, gelu=False, out_mask=None):
    import torch
    a, b = to_dev_bf16(a_bits), to_dev_bf16(b_bits)
    bias = None if bias_bits is None else to_dev_bf16(bias_bits)
    N = b_bits.shape[0]
    cm = None if out_mask is None else torch.from_numpy(out_mask.astype(np.uint8)).cuda()
    s1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    s2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    fused = H.gemm_bf16_fq(a, b, bias, gelu=gelu, out_chan_mask=cm, status=s1)
    h = H.gemm_bf16(a, b, bias, gelu=gelu, status=s2)
    ref = H.fake_quantize(h, cm, status=s2)
    torch.cuda.synchronize()
    assert torch.equal(fused.view(torch.int16), ref.view(torch.int16)), \
        "fused != gemm + fake_quantize at %s" % (fused != ref).nonzero()[:5].tolist()
    return H.get_status(s1), H.get_status(s2), N


@pytest.mark.parametrize("M,N,K", [(1, 64, 64), (130, 320, 128), (300, 512, 256), (1000, 1088, 192)])
@pytest.mark.parametrize("gelu", [False, True])
def test_fused_equals_gemm_then_fake_quantize(H, M, N, K, gelu):
    rng = np.random.default_rng(M + N + K + gelu)
    a = _bf16(rng, (M, K))
    b = _bf16(rng, (N, K), 0.1)
    bias = _bf16(rng, (N,), 0.5)
    mask = (rng.random(N) < 0.03).astype(np.uint8)
    mask[:64] = 0                      # one unit with no protected column
    if N >= 192:
        mask[64:128] = 1               # one unit entirely protected
    st1, st2, _ = fused_vs_two_kernels(H, a, b, bias, gelu, mask)
    assert st1 == st2 == 0
    fused_vs_two_kernels(H, a, b, None, gelu, None)


def test_fused_generic_path_huge_and_nonfinite(H):
    """Accumulators beyond the top scale code (> 6.5 v(254)) and beyond FP32
    range (Inf, and NaN from GELU(-Inf)) take the generic path in both."""
    rng = np.random.default_rng(5)
    M, N, K = 256, 256, 64
    a = _bf16(rng, (M, K))
    b = _bf16(rng, (N, K))
    a[:40] = wl.f32_to_bf16_bits((rng.standard_normal((40, K)) * 1e6).astype(np.float32))
    b[:, :8] = wl.f32_to_bf16_bits((rng.standard_normal((N, 8)) * 1e6).astype(np.float32))
    a[40:48] = wl.f32_to_bf16_bits(np.full((8, K), 3e38, np.float32))     # rows of Inf / NaN after GELU
    for gelu in (False, True):
        st1, st2, _ = fused_vs_two_kernels(H, a, b, None, gelu, None)
        assert st1 == st2 == 6                                              # HIF4_ERR_NONFINITE


def _quantize_w(H, w_bits, mask_idx):
    import torch
    K = w_bits.shape[1]
    cm = np.zeros(K, np.uint8)
    cm[mask_idx] = 1
    wc, wm = H.quantize(to_dev_bf16(w_bits), torch.from_numpy(cm).cuda())
    return wc, wm


def oracle_ffn(x_bits, w1_bits, w2_bits, idx1, idx2, b1_bits, b2_bits, rows):
    D, F = x_bits.shape[1], w1_bits.shape[0]
    c1 = np.zeros(D, np.uint8)
    c1[idx1] = 1
    c2 = np.zeros(F, np.uint8)
    c2[idx2] = 1
    q1c, q1m, _ = oracle.quantize(w1_bits, c1)
    q2c, q2m, _ = oracle.quantize(w2_bits, c2)
    what1 = oracle.weight_hat(q1c, q1m, F, D, idx1, np.ascontiguousarray(w1_bits[:, idx1]))
    what2 = oracle.weight_hat(q2c, q2m, D, F, idx2, np.ascontiguousarray(w2_bits[:, idx2]))
    xhat = oracle.fake_quantize(np.ascontiguousarray(x_bits[rows]), idx1)
    b1 = None if b1_bits is None else bf16_bits_to_f64(b1_bits)
    b2 = None if b2_bits is None else bf16_bits_to_f64(b2_bits)
    h = oracle.linear(xhat, what1, b1, gelu=True, threads=THREADS)
    h_bits = oracle.round_bf16(h)
    hhat = oracle.fake_quantize(h_bits, idx2)
    y = oracle.linear(hhat, what2, b2, threads=THREADS)
    return y, hhat, (q1c, q1m, q2c, q2m)


def run_ffn(H, x_bits, w1_bits, w2_bits, idx1, idx2, b1_bits=None, b2_bits=None, rows=None):
    import torch
    M, D = x_bits.shape
    F = w1_bits.shape[0]
    rows = np.arange(M) if rows is None else rows
    w1c, w1m = _quantize_w(H, w1_bits, idx1)
    w2c, w2m = _quantize_w(H, w2_bits, idx2)
    i1 = torch.from_numpy(np.asarray(idx1, np.int32)).cuda()
    i2 = torch.from_numpy(np.asarray(idx2, np.int32)).cuda()
    w1m_bf = to_dev_bf16(np.ascontiguousarray(w1_bits[:, idx1]))
    w2m_bf = to_dev_bf16(np.ascontiguousarray(w2_bits[:, idx2]))
    b1 = None if b1_bits is None else to_dev_bf16(b1_bits)
    b2 = None if b2_bits is None else to_dev_bf16(b2_bits)
    x = to_dev_bf16(x_bits)
    ws = torch.empty(H.ffn_w4a4_workspace(M, D, F), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    args = (x, w1c, w1m, F, w2c, w2m, i1, w1m_bf, b1, i2, w2m_bf, b2)
    y = H.ffn_w4a4(*args, workspace=ws, status=status)
    y32 = H.ffn_w4a4(*args, workspace=ws, status=status,
                     out=torch.empty(M, D, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    assert H.get_status(status) == 0
    assert torch.equal(y, y32.to(torch.bfloat16))
    # Hhat as the fused epilogue left it in the workspace (BF16 M x F)
    off = _a256(M * D * 2) + _a256(F * D * 2)
    hhat_dev = ws[off:off + M * F * 2].view(torch.int16).view(M, F)
    r_dev = torch.from_numpy(rows).cuda()
    hhat_rows = hhat_dev[r_dev].cpu().numpy().view(np.uint16)
    y_rows = y32[r_dev].cpu().numpy().astype(np.float64)
    y_ref, hhat_ref, (q1c, q1m, q2c, q2m) = oracle_ffn(x_bits, w1_bits, w2_bits, idx1, idx2, b1_bits, b2_bits,
                                                       rows)
    assert np.array_equal(q1c, w1c.cpu().numpy()) and np.array_equal(q1m, meta_u32(w1m))
    assert np.array_equal(q2c, w2c.cpu().numpy()) and np.array_equal(q2m, meta_u32(w2m))
    mismatch = np.mean(bf16_bits_to_f64(hhat_rows) != hhat_ref)
    assert mismatch <= 1e-3, "fused Hhat differs from the oracle's on %.2e of elements" % mismatch
    return assert_linear_close(y_rows, y_ref), mismatch


def _a256(v):
    return (v + 255) // 256 * 256


@pytest.mark.parametrize("M,D,F", [(1, 64, 64), (257, 256, 512), (600, 320, 1024)])
def test_ffn_small_vs_oracle(H, M, D, F):
    rng = np.random.default_rng(M + D + F)
    x = _bf16(rng, (M, D))
    x[:, 5] = wl.f32_to_bf16_bits((rng.standard_normal(M) * 30).astype(np.float32))
    w1 = _bf16(rng, (F, D), 1.0 / np.sqrt(D))
    w2 = _bf16(rng, (D, F), 1.0 / np.sqrt(F))
    b1, b2 = _bf16(rng, (F,), 0.1), _bf16(rng, (D,), 0.1)
    idx1 = np.array([5] if D > 5 else [], np.int32)
    idx2 = np.sort(rng.choice(F, max(1, F // 100), replace=False)).astype(np.int32)
    run_ffn(H, x, w1, w2, idx1, idx2, b1, b2)


@pytest.mark.slow
def test_ffn_full_size(H):
    """Wan2.2 FFN block (57600 x 5120 -> 13824 -> 5120, masks from the
    calibration rule), the benchmark's launch configuration: 256 sampled
    rows against the oracle."""
    import torch
    d = wl.ffn(seed=3)
    rows = wl.sample_rows(wl.WAN_TOKENS, 256)
    _, m1, _ = oracle.channel_mask(oracle.percentile(d["x"], threads=THREADS))
    h = wl.ffn_hidden(wl.WAN_TOKENS)
    _, m2, _ = oracle.channel_mask(oracle.percentile(h, threads=THREADS))
    del h
    idx1 = np.nonzero(m1)[0].astype(np.int32)
    idx2 = np.nonzero(m2)[0].astype(np.int32)
    run_ffn(H, d["x"], d["w1"], d["w2"], idx1, idx2, None, None, rows=rows)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("M,chunk", [(1000, 256), (777, 0), (300, 1000), (40000, 0)])
def test_ffn_host_pipeline_equals_device_call(H, M, chunk):
    """hif4_ffn_w4a4_host (pinned host x / y, chunked, copies overlapping
    compute) gives exactly the rows hif4_ffn_w4a4 gives on device buffers:
    per-row work and per-element accumulation order do not depend on the
    chunking.  Strided host rows, a ragged last chunk, the automatic ramped
    schedule (40000 rows: 1024, 2048, ten middle chunks, 2048, 1024) and
    FP32 output."""
    import torch
    D, F = 256, 512
    rng = np.random.default_rng(M + chunk)
    x_bits = _bf16(rng, (M, D))
    w1, w2 = _bf16(rng, (F, D), 1.0 / 16), _bf16(rng, (D, F), 1.0 / 22)
    b1, b2 = to_dev_bf16(_bf16(rng, (F,), 0.1)), to_dev_bf16(_bf16(rng, (D,), 0.1))
    idx1 = np.array([3, 77], np.int32)
    idx2 = np.sort(rng.choice(F, 6, replace=False)).astype(np.int32)
    w1c, w1m = _quantize_w(H, w1, idx1)
    w2c, w2m = _quantize_w(H, w2, idx2)
    i1 = torch.from_numpy(idx1).cuda()
    i2 = torch.from_numpy(idx2).cuda()
    w1k = to_dev_bf16(np.ascontiguousarray(w1[:, idx1]))
    w2k = to_dev_bf16(np.ascontiguousarray(w2[:, idx2]))
    args = (w1c, w1m, F, w2c, w2m, i1, w1k, b1, i2, w2k, b2)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y_dev = H.ffn_w4a4(to_dev_bf16(x_bits), *args, status=status)
    y_dev32 = H.ffn_w4a4(to_dev_bf16(x_bits), *args, status=status,
                         out=torch.empty(M, D, dtype=torch.float32, device="cuda"))
    # host rows with a leading dimension larger than D
    xh = torch.zeros(M, D + 64, dtype=torch.bfloat16, pin_memory=True)
    xh[:, :D] = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16)
    yh = torch.full((M, D + 32), float("nan"), dtype=torch.bfloat16, pin_memory=True)
    H.ffn_w4a4_host(xh[:, :D], *args, out=yh[:, :D], chunk_rows=chunk, status=status)
    yh32 = H.ffn_w4a4_host(xh[:, :D], *args, out=torch.empty(M, D, dtype=torch.float32, pin_memory=True),
                           chunk_rows=chunk, status=status)
    torch.cuda.synchronize()
    assert H.get_status(status) == 0
    assert torch.equal(yh[:, :D].view(torch.int16), y_dev.cpu().view(torch.int16))
    assert torch.isnan(yh[:, D:]).all()                       # the padding past D is untouched
    assert torch.equal(yh32.view(torch.int32), y_dev32.cpu().view(torch.int32))
