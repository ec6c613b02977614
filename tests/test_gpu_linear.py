"""GPU parity: hif4_linear_w4a4 (tcgen05 GEMM on the fake-quantized operands)
against the FP64 oracle linear on the same seeded inputs.

Tolerance, on the FP32 result (HIF4_LINEAR_OUT_F32): relative Frobenius
error <= 5e-3 and |dY| <= 2e-2 x the row's RMS, every row for small shapes, a
seeded 1024-row sample (last row included) for the Wan2.2-shaped workloads.
The BF16 output is checked to be exactly the round-to-nearest-even of that
FP32 result (BF16 rounding alone can reach 2e-2 x RMS on elements larger
than ~10 x RMS, so the bound is not applied to the rounded output).
Method: Tail-Aware HiFloat4 arXiv abstract (W4A4 HiF4 fake quantization of
the main linears, protected channels kept in high precision).
"""
import numpy as np
import pytest

import oracle
from block_floating_point_hif4_b200 import workloads as wl
from tests._util import THREADS, assert_linear_close, bf16_bits_to_f64, meta_u32, to_dev_bf16, to_host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import block_floating_point_hif4_b200 as h
    from block_floating_point_hif4_b200 import build
    build.build()
    return h


def run_case(H, x_bits, w_bits, mask_idx=None, bias_bits=None, gelu=False, rows=None):
    """GPU: quantize W (protected columns excluded), linear on X.
    Oracle: its own quantize of W, fake-quant of X rows, FP64 product."""
    import torch
    M, K = x_bits.shape
    N = w_bits.shape[0]
    chan_mask = None
    if mask_idx is not None and len(mask_idx):
        chan_mask = np.zeros(K, np.uint8)
        chan_mask[mask_idx] = 1
    wd = to_dev_bf16(w_bits)
    cm = None if chan_mask is None else torch.from_numpy(chan_mask).cuda()
    wc, wm = H.quantize(wd, cm)
    midx = None if chan_mask is None else torch.from_numpy(np.asarray(mask_idx, np.int32)).cuda()
    wmask = None if chan_mask is None else to_dev_bf16(np.ascontiguousarray(w_bits[:, mask_idx]))
    bias = None if bias_bits is None else to_dev_bf16(bias_bits)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xd = to_dev_bf16(x_bits)
    y = H.linear_w4a4(xd, wc, wm, N, midx, wmask, bias, gelu=gelu, status=status)
    y32 = H.linear_w4a4(xd, wc, wm, N, midx, wmask, bias, gelu=gelu, status=status,
                        out=torch.empty(M, N, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    assert H.get_status(status) == 0
    # the BF16 output is exactly the round-to-nearest-even of the FP32 result
    assert torch.equal(y, y32.to(torch.bfloat16))
    rows = np.arange(M) if rows is None else rows
    y_rows = y32[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    # oracle
    ref_c, ref_m, _ = oracle.quantize(w_bits, chan_mask)
    assert np.array_equal(ref_c, wc.cpu().numpy()) and np.array_equal(ref_m, meta_u32(wm))
    what = oracle.weight_hat(ref_c, ref_m, N, K, mask_idx,
                             None if chan_mask is None else np.ascontiguousarray(w_bits[:, mask_idx]))
    xhat = oracle.fake_quantize(np.ascontiguousarray(x_bits[rows]), mask_idx)
    b = None if bias_bits is None else bf16_bits_to_f64(bias_bits)
    y_ref = oracle.linear(xhat, what, b, gelu=gelu, threads=THREADS)
    return assert_linear_close(y_rows, y_ref)


def test_tiny_workload(H):
    """128x512 activations and 512x512 weights (FP32 source, 327 outliers x50):
    quantize/dequantize X and W, then the linear on the dequantized X."""
    import torch
    X, W = wl.tiny(0)
    xd = torch.from_numpy(X).cuda()
    c, m = H.quantize(xd)
    xhat_bits = to_host_bits(H.dequantize(c, m, 512))
    ref_x = oracle.dequantize(*oracle.quantize(X)[:2], 512)
    assert np.array_equal(bf16_bits_to_f64(xhat_bits), ref_x)
    w_bits = wl.f32_to_bf16_bits(W)
    # fp32 W goes through quantize (fp32 path) == bf16 of its dequantized values
    wc, wm = H.quantize(torch.from_numpy(W).cuda())
    ref_wc, ref_wm, _ = oracle.quantize(W)
    assert np.array_equal(wc.cpu().numpy(), ref_wc) and np.array_equal(meta_u32(wm), ref_wm)
    y = H.linear_w4a4(to_dev_bf16(xhat_bits), wc, wm, 512, out=torch.empty(128, 512, device="cuda"))
    what = oracle.dequantize(ref_wc, ref_wm, 512)
    y_ref = oracle.linear(ref_x, what, None, threads=THREADS)
    assert_linear_close(y.cpu().numpy().astype(np.float64), y_ref)
    del w_bits


@pytest.mark.parametrize("M,N,K", [(1, 8, 64), (5, 40, 128), (128, 256, 64), (300, 320, 192),
                                   (257, 520, 640), (1000, 768, 1024)])
def test_shapes_ragged(H, M, N, K):
    d = wl.attn_proj(M=M, K=K, N=N, seed=M + N + K)
    run_case(H, d["x"], d["w"])


@pytest.mark.parametrize("gelu", [False, True])
def test_mask_bias_gelu(H, gelu):
    d = wl.attn_proj(M=333, K=640, N=264, seed=12)
    idx = np.array(sorted(set(d["mask_idx"].tolist() + [0, 639])), np.int32)
    run_case(H, d["x"], d["w"], idx, d["bias"], gelu=gelu)


def test_bad_mask_index_flags_status(H):
    import torch
    d = wl.attn_proj(M=64, K=128, N=64, seed=3)
    wc, wm = H.quantize(to_dev_bf16(d["w"]))
    idx = torch.tensor([5, 3], dtype=torch.int32, device="cuda")          # unsorted
    wmask = torch.zeros(64, 2, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    H.linear_w4a4(to_dev_bf16(d["x"]), wc, wm, 64, idx, wmask, status=status)
    assert H.get_status(status) == 1
    H.reset_status(status)
    assert H.get_status(status) == 0


@pytest.mark.slow
def test_attn_projection_full_size(H):
    """57600 x 5120 -> 5120 with the 51 x20 outlier channels protected and a
    bias: the benchmark's launch configuration, 1024 sampled rows."""
    d = wl.attn_proj(seed=2)
    rows = wl.sample_rows(wl.WAN_TOKENS, 1024)
    run_case(H, d["x"], d["w"], d["mask_idx"], d["bias"], rows=rows)


@pytest.mark.slow
def test_ffn_full_size(H):
    """Wan2.2 FFN shapes: 57600 x 5120 -> 13824 with tanh-GELU (mask from the
    calibration rule on X), then 13824 -> 5120 on a GELU-shaped hidden input
    (mask from the rule on it); 1024 sampled rows each."""
    import torch
    d = wl.ffn(seed=3)
    rows = wl.sample_rows(wl.WAN_TOKENS, 1024)
    p = oracle.percentile(d["x"], threads=THREADS)
    _, m1, _ = oracle.channel_mask(p)
    idx1 = np.nonzero(m1)[0].astype(np.int32)
    run_case(H, d["x"], d["w1"], idx1, None, gelu=True, rows=rows)
    del d["x"]
    h = wl.ffn_hidden(wl.WAN_TOKENS)
    p2 = oracle.percentile(h, threads=THREADS)
    _, m2, n2 = oracle.channel_mask(p2)
    assert n2 == 138
    idx2 = np.nonzero(m2)[0].astype(np.int32)
    run_case(H, h, d["w2"], idx2, None, rows=rows)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("M,N,K", [(1, 8, 64), (129, 256, 128), (300, 520, 640), (512, 264, 576)])
@pytest.mark.parametrize("gelu", [False, True])
def test_linear_equals_its_stages(H, M, N, K, gelu):
    """hif4_linear_w4a4 is hif4_fake_quantize + hif4_weight_decode +
    hif4_gemm_bf16, bit for bit (the staged form a caller uses to decode a
    static weight once); protected columns at both ends of K and two
    adjacent ones inside one 64-column unit."""
    import torch
    d = wl.attn_proj(M=M, K=K, N=N, seed=M + 3 * N + K)
    idx = np.array(sorted({0, 5, 6, K // 2 + 1, K - 1}), np.int32)
    mask = np.zeros(K, np.uint8)
    mask[idx] = 1
    cm = torch.from_numpy(mask).cuda()
    wd = to_dev_bf16(d["w"])
    wc, wm = H.quantize(wd, cm)
    midx = torch.from_numpy(idx).cuda()
    wmask = to_dev_bf16(np.ascontiguousarray(d["w"][:, idx]))
    bias = to_dev_bf16(d["bias"])
    xd = to_dev_bf16(d["x"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = H.linear_w4a4(xd, wc, wm, N, midx, wmask, bias, gelu=gelu, status=status,
                      out=torch.empty(M, N, dtype=torch.float32, device="cuda"))
    xhat = H.fake_quantize(xd, cm, status=status)
    what = torch.empty(N, K, dtype=torch.bfloat16, device="cuda")
    H.weight_decode(wc, wm, N, K, midx, wmask, out=what, status=status)
    ys = H.gemm_bf16(xhat, what, bias, gelu=gelu, status=status,
                     out=torch.empty(M, N, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    assert H.get_status(status) == 0
    assert torch.equal(y, ys)
