"""GPU checks of the FP8-E4M3 remap of HiF4 and of the FP8 tensor-core
product built on it (hif4_to_e4m3, hif4_gemm_f8) [Huawei HiF4 calibration
article, section 1: an element is (-1)^s (m/4) 2^(e2+e3) S].

  * the remap is exact: E4M3 byte x unit scale, decoded here from the E4M3
    format's definition, equals the oracle's dequantized value for every
    element, and the scales are the E6M2 values;
  * the FP8 MMA is exact on these operands: with unit scales, every output
    of products of remapped values (multiples of 1/16 up to 49, 64 per unit)
    equals the exact integer-arithmetic sum, bit for bit, on adversarial
    patterns (largest product first then the smallest ones, alternating
    signs, every value of the remap) at 2, 8 and 9 units of K;
  * with real unit scales the product is the fake-quantized linear: within
    the linear tolerance of the FP64 oracle on the dequantized operands, and
    the BF16 output is the round to nearest even of the FP32 one.
"""
import numpy as np
import pytest

import oracle
from block_floating_point_hif4_b200 import workloads as wl
from tests._util import assert_linear_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import block_floating_point_hif4_b200 as h
    from block_floating_point_hif4_b200 import build
    build.build()
    return h


def e4m3_value(b):
    """FP8 E4M3 bytes -> float64 (sign, 4 exponent bits with bias 7, 3 mantissa bits)."""
    b = np.asarray(b, np.int64)
    s, e, m = b >> 7, (b >> 3) & 15, b & 7
    v = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    return np.where(s == 1, -v, v)


def e4m3_byte(v):
    """Exact E4M3 encoding of values with at most 4 significant bits in range."""
    v = np.asarray(v, np.float64)
    out = np.zeros(v.shape, np.uint8)
    nz = v != 0
    a = np.abs(v[nz])
    e = np.floor(np.log2(a)).astype(np.int64)
    man = a / np.exp2(e) - 1.0
    assert np.all(man * 8 == np.round(man * 8)) and np.all((e + 7 >= 1) & (e + 7 <= 15))
    out[nz] = ((np.signbit(v[nz]).astype(np.int64) << 7) | ((e + 7) << 3) | np.round(man * 8).astype(np.int64))
    return out


# every value a remapped HiF4 element can take: +-(m/4) 2^E, m = 0..7, E = 0..2
REMAP = np.unique(np.array([s * m / 4.0 * 2 ** E for s in (1, -1) for m in range(8) for E in range(3)]))


def test_remap_covers_fifteen_magnitudes():
    assert len(REMAP) == 31 and np.array_equal(e4m3_value(e4m3_byte(REMAP)), REMAP)


def test_remap_is_exact(H):
    import torch
    rng = np.random.default_rng(31)
    x = (rng.standard_t(3, (300, 640)) * rng.lognormal(0, 2, (300, 1))).astype(np.float32)
    x[5, :64] = 0.0                                                   # a zero unit
    x[7, 64:128] = 1e30                                               # the largest scales
    codes, meta, _ = oracle.quantize(x)
    q8, sc = H.to_e4m3(torch.from_numpy(codes).cuda(), torch.from_numpy(meta.view(np.int32)).cuda(), 640,
                       pad_rows=128)
    torch.cuda.synchronize()
    q8, sc = q8.cpu().numpy(), sc.cpu().numpy()
    assert sc.shape == (10, 384)
    scales = np.array([[oracle.e6m2_value(int(c)) for c in row] for row in (meta & 0xFF)])
    assert np.array_equal(sc[:, :300].astype(np.float64), scales.T)
    val = e4m3_value(q8) * np.repeat(sc[:, :300].T.astype(np.float64), 64, axis=1)
    assert np.array_equal(val, oracle.dequantize(codes, meta, 640))


def _patterns(rng, rows, K):
    """Adversarial rows of remapped values."""
    v = rng.choice(REMAP, size=(rows, K))
    v[0] = 7.0
    v[1] = 0.25
    v[1, ::64] = 7.0                                                  # largest product, then the smallest
    v[2] = np.where(np.arange(K) % 2, -7.0, 7.0)                      # cancellation
    v[3] = 0.25
    v[3, 63::64] = 7.0                                                # the large one last
    v[4] = np.tile(REMAP, K // len(REMAP) + 1)[:K]                    # every value
    v[5] = -v[0]
    v[6] = np.where(np.arange(K) % 64 == 0, 7.0, np.where(np.arange(K) % 2, 0.25, -0.25))
    return v


@pytest.mark.parametrize("M,N,K", [(130, 300, 128), (256, 512, 512), (200, 260, 576)])
def test_fp8_mma_is_exact_on_remapped_operands(H, M, N, K):
    import torch
    rng = np.random.default_rng(M + N + K)
    a, b = _patterns(rng, M, K), _patterns(rng, N, K)
    exact = (np.round(a * 4).astype(np.int64) @ np.round(b * 4).astype(np.int64).T)  # 16 x the result
    assert np.abs(exact).max() < 2 ** 24
    mp, np_ = -(-M // 128) * 128, -(-N // 256) * 256
    sa = torch.ones(K // 64, mp, dtype=torch.float32, device="cuda")
    sb = torch.ones(K // 64, np_, dtype=torch.float32, device="cuda")
    y = H.gemm_f8(torch.from_numpy(e4m3_byte(a)).cuda(), sa, torch.from_numpy(e4m3_byte(b)).cuda(), sb,
                  out_f32=True)
    torch.cuda.synchronize()
    got = y.cpu().numpy()
    want = (exact / 16.0).astype(np.float32)
    bad = np.argwhere(got != want)
    assert bad.size == 0, "FP8 products inexact at %s: got %r want %r" % (
        bad[:4].tolist(), got[tuple(bad[0])], want[tuple(bad[0])])


@pytest.mark.parametrize("M,N,K", [(300, 320, 576), (129, 264, 1024)])
def test_fp8_gemm_matches_oracle_linear(H, M, N, K):
    import torch
    d = wl.attn_proj(M=M, K=K, N=N, seed=2)
    cx, mx, _ = oracle.quantize(d["x"])
    cw, mw, _ = oracle.quantize(d["w"])
    dev = lambda t: torch.from_numpy(np.ascontiguousarray(t)).cuda()
    qa, sa = H.to_e4m3(dev(cx), dev(mx.view(np.int32)), K, pad_rows=128)
    qb, sb = H.to_e4m3(dev(cw), dev(mw.view(np.int32)), K, pad_rows=256)
    y32 = H.gemm_f8(qa, sa, qb, sb, out_f32=True)
    y16 = H.gemm_f8(qa, sa, qb, sb)
    torch.cuda.synchronize()
    ref = oracle.linear(oracle.dequantize(cx, mx, K), oracle.dequantize(cw, mw, K))
    assert_linear_close(y32.cpu().numpy(), ref)
    assert torch.equal(y16, y32.to(torch.bfloat16))
