"""GPU parity: hif4_quantize / hif4_dequantize / hif4_fake_quantize against the
CPU oracle, bit for bit (codes, metadata, dequantized BF16/F32 values).

Format: Huawei HiF4 calibration article (hwcomputing.csdn.net), section 1;
encode rule and decode sign convention as the library reads them.
"""
import numpy as np
import pytest

import oracle
from block_floating_point_hif4_b200 import workloads as wl
from tests._util import THREADS, meta_u32, to_dev_bf16, to_host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import torch  # noqa: F401
    import block_floating_point_hif4_b200 as h
    from block_floating_point_hif4_b200 import build
    build.build()
    return h


def _torch():
    import torch
    return torch


def gpu_quant(H, x_host, dtype, chan_mask=None, ld=None):
    torch = _torch()
    rows, cols = x_host.shape
    if dtype == "bf16":
        xd = to_dev_bf16(x_host)
    else:
        xd = torch.from_numpy(np.ascontiguousarray(x_host, np.float32)).cuda()
    if ld is not None and ld != cols:
        big = torch.zeros(rows, ld, dtype=xd.dtype, device="cuda")
        big[:, :cols] = xd
        xd = big[:, :cols]
    cm = None if chan_mask is None else torch.from_numpy(chan_mask.astype(np.uint8)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, meta = H.quantize(xd, cm, status=status)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), meta_u32(meta), int(status.item())


def check_roundtrip(H, x_host, dtype, chan_mask=None, ld=None):
    """GPU codes/meta == oracle; GPU dequantize == oracle dequantize (exact)."""
    torch = _torch()
    codes, meta, _ = gpu_quant(H, x_host, dtype, chan_mask, ld)
    ref_c, ref_m, _ = oracle.quantize(x_host if dtype == "bf16" else x_host.astype(np.float32), chan_mask)
    assert np.array_equal(meta, ref_m), "meta mismatch at %s" % (np.argwhere(meta != ref_m)[:5],)
    assert np.array_equal(codes, ref_c), "codes mismatch at %s" % (np.argwhere(codes != ref_c)[:5],)
    cols = x_host.shape[1]
    ref_y = oracle.dequantize(ref_c, ref_m, cols)
    cd = torch.from_numpy(ref_c).cuda()
    md = torch.from_numpy(ref_m.view(np.int32)).cuda()
    y32 = H.dequantize(cd, md, cols, torch.float32).cpu().numpy().astype(np.float64)
    assert np.array_equal(y32, ref_y)
    assert np.array_equal(np.signbit(y32), np.signbit(ref_y))
    yb = to_host_bits(H.dequantize(cd, md, cols, torch.bfloat16))
    assert np.array_equal(yb, wl.f32_to_bf16_bits(ref_y.astype(np.float32)))
    return codes, meta


# ------------------------------------------------------------------ tiny

def test_tiny_workload_fp32_and_bf16(H):
    X, W = wl.tiny(0)
    for arr in (X, W):
        check_roundtrip(H, arr, "f32")
        check_roundtrip(H, wl.f32_to_bf16_bits(arr), "bf16")


@pytest.mark.parametrize("rows,cols", [(1, 64), (3, 64), (5, 192), (7, 320), (33, 1024), (129, 640)])
def test_ragged_shapes(H, rows, cols):
    rng = np.random.default_rng(rows * 1000 + cols)
    x = (rng.standard_t(3, (rows, cols)) * rng.lognormal(0, 2, (rows, 1))).astype(np.float32)
    check_roundtrip(H, x, "f32")
    check_roundtrip(H, wl.f32_to_bf16_bits(x), "bf16")


def test_unaligned_view_uses_16_byte_path(H):
    """A row view starting 16 bytes past a 32-byte boundary (still 16-byte
    aligned) must give the same result through the 16-byte kernel."""
    torch = _torch()
    rng = np.random.default_rng(15)
    x = wl.f32_to_bf16_bits(rng.standard_normal((9, 192)).astype(np.float32))
    big = torch.zeros(9, 192 + 8, dtype=torch.bfloat16, device="cuda")
    big[:, 8:] = to_dev_bf16(x)
    view = big[:, 8:]
    assert view.data_ptr() % 32 == 16
    c, m = H.quantize(view)
    ref_c, ref_m, _ = oracle.quantize(x)
    assert np.array_equal(c.cpu().numpy(), ref_c) and np.array_equal(meta_u32(m), ref_m)
    y = H.fake_quantize(view)
    ref = oracle.fake_quantize(x)
    assert np.array_equal(to_host_bits(y), wl.f32_to_bf16_bits(ref.astype(np.float32)))


def test_strided_rows_and_mask(H):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((37, 256)).astype(np.float32)
    x[:, 17] *= 300
    mask = np.zeros(256, np.uint8)
    mask[[17, 64, 255]] = 1
    check_roundtrip(H, x, "f32", ld=264)
    check_roundtrip(H, wl.f32_to_bf16_bits(x), "bf16", ld=320)
    check_roundtrip(H, x, "f32", chan_mask=mask)
    check_roundtrip(H, wl.f32_to_bf16_bits(x), "bf16", chan_mask=mask, ld=264)


def adversarial_units():
    """Units whose values sit on every decision boundary of the encoder."""
    rng = np.random.default_rng(77)
    rows = []
    for c in [0, 1, 2, 3, 31, 100, 123, 124, 125, 126, 127, 128, 200, 252, 253, 254, 255]:
        S = oracle.e6m2_value(c)
        for amax_mult in [6.5, 6.5 * 1.25, 6.5 * 1.2, 6.5 * 8 / 7, 7.0, 8.125]:
            row = np.zeros(64)
            row[0] = amax_mult * S
            row[1] = np.nextafter(amax_mult * S, 0)
            E_choices = [0.25, 0.5, 1.0]
            for i in range(2, 64):
                step = S * E_choices[rng.integers(3)]
                k = rng.integers(0, 8)
                kind = rng.integers(4)
                v = (k + 0.5) * step if kind == 0 else k * step if kind == 1 else \
                    np.nextafter((k + 0.5) * step, 0) if kind == 2 else rng.uniform(0, 8 * step)
                row[i] = v * (1 if rng.random() < 0.5 else -1)
            rows.append(row)
        rows.append(np.array([1.75 * S, 3.5 * S] * 32))
    return np.array(rows)


def test_adversarial_boundaries(H):
    x = adversarial_units().astype(np.float32)
    check_roundtrip(H, x, "f32")
    check_roundtrip(H, wl.f32_to_bf16_bits(x), "bf16")


def test_special_values_and_status(H):
    x = np.zeros((4, 64), np.float32)
    x[0] = 0.0
    x[1, :] = -0.0
    x[2, 3] = np.nan
    x[2, 4] = 1.0
    x[3, 0] = np.inf
    x[3, 1] = -2.0
    x[3, 2] = 3e38
    codes, meta, st = gpu_quant(H, x, "f32")
    ref_c, ref_m, nf = oracle.quantize(x)
    assert nf == 2
    assert np.array_equal(codes, ref_c) and np.array_equal(meta, ref_m)
    assert st & 1
    bits = wl.f32_to_bf16_bits(np.where(np.isnan(x), 0, x).astype(np.float32))
    bits[2, 3] = 0x7FC0
    bits[3, 0] = 0x7F80
    codes, meta, st = gpu_quant(H, bits, "bf16")
    ref_c, ref_m, nf = oracle.quantize(bits)
    assert np.array_equal(codes, ref_c) and np.array_equal(meta, ref_m)
    assert st & 1 and nf == 2
    clean = np.ones((2, 64), np.float32)
    assert gpu_quant(H, clean, "f32")[2] == 0


def test_fp32_near_ties_exact_path(H):
    """FP32 values one ulp around every rounding half-way point."""
    rng = np.random.default_rng(8)
    rows = []
    for c in [60, 124, 125, 126, 127, 190]:
        S = oracle.e6m2_value(c)
        row = np.zeros(64)
        row[0] = 7.0 * S                           # fixes the scale at S, group E = 2
        for i in range(1, 64):
            E = 2 if i < 8 else (0 if i >= 32 else 1)
            step = S * 2.0 ** E / 4
            k = rng.integers(0, 7)
            mid = np.float32((k + 0.5) * step)
            row[i] = [np.nextafter(mid, np.float32(0)), mid, np.nextafter(mid, np.float32(np.inf))][i % 3]
        rows.append(row)
    x = np.array(rows, np.float32)
    check_roundtrip(H, x, "f32")


def test_fake_quantize_matches_oracle(H):
    torch = _torch()
    d = wl.attn_proj(M=300, K=640, N=64, seed=2)
    x, idx = d["x"], d["mask_idx"][:5]
    idx = np.array(sorted(set(list(idx) + [0, 639])), np.int32)
    mask = np.zeros(640, np.uint8)
    mask[idx] = 1
    ref = oracle.fake_quantize(x, idx)
    got = to_host_bits(H.fake_quantize(to_dev_bf16(x), torch.from_numpy(mask).cuda()))
    assert np.array_equal(got, wl.f32_to_bf16_bits(ref.astype(np.float32)))
    assert np.array_equal(got[:, idx], x[:, idx])          # protected channels pass through
    ref0 = oracle.fake_quantize(x)
    got0 = to_host_bits(H.fake_quantize(to_dev_bf16(x)))
    assert np.array_equal(got0, wl.f32_to_bf16_bits(ref0.astype(np.float32)))


@pytest.mark.parametrize("rows,cols", [
    (4001, 640),        # chunk stride a whole number of rows: lane masks built once; ragged last chunk
    (20000, 5120),      # the same with ~57 chunks per block (Wan2.2 channel count)
    (50, 64 * 997),     # no such grid (997 units per row): masks per chunk
])
def test_masked_fake_quantize_chunk_strides(H, rows, cols):
    """Masked fake quantization over many chunks per block, in both launch
    forms of the streaming kernel; rows are independent, so a spread sample
    of rows is checked against the oracle."""
    torch = _torch()
    rng = np.random.default_rng(rows + cols)
    x = rng.standard_normal((rows, cols), dtype=np.float32)
    x *= rng.lognormal(0, 0.5, cols).astype(np.float32)
    x = wl.f32_to_bf16_bits(x)
    idx = np.sort(rng.choice(cols, max(1, cols // 100), replace=False)).astype(np.int32)
    mask = np.zeros(cols, np.uint8)
    mask[idx] = 7                                           # any nonzero byte protects
    got = to_host_bits(H.fake_quantize(to_dev_bf16(x), torch.from_numpy(mask).cuda()))
    sample = np.unique(np.concatenate([np.arange(min(rows, 64)), rng.choice(rows, min(rows, 192), replace=False),
                                       [rows - 1]]))
    ref = oracle.fake_quantize(np.ascontiguousarray(x[sample]), idx)
    assert np.array_equal(got[sample], wl.f32_to_bf16_bits(ref.astype(np.float32)))
    assert np.array_equal(got[:, idx], x[:, idx])           # every protected channel passes through


def test_gpu_idempotence(H):
    torch = _torch()
    x = to_dev_bf16(wl.quant_sweep(1 << 20).reshape(-1, 1024))
    c1, m1 = H.quantize(x)
    y = H.dequantize(c1, m1, 1024)
    c2, m2 = H.quantize(y)
    assert torch.equal(c1, c2) and torch.equal(m1, m2)


# ------------------------------------------------------- bandwidth sweep

@pytest.mark.parametrize("log2n", [20, 22, 24, 26])
def test_sweep_full_compare(H, log2n):
    """Quantizer sweep workload (rows of 5120, last row partial), viewed as
    rows x 1024 exactly as the benchmark calls it; every element compared."""
    n = 1 << log2n
    x = wl.quant_sweep(n).reshape(-1, 1024)
    torch = _torch()
    xd = to_dev_bf16(x)
    codes, meta = H.quantize(xd)
    codes = codes.cpu().numpy()
    meta = meta_u32(meta)
    # oracle on row blocks in threads
    rows = x.shape[0]
    bounds = np.linspace(0, rows, THREADS + 1).astype(int)
    import threading
    out = [None] * THREADS

    def run(i):
        out[i] = oracle.quantize(x[bounds[i]:bounds[i + 1]])
    ts = [threading.Thread(target=run, args=(i,)) for i in range(THREADS)]
    [t.start() for t in ts]
    [t.join() for t in ts]
    ref_c = np.concatenate([o[0] for o in out])
    ref_m = np.concatenate([o[1] for o in out])
    assert np.array_equal(meta, ref_m)
    assert np.array_equal(codes, ref_c)
    y = to_host_bits(H.dequantize(torch.from_numpy(codes).cuda(), torch.from_numpy(meta.view(np.int32)).cuda(),
                                  1024))
    sample = wl.sample_rows(rows, 512)
    ref_y = oracle.dequantize(ref_c[sample], ref_m[sample], 1024)
    assert np.array_equal(y[sample], wl.f32_to_bf16_bits(ref_y.astype(np.float32)))


@pytest.mark.slow
@pytest.mark.parametrize("log2n", [28, 30])
def test_sweep_full_size_sampled(H, log2n):
    """2^28 and 2^30 elements, generated on the device (seeded torch RNG) in
    the benchmark's launch configuration; 1024 sampled rows of 1024 compared."""
    torch = _torch()
    n = 1 << log2n
    xd = wl.quant_sweep_torch(n, "cuda").view(-1, 1024)
    codes, meta = H.quantize(xd)
    y = H.dequantize(codes, meta, 1024)
    rows = xd.shape[0]
    sample = torch.from_numpy(wl.sample_rows(rows, 1024)).cuda()
    xs = to_host_bits(xd[sample])
    cs = codes[sample].cpu().numpy()
    ms = meta_u32(meta[sample])
    ref_c, ref_m, _ = oracle.quantize(xs)
    assert np.array_equal(ms, ref_m)
    assert np.array_equal(cs, ref_c)
    ref_y = oracle.dequantize(ref_c, ref_m, 1024)
    assert np.array_equal(to_host_bits(y[sample]), wl.f32_to_bf16_bits(ref_y.astype(np.float32)))
    del xd, codes, meta, y
    torch.cuda.empty_cache()
