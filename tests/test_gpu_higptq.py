"""GPU checks of HiGPTQ scheme one (hif4_higptq1) and of the Hessian
(hif4_hessian) against the CPU oracle [HiF4 article, section 3.1].

The oracle runs in FP64, the GPU group loop in FP32, so the error feedback
differs in the last bits and a quantization decision that sits next to a
rounding boundary can go the other way; the differences then feed forward.
So the GPU result is checked as a sequence of correct HiGPTQ steps, from
the values each 64-column group was quantized from (which the call leaves
in its workspace, hif4_higptq1_group_inputs_offset):
  * step validity, every group of every checked row: its codes and metadata
    equal the oracle's plain quantization of those FP32 values, bit for bit,
    and a protected column holds their BF16 rounding;
  * feedback: those values equal, within FP32 rounding, the FP64 GPTQ update
    W0_h - sum_{g<h} E_g U_{g,h}, with E_g = (W_g - Q_g) U_gg^-1 computed in
    FP64 from the GPU's own W_g and Q_g and U the oracle's FP64 factor.  The
    bound is 2^-12 x (|W0| + (|D| |U_gg^-1|) |U_{g,h}|) summed in absolute
    values: about twice the worst case of the GPU's arithmetic (FP32 rounding
    of U, <= 1536-term FP32 accumulations of split-TF32 products per update
    launch, <= 64-term ones for E, one rounding of W per update: about
    2^-13.3 of that sum).  A dropped term, a wrong sign or a wrong index
    moves some element by a sizeable fraction of the sum itself.
And against the oracle's own FP64 run, end to end:
  * the first 64-column group of every row has received no feedback: its
    codes and metadata are bit-exact;
  * with no cross-group coupling (identity Hessian) everything is bit-exact;
  * overall, >= 98 % of the units and >= 99 % of the element codes agree,
    and the layer-output error tr((W - Q) H (W - Q)^T) is within 2 % of the
    oracle's.
Both sides get the same FP32 Hessian, computed on the host.
"""
import numpy as np
import pytest

import oracle
from block_floating_point_hif4_b200 import workloads as wl
from tests._gptq_check import check_group_steps
from tests._util import THREADS, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import block_floating_point_hif4_b200 as h
    from block_floating_point_hif4_b200 import build
    build.build()
    return h


def _bf16(rng, shape, scale):
    return wl.f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def _factor_x(rng, T, K, rank=16, noise=0.3):
    x = rng.standard_normal((T, rank)) @ rng.standard_normal((rank, K)) + noise * rng.standard_normal((T, K))
    return x * rng.lognormal(0, 0.5, K)


def _nibbles(codes):
    return np.stack([codes & 15, codes >> 4], -1).reshape(codes.shape[0], -1)


def _objective(w_bits, wq, Hd):
    d = wl.bf16_bits_to_f32(w_bits).astype(np.float64) - wq
    return float(np.einsum("nk,kl,nl->", d, Hd, d))


def run_gpu(Hm, w_bits, Hf32, idx, damp, bs, w_dev=None):
    """-> (codes, meta, w_masked bits or None, group inputs FP32 N x K)."""
    import torch
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    i_dev = torch.from_numpy(np.asarray(idx, np.int32)).cuda() if len(idx) else None
    w_dev = to_dev_bf16(w_bits) if w_dev is None else w_dev
    N, K = w_dev.shape
    ws = torch.empty(Hm.lib().hif4_higptq1_workspace(N, K, bs), dtype=torch.uint8, device="cuda")
    codes, meta, wm = Hm.higptq1(w_dev, torch.from_numpy(Hf32).cuda(), i_dev, damp, bs, workspace=ws,
                                 status=status)
    torch.cuda.synchronize()
    assert Hm.get_status(status) == 0
    gin = Hm.higptq1_group_inputs(ws, N, K, bs).cpu().numpy()
    return (codes.cpu().numpy(), meta.cpu().numpy().view(np.uint32),
            None if wm is None else wm.view(torch.int16).cpu().numpy().view(np.uint16), gin)


def compare(w_bits, Hf32, idx, damp, bs, got, factor=None, rows=None):
    K = w_bits.shape[1]
    mask = np.zeros(K, np.uint8)
    mask[idx] = 1
    rows = np.arange(w_bits.shape[0]) if rows is None else rows
    wr = np.ascontiguousarray(w_bits[rows])
    c_o, m_o, wq_o, wm_o = oracle.higptq1(wr, Hf32.astype(np.float64), mask if len(idx) else None, damp, bs,
                                          threads=THREADS, factor=factor)
    check_group_steps(w_bits, idx, got, factor if factor is not None else oracle.gptq_factor(
        Hf32.astype(np.float64), damp), rows)
    c_g, m_g, wm_g = got[0][rows], got[1][rows], None if got[2] is None else got[2][rows]
    # the first group of every row: no feedback yet, bit-exact
    assert np.array_equal(c_g[:, :32], c_o[:, :32]) and np.array_equal(m_g[:, 0], m_o[:, 0])
    unit_agree = np.mean(m_g == m_o)
    code_agree = np.mean(_nibbles(c_g) == _nibbles(c_o))
    assert unit_agree >= 0.98 and code_agree >= 0.99, (unit_agree, code_agree)
    # layer-output error of the GPU result against the oracle's
    Hd = Hf32.astype(np.float64)
    Hd = Hd + damp * np.mean(np.diag(Hd)) * np.eye(K)
    wq_g = oracle.dequantize(c_g, m_g, K)
    if len(idx):
        wq_g[:, idx] = wl.bf16_bits_to_f32(wm_g).astype(np.float64)
    e_g, e_o = _objective(wr, wq_g, Hd), _objective(wr, wq_o, Hd)
    assert abs(e_g - e_o) <= 0.02 * e_o, (e_g, e_o)
    return unit_agree, code_agree, e_g / e_o


def test_hessian_matches_numpy(H):
    import torch
    rng = np.random.default_rng(1)
    T, K = 3001, 256
    x = wl.f32_to_bf16_bits(_factor_x(rng, T, K).astype(np.float32))
    h = H.hessian(to_dev_bf16(x))
    torch.cuda.synchronize()
    x64 = wl.bf16_bits_to_f32(x).astype(np.float64)
    ref = x64.T @ x64
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= 2e-5 * np.max(np.abs(ref))


def test_identity_hessian_is_plain_quantization(H):
    rng = np.random.default_rng(2)
    N, K = 100, 512
    w = _bf16(rng, (N, K), 0.02)
    idx = np.array([1, 64, 200, 511], np.int32)
    mask = np.zeros(K, np.uint8)
    mask[idx] = 1
    codes, meta, wm, _ = run_gpu(H, w, np.eye(K, dtype=np.float32), idx, 0.01, 128)
    rc, rm, _ = oracle.quantize(w, mask)
    assert np.array_equal(codes, rc) and np.array_equal(meta, rm)
    assert np.array_equal(wm, w[:, idx])


@pytest.mark.parametrize("bs", [64, 128, 192, 256])
def test_small_layer_vs_oracle(H, bs):
    rng = np.random.default_rng(bs)
    N, K = 96, 512
    w = _bf16(rng, (N, K), 0.02)
    x = _factor_x(rng, 2000, K)
    Hf = (x.T @ x).astype(np.float32)
    idx = np.array([3, 130, 131, 400, 511], np.int32)
    got = run_gpu(H, w, Hf, idx, 0.01, bs)
    compare(w, Hf, idx, 0.01, bs, got)


@pytest.mark.parametrize("K", [64, 128, 192, 256, 320, 448])
def test_factor_recursion_shapes(H, K):
    """The factor's recursion at its edges: a 64-row leaf alone (K = 64), a
    128-row leaf alone (128), the two leaf sizes side by side (192 = 64 +
    128), one split of 128-row leaves (256), and the splits of odd 64-row
    tile counts (320 = 128 + (64 + 128); 448 = (64 + 128) + (128 + 128))."""
    rng = np.random.default_rng(K + 7)
    N = 70
    w = _bf16(rng, (N, K), 0.02)
    x = _factor_x(rng, 1500, K, rank=8)
    Hf = (x.T @ x).astype(np.float32)
    got = run_gpu(H, w, Hf, [], 0.01, 64)
    compare(w, Hf, [], 0.01, 64, got)


def test_dead_channel_and_non_positive_definite(H):
    import torch
    rng = np.random.default_rng(4)
    N, K = 40, 256
    w = _bf16(rng, (N, K), 0.02)
    x = _factor_x(rng, 800, K)
    x[:, 17] = 0.0                                           # a channel that never fires
    Hf = (x.T @ x).astype(np.float32)
    got = run_gpu(H, w, Hf, [], 0.01, 128)
    compare(w, Hf, [], 0.01, 128, got)
    assert np.all(_nibbles(got[0])[:, 17] == 0)                 # its weights were zeroed
    # an indefinite matrix with no damping is refused through the status word
    bad = np.eye(K, dtype=np.float32)
    bad[5, 5] = -1.0
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    H.higptq1(to_dev_bf16(w), torch.from_numpy(bad).cuda(), None, 0.0, 128, status=status)
    assert H.get_status(status) == 1                            # HIF4_ERR_INVALID_ARG (NOT_SPD)


def test_many_tiles_ragged_rows(H):
    """N = 3000 rows (not a multiple of the update's 128-row tiles) and K =
    1024: each lazy update has 24 x up to 7 tiles, more than there are SMs,
    so every persistent update CTA walks several tiles and both TMEM
    accumulators; 128 sampled rows against the oracle."""
    rng = np.random.default_rng(11)
    N, K = 3000, 1024
    w = _bf16(rng, (N, K), 0.02)
    x = _factor_x(rng, 3000, K)
    Hf = (x.T @ x).astype(np.float32)
    idx = np.array([5, 300, 301, 1023], np.int32)
    got = run_gpu(H, w, Hf, idx, 0.01, 128)
    factor = oracle.gptq_factor(Hf.astype(np.float64), 0.01)
    rows = np.unique(np.concatenate([wl.sample_rows(N, 120), [0, 2943, 2944, N - 1]]))
    compare(w, Hf, idx, 0.01, 128, got, factor=factor, rows=rows)


@pytest.mark.slow
def test_wan22_w1_sampled_rows(H):
    """W1 of the Wan2.2 FFN (13824 x 5120, the bench's seeded weight) with the
    Hessian of the bench's 57600 activation tokens (the attention-projection
    input recipe, seed 3) and its 51 seeded outlier channels protected; 128
    sampled rows against the oracle, every group of them step-checked (rows
    are independent given the Hessian factor)."""
    import torch
    xd, outl = wl.device_rows(57600, 5120, seed=3, device="cuda")
    x64 = wl.bf16_bits_to_f32(xd.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    del xd
    Hf = (x64.T @ x64).astype(np.float32)
    del x64
    w1d = wl.device_weight(13824, 5120, 0.015, seed=31, device="cuda")
    w1 = w1d.view(torch.int16).cpu().numpy().view(np.uint16)
    idx = outl.cpu().numpy().astype(np.int32)
    got = run_gpu(H, w1, Hf, idx, 0.01, 128, w_dev=w1d)
    factor = oracle.gptq_factor(Hf.astype(np.float64), 0.01)
    rows = wl.sample_rows(w1.shape[0], 128)
    compare(w1, Hf, idx, 0.01, 128, got, factor=factor, rows=rows)
