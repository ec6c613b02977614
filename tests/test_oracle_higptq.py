"""CPU pins of the HiGPTQ (scheme one) oracle [HiF4 article, section 3.1].

Each pin compares the oracle with something other than itself:
  * its Hessian factor with numpy (Cholesky factor of the inverse of the
    damped Hessian, transposed);
  * an identity or 64-aligned block-diagonal Hessian leaves nothing to
    compensate, so the result is plain unit quantization (orc_quantize);
  * the error feedback of the first group equals the least-squares
    compensation w1 + D0 Hd01 Hd11^{-1} computed with numpy's solver, so the
    second group's codes are those of that compensated row;
  * the blocked (lazy) update is an exact reordering: block sizes 64, 128
    and 256 give the same codes;
  * on inputs whose channels are correlated across groups (a few shared
    factors) the layer-output error tr((W - Q) H (W - Q)^T) is well below
    that of plain rounding to the nearest HiF4 values.
The per-group step check that the GPU tests apply passes on the oracle's
own run and fails on one with a group's error left out of the feedback.
"""
import numpy as np
import pytest

import oracle
from block_floating_point_hif4_b200 import workloads as wl
from tests._gptq_check import check_group_steps


def _weights(rng, N, K, scale=0.02):
    return wl.f32_to_bf16_bits((rng.standard_normal((N, K)) * scale).astype(np.float32))


def _hessian(rng, T, K, rank=16, noise=0.3):
    """X from a few shared factors plus noise: channels correlated across
    groups (what the error feedback of scheme one can use), with lognormal
    per-channel scales."""
    x = rng.standard_normal((T, rank)) @ rng.standard_normal((rank, K)) + noise * rng.standard_normal((T, K))
    x *= rng.lognormal(0, 0.5, K)
    return x.T @ x


@pytest.mark.parametrize("K", [64, 192])
def test_factor_matches_numpy(K):
    rng = np.random.default_rng(K)
    H = _hessian(rng, 400, K)
    H[5, :] = 0
    H[:, 5] = 0                                    # a dead channel
    U, dead = oracle.gptq_factor(H, 0.01)
    assert dead[5] == 1 and dead.sum() == 1
    Hd = H.copy()
    Hd[5, 5] = 1.0
    Hd += 0.01 * np.mean(np.diag(Hd)) * np.eye(K)
    ref = np.linalg.cholesky(np.linalg.inv(Hd)).T
    assert np.allclose(U, ref, rtol=1e-9, atol=1e-12 * np.abs(ref).max())
    assert np.array_equal(np.tril(U, -1), np.zeros_like(U))


def test_large_k_factor_path_matches_the_c_routine():
    """Above K = 1024 the factor uses numpy's Cholesky and inverse; at the
    boundary both paths must agree."""
    rng = np.random.default_rng(12)
    H = _hessian(rng, 3000, 1088)
    U_np, d_np = oracle.gptq_factor(H, 0.01)                       # K = 1088: numpy path
    import ctypes
    K = H.shape[0]
    U_c = np.zeros((K, K))
    dead = np.zeros(K, np.uint8)
    rc = oracle.lib().orc_gptq_factor(H.ctypes.data_as(ctypes.c_void_p), K, 0.01,
                                      U_c.ctypes.data_as(ctypes.c_void_p), dead.ctypes.data_as(ctypes.c_void_p))
    assert rc == 0 and np.array_equal(dead, d_np)
    assert np.allclose(U_np, U_c, rtol=1e-8, atol=1e-10 * np.abs(U_c).max())


@pytest.mark.parametrize("kind", ["identity", "block_diagonal"])
def test_no_cross_group_coupling_reduces_to_plain_quantization(kind):
    rng = np.random.default_rng(3)
    N, K = 9, 256
    w = _weights(rng, N, K)
    if kind == "identity":
        H = np.eye(K)
    else:
        H = np.zeros((K, K))
        for g in range(0, K, 64):
            H[g:g + 64, g:g + 64] = _hessian(rng, 300, 64)
    mask = np.zeros(K, np.uint8)
    mask[[3, 100, 250]] = 1
    codes, meta, wq, wm = oracle.higptq1(w, H, mask, damp=0.01, blocksize=128)
    if kind == "identity":
        rc, rm, _ = oracle.quantize(w, mask)
        assert np.array_equal(codes, rc) and np.array_equal(meta, rm)
        assert np.array_equal(wm, w[:, mask.astype(bool)])
    else:
        # U is then block-diagonal as well: U_{g, later} = 0, so no group's
        # error reaches another group, and each group is quantized as it came
        rc, rm, _ = oracle.quantize(w, mask)
        assert np.array_equal(meta, rm) and np.array_equal(codes, rc)


def test_first_group_feedback_is_the_least_squares_compensation():
    rng = np.random.default_rng(5)
    N, K, damp = 7, 128, 0.01
    w = _weights(rng, N, K)
    H = _hessian(rng, 500, K)
    Hd = H + damp * np.mean(np.diag(H)) * np.eye(K)
    for bs in (64, 128):
        codes, meta, wq, _ = oracle.higptq1(w, H, None, damp=damp, blocksize=bs)
        w64 = wl.bf16_bits_to_f32(w).astype(np.float64)
        for n in range(N):
            c0, m0 = oracle.quantize_unit(w64[n, :64])
            q0 = np.array([oracle.decode_element(int(c0[i]), int(m0), i) for i in range(64)])
            d0 = w64[n, :64] - q0
            v = w64[n, 64:] + d0 @ Hd[:64, 64:] @ np.linalg.inv(Hd[64:, 64:])
            c1, m1 = oracle.quantize_unit(v)
            assert int(meta[n, 0]) == int(m0) and int(meta[n, 1]) == int(m1), (bs, n)
            got = np.stack([codes[n, 32:] & 15, codes[n, 32:] >> 4], 1).ravel()
            assert np.array_equal(got, np.asarray(c1)), (bs, n)


def test_blocksize_does_not_change_the_result():
    rng = np.random.default_rng(6)
    N, K = 6, 512
    w = _weights(rng, N, K)
    H = _hessian(rng, 800, K)
    mask = np.zeros(K, np.uint8)
    mask[[0, 77, 300]] = 1
    f = oracle.gptq_factor(H, 0.01)
    base = oracle.higptq1(w, H, mask, blocksize=64, factor=f)
    for bs in (128, 256, 512):
        other = oracle.higptq1(w, H, mask, blocksize=bs, factor=f)
        assert np.array_equal(base[0], other[0]) and np.array_equal(base[1], other[1]), bs
        assert np.allclose(base[2], other[2], rtol=0, atol=1e-12)


def test_output_error_is_well_below_plain_rounding():
    rng = np.random.default_rng(8)
    N, K = 32, 256
    w = _weights(rng, N, K)
    H = _hessian(rng, 2000, K)
    _, _, wq, _ = oracle.higptq1(w, H, None, damp=0.01, blocksize=128)
    rc, rm, _ = oracle.quantize(w)
    w_rtn = oracle.dequantize(rc, rm, K)
    w64 = wl.bf16_bits_to_f32(w).astype(np.float64)

    def err(q):
        d = w64 - q
        return float(np.einsum("nk,kl,nl->", d, H, d))
    assert err(wq) < 0.5 * err(w_rtn)


def test_group_step_check_catches_a_wrong_feedback():
    """The per-group check fails on a result whose feedback skipped one
    group's error (made on the CPU by running the oracle's steps on a
    perturbed copy), and passes on the oracle's own FP64 run."""
    rng = np.random.default_rng(21)
    N, K = 16, 256
    w = _weights(rng, N, K)
    Hd = _hessian(rng, 1000, K)
    factor = oracle.gptq_factor(Hd, 0.01)
    U = factor[0]
    c, m, wq, _ = oracle.higptq1(w, Hd, None, 0.01, 64, factor=factor)
    # the oracle's group inputs, rebuilt from its own output: W_h = W0_h - sum_{g<h} E_g U_{g,h}
    w0 = wl.bf16_bits_to_f32(w).astype(np.float64)
    gin = w0.copy()
    for h in range(1, K // 64):
        s = slice(64 * h, 64 * h + 64)
        acc = np.zeros((N, 64))
        for g in range(h):
            t = slice(64 * g, 64 * g + 64)
            e = (gin[:, t] - wq[:, t]) @ np.linalg.inv(U[t, t])
            acc += e @ U[t, s]
        gin[:, s] = w0[:, s] - acc
    ok = (c, m, None, gin.astype(np.float32))
    c2, m2, _ = oracle.quantize(gin.astype(np.float32))
    assert np.array_equal(c2, c) and np.array_equal(m2, m)     # the rebuilt inputs reproduce the codes
    check_group_steps(w, [], ok, factor)
    # group 2 never received group 0's error: its inputs (and codes) are those of a wrong feedback
    bad = gin.copy()
    e0 = (gin[:, :64] - wq[:, :64]) @ np.linalg.inv(U[:64, :64])
    bad[:, 128:192] += e0 @ U[:64, 128:192]
    cb, mb, _ = oracle.quantize(bad.astype(np.float32))
    with pytest.raises(AssertionError):
        check_group_steps(w, [], (cb, mb, None, bad.astype(np.float32)), factor)
