"""GPU test of the bounded device-side waits: a wait on a copy that is never
issued runs out, the kernel reports the time-out instead of hanging, and the
device stays usable.

hif4_debug_wait_test(1, limit) makes block 0 of every TMA-fed launch (the
tcgen05 GEMM, the 2-D TMA quantizer, the bulk-copy fake quantizer, the
calibration passes) leave its first copy un-issued and bounds every wait by
`limit`.  Each call must then raise HIF4_FLAG_TIMEOUT in its status word
(the calibration, which has no status word, poisons its outputs: ratios NaN,
mask 0, indices -1); the blocks' drains after giving up are bounded too.
Right after the switch is cleared, the same calls on the same device must
match the oracle again.  Nothing here faults, traps or hangs a GPU: every
wait involved ends by its own limit.
"""
import numpy as np
import pytest

import oracle
from block_floating_point_hif4_b200 import binding as B
from block_floating_point_hif4_b200 import workloads as wl
from tests._util import THREADS, assert_linear_close, to_dev_bf16, to_host_bits

pytestmark = pytest.mark.gpu

LIMIT_NS = 20_000_000          # 20 ms: far above every wait these sizes need, far below the defaults


@pytest.fixture(scope="module")
def H():
    import block_floating_point_hif4_b200 as h
    from block_floating_point_hif4_b200 import build
    build.build()
    return h


def _inputs():
    rng = np.random.default_rng(77)
    x = wl.f32_to_bf16_bits((rng.standard_normal((2048, 1024)) * 0.1).astype(np.float32))
    mask = np.zeros(1024, np.uint8)
    mask[[3, 500, 777]] = 1
    a = wl.f32_to_bf16_bits(rng.standard_normal((640, 512)).astype(np.float32))
    b = wl.f32_to_bf16_bits((rng.standard_normal((768, 512)) * 0.05).astype(np.float32))
    acts, _ = wl.calib(T=4096, C=256, seed=78)
    return x, mask, a, b, acts


def _run_all(H, x, mask, a, b, acts):
    """Quantize, fake-quantize, GEMM and calibration on the current stream;
    -> host results and each call's mapped status."""
    import torch
    xd, md, ad, bd = to_dev_bf16(x), torch.from_numpy(mask).cuda(), to_dev_bf16(a), to_dev_bf16(b)
    st = [torch.zeros(1, dtype=torch.int32, device="cuda") for _ in range(3)]
    codes, meta = H.quantize(xd, status=st[0])
    xh = H.fake_quantize(xd, md, status=st[1])
    y = torch.empty(a.shape[0], b.shape[0], dtype=torch.float32, device="cuda")
    H.gemm_bf16(ad, bd, out=y, status=st[2])
    pct, ratio, cmask, cidx = H.calib_percentile_mask(to_dev_bf16(acts))
    torch.cuda.synchronize()
    status = [H.get_status(s) for s in st]
    return (codes.cpu().numpy(), meta.cpu().numpy().view(np.uint32), to_host_bits(xh), y.cpu().numpy(),
            to_host_bits(pct), ratio.cpu().numpy(), cmask.cpu().numpy(), cidx.cpu().numpy()), status


def test_bounded_waits_run_out_and_the_device_recovers(H):
    L = H.lib()
    x, mask, a, b, acts = _inputs()
    L.hif4_debug_wait_test(1, LIMIT_NS)
    try:
        out, status = _run_all(H, x, mask, a, b, acts)
    finally:
        L.hif4_debug_wait_test(0, 0)
    # quantize (k_quant32), fake quantize (k_quant_tma), GEMM (k_gemm): the time-out is reported
    assert status == [B.ERR_TIMEOUT] * 3, status
    # calibration: the TMA passes gave up, so no computed mask is reported
    _, _, _, _, _, ratio, cmask, cidx = out
    assert np.all(np.isnan(ratio)) and not np.any(cmask) and np.all(cidx == -1)

    # the same device right after: every call matches the oracle again
    out, status = _run_all(H, x, mask, a, b, acts)
    assert status == [B.OK] * 3, status
    codes, meta, xh, y, pct, ratio, cmask, cidx = out
    rc, rm, _ = oracle.quantize(x)
    assert np.array_equal(codes, rc) and np.array_equal(meta, rm)
    ref_xh = oracle.round_bf16(oracle.fake_quantize(x, np.nonzero(mask)[0]))
    assert np.array_equal(xh, ref_xh)
    y_ref = wl.bf16_bits_to_f32(a).astype(np.float64) @ wl.bf16_bits_to_f32(b).astype(np.float64).T
    assert_linear_close(y, y_ref)
    p = oracle.percentile(acts, threads=THREADS)
    r, m, _ = oracle.channel_mask(p)
    assert np.array_equal(pct, p) and np.array_equal(ratio.view(np.uint32), r.view(np.uint32))
    assert np.array_equal(cmask, m) and np.array_equal(cidx, np.nonzero(m)[0].astype(np.int32))
