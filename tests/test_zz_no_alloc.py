"""GPU check of hif4_calib_percentile_mask_noalloc, the calibration entry
point for callers that cannot allocate device memory (a runtime that owns
all device memory through its own pool, a plugin host that forbids
allocation inside its enqueue callback).  Its scratch lives in a fixed
device array inside the library.

The test calls it through the C ABI twice in a row and compares every output
with the allocating entry point's, bit for bit (the calibration outputs are
exact order statistics, so the tolerance is equality).  The second call also
shows that the shared scratch is cleared between calls.  It is collected last
so that a run that stops at the first failure has run every other test
first.
"""
import ctypes

import numpy as np
import pytest

from block_floating_point_hif4_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _outputs(torch, C, n_top):
    return (torch.empty(C, dtype=torch.bfloat16, device="cuda"),
            torch.empty(C, dtype=torch.float32, device="cuda"),
            torch.empty(C, dtype=torch.uint8, device="cuda"),
            torch.full((max(n_top, 1),), -1, dtype=torch.int32, device="cuda"))


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_allocating_entry_point():
    import torch

    from block_floating_point_hif4_b200 import binding, build
    build.build()
    L = binding.lib()
    assert L.hif4_calib_noalloc_scratch_bytes() == 16 << 20
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # the last two cases sit at the Wan2.2 width and at the widest input the array admits
    cases = [(14400, 320, (999, 1000), (1, 100), 5), (3001, 130, (1, 2), (1, 10), 6),
             (4096, 5120, (999, 1000), (1, 100), 7), (4096, 5445, (999, 1000), (1, 100), 8)]
    for T, C, q, frac, seed in cases:
        acts_host, _ = wl.calib(T=T, C=C, seed=seed)
        acts = torch.from_numpy(acts_host.view(np.int16)).view(torch.bfloat16).cuda()
        n_top = C * frac[0] // frac[1]
        ref = _outputs(torch, C, n_top)
        ws = torch.empty(L.hif4_calib_workspace(T, C), dtype=torch.uint8, device="cuda")
        rc = L.hif4_calib_percentile_mask(_p(acts), T, C, C, q[0], q[1], frac[0], frac[1], _p(ref[0]), _p(ref[1]),
                                          _p(ref[2]), _p(ref[3]), _p(ws), ws.numel(), stream)
        assert rc == 0
        for _ in range(2):                                   # two calls in a row
            got = _outputs(torch, C, n_top)
            rc = L.hif4_calib_percentile_mask_noalloc(_p(acts), T, C, C, q[0], q[1], frac[0], frac[1],
                                                      _p(got[0]), _p(got[1]), _p(got[2]), _p(got[3]), stream)
            assert rc == 0
            torch.cuda.synchronize()
            assert torch.equal(got[0].view(torch.int16), ref[0].view(torch.int16))
            assert torch.equal(got[1].view(torch.int32), ref[1].view(torch.int32))
            assert torch.equal(got[2], ref[2])
            assert torch.equal(got[3][:n_top], ref[3][:n_top])


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import torch

    from block_floating_point_hif4_b200 import binding
    L = binding.lib()
    cap = L.hif4_calib_noalloc_scratch_bytes()
    # 5445 channels is the widest input whose scratch fits; one more does not
    assert L.hif4_calib_workspace(4096, 5445) <= cap < L.hif4_calib_workspace(4096, 5446)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    for T, C in ((4096, 5446), (16, 1 << 15)):
        assert L.hif4_calib_workspace(T, C) > cap
        rc = L.hif4_calib_percentile_mask_noalloc(_p(dummy), T, C, C, 999, 1000, 1, 100, _p(dummy), _p(dummy),
                                                  _p(dummy), None, stream)
        assert rc == 4                                       # HIF4_ERR_WORKSPACE, nothing launched
