"""Pins for the oracle's tail-percentile and channel-mask calibration (CPU).

The percentile rule (Tail-Aware HiFloat4 summary on agents-report.net,
"Why tail percentiles"; rank rule floor(999 (T-1) / 1000) and median over
channels are readings) is checked against numpy's sort, and the mask against
numpy's stable lexicographic ordering; tiny cases are brute-forced.
"""
import numpy as np

import oracle
from block_floating_point_hif4_b200 import workloads as wl


def keys(bits):
    return (bits & 0x7FFF).astype(np.uint16)


def test_percentile_vs_numpy_sort():
    rng = np.random.default_rng(1)
    for T, C in [(1, 3), (7, 5), (1000, 64), (2311, 33)]:
        x = wl.f32_to_bf16_bits((rng.standard_normal((T, C)) * rng.lognormal(0, 1, C)).astype(np.float32))
        got = oracle.percentile(x, threads=2)
        k = (999 * (T - 1)) // 1000
        want = np.sort(keys(x), axis=0)[k]
        assert np.array_equal(got, want)
        # the value is an order statistic of |x| in float terms too
        fx = np.abs(wl.bf16_bits_to_f32(x))
        assert np.array_equal(wl.bf16_bits_to_f32(got), np.sort(fx, axis=0)[k])


def test_percentile_rank_rule_integer():
    # floor(q (T-1)) computed in integers: T = 230400 -> k = 230168 (232nd largest)
    T = 230400
    assert (999 * (T - 1)) // 1000 == 230168
    assert T - 1 - 230168 == 231


def test_percentile_signed_zero_and_ties():
    x = np.array([[0x8000], [0x0000], [0x3F80], [0xBF80], [0x4000]], np.uint16)  # -0, 0, 1, -1, 2
    assert oracle.percentile(x, 1, 2)[0] == 0x3F80       # k = floor(4/2) = 2 -> keys 0,0,1,1,2
    assert oracle.percentile(x, 0, 1)[0] == 0x0000
    assert oracle.percentile(x, 1, 1)[0] == 0x4000


def test_percentile_brute_force_tiny():
    rng = np.random.default_rng(2)
    for _ in range(50):
        T = int(rng.integers(1, 9))
        x = rng.integers(0, 1 << 16, (T, 2)).astype(np.uint16)
        x[(x & 0x7F80) == 0x7F80] &= 0x3FFF            # finite values only
        qn, qd = int(rng.integers(0, 11)), 10
        got = oracle.percentile(x, qn, qd)
        k = qn * (T - 1) // qd
        for c in range(2):
            ks = sorted(int(v) & 0x7FFF for v in x[:, c])
            assert got[c] == ks[k]


def test_channel_mask_vs_numpy():
    rng = np.random.default_rng(3)
    for C in [1, 2, 100, 5120, 777]:
        p = keys(rng.integers(0x3000, 0x4400, C).astype(np.uint16))
        p[rng.integers(0, C, C // 7)] = p[0]            # many ties
        ratio, mask, n = oracle.channel_mask(p, 1, 100)
        assert n == C // 100 == mask.sum()
        order = np.lexsort((np.arange(C), -p.astype(np.int64)))   # p desc, idx asc
        want = np.zeros(C, np.uint8)
        want[order[:C // 100]] = 1
        assert np.array_equal(mask, want)
        med = np.sort(p)[(C - 1) // 2]
        fp = wl.bf16_bits_to_f32(p)
        assert np.array_equal(ratio, fp / wl.bf16_bits_to_f32(np.array([med], np.uint16))[0])


def test_channel_mask_zero_median():
    p = np.array([0, 0, 0, 0x3F80, 0x4000], np.uint16)
    ratio, mask, n = oracle.channel_mask(p, 2, 5)
    assert n == 2 and list(mask) == [0, 0, 0, 1, 1]
    assert list(ratio) == [0, 0, 0, np.inf, np.inf]


def test_mask_fraction_rounding():
    p = np.arange(1, 138 * 100 + 1, dtype=np.uint16)[:13824] | 0x3000
    _, _, n = oracle.channel_mask(p, 1, 100)
    assert n == 138
    _, _, n = oracle.channel_mask(p[:5120], 1, 100)
    assert n == 51
