"""Pins for the oracle's HiF4 format arithmetic (CPU only).

Every check here compares the oracle with something other than itself:
facts printed in the HiF4 format definition (Huawei HiF4 calibration article,
hwcomputing.csdn.net, section 1: 64-element unit, 32 metadata bits, S1P2
magnitudes 0.25..1.75, power-of-two levels 2 and 3), exact rational
arithmetic, brute force, hand-derived fixtures (tests/golden/hif4_units.txt)
and invariants that the encode rule provably has (idempotence, error bound).
"""
from fractions import Fraction
import itertools
import os

import numpy as np
import pytest

import oracle
from block_floating_point_hif4_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hif4_units.txt")


def frac_e6m2(code):
    """E6M2 value written from its field definition, as an exact rational."""
    E, f = code >> 2, code & 3
    return Fraction(4 + f, 4) * Fraction(2) ** (E - 31)


# ----------------------------------------------------------------- E6M2

def test_e6m2_closed_form():
    assert oracle.e6m2_value(124) == 1.0          # E = 31 = bias, f = 0
    assert oracle.e6m2_value(0) == 2.0 ** -31
    assert oracle.e6m2_value(255) == 1.75 * 2.0 ** 32
    assert oracle.e6m2_value(126) == 1.5
    vals = [oracle.e6m2_value(c) for c in range(256)]
    for c in range(256):
        assert Fraction(vals[c]) == frac_e6m2(c)
    ratios = {Fraction(vals[c + 1]) / Fraction(vals[c]) for c in range(255)}
    assert ratios == {Fraction(5, 4), Fraction(6, 5), Fraction(7, 6), Fraction(8, 7)}


def test_select_scale_exact_rationals():
    rng = np.random.default_rng(11)
    cands = list(np.exp(rng.uniform(-25, 25, 400)))
    # exact boundary values 6.5 v(c) and their float neighbours
    for c in [0, 1, 2, 3, 4, 50, 123, 124, 125, 126, 127, 200, 254, 255]:
        b = 6.5 * oracle.e6m2_value(c)
        cands += [b, np.nextafter(b, 0), np.nextafter(b, np.inf)]
    cands += [0.0, 1e-30, 1e30, 7.0, 10.0, 8.1]
    for a in cands:
        c = oracle.select_scale_code(a)
        fa = Fraction(float(a))
        if fa <= Fraction(13, 2) * frac_e6m2(0):
            assert c == 0
            continue
        assert Fraction(13, 2) * frac_e6m2(c) < fa
        if c < 255:
            assert Fraction(13, 2) * frac_e6m2(c + 1) >= fa


# ------------------------------------------------------- element rounding

def brute_round(ax, step):
    """Nearest of the 8 magnitudes m*step, ties to even m (exact)."""
    ax, step = Fraction(ax), Fraction(step)
    best = min(range(8), key=lambda m: (abs(ax - m * step), m % 2))
    return best


def test_round_magnitude_brute_force():
    rng = np.random.default_rng(12)
    steps = [0.25, 0.375, 0.3125, 0.4375, 2.0 ** -33, 1.75 * 2.0 ** 32]
    for step in steps:
        xs = list(rng.uniform(0, 9 * step, 300))
        xs += [(k + 0.5) * step for k in range(9)]                 # exact ties
        xs += [np.nextafter((k + 0.5) * step, 0) for k in range(8)]
        xs += [np.nextafter((k + 0.5) * step, np.inf) for k in range(8)]
        for x in xs:
            assert oracle.round_magnitude(x, step) == brute_round(x, step), (x, step)


# -------------------------------------------------------- decode and grid

def test_s1p2_grid():
    meta = 124                                   # S = 1, all level-2/3 bits 0
    got = [oracle.decode_element(n, meta, 0) for n in range(16)]
    want = [0, 0.25, 0.5, 0.75, 1.0, 1.25, 1.5, 1.75,
            -0.0, -0.25, -0.5, -0.75, -1.0, -1.25, -1.5, -1.75]
    assert got == want


def test_levels_are_powers_of_two_on_their_groups():
    # level-2 bit j doubles exactly elements 8j..8j+7, level-3 bit k exactly 4k..4k+3
    for j in range(8):
        meta = 124 | (1 << (8 + j))
        for i in range(64):
            y = oracle.decode_element(7, meta, i)
            assert y == (3.5 if i // 8 == j else 1.75)
    for k in range(16):
        meta = 124 | (1 << (16 + k))
        for i in range(64):
            y = oracle.decode_element(5, meta, i)
            assert y == (2.5 if i // 4 == k else 1.25)
    meta = 124 | (1 << 8) | (1 << 16)
    assert oracle.decode_element(7, meta, 0) == 7.0         # both levels: x4


def test_decoded_values_exact_in_bf16():
    for c in range(256):
        for E in range(3):
            e2 = 1 if E >= 1 else 0
            e3 = 1 if E == 2 else 0
            meta = c | (e2 << 8) | (e3 << 16)
            ys = np.array([oracle.decode_element(n, meta, 0) for n in range(16)])
            f32 = ys.astype(np.float32)
            assert np.array_equal(f32.astype(np.float64), ys)
            back = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(f32))
            assert np.array_equal(back, f32)


def test_metadata_budget():
    # 1 x 8 + 8 x 1 + 16 x 1 = 32 bits per 64 elements = 0.5 bit / element
    x = np.random.default_rng(0).standard_normal((3, 256)).astype(np.float32)
    codes, meta, _ = oracle.quantize(x)
    assert codes.nbytes * 8 == 4 * x.size
    assert meta.nbytes * 8 == 32 * (x.size // 64)
    assert meta.nbytes * 8 / x.size == 0.5


# ---------------------------------------------------------- golden units

def load_golden():
    units, cur = [], None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(" ")
        if key == "unit":
            cur = dict(name=rest)
            units.append(cur)
        elif key in ("x", "y"):
            d = {}
            for tok in rest.split():
                i, v = tok.split(":")
                d[int(i)] = float(v)
            cur[key] = d
        elif key == "meta":
            cur["meta"] = int(rest, 16)
        elif key == "codes":
            cur["codes"] = bytes.fromhex(rest.replace(" ", ""))
    return units


@pytest.mark.parametrize("u", load_golden(), ids=lambda u: u["name"])
def test_golden_units(u):
    x = np.zeros((1, 64), np.float32)
    for i, v in u["x"].items():
        x[0, i] = v
    codes, meta, nf = oracle.quantize(x)
    assert nf == 0
    assert int(meta[0, 0]) == u["meta"], hex(int(meta[0, 0]))
    assert codes[0].tobytes() == u["codes"], codes[0].tobytes().hex()
    y = oracle.dequantize(codes, meta, 64)[0]
    want = np.zeros(64)
    for i, v in u["y"].items():
        want[i] = v
    assert np.array_equal(y, want)


# ----------------------------------------------------------- invariants

def unit_batches():
    rng = np.random.default_rng(7)
    out = [rng.standard_normal((200, 64)),
           rng.standard_t(3, (200, 64)) * 0.05,
           rng.standard_cauchy((100, 64)),
           np.exp(rng.uniform(-60, 60, (100, 1))) * rng.standard_normal((100, 64))]
    # adversarial: values sitting on scale / group / rounding boundaries
    adv = []
    for c in [0, 3, 60, 124, 125, 126, 127, 250, 255]:
        S = oracle.e6m2_value(c)
        for mult in [6.5, 1.75, 3.5, 7.0, 0.125, 0.375, 0.625, 1.125, 8.125]:
            row = rng.standard_normal(64) * S
            row[rng.integers(64)] = mult * S
            row[rng.integers(64)] = np.nextafter(mult * S, 0)
            adv.append(row)
    out.append(np.array(adv))
    return [b.astype(np.float32) for b in out]


def test_idempotence():
    for b in unit_batches():
        codes, meta, _ = oracle.quantize(b)
        y = oracle.dequantize(codes, meta, 64).astype(np.float32)
        codes2, meta2, _ = oracle.quantize(y)
        assert np.array_equal(codes, codes2)
        assert np.array_equal(meta, meta2)


def test_grid_aligned_reproduction():
    rng = np.random.default_rng(8)
    for _ in range(200):
        c = int(rng.integers(0, 256))
        nib = rng.integers(0, 16, 64).astype(np.uint8)
        nib[rng.integers(64)] = 7                      # force one m = 7 element
        e2 = rng.integers(0, 2, 8)
        e3 = rng.integers(0, 2, 16)
        k0 = int(np.nonzero(nib == 7)[0][0]) // 4
        e2[k0 // 2] = 1
        e3[k0] = 1                                     # ... in an E = 2 group
        meta = c | int(sum(int(b) << (8 + j) for j, b in enumerate(e2))) \
                 | int(sum(int(b) << (16 + k) for k, b in enumerate(e3)))
        y = np.array([oracle.decode_element(int(nib[i]), meta, i) for i in range(64)], np.float32)
        codes, m2, _ = oracle.quantize(y[None])
        y2 = oracle.dequantize(codes, m2, 64)[0]
        assert np.array_equal(y2, y.astype(np.float64))


def unpack(codes, meta):
    n = codes.shape[0]
    nib = np.zeros((n, 64), np.uint8)
    nib[:, 0::2] = codes & 15
    nib[:, 1::2] = codes >> 4
    c = (meta & 0xFF).astype(np.int64)
    e2 = (meta[:, None] >> (8 + np.arange(8))) & 1
    e3 = (meta[:, None] >> (16 + np.arange(16))) & 1
    E = np.repeat(e2, 8, 1) + np.repeat(e3, 4, 1)
    return nib, c, E.astype(np.int64)


def test_error_bound_and_elementwise_optimality():
    for b in unit_batches():
        codes, meta, _ = oracle.quantize(b)
        meta = meta[:, 0]
        y = oracle.dequantize(codes, meta[:, None], 64)
        nib, c, E = unpack(codes, meta)
        S = np.array([oracle.e6m2_value(int(ci)) for ci in c])[:, None]
        step = S * 2.0 ** E / 4
        x = b.astype(np.float64)
        err = np.abs(x - y)
        sat = np.abs(x) > 7.5 * step
        # unsaturated: within half a step; saturated only in E = 2 groups
        assert np.all(err[~sat] <= step[~sat] / 2)
        assert np.all(E[sat] == 2) or np.all(c[np.any(sat, 1)] == 255)
        top = (c < 255)[:, None] & sat
        assert np.all(err[top] <= 1.125 * np.broadcast_to(S, err.shape)[top])
        # unit-wide bound for units whose scale is not clamped at either end
        ok = (c > 0) & (c < 255)
        amax = np.abs(x).max(1)
        assert np.all(err.max(1)[ok] <= 1.125 * S[ok, 0])
        assert np.all(err.max(1)[ok] < 0.1731 * amax[ok])
        # each element is the brute-force nearest magnitude for its metadata
        rng = np.random.default_rng(3)
        for r in rng.choice(b.shape[0], size=min(40, b.shape[0]), replace=False):
            for i in range(64):
                m = int(nib[r, i] & 7)
                assert m == brute_round(abs(float(x[r, i])), float(step[r, i])), (r, i)
                if m == 0:
                    assert nib[r, i] == 0                # never a negative zero
                else:
                    assert (nib[r, i] >> 3) == (1 if x[r, i] < 0 else 0)


def test_metadata_rule_properties():
    """E_k is the least exponent the level-2 sharing allows for the group."""
    for b in unit_batches():
        codes, meta, _ = oracle.quantize(b)
        meta = meta[:, 0]
        nib, c, E = unpack(codes, meta)
        S = np.array([oracle.e6m2_value(int(ci)) for ci in c])
        e2 = (meta[:, None] >> (8 + np.arange(8))) & 1
        x = np.abs(b.astype(np.float64)).reshape(-1, 16, 4).max(2)
        Ek = E[:, ::4]
        for r in range(b.shape[0]):
            for k in range(16):
                fits = x[r, k] <= 1.75 * S[r] * 2.0 ** Ek[r, k]
                assert fits or Ek[r, k] == 2
                floor = e2[r, k // 2]
                if Ek[r, k] > floor:                   # e3 = 1 only when needed
                    assert x[r, k] > 1.75 * S[r] * 2.0 ** floor
            pair_needs_4 = x[r].reshape(8, 2).max(1) > 3.5 * S[r]
            assert np.array_equal(e2[r].astype(bool), pair_needs_4)


def best_sse(x):
    """Brute force over every metadata choice (256 scales x 8^8 bit patterns,
    separable per 8-group) of the least squared error of a unit."""
    x = np.asarray(x, np.float64)
    best = np.inf
    g = np.abs(x).reshape(8, 2, 4)
    mags = np.arange(8) / 4.0
    for c in range(256):
        S = oracle.e6m2_value(c)
        tot = 0.0
        for j in range(8):
            bj = np.inf
            for e2, e3a, e3b in itertools.product((0, 1), repeat=3):
                s = 0.0
                for h, e3 in ((0, e3a), (1, e3b)):
                    grid = mags * S * 2.0 ** (e2 + e3)
                    s += np.min((g[j, h][:, None] - grid[None, :]) ** 2, 1).sum()
                bj = min(bj, s)
            tot += bj
        best = min(best, tot)
    return best


def test_encoder_against_metadata_optimum():
    rng = np.random.default_rng(21)
    ratios = []
    for _ in range(4):
        x = rng.standard_normal(64).astype(np.float32)
        codes, meta, _ = oracle.quantize(x[None])
        y = oracle.dequantize(codes, meta, 64)[0]
        sse = float(((x.astype(np.float64) - y) ** 2).sum())
        opt = best_sse(x)
        assert sse >= opt * (1 - 1e-12)
        ratios.append(sse / opt)
    assert max(ratios) < 4.0


def test_non_finite_mapping():
    x = np.zeros((1, 64), np.float32)
    x[0, 0] = np.nan
    x[0, 1] = 0.875                     # = 7 * 2^-3: on the grid, reproduced
    codes, meta, nf = oracle.quantize(x)
    assert nf == 1
    y = oracle.dequantize(codes, meta, 64)[0]
    assert y[0] == 0 and y[1] == 0.875
    x[0, 0] = -np.inf
    codes, meta, nf = oracle.quantize(x)
    assert nf == 1 and int(meta[0, 0]) & 0xFF == 255
    y = oracle.dequantize(codes, meta, 64)[0]
    assert y[0] == -7 * oracle.e6m2_value(255)


def test_mask_excludes_channel():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 128)).astype(np.float32)
    x[:, 70] = 1000.0
    mask = np.zeros(128, np.uint8)
    mask[70] = 1
    c1, m1, _ = oracle.quantize(x, mask)
    x0 = x.copy()
    x0[:, 70] = 0
    c0, m0, _ = oracle.quantize(x0)
    assert np.array_equal(c1, c0) and np.array_equal(m1, m0)


def test_bf16_input_path_matches_f32_widening():
    rng = np.random.default_rng(9)
    bits = wl.f32_to_bf16_bits(rng.standard_normal((8, 192)).astype(np.float32))
    a = oracle.quantize(bits)
    b = oracle.quantize(wl.bf16_bits_to_f32(bits))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_fake_quantize_and_weight_hat():
    rng = np.random.default_rng(6)
    x = wl.f32_to_bf16_bits(rng.standard_normal((5, 256)).astype(np.float32))
    idx = np.array([3, 64, 200], np.int32)
    xh = oracle.fake_quantize(x, idx)
    xf = wl.bf16_bits_to_f32(x).astype(np.float64)
    assert np.array_equal(xh[:, idx], xf[:, idx])
    mask = np.zeros(256, np.uint8)
    mask[idx] = 1
    codes, meta, _ = oracle.quantize(x, mask)
    deq = oracle.dequantize(codes, meta, 256)
    keep = np.ones(256, bool)
    keep[idx] = False
    assert np.array_equal(xh[:, keep], deq[:, keep])
    wm = x[:, idx]
    wh = oracle.weight_hat(codes, meta, 5, 256, idx, wm)
    assert np.array_equal(wh, xh)
