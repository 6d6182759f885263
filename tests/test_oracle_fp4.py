"""Pins of the oracle's FP4 (E2M1, per-16 fp32 scale) pack/unpack.

FP4 main-cache storage with per-group scaling: "DeepSeek-V4.1-Flash"
(visual explainer), section "Fast memory, persistent storage and
recomputation"; "Inference-Efficient LLMs", section 6.  The element format
(E2M1) and the group of 16 come from the OCP Microscaling (MX) format,
whose E2M1 value table is restated below; the amax/6 scale rule is the
reading this library takes.  Nothing here reuses the oracle's formulas:
rounding is checked by midpoint rules, packing by exactly representable
groups and by the round-to-nearest error bound.
"""
import math

import numpy as np
import pytest

import oracle

# OCP MX v1.0 E2M1 element values (positive codes 0..7); codes 8..15 negate.
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def test_e2m1_value_table():
    for c in range(16):
        v = oracle.e2m1_value(c)
        want = E2M1_TABLE[c & 7]
        assert abs(v) == want
        assert math.copysign(1.0, v) == (-1.0 if c & 8 else 1.0)


def _nearest_even_by_midpoints(y: float) -> int:
    """Round |y| to the E2M1 grid: above a midpoint goes up; exactly on a
    midpoint goes to the neighbour with an even code (mantissa bit 0)."""
    code = 0
    for i in range(7):
        mid = (E2M1_TABLE[i] + E2M1_TABLE[i + 1]) / 2.0
        if y > mid or (y == mid and (i + 1) % 2 == 0):
            code = i + 1
    return code


def _interesting_magnitudes():
    vals = set()
    for i in range(8):
        vals.add(E2M1_TABLE[i])
    for i in range(7):
        mid = np.float32((E2M1_TABLE[i] + E2M1_TABLE[i + 1]) / 2.0)
        vals.add(float(mid))
        vals.add(float(np.nextafter(mid, np.float32(0))))
        vals.add(float(np.nextafter(mid, np.float32(10))))
    vals.update([0.0, 1e-30, 6.0000005, 7.0, 1e30, float(np.float32(3.4e38))])
    rng = np.random.default_rng(11)
    vals.update(float(v) for v in rng.uniform(0, 8, 2000).astype(np.float32))
    return sorted(vals)


def test_round_to_nearest_even_matches_midpoint_rule():
    for y in _interesting_magnitudes():
        assert oracle.e2m1_round_mag(y) == _nearest_even_by_midpoints(y), y


def test_tie_cases_explicit():
    # midpoint -> expected magnitude code (even neighbour)
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for y, c in ties.items():
        assert oracle.e2m1_round_mag(y) == c


def _group_values(codes_row, scales_row, D):
    vals = []
    for i in range(D):
        byte = int(codes_row[i // 2])
        c = (byte & 0xF) if i % 2 == 0 else (byte >> 4)
        sign = -1.0 if c & 8 else 1.0
        # the exact product (fits a double) rounded once to fp32: an fp32 multiply
        vals.append(np.float32(sign * E2M1_TABLE[c & 7] * float(scales_row[i // 16])))
    return np.array(vals, np.float64)


@pytest.mark.parametrize("e", [-20, -3, 0, 5])
def test_exactly_representable_groups_roundtrip(e):
    """A group whose values are E2M1 grid points times 2**e, with 6*2**e
    present, has scale 2**e, its own grid codes and an exact round trip."""
    rng = np.random.default_rng(e + 100)
    D = 64
    codes_want = rng.integers(0, 16, size=D)
    for g in range(D // 16):
        codes_want[16 * g + rng.integers(0, 16)] = 7  # amax = 6 * 2**e in every group
    codes_want[codes_want == 8] = 0  # the format stores no negative zero
    x = np.array([(-1.0 if c & 8 else 1.0) * E2M1_TABLE[c & 7] * 2.0 ** e for c in codes_want],
                 np.float32)[None, :]
    codes, scales = oracle.pack_fp4(x)
    assert np.all(scales == np.float32(2.0 ** e))
    got_codes = [(codes[0, i // 2] >> (4 * (i % 2))) & 0xF for i in range(D)]
    assert got_codes == list(codes_want)
    assert np.array_equal(oracle.unpack_fp4(codes, scales, D), x)


def test_nibble_order_and_zero_sign():
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 6.0
    x[0, 3] = -6.0
    x[0, 5] = -0.01  # rounds to magnitude 0: stored as code 0, not 8
    codes, scales = oracle.pack_fp4(x)
    assert scales[0, 0] == np.float32(1.0)
    assert codes[0, 0] == 0x07        # element 0 low nibble, element 1 high nibble
    assert codes[0, 1] == 0xF0        # element 3 (high nibble of byte 1) = -6 -> 0xF
    assert codes[0, 2] == 0x00        # -0.01 -> +0


def test_zero_group():
    x = np.zeros((2, 32), np.float32)
    x[1, 16:] = 1.0
    codes, scales = oracle.pack_fp4(x)
    assert np.all(codes[0] == 0) and np.all(scales[0] == 0)
    assert np.all(codes[1, :8] == 0) and scales[1, 0] == 0


@pytest.mark.parametrize("D", [16, 64, 128])
def test_random_rows_error_bound_and_scale(D):
    rng = np.random.default_rng(D)
    x = (rng.standard_normal((300, D)) * np.exp(rng.uniform(-8, 8, (300, 1)))).astype(np.float32)
    codes, scales = oracle.pack_fp4(x)
    deq = oracle.unpack_fp4(codes, scales, D).astype(np.float64)
    for r in range(x.shape[0]):
        for g in range(D // 16):
            grp = x[r, 16 * g:16 * g + 16].astype(np.float64)
            s = float(scales[r, g])
            amax = np.max(np.abs(grp))
            # scale: amax / 6 rounded once to fp32 -> within half an ulp of amax/6
            assert abs(s - amax / 6.0) <= 0.5 * np.spacing(np.float32(s)) + 1e-45
            vals = _group_values(codes[r], scales[r], D)[16 * g:16 * g + 16]
            # reconstruction equals the unpack routine
            assert np.allclose(vals, deq[r, 16 * g:16 * g + 16], rtol=0, atol=0)
            # round-to-nearest bound: within half the local grid gap (+ tiny fp32 slack)
            mags = np.abs(grp) / s
            lo_gap = np.array([_gap_around(m) for m in mags])
            err = np.abs(grp - vals)
            assert np.all(err <= (0.5 * lo_gap + 1e-5) * s + 1e-30)
            # the group maximum maps to the largest magnitude
            i_max = int(np.argmax(np.abs(grp)))
            assert abs(vals[i_max]) == float(np.float32(6.0 * s))


def _gap_around(m):
    for i in range(7):
        if m <= E2M1_TABLE[i + 1]:
            return E2M1_TABLE[i + 1] - E2M1_TABLE[i]
    return 2.0
