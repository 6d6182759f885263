"""CPU pins of the oracle's FP4 index keys (E2M1 elements with one power-of-
two scale per 32 elements, stored as a biased 8-bit exponent) and of the
index score over them.  Pinned by: exactly representable blocks that must
round-trip, the shared-exponent rule checked by brute force over powers of
two, saturation and ties on the E2M1 grid, the reduction of the score to the
(pinned) int8 score when every block scale is 1, exact power-of-two scaling,
and exact small cases computed from the dequantised keys in float64."""
import numpy as np
import pytest

import oracle

GRID = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)


def _floor_log2(x: float) -> int:
    """Largest E with 2**E <= x, by brute force over exact powers of two."""
    E = -160
    while E < 130 and 2.0 ** (E + 1) <= x:
        E += 1
    return E


@pytest.mark.parametrize("k", [-20, -3, 0, 1, 7, 20])
def test_exactly_representable_blocks_round_trip(k):
    rng = np.random.default_rng(k + 50)
    vals = rng.choice(np.concatenate([GRID, -GRID[1:]]), (4, 64)).astype(np.float32)
    vals[:, 0] = 6.0            # each block's largest magnitude is 6: scale exactly 2^k
    vals[:, 32] = -6.0
    src = vals * np.float32(2.0 ** k)
    codes, exps = oracle.pack_mxfp4(src)
    assert np.all(exps == k + 127)
    assert np.array_equal(oracle.unpack_mxfp4(codes, exps, 64), src)


@pytest.mark.parametrize("amax", [5.0, 4.0, 3.99, 8.0, 7.99, 1e-30, 1.0, 2.0 ** -120, 3e38])
def test_shared_exponent_rule(amax):
    src = np.zeros((1, 32), np.float32)
    src[0, 7] = np.float32(amax)
    src[0, 8] = np.float32(amax) / 3
    _, exps = oracle.pack_mxfp4(src)
    s = min(max(_floor_log2(float(np.float32(amax))) - 2, -127), 127)
    assert exps[0, 0] == s + 127


def test_saturation_ties_and_zero_block():
    src = np.zeros((2, 32), np.float32)
    # block scale 1 (largest magnitude 7.9 -> floor(log2) = 2 -> s = 0)
    src[0, :10] = [7.9, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -5.0]
    codes, exps = oracle.pack_mxfp4(src)
    deq = oracle.unpack_mxfp4(codes, exps, 32)
    # nearest E2M1 value, ties to the even code, saturating at 6
    assert list(deq[0, :10]) == [6.0, 0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 0.0, -4.0]
    assert exps[1, 0] == 0 and np.all(codes[1] == 0)   # all-zero block
    assert np.all(deq[1] == 0.0) and not np.any(np.signbit(deq[0, [1, 8]]))


def _random_keys(rng, N, d_I):
    codes = rng.integers(0, 256, (N, d_I // 2)).astype(np.uint8)
    return codes


def _decoded_int(codes, d_I):
    """2 x E2M1 value of every element, as small integers (int8)."""
    lo, hi = codes & 0x0F, codes >> 4
    c = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], d_I)
    return (2 * np.array([oracle.e2m1_value(int(v)) for v in range(16)],
                         np.float32)[c]).astype(np.int8)


@pytest.mark.parametrize("d_I,H_I", [(32, 4), (64, 4), (64, 8), (128, 2)])
def test_score_with_unit_scales_equals_the_int8_score(d_I, H_I):
    rng = np.random.default_rng(d_I + H_I)
    N = 300
    q = rng.integers(-127, 128, (H_I, d_I)).astype(np.int8)
    w = rng.random(H_I, dtype=np.float32)
    codes = _random_keys(rng, N, d_I)
    exps = np.full((N, d_I // 32), 128, np.uint8)       # every block scale 2^(128-128) = 1
    got = oracle.index_score_fp4k_row(q, w, codes, exps)
    ref = oracle.index_score_row(q, w, _decoded_int(codes, d_I))
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("k", [-9, -1, 3, 11])
def test_score_scales_exactly_by_a_common_power_of_two(k):
    rng = np.random.default_rng(k + 100)
    H_I, d_I, N = 4, 64, 200
    q = rng.integers(-127, 128, (H_I, d_I)).astype(np.int8)
    w = rng.random(H_I, dtype=np.float32)
    codes = _random_keys(rng, N, d_I)
    base = oracle.index_score_fp4k_row(q, w, codes, np.full((N, 2), 128, np.uint8))
    got = oracle.index_score_fp4k_row(q, w, codes, np.full((N, 2), 128 + k, np.uint8))
    assert np.array_equal(got, base * np.float32(2.0 ** k))


def test_score_exact_small_cases_from_dequantised_keys():
    # unit weights and small integers: every rounding is exact, so the score
    # is the exact dot product of the query with the dequantised key
    rng = np.random.default_rng(7)
    H_I, d_I, N = 2, 64, 50
    q = rng.integers(-3, 4, (H_I, d_I)).astype(np.int8)
    w = np.ones(H_I, np.float32)
    codes = _random_keys(rng, N, d_I)
    exps = rng.integers(125, 131, (N, 2)).astype(np.uint8)
    got = oracle.index_score_fp4k_row(q, w, codes, exps)
    deq = oracle.unpack_mxfp4(codes, exps, d_I).astype(np.float64)
    exact = (q.astype(np.float64).sum(axis=0)[None, :] * deq).sum(axis=1)
    assert np.array_equal(got.astype(np.float64), exact)


def test_topk_over_fp4_keys_is_the_full_sort():
    rng = np.random.default_rng(2)
    B, H_I, d_I, N, k = 2, 4, 64, 700, 50
    q = rng.integers(-127, 128, (B, H_I, d_I)).astype(np.int8)
    w = rng.random((B, H_I), dtype=np.float32)
    src = rng.standard_normal((B * N, d_I)).astype(np.float32)
    codes, exps = oracle.pack_mxfp4(src)
    codes, exps = codes.reshape(B, N, -1), exps.reshape(B, N, -1)
    idx, sc = oracle.index_topk_fp4k(q, w, codes, exps, k, want_scores=True)
    for b in range(B):
        order = sorted(range(N), key=lambda n: (-float(sc[b, n]), n))[:k]
        assert list(idx[b]) == sorted(order)
        assert np.array_equal(sc[b], oracle.index_score_fp4k_row(q[b], w[b], codes[b], exps[b]))
