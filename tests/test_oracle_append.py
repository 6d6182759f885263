"""CPU pins of the oracle's entry append (the per-token write side of the
cache: a completed entry packed to FP4 into its row of the store, with its
int8 index key beside it).  Pinned by facts outside the function: the bulk
pack of the same rows, exactly representable entries that must come back
unchanged, untouched neighbour rows, and the error case."""
import numpy as np
import pytest

import oracle


def _store(B, N, D, d_I, fill=0x5A):
    codes = np.full((B, N, D // 2), fill, np.uint8)
    scales = np.full((B, N, D // 16), np.float32(-3.0), np.float32)
    keys = np.full((B, N, d_I), np.int8(-7), np.int8)
    return codes, scales, keys


def test_appending_rows_one_by_one_equals_the_bulk_pack():
    rng = np.random.default_rng(3)
    B, N, D, d_I = 3, 9, 64, 32
    src = rng.standard_normal((B, N, D)).astype(np.float32)
    src[1, 4] *= np.float32(1e-30)                    # tiny groups
    src[2, 5, :16] = 0.0                              # a zero group
    key = rng.integers(-127, 128, (B, N, d_I)).astype(np.int8)
    codes, scales, keys = _store(B, N, D, d_I)
    for n in range(N):                                # one decode step per entry
        oracle.append_entry(src[:, n], key[:, n], np.full(B, n, np.int64), codes, scales, keys)
    bulk_c, bulk_s = oracle.pack_fp4(src.reshape(B * N, D))
    assert np.array_equal(codes.reshape(B * N, -1), bulk_c)
    assert np.array_equal(scales.reshape(B * N, -1).view(np.uint32), bulk_s.view(np.uint32))
    assert np.array_equal(keys, key)


def test_exactly_representable_entry_comes_back_unchanged():
    # values on the E2M1 grid times 2^e with the group's largest magnitude 6:
    # scale 2^e exactly, every code exact, so unpacking returns the entry
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -.5, -1, -1.5, -2, -3, -4, -6, 6], np.float32)
    D, d_I = 32, 16
    src = np.stack([grid * np.float32(2.0 ** -3), grid[::-1] * np.float32(2.0 ** 5)]).reshape(1, D)
    codes, scales, keys = _store(1, 4, D, d_I)
    oracle.append_entry(src, np.arange(d_I, dtype=np.int8)[None], np.array([2], np.int64), codes,
                        scales, keys)
    assert np.array_equal(scales[0, 2], np.float32([2.0 ** -3, 2.0 ** 5]))
    assert np.array_equal(oracle.unpack_fp4(codes[0, 2], scales[0, 2], D)[0], src[0])
    assert np.array_equal(keys[0, 2], np.arange(d_I, dtype=np.int8))


def test_only_the_appended_row_changes_and_negative_positions_skip():
    rng = np.random.default_rng(5)
    B, N, D, d_I = 4, 6, 64, 32
    codes, scales, keys = _store(B, N, D, d_I)
    before = (codes.copy(), scales.copy(), keys.copy())
    src = rng.standard_normal((B, D)).astype(np.float32)
    key = rng.integers(-127, 128, (B, d_I)).astype(np.int8)
    pos = np.array([5, -1, 0, 3], np.int64)
    oracle.append_entry(src, key, pos, codes, scales, keys)
    for b in range(B):
        for n in range(N):
            same = (np.array_equal(codes[b, n], before[0][b, n])
                    and np.array_equal(scales[b, n], before[1][b, n])
                    and np.array_equal(keys[b, n], before[2][b, n]))
            assert same == (n != pos[b]), (b, n)
    c1, s1 = oracle.pack_fp4(src[[0]])
    assert np.array_equal(codes[0, 5], c1[0]) and np.array_equal(keys[0, 5], key[0])


def test_position_past_the_store_is_an_error_and_writes_nothing():
    codes, scales, keys = _store(2, 4, 64, 32)
    before = codes.copy()
    with pytest.raises(oracle.OracleError):
        oracle.append_entry(np.ones((2, 64), np.float32), np.ones((2, 32), np.int8),
                            np.array([1, 4], np.int64), codes, scales, keys)
    assert np.array_equal(codes, before)
