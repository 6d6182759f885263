"""Pins of the oracle's indexer score, visibility rule and top-k.

Indexer and Top-K: "Why Is DeepSeek V4.1 Flash So Fast?", section 4 ("The
indexer": index heads score compressed positions cheaply, the Top-K best
go on to attention).  The score reading (exact int8 dot per head, heads
summed left to right with fp32 weights, each product and sum rounded on
its own) and the tie rule (lower index first) are this library's
readings.  Pins: exact integer brute force, a hand-worked rounding example
that only the stated summation order produces, the recursive-summation
error bound, and top-k properties checked without sorting.
"""
import numpy as np
import pytest

import oracle


def _brute_dots(q, keys):
    """Exact per-head integer dot products with Python ints."""
    H_I, d_I = q.shape
    return [[sum(int(q[h, i]) * int(k[i]) for i in range(d_I)) for h in range(H_I)] for k in keys]


@pytest.mark.parametrize("d_I", [16, 32, 64])
def test_single_head_unit_weight_is_exact_int_dot(d_I):
    rng = np.random.default_rng(d_I)
    q = rng.integers(-127, 128, (1, d_I), dtype=np.int8)
    keys = rng.integers(-127, 128, (200, d_I), dtype=np.int8)
    keys[0] = 127
    keys[1] = -127
    q_ext = np.full((1, d_I), 127, np.int8)
    got = oracle.index_score_row(q, np.ones(1, np.float32), keys)
    want = [d[0] for d in _brute_dots(q, keys)]
    assert got.tolist() == [float(v) for v in want]
    # the extreme dot 64*127*127 is still exact in fp32 (< 2**24)
    ext = oracle.index_score_row(q_ext, np.ones(1, np.float32), keys[:2])
    assert ext.tolist() == [float(d_I * 127 * 127), float(-d_I * 127 * 127)]


def test_single_head_weighted_is_one_rounding():
    rng = np.random.default_rng(5)
    q = rng.integers(-127, 128, (1, 64), dtype=np.int8)
    keys = rng.integers(-127, 128, (300, 64), dtype=np.int8)
    w = rng.random(1, dtype=np.float32)
    got = oracle.index_score_row(q, w, keys)
    dots = [d[0] for d in _brute_dots(q, keys)]
    # w * dot is exact in double (24 + 21 bits), so one cast is one rounding
    want = [np.float32(float(w[0]) * d) for d in dots]
    assert np.array_equal(got, np.array(want, np.float32))


def test_heads_summed_left_to_right():
    """Worked example: terms 2**24, 1, 1.  Left to right, each +1 is a tie
    at 2**24 + 1 and rounds back to 2**24 (even); any order that adds the
    two ones first gives 2**24 + 2."""
    d_I = 16
    q = np.zeros((3, d_I), np.int8)
    q[0, 0] = q[1, 1] = q[2, 2] = 1
    key = np.zeros((1, d_I), np.int8)
    key[0, 0], key[0, 1], key[0, 2] = 64, 1, 1
    w = np.array([2.0 ** 18, 1.0, 1.0], np.float32)      # 2**18 * 64 = 2**24
    assert oracle.index_score_row(q, w, key)[0] == np.float32(16777216.0)
    w_rev = np.array([1.0, 1.0, 2.0 ** 18], np.float32)
    key_rev = np.zeros((1, d_I), np.int8)
    key_rev[0, 0], key_rev[0, 1], key_rev[0, 2] = 1, 1, 64
    assert oracle.index_score_row(q, w_rev, key_rev)[0] == np.float32(16777218.0)


def test_random_scores_within_summation_bound_and_never_negative_zero():
    rng = np.random.default_rng(9)
    H_I, d_I = 4, 64
    q = rng.integers(-127, 128, (H_I, d_I), dtype=np.int8)
    keys = rng.integers(-127, 128, (500, d_I), dtype=np.int8)
    keys[10] = 0
    w = np.concatenate([rng.random(3, dtype=np.float32), np.float32([-0.75])])
    got = oracle.index_score_row(q, w, keys).astype(np.float64)
    dots = _brute_dots(q, keys)
    u = 2.0 ** -24
    for n, dn in enumerate(dots):
        terms = [float(w[h]) * dn[h] for h in range(H_I)]
        exact = sum(terms)
        bound = (2 * H_I) * u * sum(abs(t) for t in terms)
        assert abs(got[n] - exact) <= bound + 1e-30
    assert got[10] == 0.0 and np.signbit(np.float32(got[10])) == False  # noqa: E712


def test_visibility_rule_brute_force():
    """Prefill chunk entry j compresses tokens ratio*j .. ratio*j+ratio-1;
    query t sees it once all of them are at or before t."""
    for ratio in (1, 2, 4):
        n_prior, chunk_entries = 7, 9
        N = n_prior + chunk_entries
        for t in range(ratio * chunk_entries + 3):
            want = n_prior + sum(
                1 for j in range(chunk_entries) if all(ratio * j + r <= t for r in range(ratio)))
            assert oracle.visible_count(N, n_prior, ratio, t) == min(want, N)
        assert oracle.visible_count(N, -1, ratio, 0) == N


def _check_topk_valid(scores, V, k, idx):
    m = min(k, V)
    sel = idx[:m]
    assert np.all(idx[m:] == -1)
    assert np.all(sel >= 0) and np.all(sel < V)
    assert np.all(np.diff(sel) > 0)  # ascending, unique
    chosen = np.zeros(V, bool)
    chosen[sel] = True
    if m == V:
        return
    worst_in = scores[:V][chosen].min()
    best_out = scores[:V][~chosen].max()
    assert worst_in >= best_out
    # on the boundary value, every kept index is below every dropped one
    tie_in = np.nonzero(chosen & (scores[:V] == worst_in))[0]
    tie_out = np.nonzero(~chosen & (scores[:V] == worst_in))[0]
    if tie_in.size and tie_out.size:
        assert tie_in.max() < tie_out.min()


def test_topk_all_equal_gives_first_k():
    for N, k in [(10, 3), (1000, 64), (5, 5)]:
        assert oracle.topk_row(np.full(N, 1.5, np.float32), k).tolist() == list(range(k))


def test_topk_k_at_least_visible_pads():
    got = oracle.topk_row(np.arange(5, dtype=np.float32), 8)
    assert got.tolist() == [0, 1, 2, 3, 4, -1, -1, -1]
    assert oracle.topk_row(np.zeros(0, np.float32), 3).tolist() == [-1, -1, -1]


def test_topk_permutation_scores_exact_set():
    rng = np.random.default_rng(3)
    N, k = 4096, 300
    perm = rng.permutation(N).astype(np.float32)
    got = oracle.topk_row(perm, k)
    assert got.tolist() == sorted(np.nonzero(perm >= N - k)[0].tolist())


@pytest.mark.parametrize("levels", [3, 50, 100000])
def test_topk_random_with_ties_valid(levels):
    rng = np.random.default_rng(levels)
    N, k = 3000, 257
    scores = rng.integers(-levels, levels, N).astype(np.float32) * np.float32(0.5)
    idx = oracle.topk_row(scores, k)
    _check_topk_valid(scores, N, k, idx)


def test_index_topk_prefill_visibility_and_padding():
    rng = np.random.default_rng(21)
    B, T, H_I, d_I, topk, ratio, n_prior = 2, 12, 2, 16, 6, 4, 3
    N = n_prior + T // ratio
    q = rng.integers(-127, 128, (B, T, H_I, d_I), dtype=np.int8)
    w = rng.random((B, T, H_I), dtype=np.float32)
    keys = rng.integers(-127, 128, (B, N, d_I), dtype=np.int8)
    idx, scores = oracle.index_topk(q, w, keys, topk, n_prior, ratio, want_scores=True)
    for r in range(B * T):
        b, t = divmod(r, T)
        V = n_prior + (t + 1) // ratio
        assert np.all(np.isneginf(scores[r, V:])) and np.all(np.isfinite(scores[r, :V]))
        assert np.array_equal(scores[r, :V], oracle.index_score_row(q[b, t], w[b, t], keys[b])[:V])
        _check_topk_valid(scores[r], V, topk, idx[r])
