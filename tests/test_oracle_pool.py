"""Pins of the oracle's hierarchical indexer: the candidate pool of a Full
layer and the top-k of a Reindex layer within it.

"Inference-Efficient LLMs: How Sparse Compute and Compressed Memory Work",
section 5 ("Hierarchical Sparse Indexing"): an earlier Full layer keeps a
candidate pool (the example: 2,048 blocks of eight positions, 16,384
candidates) and later Reindex layers search only within it.  The block
score (the block's largest score), the tie rule (lower block, lower
position) and the ascending pool order are this library's readings.  Pins:
the example's pool size, planted blocks whose answer is known by
construction, ties, a partial last block, the reduction to the pinned
full-store top-k when the pool covers every block, and pairwise properties
of the pool top-k checked without sorting.
"""
import numpy as np
import pytest

import oracle


def _blocks_of(pool, block):
    return sorted(set(int(n) // block for n in pool))


def test_pool_of_the_pages_example_holds_16384_candidates():
    rng = np.random.default_rng(1)
    scores = rng.standard_normal(100_000).astype(np.float32)
    pool = oracle.block_pool(scores, 8, 2048)
    assert pool.shape == (16_384,)
    assert np.all(np.diff(pool) > 0)
    blocks = _blocks_of(pool, 8)
    assert len(blocks) == 2048
    # whole blocks: every kept block contributes its 8 positions
    assert set(pool.tolist()) == {8 * j + i for j in blocks for i in range(8)}


@pytest.mark.parametrize("block,n_blocks", [(8, 5), (4, 3), (16, 1)])
def test_planted_blocks_are_the_pool(block, n_blocks):
    rng = np.random.default_rng(block * 10 + n_blocks)
    V = 40 * block + 3
    scores = np.full(V, -1.0, np.float32)
    chosen = sorted(rng.choice(V // block, n_blocks, replace=False).tolist())
    for j in chosen:
        # one position of the block far above every other score
        scores[j * block + int(rng.integers(block))] = 10.0 + j
    pool = oracle.block_pool(scores, block, n_blocks)
    assert pool.tolist() == [j * block + i for j in chosen for i in range(block)]


def test_equal_scores_keep_the_lowest_blocks():
    pool = oracle.block_pool(np.zeros(100, np.float32), 8, 3)
    assert pool.tolist() == list(range(24))


def test_partial_last_block_contributes_its_visible_positions():
    scores = np.zeros(8 * 10 + 3, np.float32)
    scores[81] = 5.0   # in the last block, which holds positions 80..82 only
    scores[17] = 4.0   # block 2
    pool = oracle.block_pool(scores, 8, 2)
    assert pool.tolist() == list(range(16, 24)) + [80, 81, 82]


def test_one_large_score_outranks_a_block_of_many_good_ones():
    # a block's score is its best position, not the sum of its positions
    scores = np.zeros(64, np.float32)
    scores[0:8] = 3.0        # block 0: eight good positions
    scores[40] = 3.5         # block 5: one better position
    assert oracle.block_pool(scores, 8, 1).tolist() == list(range(40, 48))


def test_empty_store_gives_an_empty_pool():
    assert oracle.block_pool(np.zeros(0, np.float32), 8, 4).shape == (0,)


@pytest.mark.parametrize("N,k", [(200, 16), (203, 64), (97, 200)])
def test_pool_covering_every_block_reduces_to_the_full_topk(N, k):
    rng = np.random.default_rng(N + k)
    q = rng.integers(-127, 128, (1, 1, 4, 32), dtype=np.int8)
    w = rng.random((1, 1, 4), dtype=np.float32)
    keys = rng.integers(-127, 128, (1, N, 32), dtype=np.int8)
    scores = oracle.index_score_row(q[0, 0], w[0, 0], keys[0])
    pool = oracle.block_pool(scores, 8, (N + 7) // 8)
    assert pool.tolist() == list(range(N))
    got = oracle.pool_topk(q[0, 0], w[0, 0], keys[0], pool, k)
    assert got.tolist() == oracle.index_topk(q, w, keys, k)[0].tolist()


@pytest.mark.parametrize("seed", range(6))
def test_pool_topk_keeps_the_best_of_the_pool_only(seed):
    rng = np.random.default_rng(100 + seed)
    N, k = 300, int(rng.integers(1, 40))
    q = rng.integers(-127, 128, (2, 16), dtype=np.int8)
    w = rng.random(2, dtype=np.float32)
    levels = int(rng.integers(1, 4))   # few key values: many equal scores
    keys = rng.integers(-levels, levels + 1, (N, 16), dtype=np.int8)
    pool = np.sort(rng.choice(N, int(rng.integers(1, 120)), replace=False)).astype(np.int32)
    got = oracle.pool_topk(q, w, keys, pool, k)
    m = min(k, pool.shape[0])
    sel, pad = got[:m], got[m:]
    assert np.all(pad == -1)
    assert np.all(np.diff(sel) > 0)
    assert set(sel.tolist()) <= set(pool.tolist())
    score = dict(zip(pool.tolist(), oracle.index_score_row(q, w, keys[pool]).tolist()))
    rest = [n for n in pool.tolist() if n not in set(sel.tolist())]
    for s in sel.tolist():
        for u in rest:
            assert score[s] > score[u] or (score[s] == score[u] and s < u)


def test_pool_topk_rejects_positions_outside_the_store():
    q = np.ones((1, 16), np.int8)
    w = np.ones(1, np.float32)
    keys = np.ones((10, 16), np.int8)
    with pytest.raises(Exception):
        oracle.pool_topk(q, w, keys, np.array([3, 10], np.int32), 2)
