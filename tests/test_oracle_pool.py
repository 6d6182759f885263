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


# ---------------------------------------------------------------------------
# The mode-table walk with a Reindex layer that searches its Full source's
# pool (oracle.REINDEX_POOL).
# ---------------------------------------------------------------------------

def _pool_group(B=2, N=3000, topk=64, seed=3):
    from compressed_sparse_attention_topk_b200 import workloads as wl
    w0 = wl.with_sizes(wl.LONG, name="pool_walk", B=B, N=N, topk=topk, seed=seed)
    layers = wl.all_layer_inputs(w0)
    c, s_ = oracle.pack_fp4(layers[0]["entries"].reshape(B * N, -1))
    layers[0]["codes"], layers[0]["scales"] = c.reshape(B, N, -1), s_.reshape(B, N, -1)
    return w0, layers


def test_pool_layer_with_a_pool_covering_the_store_equals_reindex():
    w0, layers = _pool_group()
    plain = oracle.layer_group([(0, 0, 0), (1, 0, 1)], layers, w0.topk)
    pooled = oracle.layer_group([(0, 0, 0), (oracle.REINDEX_POOL, 0, 1)], layers, w0.topk,
                                pool=(8, (w0.N + 7) // 8))
    assert np.array_equal(pooled[1]["idx"], plain[1]["idx"])
    assert np.array_equal(pooled[1]["out"], plain[1]["out"])
    assert np.array_equal(pooled[0]["idx"], plain[0]["idx"])


def test_pool_layer_selects_within_the_full_layers_best_blocks():
    w0, layers = _pool_group(N=5000, topk=100, seed=4)
    block, n_blocks = 8, 40
    res = oracle.layer_group([(0, 0, 0), (oracle.REINDEX_POOL, 0, 1), (2, 0, 1)], layers + [
        dict(layers[1])], w0.topk, pool=(block, n_blocks))
    for b in range(w0.B):
        full = oracle.index_score_row(layers[0]["q_idx"][b, 0], layers[0]["w"][b, 0],
                                      layers[0]["k_idx"][b])
        # the kept blocks: the n_blocks largest block maxima (no ties here)
        bmax = full.reshape(-1, block).max(axis=1)
        kept = set(np.argsort(-bmax, kind="stable")[:n_blocks].tolist())
        sel = res[1]["idx"][b, 0]
        assert all(int(n) // block in kept for n in sel if n >= 0)
        # within the pool the selection is the exact top-k of the layer's own scores
        mine = oracle.index_score_row(layers[1]["q_idx"][b, 0], layers[1]["w"][b, 0],
                                      layers[0]["k_idx"][b])
        pool = [n for n in range(w0.N) if n // block in kept]
        best = sorted(pool, key=lambda n: (-float(mine[n]), n))[:w0.topk]
        assert sel.tolist() == sorted(best)
    # a Reuse layer after it copies its selection
    assert np.array_equal(res[2]["idx"], res[1]["idx"])
