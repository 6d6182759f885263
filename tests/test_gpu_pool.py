"""GPU parity of the hierarchical indexer ("Inference-Efficient LLMs",
section 5): the candidate pool of a Full layer (csa2_index_pool) and the
top-k of a Reindex layer within a pool (csa2_pool_topk), bit-exact against
the oracle's block_pool / pool_topk on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
import compressed_sparse_attention_topk_b200 as csa2
from compressed_sparse_attention_topk_b200 import build as csa2_build
from compressed_sparse_attention_topk_b200 import workloads as wl
from tests._parity import assert_bits_equal, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    csa2_build.build()
    csa2.lib()
    assert csa2.get_device_status() == 0


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert csa2.get_device_status() == 0


def _case(B, H_I, d_I, N, seed, levels=None):
    rng = np.random.default_rng(seed)
    q = wl.int8_uniform(rng, (B, H_I, d_I))
    w = rng.random((B, H_I), dtype=np.float32)
    if levels is None:
        k = wl.int8_uniform(rng, (B, N, d_I))
    else:
        k = rng.integers(-levels, levels + 1, (B, N, d_I)).astype(np.int8)
    return q, w, k


def _oracle_pool(q, w, k, block, n_blocks):
    rows = []
    for b in range(q.shape[0]):
        scores = oracle.index_score_row(q[b], w[b], k[b])
        p = oracle.block_pool(scores, block, n_blocks)
        rows.append(np.concatenate([p, np.full(n_blocks * block - p.shape[0], -1, np.int32)]))
    return np.stack(rows)


def _oracle_pool_topk(q, w, k, pool, topk):
    rows = []
    for b in range(q.shape[0]):
        valid = pool[b][(pool[b] >= 0) & (pool[b] < k.shape[1])]
        rows.append(oracle.pool_topk(q[b], w[b], k[b], valid, topk))
    return np.stack(rows)


@pytest.mark.parametrize("N", [1, 7, 100, 5000, 70001])
@pytest.mark.parametrize("block,n_blocks", [(8, 2048), (8, 5), (1, 300), (16, 40), (64, 3)])
def test_index_pool_matches_oracle(N, block, n_blocks):
    q, w, k = _case(3, 4, 32, N, seed=N + 7 * block + n_blocks)
    got = host(csa2.index_pool(dev(q), dev(w), dev(k), block, n_blocks))
    assert_bits_equal(got, _oracle_pool(q, w, k, block, n_blocks), "pool")


@pytest.mark.parametrize("d_I,H_I", [(16, 8), (64, 1), (64, 4), (128, 4)])
def test_index_pool_index_shapes(d_I, H_I):
    q, w, k = _case(2, H_I, d_I, 9000, seed=d_I + H_I)
    got = host(csa2.index_pool(dev(q), dev(w), dev(k), 8, 64))
    assert_bits_equal(got, _oracle_pool(q, w, k, 8, 64), "pool")


def test_index_pool_ties_take_the_lowest_blocks():
    q, w, k = _case(2, 2, 16, 4000, seed=3, levels=1)
    q[:] = 0   # every score 0: every block ties
    got = host(csa2.index_pool(dev(q), dev(w), dev(k), 8, 10))
    assert np.array_equal(got, np.tile(np.arange(80, dtype=np.int32), (2, 1)))
    assert_bits_equal(got, _oracle_pool(q, w, k, 8, 10), "pool")


def test_index_pool_empty_store():
    q, w, _ = _case(2, 4, 64, 0, seed=1)
    import torch
    got = host(csa2.index_pool(dev(q), dev(w), torch.empty((2, 0, 64), dtype=torch.int8,
                                                           device="cuda"), 8, 4))
    assert np.all(got == -1)


def test_index_pool_of_the_pages_example_at_the_decode_shape():
    # 2,048 blocks of eight positions (16,384 candidates) at N = 262,144
    q, w, k = _case(4, 4, 64, 262144, seed=41)
    got = host(csa2.index_pool(dev(q), dev(w), dev(k), 8, 2048))
    assert np.all(got >= 0) and got.shape == (4, 16384)
    assert_bits_equal(got, _oracle_pool(q, w, k, 8, 2048), "pool")


@pytest.mark.parametrize("N,block,n_blocks,topk", [(5000, 8, 64, 100), (70001, 8, 2048, 2048),
                                                   (3000, 16, 10, 500), (900, 1, 50, 64)])
def test_pool_topk_of_a_reindex_query_in_a_full_layers_pool(N, block, n_blocks, topk):
    q_full, w_full, k = _case(3, 4, 32, N, seed=N + topk)
    q_re, w_re, _ = _case(3, 4, 32, 0, seed=N + topk + 1)
    pool = csa2.index_pool(dev(q_full), dev(w_full), dev(k), block, n_blocks)
    got = host(csa2.pool_topk(dev(q_re), dev(w_re), dev(k), pool, topk))
    assert_bits_equal(got, _oracle_pool_topk(q_re, w_re, k, host(pool), topk), "indices")


def test_pool_topk_heavy_ties_and_padding():
    q, w, k = _case(2, 2, 16, 3000, seed=9, levels=1)
    rng = np.random.default_rng(10)
    pool = np.full((2, 600), -1, np.int32)
    for b in range(2):
        n = 400 + 50 * b
        pool[b, :n] = np.sort(rng.choice(3000, n, replace=False))
    for topk in (1, 37, 450, 700):
        got = host(csa2.pool_topk(dev(q), dev(w), dev(k), dev(pool), topk))
        assert_bits_equal(got, _oracle_pool_topk(q, w, k, pool, topk), f"indices k={topk}")


def test_pool_topk_over_every_block_equals_the_full_topk():
    q, w, k = _case(2, 4, 64, 4000, seed=12)
    pool = csa2.index_pool(dev(q), dev(w), dev(k), 8, 500)   # 500 blocks cover all 4,000
    got = host(csa2.pool_topk(dev(q), dev(w), dev(k), pool, 256))
    full = host(csa2.index_topk(dev(q[:, None]), dev(w[:, None]), dev(k), 256)).reshape(2, 256)
    assert np.array_equal(got, full)


def test_pool_topk_entry_beyond_the_store_is_recorded_and_skipped():
    q, w, k = _case(1, 4, 32, 1000, seed=13)
    pool = np.concatenate([np.arange(0, 1000, 3, dtype=np.int32),
                           np.array([1000, 5000], np.int32)])[None]
    got = host(csa2.pool_topk(dev(q), dev(w), dev(k), dev(pool), 400))
    assert csa2.get_device_status() & 1   # reading clears it
    assert_bits_equal(got, _oracle_pool_topk(q, w, k, pool, 400), "indices")


# ---------------------------------------------------------------------------
# Pool layers in the layer call: a Full layer keeps its candidate pool from
# the same scan as its own selection, a CSA2_REINDEX_POOL layer selects
# within it, a Reuse layer takes that selection.
# ---------------------------------------------------------------------------

def _pool_layers(w0, layers, block, n_blocks):
    from tests._parity import gpu_store
    tens = []
    P = block * n_blocks
    for lay in layers:
        d = {k: dev(v) for k, v in lay.items() if k != "entries"}
        d["q"] = d["q"][:, 0].contiguous()
        if "entries" in lay:
            d["codes"], d["scales"] = gpu_store(lay["entries"])
            d["pool"] = torch.full((w0.B, P), -9, dtype=torch.int32, device="cuda")
        d["idx"] = torch.empty((w0.B, 1, w0.topk), dtype=torch.int32, device="cuda")
        d["out"] = torch.empty((w0.B, w0.H, w0.D), dtype=torch.float32, device="cuda")
        d["lse"] = torch.empty((w0.B, w0.H), dtype=torch.float32, device="cuda")
        tens.append(d)
    return tens


@pytest.mark.parametrize("B,N,block,n_blocks,topk,d_I", [(4, 262144, 8, 2048, 2048, 64),
                                                         (3, 20001, 8, 300, 512, 64),
                                                         (2, 5000, 16, 40, 100, 64),
                                                         (2, 3000, 8, 400, 64, 64),
                                                         (3, 9999, 4, 500, 256, 64),
                                                         (2, 4097, 2, 1000, 128, 32),
                                                         (2, 3001, 1, 1500, 64, 32),
                                                         (2, 5003, 32, 50, 128, 64)])
def test_pool_layers_in_the_layer_call(B, N, block, n_blocks, topk, d_I, decode_kernel):
    """Blocks of 2^i <= 16 positions take their maxima in the Full layer's
    scan itself; other block sizes in a pass over the scores after it."""
    from tests._parity import assert_close, oracle_store
    w0 = wl.with_sizes(wl.LONG, name=f"pool_layers_{N}", B=B, N=N, topk=topk, d_I=d_I,
                       seed=N + B, modes=((0, 0, 0), (csa2.REINDEX_POOL, 0, 1), (2, 0, 1)))
    layers = wl.all_layer_inputs(w0)
    tens = _pool_layers(w0, layers, block, n_blocks)
    dims = csa2.make_dims(B, 1, w0.H, w0.D, N, w0.H_I, w0.d_I, topk, w0.W, pool_block=block,
                          pool_blocks=n_blocks)
    csa2.layer_group_run(list(w0.modes), tens, dims)
    layers[0]["codes"], layers[0]["scales"] = oracle_store(layers[0]["entries"])
    ref = oracle.layer_group(list(w0.modes), layers, topk, pool=(block, n_blocks))
    # the Full layer's pool, from the same scan as its own selection
    for b in range(B):
        full = oracle.index_score_row(layers[0]["q_idx"][b, 0], layers[0]["w"][b, 0],
                                      layers[0]["k_idx"][b])
        want = oracle.block_pool(full, block, n_blocks)
        got = host(tens[0]["pool"])[b]
        assert_bits_equal(got[: len(want)], want, "pool")
        assert np.all(got[len(want):] == -1)
    for l in range(3):
        src = w0.modes[l][2]
        assert_bits_equal(host(tens[src]["idx"]).reshape(B, -1), ref[l]["idx"].reshape(B, -1),
                          f"layer {l} idx")
        assert_close(host(tens[l]["out"]).reshape(ref[l]["out"].shape), ref[l]["out"],
                     f"layer {l} out")
        assert_close(host(tens[l]["lse"]).reshape(ref[l]["lse"].shape), ref[l]["lse"],
                     f"layer {l} lse")
    assert csa2.get_device_status() == 0
