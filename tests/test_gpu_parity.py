"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  FP4 codes/scales, unpacked values, indexer scores and
top-k indices must be bit-exact; attention outputs within 2e-3 absolute +
1e-2 relative of the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import compressed_sparse_attention_topk_b200 as csa2
from compressed_sparse_attention_topk_b200 import build as csa2_build
from compressed_sparse_attention_topk_b200 import workloads as wl
from tests._parity import (DECODE_KERNELS, assert_bits_equal, assert_close, dev, gpu_store,
                           group_tensors, host, oracle_store, run_group_and_compare,
                           use_decode_kernel)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    csa2_build.build()
    csa2.lib()
    assert csa2.get_device_status() == 0


# ---------------------------------------------------------------------------
# FP4 pack / unpack
# ---------------------------------------------------------------------------

def _fp4_sources(D, rows=2000, seed=1):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((rows, D)) * np.exp(rng.uniform(-30, 30, (rows, 1)))).astype(
        np.float32)
    x[:rows // 100] *= np.float32(8.0)            # outliers
    x[5] = 0.0                                     # zero row
    x[6, :16] = np.float32(1e-41)                  # subnormal group
    x[7, :16] = -np.float32(3e-39)
    mids = np.array([6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5,
                     -3.5, -5.0, -6.0], np.float32)
    for i, e in enumerate(range(-10, 10)):         # exact midpoints: ties
        x[10 + i, :16] = mids * np.float32(2.0 ** e)
        if D >= 32:
            x[10 + i, 16:32] = -mids * np.float32(2.0 ** e)
    x[40, :16] = np.float32([6, 5.9999995, 6.0000005, 0.2499999, 0.2500001] + [0] * 11)
    return x


@pytest.mark.parametrize("D", [16, 64, 128])
def test_pack_unpack_bit_exact(D):
    x = _fp4_sources(D, seed=D)
    oc, os_ = oracle.pack_fp4(x)
    gc, gs = csa2.pack_fp4(dev(x))
    assert_bits_equal(host(gc), oc, "codes")
    assert_bits_equal(host(gs), os_, "scales")
    ou = oracle.unpack_fp4(oc, os_, D)
    gu = csa2.unpack_fp4(gc, gs, D)
    assert_bits_equal(host(gu), ou, "unpacked")


# ---------------------------------------------------------------------------
# Indexer scores + top-k
# ---------------------------------------------------------------------------

def _index_case(B, T, H_I, d_I, N, seed, key_levels=None, q_zero=False):
    rng = np.random.default_rng(seed)
    q = wl.int8_uniform(rng, (B, T, H_I, d_I))
    if q_zero:
        q[:] = 0
    w = rng.random((B, T, H_I), dtype=np.float32)
    if key_levels is None:
        k = wl.int8_uniform(rng, (B, N, d_I))
    else:
        k = rng.integers(-key_levels, key_levels + 1, (B, N, d_I)).astype(np.int8)
    return q, w, k


def _check_index(q, w, k, topk, n_prior=-1, ratio=4, rows=None, check_scores=True):
    B, T = q.shape[:2]
    N = k.shape[1]
    res = csa2.index_topk(dev(q), dev(w), dev(k), topk, n_prior, ratio,
                          want_scores=check_scores)
    g_idx, g_sc = res if check_scores else (res, None)
    g_idx = host(g_idx).reshape(B * T, topk)
    if rows is not None:
        g_idx = g_idx[rows]
    o_idx, o_sc = oracle.index_topk(q, w, k, topk, n_prior, ratio, rows=rows, want_scores=True)
    if check_scores:
        g_sc = host(g_sc).reshape(B * T, N)
        if rows is not None:
            g_sc = g_sc[rows]
        assert_bits_equal(g_sc, o_sc, "scores")
        # the same call without a score output, under each decode kernel
        # (with one query per sequence the fused kernel keeps the scores on
        # chip)
        for kernel, name in DECODE_KERNELS:
            prev = use_decode_kernel(kernel)
            try:
                g2 = host(csa2.index_topk(dev(q), dev(w), dev(k), topk, n_prior, ratio))
            finally:
                use_decode_kernel(prev)
            g2 = g2.reshape(B * T, topk)
            if rows is not None:
                g2 = g2[rows]
            assert_bits_equal(g2, o_idx, f"indices without score output ({name})")
    assert_bits_equal(g_idx, o_idx, "indices")
    return g_idx


@pytest.mark.parametrize("d_I,H_I", [(16, 1), (16, 8), (32, 2), (32, 4), (32, 8), (64, 1),
                                     (64, 4), (64, 8), (128, 2), (128, 4)])
@pytest.mark.parametrize("N", [1, 777, 5000])
def test_index_topk_shapes(d_I, H_I, N):
    q, w, k = _index_case(3, 1, H_I, d_I, N, seed=d_I * 100 + H_I + N)
    _check_index(q, w, k, topk=64)


@pytest.mark.parametrize("topk", [1, 7, 64, 2048, 5000])
def test_index_topk_k_sweep_and_padding(topk):
    q, w, k = _index_case(2, 1, 4, 64, 3001, seed=topk)
    _check_index(q, w, k, topk)


def test_topk_all_equal_scores_take_lowest_indices():
    q, w, k = _index_case(2, 1, 4, 32, 9000, seed=3, q_zero=True)
    idx = _check_index(q, w, k, 300)
    assert np.array_equal(idx, np.tile(np.arange(300, dtype=np.int32), (2, 1)))


@pytest.mark.parametrize("levels", [1, 2])
def test_topk_heavy_ties_at_boundary(levels):
    q, w, k = _index_case(4, 1, 2, 16, 20000, seed=levels, key_levels=levels)
    w[:] = 1.0
    _check_index(q, w, k, 1000)


def test_topk_crowded_into_few_slices():
    # The top-k sits in the last 3,000 entries (their head-0 dot product is
    # |q_0|^2), i.e. in the last one or two of the row's slices: the per-row
    # cluster kernel's last CTAs select nearly every entry while the others
    # select none, so the output offsets of the other slices are all zero.
    q, w, k = _index_case(2, 1, 4, 64, 60000, seed=11)
    for b in range(2):
        k[b, -3000:, :] = q[b, 0, 0, :]
    _check_index(q, w, k, 2048)


@pytest.mark.parametrize("N", [4096, 70000, 262144])
def test_topk_one_row_many_scan_slices(N):
    # one row scanned by many CTAs (about two per SM), whose digit-1
    # histograms the selection sums; at N = 262,144 each of the row
    # kernel's 16 CTAs selects from 16,384 staged scores
    q, w, k = _index_case(1, 1, 4, 64, N, seed=N)
    _check_index(q, w, k, 2048)


def test_topk_all_equal_scores_beyond_on_chip_list():
    # every entry is a candidate: the list of a row exceeds what a CTA keeps
    # in shared memory, so the exact selection reads it from L2
    q, w, k = _index_case(2, 1, 4, 64, 60000, seed=4, q_zero=True)
    idx = _check_index(q, w, k, 300)
    assert np.array_equal(idx, np.tile(np.arange(300, dtype=np.int32), (2, 1)))


def test_topk_heavy_ties_fused_shapes():
    q, w, k = _index_case(4, 1, 4, 32, 20000, seed=8, key_levels=1)
    w[:] = 1.0
    _check_index(q, w, k, 1000)


def test_topk_more_rows_than_one_launch():
    # 40 sequences: more rows than one fused launch takes (about a quarter of
    # the SMs), so the rows go in several launches
    q, w, k = _index_case(40, 1, 4, 64, 3000, seed=40)
    _check_index(q, w, k, 256)


def test_topk_empty_store():
    q, w, k = _index_case(2, 1, 4, 64, 0, seed=1)
    idx = csa2.index_topk(dev(q), dev(w), torch.empty((2, 0, 64), dtype=torch.int8,
                                                       device="cuda"), 5)
    assert np.all(host(idx) == -1)


def test_prefill_visibility():
    B, T, H_I, d_I, n_prior, ratio = 2, 67, 4, 64, 301, 4
    N = n_prior + T // ratio
    q, w, k = _index_case(B, T, H_I, d_I, N, seed=9)
    _check_index(q, w, k, 320, n_prior=n_prior, ratio=ratio)


# ---------------------------------------------------------------------------
# Chunked prefill through the tensor-core indexer: T >= 64 queries per
# sequence and no score output select this path (approximate two-level int8
# products on tcgen05, exact rescoring of the candidates, exact fallback).
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d_I,H_I", [(32, 4), (32, 8), (64, 1), (64, 4), (64, 8), (128, 2),
                                     (128, 4)])
def test_prefill_tensor_core_shapes(d_I, H_I):
    B, T, n_prior, ratio = 2, 130, 12000, 4
    N = n_prior + T // ratio
    q, w, k = _index_case(B, T, H_I, d_I, N, seed=7 * d_I + H_I)
    _check_index(q, w, k, 512, n_prior=n_prior, ratio=ratio, check_scores=False)


@pytest.mark.parametrize("topk", [64, 2048, 4096])
def test_prefill_tensor_core_all_visible(topk):
    q, w, k = _index_case(1, 128, 4, 64, 30000, seed=topk)
    _check_index(q, w, k, topk, check_scores=False)


@pytest.mark.parametrize("N,topk", [(3000, 64), (3000, 2999), (3000, 4000), (8192, 2048)])
def test_prefill_tensor_core_every_entry_a_candidate(N, topk):
    q, w, k = _index_case(1, 129, 4, 64, N, seed=N + topk)
    _check_index(q, w, k, topk, check_scores=False)


def test_prefill_tensor_core_padding_and_empty_rows():
    B, T, n_prior, ratio = 2, 300, 0, 4        # rows t < 3 see nothing; V_t = (t+1)//4
    N = T // ratio
    q, w, k = _index_case(B, T, 4, 64, N, seed=11)
    idx = _check_index(q, w, k, 100, n_prior=n_prior, ratio=ratio, check_scores=False)
    assert np.all(idx[:3] == -1)


def test_prefill_tensor_core_heavy_ties():
    q, w, k = _index_case(1, 64, 4, 64, 20000, seed=5, key_levels=1)
    w[:] = 1.0                                 # integer scores in [-256, 256]: many ties
    _check_index(q, w, k, 1000, check_scores=False)


def test_prefill_tensor_core_all_equal_scores():
    q, w, k = _index_case(1, 64, 4, 64, 20000, seed=6, q_zero=True)
    idx = _check_index(q, w, k, 700, check_scores=False)
    assert np.array_equal(idx, np.tile(np.arange(700, dtype=np.int32), (64, 1)))


def _aligned_keys(q, w, n_keys):
    """Keys that maximise the score of every row (all rows share q and w)."""
    comb = (w[0, 0][:, None].astype(np.float64) * q[0, 0].astype(np.float64)).sum(axis=0)
    return np.where(comb >= 0, 127, -127).astype(np.int8)[None, :].repeat(n_keys, axis=0)


@pytest.mark.parametrize("where", ["sampled", "between_samples"])
def test_prefill_tensor_core_misleading_sample(where):
    """Top entries placed only on, or only between, the strided sample
    positions (every 3rd entry for N = 20000): the sampled threshold then
    misjudges the row (too few candidates, or more than the selection
    capacity), and the exact fallback must still return the exact top-k."""
    T, N, topk = 64, 20000, 2048
    q, w, k = _index_case(1, T, 4, 64, N, seed=17)
    q[:] = q[:, :1]
    w[:] = w[:, :1]
    n = np.arange(N)
    pos = n[(n % 3 == 0)][:1400] if where == "sampled" else n[(n % 3 != 0)][:9000]
    k[0, pos] = _aligned_keys(q, w, len(pos))
    _check_index(q, w, k, topk, check_scores=False)


# ---------------------------------------------------------------------------
# Several query rows per sequence (2 <= T <= 8, d_I <= 64): one shared key
# scan scores every row of the sequence.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T", [2, 3, 5, 8])
@pytest.mark.parametrize("d_I,H_I", [(32, 4), (64, 4), (64, 1), (16, 8)])
def test_multi_query_shared_scan(T, d_I, H_I):
    q, w, k = _index_case(3, T, H_I, d_I, 9001, seed=100 * T + d_I + H_I)
    _check_index(q, w, k, 300)                     # scores bit-exact too
    _check_index(q, w, k, 300, check_scores=False)


@pytest.mark.parametrize("T,d_I,N,topk", [(4, 32, 1, 1), (6, 64, 15, 20), (7, 32, 17, 16),
                                           (4, 64, 300, 64), (8, 32, 4097, 512),
                                           (3, 64, 131, 131), (2, 32, 257, 300)])
def test_multi_query_tensor_core_scan_edges(T, d_I, N, topk):
    """The tensor-core multi-token scan (4 index heads): fewer keys than one
    16-key block, a ragged last block and tile, k >= N, every token count
    of the three n-tile widths; scores and indices bit-exact."""
    q, w, k = _index_case(2, T, 4, d_I, N, seed=T * 1000 + N)
    _check_index(q, w, k, topk)


def test_multi_query_tensor_core_scan_extreme_values():
    """Index queries and keys at the int8 extremes (dots up to 64 x 127 x 128
    in one int32 accumulator) and negative weights."""
    q, w, k = _index_case(2, 5, 4, 64, 5000, seed=5)
    q[0] = -128
    k[0, ::2] = -128
    k[0, 1::2] = 127
    w[1] = -np.abs(w[1])
    _check_index(q, w, k, 700)


def test_multi_query_shared_scan_visibility():
    B, T, n_prior, ratio = 2, 7, 5000, 2         # each row sees a different prefix
    N = n_prior + T // ratio
    q, w, k = _index_case(B, T, 4, 64, N, seed=77)
    _check_index(q, w, k, 1024, n_prior=n_prior, ratio=ratio)


def test_multi_token_decode_workload_full_size():
    """5 query tokens per sequence at the 1M-context shape (B=4, N=262,144,
    Full + Reindex): shared scans, per-row top-k, attention; every row."""
    run_group_and_compare(wl.MTP5)


@pytest.mark.parametrize("wl_name", ["tiny_decode_n1024", "decode_b32_n131072"])
def test_index_topk_workload(wl_name):
    w0 = wl.ALL[wl_name]
    lay = wl.layer_inputs(w0, 0)
    _check_index(lay["q_idx"], lay["w"], lay["k_idx"], w0.topk)


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def _attn_inputs(B, T, H, D, N, topk, W, seed, idx_mode="random"):
    rng = np.random.default_rng(seed)
    entries = rng.standard_normal((B, N, D)).astype(np.float32)
    q = wl.bf16_bits(rng.standard_normal((B, T, H, D)).astype(np.float32))
    wk = wl.bf16_bits(rng.standard_normal((B, W - 1 + T, D)).astype(np.float32)) if W else None
    wv = wl.bf16_bits(rng.standard_normal((B, W - 1 + T, D)).astype(np.float32)) if W else None
    if idx_mode == "random":
        idx = np.stack([np.sort(rng.choice(N, min(topk, N), replace=False))
                        for _ in range(B * T)]).astype(np.int32)
        if topk > N:
            idx = np.concatenate([idx, np.full((B * T, topk - N), -1, np.int32)], axis=1)
    else:
        idx = np.full((B * T, topk), -1, np.int32)
    return entries, q, wk, wv, idx.reshape(B, T, topk)


def _check_attn(entries, q, wk, wv, idx, decode):
    B, T, H, D = q.shape
    oc, os_ = oracle_store(entries)
    gc, gs = gpu_store(entries)
    ref_out, ref_lse = oracle.sparse_attn(q, oc, os_, idx, wk, wv)
    if decode:
        out, lse = csa2.sparse_attn_decode(dev(q[:, 0]), gc, gs, dev(idx[:, 0]),
                                           None if wk is None else dev(wk),
                                           None if wv is None else dev(wv))
    else:
        out, lse = csa2.sparse_attn_prefill(dev(q), gc, gs, dev(idx),
                                            None if wk is None else dev(wk),
                                            None if wv is None else dev(wv))
    assert_close(host(out).reshape(B * T, H, D), ref_out, "out")
    assert_close(host(lse).reshape(B * T, H), ref_lse, "lse")


@pytest.mark.parametrize("D,H,topk,W", [(64, 8, 64, 128), (128, 16, 2048, 128), (128, 16, 100, 0),
                                        (128, 20, 130, 70), (64, 3, 0, 5), (128, 16, 37, 1)])
def test_attention_decode(D, H, topk, W):
    entries, q, wk, wv, idx = _attn_inputs(3, 1, H, D, 4000, topk, W, seed=D + H + topk + W)
    _check_attn(entries, q, wk, wv, idx, decode=True)


def test_attention_padding_and_nothing_to_attend():
    entries, q, wk, wv, idx = _attn_inputs(2, 1, 16, 128, 500, 64, 0, seed=5)
    idx[0, 0, ::3] = -1
    idx[1, 0, :] = -1          # sequence 1: nothing to attend to
    _check_attn(entries, q, wk, wv, idx, decode=True)


def test_attention_bad_index_recorded_and_skipped():
    entries, q, wk, wv, idx = _attn_inputs(2, 1, 16, 128, 300, 32, 16, seed=7)
    bad = idx.copy()
    bad[0, 0, 4] = 300 + 5
    skipped = bad.copy()
    skipped[0, 0, 4] = -1
    oc, os_ = oracle_store(entries)
    gc, gs = gpu_store(entries)
    ref_out, _ = oracle.sparse_attn(q, oc, os_, skipped, wk, wv)
    out, _ = csa2.sparse_attn_decode(dev(q[:, 0]), gc, gs, dev(bad[:, 0]), dev(wk), dev(wv))
    assert_close(host(out), ref_out, "out")
    assert csa2.get_device_status() & 1
    assert csa2.get_device_status() == 0   # reading clears it


@pytest.mark.parametrize("T,W", [(37, 16), (5, 128), (64, 1)])
def test_attention_prefill(T, W):
    entries, q, wk, wv, idx = _attn_inputs(2, T, 16, 128, 700, 96, W, seed=T + W)
    _check_attn(entries, q, wk, wv, idx, decode=False)


@pytest.mark.parametrize("D,H,topk,W", [(128, 16, 2048, 128), (64, 8, 100, 5), (128, 20, 64, 0),
                                        (128, 16, 37, 17)])
def test_attention_many_rows(D, H, topk, W):
    """320 query rows (more than two per SM) take the one-CTA-per-row kernel:
    ragged key chunks, a second head pass, padding inside a row and a row
    with no selected entry."""
    entries, q, wk, wv, idx = _attn_inputs(2, 160, H, D, 3000, topk, W, seed=D * 7 + H + topk + W)
    idx[0, 3, ::5] = -1
    idx[1, 7, :] = -1
    _check_attn(entries, q, wk, wv, idx, decode=False)


def test_attention_many_rows_bad_index_recorded_and_skipped():
    entries, q, wk, wv, idx = _attn_inputs(2, 160, 16, 128, 900, 64, 16, seed=9)
    bad = idx.copy()
    bad[1, 100, 7] = 900 + 3
    skipped = bad.copy()
    skipped[1, 100, 7] = -1
    oc, os_ = oracle_store(entries)
    gc, gs = gpu_store(entries)
    ref_out, ref_lse = oracle.sparse_attn(q, oc, os_, skipped, wk, wv)
    out, lse = csa2.sparse_attn_prefill(dev(q), gc, gs, dev(bad), dev(wk), dev(wv))
    assert_close(host(out).reshape(ref_out.shape), ref_out, "out")
    assert_close(host(lse).reshape(ref_lse.shape), ref_lse, "lse")
    assert csa2.get_device_status() & 1
    assert csa2.get_device_status() == 0


# ---------------------------------------------------------------------------
# Whole workloads through the C ABI
# ---------------------------------------------------------------------------

def _store_for(lay):
    return oracle_store(lay["entries"]), gpu_store(lay["entries"])


def test_tiny_workload_end_to_end():
    w0 = wl.TINY
    lay = wl.layer_inputs(w0, 0)
    (oc, os_), (gc, gs) = _store_for(lay)
    assert_bits_equal(host(gc), oc, "codes")
    g_idx = csa2.index_topk(dev(lay["q_idx"]), dev(lay["w"]), dev(lay["k_idx"]), w0.topk)
    o_idx = oracle.index_topk(lay["q_idx"], lay["w"], lay["k_idx"], w0.topk)
    assert_bits_equal(host(g_idx).reshape(1, -1), o_idx, "idx")
    out, lse = csa2.sparse_attn_decode(dev(lay["q"][:, 0]), gc, gs, g_idx[:, 0],
                                       dev(lay["win_k"]), dev(lay["win_v"]))
    ref_out, ref_lse = oracle.sparse_attn(lay["q"], oc, os_, o_idx.reshape(1, 1, -1),
                                          lay["win_k"], lay["win_v"])
    assert_close(host(out), ref_out, "out")
    assert_close(host(lse), ref_lse, "lse")


@pytest.mark.parametrize("B,N,topk,W,H,D,H_I,d_I", [
    (2, 5000, 2048, 128, 16, 128, 4, 64),
    (3, 1000, 2048, 128, 16, 128, 4, 64),     # fewer entries than k: padding
    (1, 3000, 100, 0, 16, 128, 4, 64),        # no window
    (2, 7777, 512, 1, 5, 64, 8, 32),          # one window row, 5 heads
    (5, 20000, 4096, 70, 16, 128, 8, 64),
    (2, 100, 7, 128, 16, 128, 4, 32),
])
def test_decode_layer_shapes(B, N, topk, W, H, D, H_I, d_I, decode_kernel):
    """Full + Reindex decode layers through the layer call (fused decode
    kernel): selection bit-exact, attention within tolerance."""
    w0 = wl.with_sizes(wl.LONG, name=f"decode_{B}_{N}_{topk}", B=B, N=N, topk=topk, W=W, H=H,
                       D=D, H_I=H_I, d_I=d_I, seed=B * 1000 + N)
    run_group_and_compare(w0)


def test_decode_layer_heavy_ties(decode_kernel):
    """Layers whose index scores take a few integer values (keys in {-1, 0, 1},
    unit weights): the keys equal to the threshold outnumber the slots left,
    so only the lowest-indexed of them are taken and each CTA's share depends
    on the other ranks' counts before it attends."""
    w0 = wl.with_sizes(wl.LONG, name="decode_ties", B=3, N=20000, seed=77)

    def mutate(layers):
        rng = np.random.default_rng(9)
        layers[0]["k_idx"] = rng.integers(-1, 2, layers[0]["k_idx"].shape).astype(np.int8)
        for lay in layers:
            lay["q_idx"] = rng.integers(0, 2, lay["q_idx"].shape).astype(np.int8)
            lay["w"][:] = 1.0

    run_group_and_compare(w0, mutate=mutate)


def test_decode_layer_selection_crowded_into_one_slice(decode_kernel):
    """A top-k of 6,000 whose entries all lie in the first 6,000 positions of
    100,000: one CTA selects more than its on-chip list holds and attends over
    the rest from the written output row."""
    w0 = wl.with_sizes(wl.LONG, name="decode_crowded", B=1, N=100000, topk=6000, seed=78)

    def mutate(layers):
        k = layers[0]["k_idx"]
        k[:, :6000] = np.abs(k[:, :6000]) // 2 + 60          # high keys first
        k[:, 6000:] = k[:, 6000:] // 4                        # the rest small
        for lay in layers:
            lay["q_idx"] = np.abs(lay["q_idx"]) // 2 + 1      # positive queries

    run_group_and_compare(w0, mutate=mutate)


def test_decode_layer_cuda_graph_replay(decode_kernel):
    """The layer call captured into a CUDA graph (as the benchmark runs it)
    and replayed gives the eager results, bit for bit, on every replay."""
    w0 = wl.with_sizes(wl.LONG, name="graph_replay", B=4, N=20000, seed=77)
    layers = wl.all_layer_inputs(w0)
    tens = group_tensors(w0, layers)
    dims = csa2.make_dims(w0.B, w0.T, w0.H, w0.D, w0.N, w0.H_I, w0.d_I, w0.topk, w0.W)
    group = csa2.LayerGroup(list(w0.modes), tens, dims)
    group.run()
    torch.cuda.synchronize()
    eager = [(t["idx"].clone(), t["out"].clone(), t["lse"].clone()) for t in tens]
    for t in tens:
        t["idx"].fill_(-5)
        t["out"].fill_(7.0)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        group.run()
    for _ in range(2):
        for t in tens:
            t["idx"].fill_(-5)
            t["out"].fill_(7.0)
        g.replay()
        torch.cuda.synchronize()
        for (i0, o0, l0), t in zip(eager, tens):
            assert torch.equal(t["idx"], i0)
            assert torch.equal(t["out"], o0)
            assert torch.equal(t["lse"], l0)
    del g
    assert csa2.get_device_status() == 0


def test_group_workload_16_layers():
    """4 groups of (Full, Reindex, Reuse, Reuse), B=8, N=4096, k=512."""
    w0 = wl.GROUP
    tens = run_group_and_compare(w0)
    assert csa2.group_cache_bytes(list(w0.modes), w0.N, 128, 8) == 2 * 1024 * 1024


def test_long_decode_workload_full_size(decode_kernel):
    """The 1M-token decode workload at full size (B=4, N=262144, Full +
    Reindex), in the launch configuration the benchmark times."""
    run_group_and_compare(wl.LONG)


def test_decode_workload_full_size():
    """B=32, N=131072, d_I=32, k=2048, with salient outlier entries."""
    run_group_and_compare(wl.DECODE)


def test_prefill_workload_sampled_rows():
    """Chunked prefill at full size (T=4096 after 262,144 prior entries):
    every row computed on the GPU, a spread sample checked against the
    oracle (first 64, last 64, 128 seeded): the tensor-core filter certifies
    each row on its own, so the sample spans the chunk."""
    w0 = wl.PREFILL
    rng = np.random.default_rng(1234)
    rows = np.unique(np.concatenate([np.arange(64), np.arange(w0.T - 64, w0.T),
                                     rng.choice(w0.T, 128, replace=False)])).astype(np.int64)
    run_group_and_compare(w0, rows=rows)
