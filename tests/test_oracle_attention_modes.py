"""Pins of the oracle's sparse attention and of the cross-layer mode walk.

Attention over the selected compressed entries plus a 128-token local
window: "Why Is DeepSeek V4.1 Flash So Fast?", section 3; local keys and
values are per layer: "Inference-Efficient LLMs", section 3.  Modes and
cache accounting: "DeepSeek-V4.1-Flash" (visual explainer), sections
"Sharing the cache across layers" and "Several mechanisms in one release".

Pins: dense attention from a library routine (torch's scaled dot-product
attention in float64) when the selection covers every entry, closed forms
(one key, two keys, nothing to attend to), invariances, and the page's
worked 8 MiB -> 2 MiB cache example stored under tests/golden.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_attention_topk_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _store(rng, B, N, D):
    x = rng.standard_normal((B, N, D)).astype(np.float32)
    codes, scales = oracle.pack_fp4(x.reshape(B * N, D))
    return codes.reshape(B, N, D // 2), scales.reshape(B, N, D // 16)


def _bf16(rng, shape):
    return wl.bf16_bits(rng.standard_normal(shape).astype(np.float32))


@pytest.mark.parametrize("W", [0, 5])
def test_full_selection_equals_dense_attention(W):
    rng = np.random.default_rng(W + 1)
    B, T, H, D, N = 2, 3, 4, 32, 40
    codes, scales = _store(rng, B, N, D)
    q = _bf16(rng, (B, T, H, D))
    win_k = _bf16(rng, (B, W - 1 + T, D)) if W else None
    win_v = _bf16(rng, (B, W - 1 + T, D)) if W else None
    idx = np.tile(np.arange(N, dtype=np.int32), (B, T, 1))
    out, lse = oracle.sparse_attn(q, codes, scales, idx, win_k, win_v)
    deq = oracle.unpack_fp4(codes.reshape(-1, D // 2), scales.reshape(-1, D // 16), D)
    deq = torch.from_numpy(deq.reshape(B, N, D).astype(np.float64))
    qf = torch.from_numpy(wl.bf16_to_f32(q).astype(np.float64))
    sm = float(np.float32(1.0 / math.sqrt(D)))   # the scale travels as an fp32 argument
    for b in range(B):
        for t in range(T):
            K, V = deq[b], deq[b]
            if W:
                wk = torch.from_numpy(wl.bf16_to_f32(win_k[b, t:t + W]).astype(np.float64))
                wv = torch.from_numpy(wl.bf16_to_f32(win_v[b, t:t + W]).astype(np.float64))
                K, V = torch.cat([K, wk]), torch.cat([V, wv])
            ref = torch.nn.functional.scaled_dot_product_attention(
                qf[b, t][None], K[None], V[None], scale=sm)[0]
            r = b * T + t
            assert np.allclose(out[r], ref.numpy(), rtol=1e-12, atol=1e-12)
            ref_lse = torch.logsumexp(sm * qf[b, t] @ K.T, dim=-1)
            assert np.allclose(lse[r], ref_lse.numpy(), rtol=1e-12, atol=1e-12)


def test_single_entry_no_window_is_that_entry():
    rng = np.random.default_rng(2)
    B, T, H, D, N = 1, 1, 3, 64, 9
    codes, scales = _store(rng, B, N, D)
    q = _bf16(rng, (B, T, H, D))
    idx = np.full((B, T, 4), -1, np.int32)
    idx[0, 0, 2] = 5
    out, lse = oracle.sparse_attn(q, codes, scales, idx, None, None)
    e = oracle.unpack_fp4(codes[0, 5:6], scales[0, 5:6], D)[0].astype(np.float64)
    for h in range(H):
        assert np.array_equal(out[0, h], e)
        z = float(np.dot(wl.bf16_to_f32(q[0, 0, h]).astype(np.float64), e)) * float(
            np.float32(1.0 / math.sqrt(D)))
        assert lse[0, h] == pytest.approx(z, rel=1e-14, abs=1e-14)


def test_two_keys_closed_form():
    rng = np.random.default_rng(4)
    D = 16
    codes, scales = _store(rng, 1, 2, D)
    q = _bf16(rng, (1, 1, 1, D))
    idx = np.array([[[0, 1]]], np.int32)
    out, _ = oracle.sparse_attn(q, codes, scales, idx, None, None, sm_scale=0.375)
    e = oracle.unpack_fp4(codes[0], scales[0], D).astype(np.float64)
    qq = wl.bf16_to_f32(q[0, 0, 0]).astype(np.float64)
    z0, z1 = 0.375 * qq @ e[0], 0.375 * qq @ e[1]
    p0 = 1.0 / (1.0 + math.exp(z1 - z0))   # logistic of the logit gap
    assert np.allclose(out[0, 0], p0 * e[0] + (1 - p0) * e[1], rtol=1e-13, atol=1e-13)


def test_permutation_and_padding_invariance():
    rng = np.random.default_rng(6)
    B, T, H, D, N, k, W = 2, 1, 4, 64, 100, 12, 7
    codes, scales = _store(rng, B, N, D)
    q = _bf16(rng, (B, T, H, D))
    win_k, win_v = _bf16(rng, (B, W, D)), _bf16(rng, (B, W, D))
    idx = np.stack([np.sort(rng.choice(N, k, replace=False)) for _ in range(B)])[:, None, :]
    idx = idx.astype(np.int32)
    out0, lse0 = oracle.sparse_attn(q, codes, scales, idx, win_k, win_v)
    perm = idx[:, :, rng.permutation(k)]
    out1, lse1 = oracle.sparse_attn(q, codes, scales, perm, win_k, win_v)
    padded = np.full((B, T, k + 5), -1, np.int32)
    padded[:, :, 3:3 + k] = idx
    out2, lse2 = oracle.sparse_attn(q, codes, scales, padded, win_k, win_v)
    assert np.allclose(out0, out1, rtol=1e-12, atol=1e-13)
    assert np.allclose(out0, out2, rtol=1e-12, atol=1e-13)
    assert np.allclose(lse0, lse2, rtol=1e-12, atol=1e-13)


def test_nothing_to_attend():
    rng = np.random.default_rng(8)
    codes, scales = _store(rng, 1, 4, 16)
    q = _bf16(rng, (1, 1, 2, 16))
    out, lse = oracle.sparse_attn(q, codes, scales, np.full((1, 1, 3), -1, np.int32), None, None)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_window_ends_at_the_query_token():
    """Query t of a chunk reads window rows t .. t+W-1; row t+W-1 is token t
    itself and row t+W (a later token) is never read."""
    rng = np.random.default_rng(10)
    T, W, D, H = 4, 3, 16, 1
    codes, scales = _store(rng, 1, 1, D)
    q = wl.bf16_bits(np.ones((1, T, H, D), np.float32))
    win_k = wl.bf16_bits(np.zeros((1, W - 1 + T, D), np.float32))
    win_v = wl.bf16_bits(np.tile(np.arange(W - 1 + T, dtype=np.float32)[None, :, None], (1, 1, D)))
    idx = np.full((1, T, 1), -1, np.int32)
    out, _ = oracle.sparse_attn(q, codes, scales, idx, win_k, win_v)
    for t in range(T):
        assert np.allclose(out[t, 0], np.mean(np.arange(t, t + W)))   # equal logits: mean of rows
    for t in range(T):   # make the query's own row dominate: it must be row t + W - 1
        wk = np.zeros((1, W - 1 + T, D), np.float32)
        wk[0, t + W - 1] = 4.0
        if t + W < W - 1 + T:
            wk[0, t + W] = 8.0   # a future row with an even larger logit must be ignored
        o, _ = oracle.sparse_attn(q, codes, scales, idx, wl.bf16_bits(wk), win_v)
        assert abs(o[t, 0, 0] - (t + W - 1)) < 1e-6


def test_cache_sharing_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "cache_sharing_example.json")))
    L = g["layers"]
    all_full = [(0, l, l) for l in range(L)]
    grouped = []
    for gi in range(L // g["layers_per_shared_copy"]):
        f = 4 * gi
        grouped += [(0, f, f), (1, f, f + 1), (2, f, f + 1), (2, f, f + 1)]
    args = (g["entries"], g["numbers_per_entry"], g["bits_per_number"])
    assert oracle.group_cache_bytes(all_full, *args) == g["bytes_every_layer_own_copy"]
    assert oracle.group_cache_bytes(grouped, *args) == g["bytes_one_copy_per_group_of_four"]
    # the group workload's own table stores one copy per four layers as well
    assert oracle.group_cache_bytes(list(wl.GROUP.modes), *args) == g[
        "bytes_one_copy_per_group_of_four"]


@pytest.mark.parametrize("table", [
    [(1, 0, 0)],                          # Reindex with nothing before it
    [(0, 0, 0), (0, 0, 1)],               # Full naming another layer
    [(0, 0, 0), (2, 0, 1)],               # Reuse naming itself / forward
    [(0, 0, 0), (1, 0, 1), (1, 1, 2)],    # Reindex of a Reindex layer's entries
    [(0, 0, 0), (0, 1, 1), (2, 0, 1)],    # Reuse whose entries differ from its selection's
    [(0, 0, 0), (2, 0, 0), (2, 0, 1)],    # Reuse of a Reuse layer's selection
    [(0, 0, 0), (3, 0, 0)],               # unknown mode
])
def test_invalid_mode_tables_rejected(table):
    assert not oracle.validate_modes(table)


def _small_group_inputs(seed=12):
    w0 = wl.with_sizes(wl.GROUP, B=2, N=300, topk=40, W=9, seed=seed,
                       modes=((0, 0, 0), (1, 0, 1), (2, 0, 1), (2, 0, 1), (0, 4, 4), (2, 4, 4)))
    layers = wl.all_layer_inputs(w0)
    for lay in layers:
        if "entries" in lay:
            B, N, D = lay["entries"].shape
            c, s = oracle.pack_fp4(lay["entries"].reshape(B * N, D))
            lay["codes"], lay["scales"] = c.reshape(B, N, D // 2), s.reshape(B, N, D // 16)
    return w0, layers


def test_mode_invariants():
    w0, layers = _small_group_inputs()
    res = oracle.layer_group(list(w0.modes), layers, w0.topk)
    # Reuse layers take the selection of their source verbatim
    assert np.array_equal(res[2]["idx"], res[1]["idx"])
    assert np.array_equal(res[3]["idx"], res[1]["idx"])
    assert np.array_equal(res[5]["idx"], res[4]["idx"])
    # Reindex and Reuse read their source's entries
    assert [r["store"] for r in res] == [0, 0, 0, 0, 4, 4]
    # a Reindex layer == a Full layer run on its source's store with its own queries
    lay1 = dict(layers[1])
    for key in ("codes", "scales", "k_idx"):
        lay1[key] = layers[0][key]
    full_equiv = oracle.layer_group([(0, 0, 0)], [lay1], w0.topk)[0]
    assert np.array_equal(full_equiv["idx"], res[1]["idx"])
    assert np.array_equal(full_equiv["out"], res[1]["out"])
    # every layer keeps its own queries and window: Reuse output differs from its source's
    assert not np.allclose(res[2]["out"], res[1]["out"])
