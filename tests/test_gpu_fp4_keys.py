"""GPU parity of FP4 index keys (E2M1 with one power-of-two scale per 32
elements) through the C ABI: packing bit-exact against the oracle, the index
score + top-k bit-exact, and whole decode layers over FP4 keys (selection
bit-exact, attention within tolerance).  Also the entry append run inside a
layer call."""
import numpy as np
import pytest
import torch

import oracle
import compressed_sparse_attention_topk_b200 as csa2
from compressed_sparse_attention_topk_b200 import build as csa2_build
from compressed_sparse_attention_topk_b200 import workloads as wl
from tests._parity import assert_bits_equal, assert_close, dev, host, oracle_store

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    csa2_build.build()
    csa2.lib()
    assert csa2.get_device_status() == 0


def _key_sources(rng, rows, d_I):
    x = (rng.standard_normal((rows, d_I)) * np.exp(rng.uniform(-40, 40, (rows, 1)))).astype(
        np.float32)
    x[0] = 0.0                                             # zero blocks
    x[1, :32] = np.float32(1e-42)                          # subnormal block
    grid = np.array([7.9, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    x[2, :8] = grid                                        # ties and saturation at scale 1
    x[2, 8:16] = -grid
    x[3, :32] = np.float32(3e38)                           # near the top of the range
    return x


@pytest.mark.parametrize("d_I", [32, 64, 128])
def test_pack_index_keys_bit_exact(d_I):
    rng = np.random.default_rng(d_I)
    x = _key_sources(rng, 3000, d_I)
    oc, oe = oracle.pack_mxfp4(x)
    gc, ge = csa2.pack_index_keys_fp4(dev(x))
    assert_bits_equal(host(gc), oc, "codes")
    assert_bits_equal(host(ge), oe, "exponents")


def _fp4_case(seed, B, H_I, d_I, N):
    rng = np.random.default_rng(seed)
    q = wl.int8_uniform(rng, (B, H_I, d_I))
    w = rng.random((B, H_I), dtype=np.float32)
    src = rng.standard_normal((B * N, d_I)).astype(np.float32)
    src[: N // 7] *= np.float32(16.0)                      # blocks at several scales
    codes, exps = oracle.pack_mxfp4(src)
    return q, w, codes.reshape(B, N, -1), exps.reshape(B, N, -1)


@pytest.mark.parametrize("B,d_I,N,topk", [(1, 64, 16, 5), (4, 64, 3008, 2048), (3, 32, 20000, 64),
                                          (2, 64, 262144, 2048), (5, 64, 4096, 4096),
                                          (40, 32, 4000, 256)])
def test_index_topk_fp4_keys_bit_exact(B, d_I, N, topk, decode_kernel):
    q, w, codes, exps = _fp4_case(B * 10 + N, B, 4, d_I, N)
    got = host(csa2.index_topk_fp4k(dev(q), dev(w), dev(codes), dev(exps), topk))
    ref = oracle.index_topk_fp4k(q, w, codes, exps, topk)
    assert_bits_equal(got, ref, "indices")
    assert csa2.get_device_status() == 0


def test_index_topk_fp4_keys_ties(decode_kernel):
    # keys from a few levels only: many equal scores at the threshold
    rng = np.random.default_rng(4)
    B, H_I, d_I, N, topk = 3, 4, 64, 9008, 1000
    q = wl.int8_uniform(rng, (B, H_I, d_I))
    w = np.ones((B, H_I), np.float32)
    src = rng.integers(-1, 2, (B * N, d_I)).astype(np.float32)
    codes, exps = oracle.pack_mxfp4(src)
    codes, exps = codes.reshape(B, N, -1), exps.reshape(B, N, -1)
    got = host(csa2.index_topk_fp4k(dev(q), dev(w), dev(codes), dev(exps), topk))
    assert_bits_equal(got, oracle.index_topk_fp4k(q, w, codes, exps, topk), "indices")


def _layers_fp4(w0, layers):
    """Device tensors of a Full + Reindex pair whose store keeps FP4 index keys."""
    tens = []
    for lay in layers:
        d = {k: dev(v) for k, v in lay.items() if k not in ("entries", "k_idx", "key_src")}
        d["q"] = d["q"][:, 0].contiguous()
        if "entries" in lay:
            d["codes"], d["scales"] = csa2.pack_fp4(dev(lay["entries"]))
            d["k_idx"], d["k_exps"] = csa2.pack_index_keys_fp4(dev(lay["key_src"]))
        d["idx"] = torch.empty((w0.B, 1, w0.topk), dtype=torch.int32, device="cuda")
        d["out"] = torch.empty((w0.B, w0.H, w0.D), dtype=torch.float32, device="cuda")
        d["lse"] = torch.empty((w0.B, w0.H), dtype=torch.float32, device="cuda")
        tens.append(d)
    return tens


@pytest.mark.parametrize("B,N,W", [(4, 262144, 128), (2, 5008, 0), (3, 1008, 128)])
def test_decode_layers_over_fp4_keys(B, N, W, decode_kernel):
    w0 = wl.with_sizes(wl.LONG, name=f"fp4k_{B}_{N}", B=B, N=N, W=W, seed=B + N)
    layers = wl.all_layer_inputs(w0)
    rng = np.random.default_rng(N)
    layers[0]["key_src"] = rng.standard_normal((B, N, w0.d_I)).astype(np.float32)
    tens = _layers_fp4(w0, layers)
    dims = csa2.make_dims(w0.B, 1, w0.H, w0.D, w0.N, w0.H_I, w0.d_I, w0.topk, w0.W)
    csa2.layer_group_run(list(w0.modes), tens, dims)
    oc, os_ = oracle_store(layers[0]["entries"])
    kc, ke = oracle.pack_mxfp4(layers[0]["key_src"].reshape(B * N, -1))
    kc, ke = kc.reshape(B, N, -1), ke.reshape(B, N, -1)
    for l, lay in enumerate(layers):
        idx = oracle.index_topk_fp4k(lay["q_idx"], lay["w"], kc, ke, w0.topk)
        assert_bits_equal(host(tens[l]["idx"]).reshape(B, -1), idx, f"layer {l} idx")
        out, lse = oracle.sparse_attn(lay["q"], oc, os_, idx.reshape(B, 1, -1), lay["win_k"],
                                      lay["win_v"])
        assert_close(host(tens[l]["out"]).reshape(out.shape), out, f"layer {l} out")
        assert_close(host(tens[l]["lse"]).reshape(lse.shape), lse, f"layer {l} lse")
    assert csa2.get_device_status() == 0


def test_layer_call_appends_the_step_entry_before_its_scan(decode_kernel):
    """A Full layer given this step's entry appends it (FP4 entry + int8 key)
    into its store before scanning: bit-exact store, and the selection and
    attention of both layers see the new entry."""
    w0 = wl.with_sizes(wl.LONG, name="append_in_layer", B=3, N=6000, seed=31)
    layers = wl.all_layer_inputs(w0)
    B, N, D, d_I = w0.B, w0.N, w0.D, w0.d_I
    rng = np.random.default_rng(5)
    src = rng.standard_normal((B, D)).astype(np.float32) * np.float32(3.0)
    key = wl.int8_uniform(rng, (B, d_I))
    pos = np.array([N - 1, 17, -1], np.int64)
    tens = []
    for lay in layers:
        d = {k: dev(v) for k, v in lay.items() if k != "entries"}
        d["q"] = d["q"][:, 0].contiguous()
        if "entries" in lay:
            d["codes"], d["scales"] = csa2.pack_fp4(dev(lay["entries"]))
            d["app_src"], d["app_key"], d["app_pos"] = dev(src), dev(key), dev(pos)
        d["idx"] = torch.empty((B, 1, w0.topk), dtype=torch.int32, device="cuda")
        d["out"] = torch.empty((B, w0.H, D), dtype=torch.float32, device="cuda")
        d["lse"] = torch.empty((B, w0.H), dtype=torch.float32, device="cuda")
        tens.append(d)
    dims = csa2.make_dims(B, 1, w0.H, D, N, w0.H_I, d_I, w0.topk, w0.W)
    csa2.layer_group_run(list(w0.modes), tens, dims)
    codes, scales = oracle_store(layers[0]["entries"])
    keys = layers[0]["k_idx"].copy()
    oracle.append_entry(src, key, pos, codes, scales, keys)
    assert_bits_equal(host(tens[0]["codes"]), codes, "codes")
    assert_bits_equal(host(tens[0]["scales"]), scales, "scales")
    assert_bits_equal(host(tens[0]["k_idx"]), keys, "keys")
    layers[0]["codes"], layers[0]["scales"], layers[0]["k_idx"] = codes, scales, keys
    ref = oracle.layer_group(list(w0.modes), layers, w0.topk)
    for l in range(2):
        assert_bits_equal(host(tens[l]["idx"]).reshape(B, -1), ref[l]["idx"].reshape(B, -1),
                          f"layer {l} idx")
        assert_close(host(tens[l]["out"]).reshape(ref[l]["out"].shape), ref[l]["out"], "out")
    assert csa2.get_device_status() == 0
