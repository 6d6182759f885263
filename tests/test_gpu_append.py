"""GPU parity of the per-token entry append (csa2_append_entry through the C
ABI) against the oracle's append: FP4 codes, scales and index keys of the
written rows bit-exact, every other row untouched."""
import numpy as np
import pytest
import torch

import oracle
import compressed_sparse_attention_topk_b200 as csa2
from compressed_sparse_attention_topk_b200 import build as csa2_build
from tests._parity import assert_bits_equal, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    csa2_build.build()
    csa2.lib()
    assert csa2.get_device_status() == 0


def _stores(rng, B, N, D, d_I):
    codes = rng.integers(0, 256, (B, N, D // 2)).astype(np.uint8)
    scales = rng.standard_normal((B, N, D // 16)).astype(np.float32)
    keys = rng.integers(-127, 128, (B, N, d_I)).astype(np.int8)
    return codes, scales, keys


@pytest.mark.parametrize("B,N,D,d_I", [(4, 1000, 128, 64), (3, 17, 64, 32), (1, 5, 16, 16),
                                       (32, 4096, 128, 32)])
def test_append_matches_oracle_over_steps(B, N, D, d_I):
    rng = np.random.default_rng(B * 100 + N)
    codes, scales, keys = _stores(rng, B, N, D, d_I)
    g_codes, g_scales, g_keys = dev(codes), dev(scales), dev(keys)
    for step in range(3):
        src = (rng.standard_normal((B, D)) * np.exp(rng.uniform(-20, 20, (B, 1)))).astype(
            np.float32)
        src[0, :16] = 0.0                                 # a zero group
        key = rng.integers(-127, 128, (B, d_I)).astype(np.int8)
        pos = rng.integers(-1, N, B).astype(np.int64)     # some sequences append nothing
        pos[-1] = N - 1
        oracle.append_entry(src, key, pos, codes, scales, keys)
        csa2.append_entry(dev(src), dev(key), dev(pos), g_codes, g_scales, g_keys)
        assert_bits_equal(host(g_codes), codes, f"codes step {step}")
        assert_bits_equal(host(g_scales), scales, f"scales step {step}")
        assert_bits_equal(host(g_keys), keys, f"keys step {step}")
    assert csa2.get_device_status() == 0


def test_append_position_past_the_store_is_skipped_and_recorded():
    rng = np.random.default_rng(9)
    B, N, D, d_I = 2, 8, 64, 32
    codes, scales, keys = _stores(rng, B, N, D, d_I)
    g = [dev(codes), dev(scales), dev(keys)]
    src = rng.standard_normal((B, D)).astype(np.float32)
    key = rng.integers(-127, 128, (B, d_I)).astype(np.int8)
    pos = np.array([3, N], np.int64)                      # sequence 1 is out of range
    csa2.append_entry(dev(src), dev(key), dev(pos), *g)
    assert csa2.get_device_status() & 1
    ok = pos.copy()
    ok[1] = -1                                            # the oracle's view: only b = 0
    oracle.append_entry(src, key, ok, codes, scales, keys)
    assert_bits_equal(host(g[0]), codes, "codes")
    assert_bits_equal(host(g[1]), scales, "scales")
    assert_bits_equal(host(g[2]), keys, "keys")
    assert csa2.get_device_status() == 0


def test_append_then_decode_sees_the_new_entry():
    """An entry appended at the last row becomes selectable at once: its
    index key is the query's best match, so the top-k must contain it."""
    rng = np.random.default_rng(11)
    B, N, H_I, d_I, topk = 2, 5000, 4, 64, 64
    q = rng.integers(-127, 128, (B, 1, H_I, d_I)).astype(np.int8)
    w = np.ones((B, 1, H_I), np.float32)
    keys = rng.integers(-20, 21, (B, N, d_I)).astype(np.int8)
    best = np.where(q[:, 0].astype(np.int64).sum(axis=1) >= 0, 127, -127).astype(np.int8)
    g_keys = dev(keys)
    g_codes = torch.zeros((B, N, 64), dtype=torch.uint8, device="cuda")
    g_scales = torch.zeros((B, N, 8), dtype=torch.float32, device="cuda")
    src = rng.standard_normal((B, 128)).astype(np.float32)
    pos = np.full(B, N - 1, np.int64)
    csa2.append_entry(dev(src), dev(best), dev(pos), g_codes, g_scales, g_keys)
    keys[:, N - 1] = best
    idx = host(csa2.index_topk(dev(q), dev(w), g_keys, topk)).reshape(B, topk)
    assert np.all(idx[:, -1] == N - 1)
    ref = oracle.index_topk(q, w, keys, topk)
    assert_bits_equal(idx, ref, "indices")


def test_bounded_waits_give_up_and_the_device_keeps_working():
    """The library's bounded waits, run against a barrier phase that never
    completes and a counter that nothing raises with a short limit (2^20
    cycles, under a millisecond): they give up, record bit 1 of the status
    word, and the next call on the same context works and is exact."""
    assert csa2.get_device_status() == 0
    rc = csa2.lib().csa2_wait_timeout_selftest(1 << 20, torch.cuda.current_stream().cuda_stream)
    assert rc == csa2.CSA2_OK
    assert csa2.get_device_status() == 2
    assert csa2.get_device_status() == 0          # reading clears it
    rng = np.random.default_rng(1)
    q = rng.integers(-127, 128, (2, 1, 4, 64)).astype(np.int8)
    w = rng.random((2, 1, 4), dtype=np.float32)
    k = rng.integers(-127, 128, (2, 5000, 64)).astype(np.int8)
    idx = host(csa2.index_topk(dev(q), dev(w), dev(k), 100)).reshape(2, 100)
    assert_bits_equal(idx, oracle.index_topk(q, w, k, 100), "indices after the self-test")
