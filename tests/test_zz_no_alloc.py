"""csa2_index_topk_noalloc: the index + top-k call for callers that cannot
allocate device memory (e.g. a host runtime that owns all device memory and
gives extensions no workspace).  It must return exactly what the workspace
version returns, on consecutive calls that reuse its built-in scratch.

This file is collected last on purpose: it also passes when run alone in a
fresh process (the first call sets the scratch up), and after every other
test (scratch left behind by earlier calls must not leak into results)."""
import ctypes

import numpy as np
import pytest
import torch

import compressed_sparse_attention_topk_b200 as csa2
import oracle
from compressed_sparse_attention_topk_b200 import build as csa2_build
from compressed_sparse_attention_topk_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _case(seed, B, H_I, d_I, N, T=1):
    rng = np.random.default_rng(seed)
    q = torch.from_numpy(wl.int8_uniform(rng, (B, T, H_I, d_I))).cuda()
    w = torch.from_numpy(rng.random((B, T, H_I), dtype=np.float32)).cuda()
    k = torch.from_numpy(wl.int8_uniform(rng, (B, N, d_I))).cuda()
    return q, w, k


def _noalloc(q, w, k, topk, want_scores=True):
    B, T, H_I, d_I = q.shape
    N = k.shape[1]
    idx = torch.full((B, T, topk), -7, dtype=torch.int32, device="cuda")
    scores = (torch.full((B, T, N), 7.0, dtype=torch.float32, device="cuda") if want_scores
              else None)
    stream = torch.cuda.current_stream().cuda_stream
    rc = csa2.lib().csa2_index_topk_noalloc(
        q.data_ptr(), w.data_ptr(), k.data_ptr(), B, T, H_I, d_I, N, -1, 4, topk,
        idx.data_ptr(), None if scores is None else scores.data_ptr(), ctypes.c_void_p(stream))
    assert rc == csa2.CSA2_OK, csa2.lib().csa2_status_string(rc)
    torch.cuda.synchronize()
    return idx, scores


def test_noalloc_matches_workspace_version_on_consecutive_calls():
    csa2_build.build()
    topk = 2048
    # two different inputs in a row: the second call reuses the scratch the
    # first one left behind
    for seed, (B, H_I, d_I, N) in [(31, (4, 4, 64, 100_000)), (32, (3, 4, 32, 150_001))]:
        q, w, k = _case(seed, B, H_I, d_I, N)
        ref_idx, ref_scores = csa2.index_topk(q, w, k, topk, want_scores=True)
        idx, scores = _noalloc(q, w, k, topk)
        assert torch.equal(idx, ref_idx)
        assert torch.equal(scores.view(torch.int32), ref_scores.view(torch.int32))
    assert csa2.get_device_status() == 0


def test_noalloc_many_queries_tensor_core_path_matches_oracle():
    """64 queries per sequence and no score output take the tensor-core
    indexer, whose scratch differs from the per-row scan's; two calls in a
    row, the second after a decode-shape call has left the scratch dirty."""
    csa2_build.build()
    topk = 512
    for seed in (41, 42):
        q, w, k = _case(seed, 1, 4, 64, 10_000, T=64)
        assert csa2.index_topk_workspace_size(1, 64, 4, 64, 10_000, topk) <= 16 << 20
        idx, _ = _noalloc(q, w, k, topk, want_scores=False)
        ref = oracle.index_topk(q.cpu().numpy(), w.cpu().numpy(), k.cpu().numpy(), topk)
        assert np.array_equal(idx.cpu().numpy().reshape(64, topk), ref)
        ref_idx = csa2.index_topk(q, w, k, topk)
        assert torch.equal(idx, ref_idx)
        _noalloc(*_case(seed + 100, 2, 4, 64, 50_000), 2048)   # leaves other scratch behind
    assert csa2.get_device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    csa2_build.build()
    # 4 x 1,000,000 entries need ~48 MB of scratch: refused before any launch
    fake = ctypes.c_void_p(256)
    rc = csa2.lib().csa2_index_topk_noalloc(fake, fake, fake, 4, 1, 4, 64, 1_000_000, -1, 4,
                                            2048, fake, None, None)
    assert rc == csa2.CSA2_ERR_UNSUPPORTED
