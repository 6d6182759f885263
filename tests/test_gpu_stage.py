"""Staging copies (csa2_stage_copies) on the GPU: bytes moved exactly between
pinned host memory and device memory, strided rows (a window's new row into
its slot), several copies per launch, CUDA graph replay reading the host
buffer afresh, and pageable memory refused on the host."""
import ctypes

import numpy as np
import pytest

import compressed_sparse_attention_topk_b200 as csa2

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _bytes(torch, n, seed, pinned=False, cuda=False):
    g = torch.Generator().manual_seed(seed)
    t = torch.randint(0, 256, (n,), dtype=torch.uint8, generator=g)
    if pinned:
        t = t.pin_memory()
    return t.cuda() if cuda else t


@pytest.mark.parametrize("n", [16, 48, 39424, 131584, 8 << 20])
def test_host_to_device_and_back(n):
    torch = _torch()
    h_src = _bytes(torch, n, n, pinned=True)
    d = torch.zeros(n, dtype=torch.uint8, device="cuda")
    csa2.stage_copies([(h_src, d)])
    h_dst = torch.zeros(n, dtype=torch.uint8).pin_memory()
    csa2.stage_copies([(d, h_dst)])
    torch.cuda.synchronize()
    assert torch.equal(d.cpu(), h_src)
    assert torch.equal(h_dst, h_src)


def test_window_rows_into_their_slots():
    """New rows (host, contiguous) and the same from device memory into
    slot W-1 of each [W, D] window; every other slot untouched."""
    torch = _torch()
    L2, B, W, D = 4, 5, 128, 128
    win = torch.randn(L2, B, W, D, dtype=torch.float32).to(torch.bfloat16).cuda()
    before = win.clone()
    rows_h = torch.randn(L2, B, D).to(torch.bfloat16).pin_memory()
    csa2.stage_copies([(rows_h, win[:, :, -1])])
    torch.cuda.synchronize()
    assert torch.equal(win[:, :, -1].cpu(), rows_h)
    assert torch.equal(win[:, :, :-1], before[:, :, :-1])
    rows_d = torch.randn(L2, B, D).to(torch.bfloat16).cuda()
    csa2.stage_copies([(rows_d, win[:, :, 7])])
    torch.cuda.synchronize()
    assert torch.equal(win[:, :, 7], rows_d)
    assert torch.equal(win[:, :, -1].cpu(), rows_h)


def test_sixteen_copies_in_one_launch():
    torch = _torch()
    sizes = [16 * (1 + 37 * i) for i in range(16)]
    srcs, dsts = [], []
    for i, n in enumerate(sizes):
        if i % 2 == 0:  # host -> device
            srcs.append(_bytes(torch, n, i, pinned=True))
            dsts.append(torch.zeros(n, dtype=torch.uint8, device="cuda"))
        else:           # device -> host
            srcs.append(_bytes(torch, n, i, cuda=True))
            dsts.append(torch.zeros(n, dtype=torch.uint8).pin_memory())
    csa2.stage_copies(list(zip(srcs, dsts)))
    torch.cuda.synchronize()
    for s, d in zip(srcs, dsts):
        assert torch.equal(s.cpu(), d.cpu())
    with pytest.raises(ValueError):
        csa2.stage_copies(list(zip(srcs, dsts)) + [(srcs[0], dsts[0])])


def test_graph_replay_reads_the_host_buffer_again():
    """A captured staging launch, replayed after the host rewrote its pinned
    source, delivers the new bytes (host memory is read uncached)."""
    torch = _torch()
    n = 39424
    h_in = _bytes(torch, n, 1, pinned=True)
    d = torch.zeros(n, dtype=torch.uint8, device="cuda")
    h_out = torch.zeros(n, dtype=torch.uint8).pin_memory()
    g_in, g_out = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_in):
        csa2.stage_copies([(h_in, d)])
    with torch.cuda.graph(g_out):
        csa2.stage_copies([(d, h_out)])
    torch.cuda.synchronize()
    for seed in (2, 3, 4):
        h_in.copy_(_bytes(torch, n, seed))
        g_in.replay()
        g_out.replay()
        torch.cuda.synchronize()
        assert torch.equal(h_out, h_in)
    del g_in, g_out


def test_pageable_host_memory_refused_before_launch():
    torch = _torch()
    lib = csa2.lib()
    a = np.zeros(4096, dtype=np.uint8)  # pageable (malloc'd) host memory
    d = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    for src, dst in ((a.ctypes.data, d.data_ptr()), (d.data_ptr(), a.ctypes.data)):
        arr = (csa2.Copy2D * 1)(csa2.Copy2D(src, dst, 1, 4096, 4096, 4096))
        rc = lib.csa2_stage_copies(arr, 1, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == csa2.CSA2_ERR_INVALID_ARG
    assert not a.any()
    assert csa2.get_device_status() == 0
