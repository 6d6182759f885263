"""GPU parity of the decode path that hands each selecting CTA's list to a
separate attention kernel: layer calls whose passes have 8 or fewer selecting
CTAs per row (more decode rows than the device holds 16-CTA clusters of the
row kernel at once: 8 or more on a 148-SM B200; clusters of 8 while they all
fit, else of 4).  Indices bit-exact, attention within 2e-3 absolute + 1e-2
relative of the fp64 oracle."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_topk_b200 as csa2
from compressed_sparse_attention_topk_b200 import build as csa2_build
from compressed_sparse_attention_topk_b200 import workloads as wl
from tests._parity import group_tensors, run_group_and_compare, use_decode_kernel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _scan_cluster():
    csa2_build.build()
    csa2.lib()
    prev = use_decode_kernel(csa2.DECODE_SCAN_CLUSTER)
    yield
    use_decode_kernel(prev)


@pytest.mark.parametrize("B,N,topk,W,H,D,H_I,d_I", [
    (10, 5000, 512, 128, 16, 128, 4, 64),    # 8 selecting CTAs per row
    (40, 3000, 256, 128, 16, 128, 4, 32),    # 4 per row
    (24, 1000, 2048, 128, 16, 128, 4, 64),   # fewer entries than k: every entry, padding
    (9, 16, 64, 5, 16, 128, 4, 64),          # 16 entries: seven of a row's eight lists empty
    (20, 9000, 1024, 64, 32, 128, 4, 64),    # two head passes
    (12, 9000, 1024, 64, 32, 128, 4, 64),    # two head passes, 8 lists per row
    (21, 6000, 700, 33, 8, 64, 8, 32),       # D = 64, 8 heads, uneven window shares
    (11, 6000, 700, 33, 8, 64, 8, 32),       # the same with 8 lists per row
])
def test_handoff_decode_layer_shapes(B, N, topk, W, H, D, H_I, d_I):
    w0 = wl.with_sizes(wl.LONG, name=f"handoff_{B}_{N}_{topk}", B=B, N=N, topk=topk, W=W, H=H,
                       D=D, H_I=H_I, d_I=d_I, seed=B * 1000 + N + 7)
    csa2.trace_enable(True)
    try:
        run_group_and_compare(w0)
        names = {name for name, _ in csa2.trace_records()}
    finally:
        csa2.trace_enable(False)
    assert "attend_handoff" in names and "topk_select" in names, names


@pytest.mark.parametrize("B", [10, 20])
def test_handoff_heavy_ties(B):
    """Scores that take a few integer values: the keys equal to the threshold
    outnumber the slots left, so a CTA's list is known only after every rank's
    counts are in, and it is published then."""
    w0 = wl.with_sizes(wl.LONG, name=f"handoff_ties_{B}", B=B, N=20000, topk=1000, seed=91)

    def mutate(layers):
        rng = np.random.default_rng(19)
        layers[0]["k_idx"] = rng.integers(-1, 2, layers[0]["k_idx"].shape).astype(np.int8)
        for lay in layers:
            lay["q_idx"] = rng.integers(0, 2, lay["q_idx"].shape).astype(np.int8)
            lay["w"][:] = 1.0

    run_group_and_compare(w0, mutate=mutate)


@pytest.mark.parametrize("B", [10, 20])
def test_handoff_selection_crowded_into_one_slice(B):
    """The top-k of every row lies in its first positions: one CTA's list
    holds the whole selection, the others publish empty lists."""
    w0 = wl.with_sizes(wl.LONG, name=f"handoff_crowded_{B}", B=B, N=40000, topk=2000, seed=92)

    def mutate(layers):
        k = layers[0]["k_idx"]
        k[:, :2000] = np.abs(k[:, :2000]) // 2 + 60
        k[:, 2000:] = k[:, 2000:] // 4
        for lay in layers:
            lay["q_idx"] = np.abs(lay["q_idx"]) // 2 + 1

    run_group_and_compare(w0, mutate=mutate)


def test_handoff_cuda_graph_replay():
    """Captured into a CUDA graph and replayed (the flags and counters are
    cleared in every replay): the eager results, bit for bit, every time."""
    w0 = wl.with_sizes(wl.LONG, name="handoff_graph", B=20, N=8000, topk=512, seed=93)
    layers = wl.all_layer_inputs(w0)
    tens = group_tensors(w0, layers)
    dims = csa2.make_dims(w0.B, w0.T, w0.H, w0.D, w0.N, w0.H_I, w0.d_I, w0.topk, w0.W)
    group = csa2.LayerGroup(list(w0.modes), tens, dims)
    group.run()
    torch.cuda.synchronize()
    eager = [(t["idx"].clone(), t["out"].clone(), t["lse"].clone()) for t in tens]
    graphs = []
    for l in range(w0.L):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            group.run_layer(l)
        graphs.append(g)
    for _ in range(3):
        for t in tens:
            t["idx"].fill_(-7)
            t["out"].fill_(float("nan"))
            t["lse"].fill_(float("nan"))
        for g in graphs:
            g.replay()
        torch.cuda.synchronize()
        for (i0, o0, l0), t in zip(eager, tens):
            assert torch.equal(t["idx"], i0)
            assert torch.equal(t["out"], o0)
            assert torch.equal(t["lse"], l0)
    assert csa2.get_device_status() == 0
