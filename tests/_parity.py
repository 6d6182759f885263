"""Helpers shared by the GPU parity tests: host->device marshalling of the
seeded inputs, each side's own FP4 store, the tolerance check and the
layer-group comparison against the oracle's layer walk."""
import numpy as np
import torch

import oracle
import compressed_sparse_attention_topk_b200 as csa2
from compressed_sparse_attention_topk_b200 import workloads as wl

# Attention agreement: |gpu - oracle| <= ATOL + RTOL * |oracle| (fp32 accumulation
# against the fp64 oracle).
ATOL, RTOL = 2e-3, 1e-2


def dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:  # bf16 bit patterns
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    torch.cuda.synchronize()
    return t.cpu().numpy()


def oracle_store(entries: np.ndarray):
    B, N, D = entries.shape
    c, s = oracle.pack_fp4(entries.reshape(B * N, D))
    return c.reshape(B, N, D // 2), s.reshape(B, N, D // 16)


def gpu_store(entries: np.ndarray):
    return csa2.pack_fp4(dev(entries))


def assert_close(gpu: np.ndarray, ref: np.ndarray, what: str = ""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    both_inf = np.isneginf(gpu) & np.isneginf(ref)
    with np.errstate(invalid="ignore"):
        diff = np.where(both_inf, 0.0, np.abs(gpu - ref))
    bound = ATOL + RTOL * np.where(both_inf, 0.0, np.abs(ref))
    bad = ~(diff <= bound)
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance, worst excess "
                           f"{np.nanmax(np.where(bad, diff - bound, 0))}")


def assert_bits_equal(gpu: np.ndarray, ref: np.ndarray, what: str = ""):
    g = np.ascontiguousarray(gpu)
    r = np.ascontiguousarray(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    gv = g.view(np.uint8).reshape(-1)
    rv = r.view(np.uint8).reshape(-1)
    if not np.array_equal(gv, rv):
        nbad = int(np.sum(g.reshape(-1) != r.reshape(-1)))
        raise AssertionError(f"{what}: {nbad} elements differ")


DECODE_KERNELS = [(csa2.DECODE_SCAN_CLUSTER, "scan_cluster"), (csa2.DECODE_FUSED, "fused")]


def use_decode_kernel(kernel):
    """Select the decode kernels (process-wide); returns the previous choice."""
    prev = csa2.get_decode_kernel()
    csa2.set_decode_kernel(kernel)
    return prev


def group_tensors(w0, layers):
    """Device tensors of a layer group's inputs (each Full layer's FP4 store
    packed on the GPU) and its outputs."""
    tens = []
    for l, lay in enumerate(layers):
        d = {k: dev(v) for k, v in lay.items() if k != "entries"}
        d["q"] = d["q"] if w0.T > 1 else d["q"][:, 0].contiguous()
        if "entries" in lay:
            d["codes"], d["scales"] = gpu_store(lay["entries"])
        d["idx"] = torch.empty((w0.B, w0.T, w0.topk), dtype=torch.int32, device="cuda")
        shape = (w0.B, w0.T, w0.H) if w0.T > 1 else (w0.B, w0.H)
        d["out"] = torch.empty(shape + (w0.D,), dtype=torch.float32, device="cuda")
        d["lse"] = torch.empty(shape, dtype=torch.float32, device="cuda")
        tens.append(d)
    return tens


def run_group_and_compare(w0, rows=None, mutate=None):
    """The layer group of workload w0 through the layer call against the
    oracle's layer walk: indices bit-exact, out and lse within tolerance;
    `mutate` edits the seeded inputs first, `rows` restricts the comparison."""
    layers = wl.all_layer_inputs(w0)
    if mutate is not None:
        mutate(layers)
    tens = group_tensors(w0, layers)
    dims = csa2.make_dims(w0.B, w0.T, w0.H, w0.D, w0.N, w0.H_I, w0.d_I, w0.topk, w0.W,
                          w0.n_prior, w0.ratio)
    csa2.layer_group_run(list(w0.modes), tens, dims)
    for lay in layers:
        if "entries" in lay:
            lay["codes"], lay["scales"] = oracle_store(lay["entries"])
    ref = oracle.layer_group(list(w0.modes), layers, w0.topk, w0.n_prior, w0.ratio, rows=rows)
    for l, (mode, kv, ix) in enumerate(w0.modes):
        g_idx = host(tens[ix]["idx"]).reshape(w0.B * w0.T, w0.topk)
        o_idx = ref[l]["idx"].reshape(w0.B * w0.T, w0.topk)
        if rows is not None:
            g_idx, o_idx = g_idx[rows], o_idx[rows]
        assert_bits_equal(g_idx, o_idx, f"layer {l} idx")
        out = host(tens[l]["out"]).reshape(w0.B * w0.T, w0.H, w0.D)
        lse = host(tens[l]["lse"]).reshape(w0.B * w0.T, w0.H)
        if rows is not None:
            out, lse = out[rows], lse[rows]
        assert_close(out, ref[l]["out"], f"layer {l} out")
        assert_close(lse, ref[l]["lse"], f"layer {l} lse")
    assert csa2.get_device_status() == 0
    return tens
