"""Helpers shared by the GPU parity tests: host->device marshalling of the
seeded inputs, each side's own FP4 store, and the tolerance check."""
import numpy as np
import torch

import oracle
import compressed_sparse_attention_topk_b200 as csa2

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
