"""Seeded synthetic workloads for the CSA2 hot path.

This module only draws random inputs and states shapes; it holds none of
the method's arithmetic (no packing, scoring, selection or attention).  The
same arrays feed the CUDA library and the CPU oracle.

Shapes and value structure follow the pages' long-context decode and
prefill workloads ("Why Is DeepSeek V4.1 Flash So Fast?", section 3:
1M-token context, 128-token window; section 4: indexer + Top-K) with every
size fixed explicitly below, since the pages fix none of them:

* entries: fp32 sources N(0,1) [B, N, D], stored as FP4 by the path under
  test; the decode workload scales a seeded 1% of entries by 8 (salient
  outliers);
* index keys / index queries: int8 uniform on [-127, 127];
* index head weights: fp32 U(0, 1);
* attention queries and window keys/values: bf16 of N(0,1) draws.

Random draws use numpy's PCG64 with one SeedSequence stream per tensor
(``[seed, tensor id, layer]``), so inputs are bit-identical on any machine.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

import numpy as np

FULL, REINDEX, REUSE = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    D: int
    N: int             # stored entries per sequence (incl. the chunk's own for prefill)
    H_I: int
    d_I: int
    topk: int
    W: int
    seed: int
    modes: Tuple[Tuple[int, int, int], ...]   # per layer (mode, kv_src, idx_src)
    n_prior: int = -1  # -1: decode, all N visible; >= 0: prefill chunk after n_prior entries
    ratio: int = 4     # tokens per compressed entry (prefill visibility)
    outlier_frac: float = 0.0
    outlier_scale: float = 8.0

    @property
    def L(self) -> int:
        return len(self.modes)

    @property
    def sm_scale(self) -> float:
        return float(1.0 / np.sqrt(self.D))

    @property
    def win_rows(self) -> int:
        return self.W - 1 + self.T


def _group(n_groups: int) -> Tuple[Tuple[int, int, int], ...]:
    modes = []
    for g in range(n_groups):
        f = 4 * g
        modes += [(FULL, f, f), (REINDEX, f, f + 1), (REUSE, f, f + 1), (REUSE, f, f + 1)]
    return tuple(modes)


TINY = Workload("tiny_decode_n1024", B=1, T=1, H=8, D=64, N=1024, H_I=8, d_I=32, topk=64,
                W=128, seed=0, modes=((FULL, 0, 0),))
DECODE = Workload("decode_b32_n131072", B=32, T=1, H=16, D=128, N=131072, H_I=4, d_I=32,
                  topk=2048, W=128, seed=2, modes=((FULL, 0, 0),), outlier_frac=0.01)
GROUP = Workload("group16_b8_n4096", B=8, T=1, H=16, D=128, N=4096, H_I=4, d_I=32, topk=512,
                 W=128, seed=3, modes=_group(4))
LONG = Workload("long_decode_1m_b4_n262144", B=4, T=1, H=16, D=128, N=262144, H_I=4, d_I=64,
                topk=2048, W=128, seed=4, modes=((FULL, 0, 0), (REINDEX, 0, 1)))
PREFILL = Workload("prefill_t4096_nprior262144", B=1, T=4096, H=16, D=128, N=262144 + 1024,
                   H_I=4, d_I=64, topk=2048, W=128, seed=5, modes=((FULL, 0, 0),),
                   n_prior=262144, ratio=4)

# Multi-token decode: 5 query tokens per sequence (draft tokens verified
# together) at the 1M-context shape; every token sees all N entries.
MTP5 = Workload("mtp5_decode_1m_b4_n262144", B=4, T=5, H=16, D=128, N=262144, H_I=4, d_I=64,
                topk=2048, W=128, seed=6, modes=((FULL, 0, 0), (REINDEX, 0, 1)))

ALL = {w.name: w for w in (TINY, DECODE, GROUP, LONG, PREFILL, MTP5)}

_TENSOR_IDS = {"entries": 1, "k_idx": 2, "q_idx": 3, "w": 4, "q": 5, "win_k": 6, "win_v": 7,
               "outliers": 8, "key_src": 9, "app_src": 10, "app_key": 11}


def rng_for(seed: int, tensor: str, layer: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(
        [seed, _TENSOR_IDS[tensor], layer])))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 draws -> bf16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    rounded = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << np.uint32(16)).view(
        np.float32)


def int8_uniform(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.integers(-127, 128, size=shape, dtype=np.int8)


def entry_sources(wl: Workload, layer: int = 0, B: Optional[int] = None,
                  N: Optional[int] = None) -> np.ndarray:
    """fp32 [B, N, D] sources of the FP4 entries of one entry store."""
    B = wl.B if B is None else B
    N = wl.N if N is None else N
    x = rng_for(wl.seed, "entries", layer).standard_normal((B, N, wl.D), dtype=np.float32)
    if wl.outlier_frac > 0.0:
        r = rng_for(wl.seed, "outliers", layer)
        n_out = max(1, int(round(wl.outlier_frac * N)))
        for b in range(B):
            rows = r.choice(N, size=n_out, replace=False)
            x[b, rows, :] *= np.float32(wl.outlier_scale)
    return x


def layer_inputs(wl: Workload, layer: int, B: Optional[int] = None) -> dict:
    """A layer's own inputs: q, q_idx, w, win_k, win_v and, for a layer that
    keeps its own entries (Full), its store's entry sources and index keys."""
    B = wl.B if B is None else B
    mode, kv_src, _ = wl.modes[layer]
    d = {
        "q": bf16_bits(rng_for(wl.seed, "q", layer).standard_normal(
            (B, wl.T, wl.H, wl.D), dtype=np.float32)),
        "q_idx": int8_uniform(rng_for(wl.seed, "q_idx", layer), (B, wl.T, wl.H_I, wl.d_I)),
        "w": rng_for(wl.seed, "w", layer).random((B, wl.T, wl.H_I), dtype=np.float32),
        "win_k": bf16_bits(rng_for(wl.seed, "win_k", layer).standard_normal(
            (B, wl.win_rows, wl.D), dtype=np.float32)),
        "win_v": bf16_bits(rng_for(wl.seed, "win_v", layer).standard_normal(
            (B, wl.win_rows, wl.D), dtype=np.float32)),
    }
    if mode == FULL:
        d["entries"] = entry_sources(wl, layer, B)
        d["k_idx"] = int8_uniform(rng_for(wl.seed, "k_idx", layer), (B, wl.N, wl.d_I))
    return d


def all_layer_inputs(wl: Workload, B: Optional[int] = None) -> List[dict]:
    return [layer_inputs(wl, l, B) for l in range(wl.L)]


def with_sizes(wl: Workload, **kw) -> Workload:
    """A copy of a workload with some sizes changed (smaller parity cases)."""
    return dataclasses.replace(wl, **kw)


def index_key_sources(wl: Workload, layer: int = 0, B: Optional[int] = None) -> np.ndarray:
    """fp32 [B, N, d_I] N(0,1) sources of a store's index keys, for stores that
    keep them in FP4 (each side packs them on its own)."""
    B = wl.B if B is None else B
    return rng_for(wl.seed, "key_src", layer).standard_normal((B, wl.N, wl.d_I),
                                                              dtype=np.float32)


def append_inputs(wl: Workload, step: int = 0, B: Optional[int] = None) -> dict:
    """One decode step's completed entries: fp32 [B, D] N(0,1) entry values
    and int8 [B, d_I] uniform index keys (the compressor's and the indexer
    key projection's outputs, which this library does not model)."""
    B = wl.B if B is None else B
    return {"src": rng_for(wl.seed, "app_src", step).standard_normal((B, wl.D),
                                                                     dtype=np.float32),
            "key": int8_uniform(rng_for(wl.seed, "app_key", step), (B, wl.d_I))}
