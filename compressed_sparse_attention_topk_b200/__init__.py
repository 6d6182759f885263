"""CSA2 hot path on B200: a thin ctypes binding over libcsa2.so.

Every function here only marshals arguments (torch tensors -> device
pointers, sizes, the current CUDA stream) and calls the C ABI declared in
``include/csa2.h``; all computation runs in the library's sm_100a kernels.
There is no CPU fallback: if the library is missing or a tensor is not on
a CUDA device, the call raises.

Functions mirror the C entry points: ``pack_fp4``, ``unpack_fp4``,
``index_topk``, ``sparse_attn_decode``, ``sparse_attn_prefill``,
``layer_group_run``, plus ``validate_modes``, ``group_cache_bytes`` and
``get_device_status``.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Dict, List, Optional, Sequence, Tuple

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcsa2.so")

CSA2_OK, CSA2_ERR_INVALID_ARG, CSA2_ERR_UNSUPPORTED, CSA2_ERR_CUDA = 0, 1, 2, 3
CSA2_ERR_WORKSPACE, CSA2_ERR_DEVICE_STATUS = 4, 5
FULL, REINDEX, REUSE, REINDEX_POOL = 0, 1, 2, 3

EXPORTED = (
    "csa2_status_string", "csa2_version", "csa2_pack_fp4", "csa2_unpack_fp4",
    "csa2_index_topk_workspace_size", "csa2_index_topk", "csa2_sparse_attn_workspace_size",
    "csa2_sparse_attn_decode", "csa2_sparse_attn_prefill", "csa2_validate_modes",
    "csa2_group_cache_bytes", "csa2_layer_group_workspace_size", "csa2_layer_group_run",
    "csa2_get_device_status", "csa2_trace_enable", "csa2_trace_count", "csa2_trace_get",
    "csa2_layer_run", "csa2_index_topk_noalloc", "csa2_index_pool_workspace_size",
    "csa2_index_pool", "csa2_pool_topk_workspace_size", "csa2_pool_topk", "csa2_append_entry",
    "csa2_pack_index_keys_fp4", "csa2_index_topk_fp4k_workspace_size", "csa2_index_topk_fp4k",
    "csa2_wait_timeout_selftest", "csa2_set_decode_kernel", "csa2_get_decode_kernel",
    "csa2_stage_copies",
)
DECODE_SCAN_CLUSTER, DECODE_FUSED = 0, 1


class CSA2Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().csa2_status_string(status).decode()}")


class LayerMode(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("kv_src", ctypes.c_int32), ("idx_src", ctypes.c_int32)]


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32),
                ("D", ctypes.c_int32), ("N", ctypes.c_int64), ("H_I", ctypes.c_int32),
                ("d_I", ctypes.c_int32), ("topk", ctypes.c_int32), ("W", ctypes.c_int32),
                ("n_prior", ctypes.c_int64), ("ratio", ctypes.c_int32),
                ("sm_scale", ctypes.c_float), ("pool_block", ctypes.c_int32),
                ("pool_blocks", ctypes.c_int32)]


class Copy2D(ctypes.Structure):
    _fields_ = [("src", ctypes.c_void_p), ("dst", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("row_bytes", ctypes.c_int64), ("src_stride", ctypes.c_int64),
                ("dst_stride", ctypes.c_int64)]


MAX_STAGE_COPIES = 16


class LayerIO(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "q", "q_idx", "w", "win_k", "win_v", "codes", "scales", "k_idx", "idx", "out", "lse",
        "k_exps", "app_src", "app_key", "app_pos", "pool")]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libcsa2.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m compressed_sparse_attention_topk_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                            ctypes.c_size_t)
    sig = {
        "csa2_status_string": ([i32], ctypes.c_char_p),
        "csa2_version": ([], i32),
        "csa2_pack_fp4": ([P, i64, i32, P, P, P], i32),
        "csa2_unpack_fp4": ([P, P, i64, i32, P, P], i32),
        "csa2_append_entry": ([P, P, P, i32, i32, i32, i64, P, P, P, P], i32),
        "csa2_pack_index_keys_fp4": ([P, i64, i32, P, P, P], i32),
        "csa2_index_topk_fp4k_workspace_size": ([i32, i32, i32, i64, i32], sz),
        "csa2_index_topk_fp4k": ([P, P, P, P, i32, i32, i32, i64, i32, P, P, sz, P], i32),
        "csa2_index_topk_workspace_size": ([i32, i32, i32, i32, i64, i32], sz),
        "csa2_index_topk": ([P, P, P, i32, i32, i32, i32, i64, i64, i32, i32, P, P, P, sz, P], i32),
        "csa2_sparse_attn_workspace_size": ([i32, i32, i32, i32, i32, i32], sz),
        "csa2_sparse_attn_decode": ([P, P, P, P, P, P, i32, i32, i32, i64, i32, i32, f32, P, P, P,
                                     sz, P], i32),
        "csa2_sparse_attn_prefill": ([P, P, P, P, P, P, i32, i32, i32, i32, i64, i32, i32, f32, P,
                                      P, P, sz, P], i32),
        "csa2_validate_modes": ([P, i32], i32),
        "csa2_group_cache_bytes": ([P, i32, i64, i64, i64, P], i32),
        "csa2_layer_group_workspace_size": ([P], sz),
        "csa2_layer_group_run": ([P, P, i32, P, P, sz, P], i32),
        "csa2_layer_run": ([P, P, i32, i32, P, P, sz, P], i32),
        "csa2_index_topk_noalloc": ([P, P, P, i32, i32, i32, i32, i64, i64, i32, i32, P, P, P],
                                    i32),
        "csa2_index_pool_workspace_size": ([i32, i32, i32, i64, i32, i32], sz),
        "csa2_index_pool": ([P, P, P, i32, i32, i32, i64, i32, i32, P, P, sz, P], i32),
        "csa2_pool_topk_workspace_size": ([i32, i32, i32], sz),
        "csa2_pool_topk": ([P, P, P, i32, i32, i32, i64, P, i32, i32, P, P, sz, P], i32),
        "csa2_stage_copies": ([P, i32, P], i32),
        "csa2_get_device_status": ([P, P], i32),
        "csa2_wait_timeout_selftest": ([i64, P], i32),
        "csa2_set_decode_kernel": ([i32], i32),
        "csa2_get_decode_kernel": ([], i32),
        "csa2_trace_enable": ([i32], i32),
        "csa2_trace_count": ([], i32),
        "csa2_trace_get": ([i32, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(f32)], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def _check(rc: int, what: str):
    if rc != CSA2_OK:
        raise CSA2Error(rc, what)


# --- torch marshalling --------------------------------------------------------

def _torch():
    import torch
    return torch


def _dev(t, name, dtype=None):
    torch = _torch()
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(device=None) -> int:
    return _torch().cuda.current_stream(device).cuda_stream


_ws_cache: Dict[int, object] = {}


def workspace(nbytes: int, device=None):
    """A cached uint8 device buffer of at least nbytes (grown on demand)."""
    torch = _torch()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < max(nbytes, 1):
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
        _ws_cache[key] = buf
    return buf


# --- staging copies -----------------------------------------------------------

def _rows_of(t, name):
    """(rows, row bytes, row stride in bytes) of a tensor whose last dim is
    contiguous and whose leading dims collapse to rows of one stride."""
    es = t.element_size()
    if t.dim() == 0:
        return 1, es, es
    if t.shape[-1] > 1 and t.stride(-1) != 1:
        raise ValueError(f"{name}: the last dim must be contiguous")
    if t.dim() == 1:
        return 1, t.shape[0] * es, t.shape[0] * es
    for i in range(t.dim() - 2):
        if t.shape[i] > 1 and t.stride(i) != t.stride(i + 1) * t.shape[i + 1]:
            raise ValueError(f"{name}: the leading dims must collapse to rows of one stride")
    rows = 1
    for n in t.shape[:-1]:
        rows *= n
    return rows, t.shape[-1] * es, t.stride(-2) * es


def stage_copies(pairs):
    """One launch copying each (src, dst) tensor pair (same shape and dtype;
    each a CUDA tensor of the current device or a pinned CPU tensor; last
    dim contiguous, leading dims collapsing to rows of one stride; 16-byte
    aligned rows), at most MAX_STAGE_COPIES pairs, on the current stream."""
    torch = _torch()
    pairs = list(pairs)
    if len(pairs) > MAX_STAGE_COPIES:
        raise ValueError(f"at most {MAX_STAGE_COPIES} copies per launch")
    arr = (Copy2D * max(len(pairs), 1))()
    for i, (src, dst) in enumerate(pairs):
        for name, t in (("src", src), ("dst", dst)):
            if not isinstance(t, torch.Tensor) or not (t.is_cuda or t.is_pinned()):
                raise TypeError(f"pairs[{i}].{name} must be a CUDA or pinned CPU tensor")
        if src.shape != dst.shape or src.dtype != dst.dtype:
            raise ValueError(f"pairs[{i}]: src and dst differ in shape or dtype")
        rows, rb, ss = _rows_of(src, f"pairs[{i}].src")
        _, _, ds = _rows_of(dst, f"pairs[{i}].dst")
        arr[i] = Copy2D(src.data_ptr(), dst.data_ptr(), rows, rb, ss, ds)
    _check(lib().csa2_stage_copies(arr, len(pairs), _stream()), "csa2_stage_copies")


# --- FP4 ----------------------------------------------------------------------

def pack_fp4(src, codes=None, scales=None) -> Tuple[object, object]:
    """fp32 [..., D] -> (uint8 [..., D/2] codes, fp32 [..., D/16] scales)."""
    torch = _torch()
    src = _dev(src, "src", torch.float32)
    D = src.shape[-1]
    rows = src.numel() // D if D else 0
    if codes is None:
        codes = torch.empty(src.shape[:-1] + (D // 2,), dtype=torch.uint8, device=src.device)
    if scales is None:
        scales = torch.empty(src.shape[:-1] + (D // 16,), dtype=torch.float32, device=src.device)
    _check(lib().csa2_pack_fp4(_ptr(src), rows, D, _ptr(codes), _ptr(scales), _stream()),
           "csa2_pack_fp4")
    return codes, scales


def append_entry(src, key, pos, codes, scales, k_idx):
    """One decode step's entry append, in place: for each sequence b with
    pos[b] >= 0, src[b] (fp32 [B, D]) packed to FP4 into row pos[b] of
    codes [B, N, D/2] / scales [B, N, D/16] and key[b] (int8 [B, d_I]) into
    row pos[b] of k_idx [B, N, d_I]; pos is int64 [B] on the device."""
    torch = _torch()
    src = _dev(src, "src", torch.float32)
    key = _dev(key, "key", torch.int8)
    pos = _dev(pos, "pos", torch.int64)
    codes = _dev(codes, "codes", torch.uint8)
    scales = _dev(scales, "scales", torch.float32)
    k_idx = _dev(k_idx, "k_idx", torch.int8)
    B, D = src.shape
    d_I = key.shape[1]
    N = codes.shape[1]
    _check(lib().csa2_append_entry(_ptr(src), _ptr(key), _ptr(pos), B, D, d_I, N, _ptr(codes),
                                   _ptr(scales), _ptr(k_idx), _stream()), "csa2_append_entry")


def unpack_fp4(codes, scales, D: int, out=None):
    torch = _torch()
    codes = _dev(codes, "codes", torch.uint8)
    scales = _dev(scales, "scales", torch.float32)
    rows = codes.numel() // (D // 2)
    if out is None:
        out = torch.empty(codes.shape[:-1] + (D,), dtype=torch.float32, device=codes.device)
    _check(lib().csa2_unpack_fp4(_ptr(codes), _ptr(scales), rows, D, _ptr(out), _stream()),
           "csa2_unpack_fp4")
    return out


# --- indexer + top-k ----------------------------------------------------------

def index_topk_workspace_size(B, T, H_I, d_I, N, topk) -> int:
    return int(lib().csa2_index_topk_workspace_size(B, T, H_I, d_I, N, topk))


def index_topk(q_idx, w, k_idx, topk: int, n_prior: int = -1, ratio: int = 4, idx_out=None,
               want_scores: bool = False, ws=None):
    """q_idx int8 [B,T,H_I,d_I], w fp32 [B,T,H_I], k_idx int8 [B,N,d_I] ->
    idx int32 [B,T,topk] (and fp32 scores [B,T,N] when want_scores)."""
    torch = _torch()
    q_idx = _dev(q_idx, "q_idx", torch.int8)
    w = _dev(w, "w", torch.float32)
    k_idx = _dev(k_idx, "k_idx", torch.int8)
    B, T, H_I, d_I = q_idx.shape
    N = k_idx.shape[1]
    if idx_out is None:
        idx_out = torch.empty((B, T, topk), dtype=torch.int32, device=q_idx.device)
    scores = (torch.empty((B, T, N), dtype=torch.float32, device=q_idx.device)
              if want_scores else None)
    need = index_topk_workspace_size(B, T, H_I, d_I, N, topk)
    if ws is None:
        ws = workspace(need)
    _check(lib().csa2_index_topk(_ptr(q_idx), _ptr(w), _ptr(k_idx), B, T, H_I, d_I, N, n_prior,
                                 ratio, topk, _ptr(idx_out), _ptr(scores), _ptr(ws), ws.numel(),
                                 _stream()), "csa2_index_topk")
    return (idx_out, scores) if want_scores else idx_out


# --- FP4 index keys -----------------------------------------------------------

def pack_index_keys_fp4(src, codes=None, exps=None):
    """fp32 [..., d_I] -> (uint8 [..., d_I/2] E2M1 codes, uint8 [..., d_I/32]
    biased block exponents): FP4 index keys with one power-of-two scale per
    32 elements."""
    torch = _torch()
    src = _dev(src, "src", torch.float32)
    d_I = src.shape[-1]
    rows = src.numel() // d_I if d_I else 0
    if codes is None:
        codes = torch.empty(src.shape[:-1] + (d_I // 2,), dtype=torch.uint8, device=src.device)
    if exps is None:
        exps = torch.empty(src.shape[:-1] + (d_I // 32,), dtype=torch.uint8, device=src.device)
    _check(lib().csa2_pack_index_keys_fp4(_ptr(src), rows, d_I, _ptr(codes), _ptr(exps),
                                          _stream()), "csa2_pack_index_keys_fp4")
    return codes, exps


def index_topk_fp4k(q_idx, w, codes, exps, topk: int, idx_out=None, ws=None):
    """Decode rows over FP4 index keys: q_idx int8 [B,H_I,d_I] (or
    [B,1,H_I,d_I]), w fp32 [B,H_I], codes uint8 [B,N,d_I/2], exps uint8
    [B,N,d_I/32] -> idx int32 [B, topk]."""
    torch = _torch()
    q_idx = _dev(q_idx, "q_idx", torch.int8)
    w = _dev(w, "w", torch.float32)
    codes = _dev(codes, "codes", torch.uint8)
    exps = _dev(exps, "exps", torch.uint8)
    B = q_idx.shape[0]
    H_I, d_I = q_idx.shape[-2:]
    N = codes.shape[1]
    if idx_out is None:
        idx_out = torch.empty((B, topk), dtype=torch.int32, device=q_idx.device)
    if ws is None:
        ws = workspace(int(lib().csa2_index_topk_fp4k_workspace_size(B, H_I, d_I, N, topk)))
    _check(lib().csa2_index_topk_fp4k(_ptr(q_idx), _ptr(w), _ptr(codes), _ptr(exps), B, H_I, d_I,
                                      N, topk, _ptr(idx_out), _ptr(ws), ws.numel(), _stream()),
           "csa2_index_topk_fp4k")
    return idx_out


# --- hierarchical indexer -----------------------------------------------------

def index_pool_workspace_size(B, H_I, d_I, N, block, n_blocks) -> int:
    return int(lib().csa2_index_pool_workspace_size(B, H_I, d_I, N, block, n_blocks))


def index_pool(q_idx, w, k_idx, block: int = 8, n_blocks: int = 2048, ws=None):
    """Candidate pool of each sequence's Full-layer query: q_idx int8
    [B,H_I,d_I], w fp32 [B,H_I], k_idx int8 [B,N,d_I] -> int32
    [B, n_blocks*block] positions ascending, then -1."""
    torch = _torch()
    q_idx = _dev(q_idx, "q_idx", torch.int8)
    w = _dev(w, "w", torch.float32)
    k_idx = _dev(k_idx, "k_idx", torch.int8)
    B, H_I, d_I = q_idx.shape
    N = k_idx.shape[1]
    pool = torch.empty((B, n_blocks * block), dtype=torch.int32, device=q_idx.device)
    if ws is None:
        ws = workspace(index_pool_workspace_size(B, H_I, d_I, N, block, n_blocks))
    _check(lib().csa2_index_pool(_ptr(q_idx), _ptr(w), _ptr(k_idx), B, H_I, d_I, N, block,
                                 n_blocks, _ptr(pool), _ptr(ws), ws.numel(), _stream()),
           "csa2_index_pool")
    return pool


def pool_topk_workspace_size(B, P, topk) -> int:
    return int(lib().csa2_pool_topk_workspace_size(B, P, topk))


def pool_topk(q_idx, w, k_idx, pool, topk: int, ws=None):
    """Top-k of each sequence's query within its pool (int32 [B, P],
    positions ascending then -1) -> int32 [B, topk] positions ascending,
    then -1."""
    torch = _torch()
    q_idx = _dev(q_idx, "q_idx", torch.int8)
    w = _dev(w, "w", torch.float32)
    k_idx = _dev(k_idx, "k_idx", torch.int8)
    pool = _dev(pool, "pool", torch.int32)
    B, H_I, d_I = q_idx.shape
    N = k_idx.shape[1]
    P = pool.shape[1]
    out = torch.empty((B, topk), dtype=torch.int32, device=q_idx.device)
    if ws is None:
        ws = workspace(pool_topk_workspace_size(B, P, topk))
    _check(lib().csa2_pool_topk(_ptr(q_idx), _ptr(w), _ptr(k_idx), B, H_I, d_I, N, _ptr(pool), P,
                                topk, _ptr(out), _ptr(ws), ws.numel(), _stream()),
           "csa2_pool_topk")
    return out


# --- attention ----------------------------------------------------------------

def sparse_attn_workspace_size(B, T, H, D, topk, W) -> int:
    return int(lib().csa2_sparse_attn_workspace_size(B, T, H, D, topk, W))


def _attn_common(q, codes, scales, idx, win_k, win_v):
    torch = _torch()
    q = _dev(q, "q", torch.bfloat16)
    codes = _dev(codes, "codes", torch.uint8)
    scales = _dev(scales, "scales", torch.float32)
    idx = _dev(idx, "idx", torch.int32)
    win_k = _dev(win_k, "win_k", torch.bfloat16)
    win_v = _dev(win_v, "win_v", torch.bfloat16)
    return q, codes, scales, idx, win_k, win_v


def sparse_attn_decode(q, codes, scales, idx, win_k, win_v, sm_scale: Optional[float] = None,
                       out=None, lse=None, ws=None):
    """q bf16 [B,H,D]; codes u8 [B,N,D/2]; scales fp32 [B,N,D/16]; idx int32
    [B,topk]; win_k/win_v bf16 [B,W,D] (or None) -> (out fp32 [B,H,D], lse fp32 [B,H])."""
    torch = _torch()
    q, codes, scales, idx, win_k, win_v = _attn_common(q, codes, scales, idx, win_k, win_v)
    B, H, D = q.shape
    N = codes.shape[1]
    topk = idx.shape[-1]
    W = 0 if win_k is None else win_k.shape[1]
    sm_scale = 1.0 / math.sqrt(D) if sm_scale is None else sm_scale
    if out is None:
        out = torch.empty((B, H, D), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    need = sparse_attn_workspace_size(B, 1, H, D, topk, W)
    if ws is None:
        ws = workspace(need)
    _check(lib().csa2_sparse_attn_decode(_ptr(q), _ptr(codes), _ptr(scales), _ptr(idx),
                                         _ptr(win_k), _ptr(win_v), B, H, D, N, topk, W,
                                         sm_scale, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                         _stream()), "csa2_sparse_attn_decode")
    return out, lse


def sparse_attn_prefill(q, codes, scales, idx, win_k, win_v, sm_scale: Optional[float] = None,
                        out=None, lse=None, ws=None):
    """q bf16 [B,T,H,D]; idx int32 [B,T,topk]; win_k/win_v bf16 [B,W-1+T,D]
    -> (out fp32 [B,T,H,D], lse fp32 [B,T,H])."""
    torch = _torch()
    q, codes, scales, idx, win_k, win_v = _attn_common(q, codes, scales, idx, win_k, win_v)
    B, T, H, D = q.shape
    N = codes.shape[1]
    topk = idx.shape[-1]
    W = 0 if win_k is None else win_k.shape[1] - T + 1
    sm_scale = 1.0 / math.sqrt(D) if sm_scale is None else sm_scale
    if out is None:
        out = torch.empty((B, T, H, D), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, T, H), dtype=torch.float32, device=q.device)
    need = sparse_attn_workspace_size(B, T, H, D, topk, W)
    if ws is None:
        ws = workspace(need)
    _check(lib().csa2_sparse_attn_prefill(_ptr(q), _ptr(codes), _ptr(scales), _ptr(idx),
                                          _ptr(win_k), _ptr(win_v), B, T, H, D, N, topk, W,
                                          sm_scale, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                          _stream()), "csa2_sparse_attn_prefill")
    return out, lse


# --- cross-layer groups ---------------------------------------------------------

def _modes_array(modes: Sequence[Tuple[int, int, int]]):
    arr = (LayerMode * len(modes))()
    for i, (m, kv, ix) in enumerate(modes):
        arr[i].mode, arr[i].kv_src, arr[i].idx_src = m, kv, ix
    return arr


def validate_modes(modes) -> bool:
    arr = _modes_array(modes)
    return lib().csa2_validate_modes(arr, len(modes)) == CSA2_OK


def group_cache_bytes(modes, entries: int, numbers_per_entry: int, bits_per_number: int) -> int:
    arr = _modes_array(modes)
    out = ctypes.c_uint64(0)
    _check(lib().csa2_group_cache_bytes(arr, len(modes), entries, numbers_per_entry,
                                        bits_per_number, ctypes.byref(out)),
           "csa2_group_cache_bytes")
    return int(out.value)


def make_dims(B, T, H, D, N, H_I, d_I, topk, W, n_prior=-1, ratio=4, sm_scale=None,
              pool_block=0, pool_blocks=0) -> Dims:
    return Dims(B, T, H, D, N, H_I, d_I, topk, W, n_prior, ratio,
                1.0 / math.sqrt(D) if sm_scale is None else sm_scale, pool_block, pool_blocks)


def layer_group_workspace_size(dims: Dims) -> int:
    return int(lib().csa2_layer_group_workspace_size(ctypes.byref(dims)))


def layer_group_run(modes, layers: List[dict], dims: Dims, ws=None):
    """Run a mode table.  ``layers[l]`` holds the layer's device tensors
    (q, q_idx, w, win_k, win_v, idx, out, lse and, for Full layers, codes,
    scales, k_idx)."""
    arr = _modes_array(modes)
    io = (LayerIO * len(layers))()
    for i, lay in enumerate(layers):
        for name, _ in LayerIO._fields_:
            t = lay.get(name)
            if t is not None:
                _dev(t, f"layers[{i}].{name}")
            setattr(io[i], name, _ptr(t))
    need = layer_group_workspace_size(dims)
    if ws is None:
        ws = workspace(need)
    _check(lib().csa2_layer_group_run(arr, io, len(layers), ctypes.byref(dims), _ptr(ws),
                                      ws.numel(), _stream()), "csa2_layer_group_run")


class LayerGroup:
    """A mode table with its layers' device tensors, marshalled once, so a
    layer (or the whole group) can be launched repeatedly with one C call
    (e.g. inside CUDA graph capture)."""

    def __init__(self, modes, layers: List[dict], dims: Dims, ws=None):
        self.modes = _modes_array(modes)
        self.L = len(layers)
        self.layers = layers
        self.io = (LayerIO * self.L)()
        for i, lay in enumerate(layers):
            for name, _ in LayerIO._fields_:
                t = lay.get(name)
                if t is not None:
                    _dev(t, f"layers[{i}].{name}")
                setattr(self.io[i], name, _ptr(t))
        self.dims = dims
        need = layer_group_workspace_size(dims)
        self.ws = workspace(need) if ws is None else ws

    def run_layer(self, layer: int):
        _check(lib().csa2_layer_run(self.modes, self.io, self.L, layer, ctypes.byref(self.dims),
                                    _ptr(self.ws), self.ws.numel(), _stream()), "csa2_layer_run")

    def run(self):
        _check(lib().csa2_layer_group_run(self.modes, self.io, self.L, ctypes.byref(self.dims),
                                          _ptr(self.ws), self.ws.numel(), _stream()),
               "csa2_layer_group_run")


def set_decode_kernel(kernel: int):
    """DECODE_SCAN_CLUSTER (default) or DECODE_FUSED: which kernels serve
    decode rows (process-wide)."""
    _check(lib().csa2_set_decode_kernel(kernel), "csa2_set_decode_kernel")


def get_decode_kernel() -> int:
    return int(lib().csa2_get_decode_kernel())


def get_device_status() -> int:
    code = ctypes.c_int32(0)
    rc = lib().csa2_get_device_status(_stream(), ctypes.byref(code))
    if rc not in (CSA2_OK, CSA2_ERR_DEVICE_STATUS):
        raise CSA2Error(rc, "csa2_get_device_status")
    return int(code.value)


# --- kernel timing trace -----------------------------------------------------------

def trace_enable(on: bool = True):
    _check(lib().csa2_trace_enable(1 if on else 0), "csa2_trace_enable")


def trace_records() -> List[Tuple[str, float]]:
    """(kernel name, device ms) of every launch recorded since trace_enable."""
    out = []
    name = ctypes.c_char_p()
    ms = ctypes.c_float()
    for i in range(lib().csa2_trace_count()):
        _check(lib().csa2_trace_get(i, ctypes.byref(name), ctypes.byref(ms)), "csa2_trace_get")
        out.append((name.value.decode(), float(ms.value)))
    return out
