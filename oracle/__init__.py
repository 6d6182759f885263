"""CSA2 CPU oracle -- test infrastructure, not part of the product.

A thin numpy/ctypes wrapper over ``csa2_oracle.c`` (plain C, fp64
attention) plus the per-layer mode-table walk.  Only the test suite,
``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import this package.  The CUDA library never imports,
links or calls it; the two share no code.

Citations (page title, section) are on each function of the C source; the
mode walk below follows "DeepSeek-V4.1-Flash", section "Sharing the cache
across layers" (Full: own entries and selection; Reindex: another layer's
entries, fresh selection; Reuse: another layer's entries and selection;
every layer keeps its own queries and local window).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa2_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

OK, EINVAL, ENOMEM, ERANGE = 0, 1, 2, 3
FULL, REINDEX, REUSE = 0, 1, 2
# A Reindex layer that searches only its Full source's candidate pool
# ("Inference-Efficient LLMs", section 5: later Reindex layers search within
# the pool an earlier Full layer kept).  Same table rules as REINDEX.
REINDEX_POOL = 3


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fused multiply-add, no fast math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
           "-fexcess-precision=standard", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float
        lib.orc_e2m1_value.argtypes = [ctypes.c_uint32]
        lib.orc_e2m1_value.restype = f32
        lib.orc_e2m1_round_mag.argtypes = [f32]
        lib.orc_e2m1_round_mag.restype = ctypes.c_uint32
        lib.orc_pack_fp4.argtypes = [P, i64, i32, P, P]
        lib.orc_unpack_fp4.argtypes = [P, P, i64, i32, P]
        lib.orc_index_score_row.argtypes = [P, P, P, i32, i32, i64, P]
        lib.orc_index_score_row.restype = None
        lib.orc_visible_count.argtypes = [i64, i64, i32, i64]
        lib.orc_visible_count.restype = i64
        lib.orc_topk_row.argtypes = [P, i64, i32, P]
        lib.orc_index_topk.argtypes = [P, P, P, i32, i32, i32, i32, i64, i64, i32, i32, P, i64,
                                       P, P]
        lib.orc_sparse_attn.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i64, i32, i32, f32,
                                        P, i64, P, P]
        lib.orc_validate_modes.argtypes = [P, i32]
        lib.orc_group_cache_bytes.argtypes = [P, i32, i64, i64, i64, P]
        lib.orc_block_pool.argtypes = [P, i64, i32, i32, P, P]
        lib.orc_pool_topk.argtypes = [P, P, P, i32, i32, i64, P, i64, i32, P]
        lib.orc_append_entry.argtypes = [P, P, P, i32, i32, i32, i64, P, P, P]
        lib.orc_pack_mxfp4.argtypes = [P, i64, i32, P, P]
        lib.orc_unpack_mxfp4.argtypes = [P, P, i64, i32, P]
        lib.orc_index_score_fp4k_row.argtypes = [P, P, P, P, i32, i32, i64, P]
        lib.orc_index_score_fp4k_row.restype = None
        lib.orc_index_topk_fp4k.argtypes = [P, P, P, P, i32, i32, i32, i64, i32, P, P]
        for name in ("orc_pack_fp4", "orc_unpack_fp4", "orc_topk_row", "orc_index_topk",
                     "orc_sparse_attn", "orc_validate_modes", "orc_group_cache_bytes",
                     "orc_block_pool", "orc_pool_topk", "orc_append_entry",
                     "orc_pack_mxfp4", "orc_unpack_mxfp4", "orc_index_topk_fp4k"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    pass


def _check(rc, what):
    if rc != OK:
        raise OracleError(f"{what} failed with oracle status {rc}")


# --- FP4 --------------------------------------------------------------------

def e2m1_value(code: int) -> float:
    return float(_load().orc_e2m1_value(code))


def e2m1_round_mag(y: float) -> int:
    return int(_load().orc_e2m1_round_mag(y))


def pack_fp4(src: np.ndarray):
    """fp32 [rows, D] -> (codes u8 [rows, D/2], scales fp32 [rows, D/16])."""
    src = _c(src, np.float32)
    rows, D = src.shape
    codes = np.zeros((rows, D // 2), np.uint8)
    scales = np.zeros((rows, max(D // 16, 0)), np.float32)
    _check(_load().orc_pack_fp4(_ptr(src), rows, D, _ptr(codes), _ptr(scales)), "pack_fp4")
    return codes, scales


def unpack_fp4(codes: np.ndarray, scales: np.ndarray, D: int) -> np.ndarray:
    codes = _c(codes, np.uint8).reshape(-1, D // 2)
    scales = _c(scales, np.float32).reshape(-1, D // 16)
    out = np.empty((codes.shape[0], D), np.float32)
    _check(_load().orc_unpack_fp4(_ptr(codes), _ptr(scales), codes.shape[0], D, _ptr(out)),
           "unpack_fp4")
    return out


def append_entry(src, key, pos, codes, scales, k_idx):
    """One decode step's entry append, in place: for each sequence b with
    pos[b] >= 0, src[b] (fp32 [D]) packed to FP4 into row pos[b] of codes
    [B, N, D/2] / scales [B, N, D/16], and key[b] (int8 [d_I]) into row
    pos[b] of k_idx [B, N, d_I].  The arrays must be C-contiguous numpy
    arrays of those dtypes (they are modified)."""
    src, key, pos = _c(src, np.float32), _c(key, np.int8), _c(pos, np.int64)
    B, D = src.shape
    d_I = key.shape[1]
    N = codes.shape[1]
    for a, dt in ((codes, np.uint8), (scales, np.float32), (k_idx, np.int8)):
        if a.dtype != dt or not a.flags["C_CONTIGUOUS"]:
            raise OracleError("append_entry: stores must be C-contiguous arrays of their dtype")
    _check(_load().orc_append_entry(_ptr(src), _ptr(key), _ptr(pos), B, D, d_I, N, _ptr(codes),
                                    _ptr(scales), _ptr(k_idx)), "append_entry")


# --- indexer + top-k --------------------------------------------------------

def index_score_row(q: np.ndarray, w: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """q int8 [H_I, d_I], w fp32 [H_I], keys int8 [N, d_I] -> fp32 [N]."""
    q, w, keys = _c(q, np.int8), _c(w, np.float32), _c(keys, np.int8)
    H_I, d_I = q.shape
    N = keys.shape[0]
    out = np.empty(N, np.float32)
    _load().orc_index_score_row(_ptr(q), _ptr(w), _ptr(keys), H_I, d_I, N, _ptr(out))
    return out


def visible_count(N: int, n_prior: int, ratio: int, t: int) -> int:
    return int(_load().orc_visible_count(N, n_prior, ratio, t))


def topk_row(scores: np.ndarray, k: int) -> np.ndarray:
    scores = _c(scores, np.float32)
    out = np.empty(k, np.int32)
    _check(_load().orc_topk_row(_ptr(scores), scores.shape[0], k, _ptr(out)), "topk_row")
    return out


def index_topk(q_idx, w, k_idx, topk, n_prior=-1, ratio=4, rows=None, want_scores=False):
    """q_idx int8 [B,T,H_I,d_I], w fp32 [B,T,H_I], k_idx int8 [B,N,d_I].

    Returns idx int32 [nrows, topk] (and scores fp32 [nrows, N] with -inf
    where a row may not see the entry) for the flattened rows b*T+t given
    in ``rows`` (all rows when None).
    """
    q_idx, w, k_idx = _c(q_idx, np.int8), _c(w, np.float32), _c(k_idx, np.int8)
    B, T, H_I, d_I = q_idx.shape
    N = k_idx.shape[1]
    rows_arr = None if rows is None else _c(rows, np.int64)
    nrows = B * T if rows is None else rows_arr.shape[0]
    idx = np.empty((nrows, topk), np.int32)
    scores = np.empty((nrows, N), np.float32) if want_scores else None
    _check(_load().orc_index_topk(_ptr(q_idx), _ptr(w), _ptr(k_idx), B, T, H_I, d_I, N, n_prior,
                                  ratio, topk, _ptr(rows_arr), nrows, _ptr(idx), _ptr(scores)),
           "index_topk")
    return (idx, scores) if want_scores else idx


# --- FP4 index keys (E2M1 with a power-of-two scale per 32 elements) ------------

def pack_mxfp4(src: np.ndarray):
    """fp32 [rows, d] -> (codes u8 [rows, d/2], biased exponents u8 [rows, d/32])."""
    src = _c(src, np.float32)
    rows, d = src.shape
    codes = np.zeros((rows, d // 2), np.uint8)
    exps = np.zeros((rows, d // 32), np.uint8)
    _check(_load().orc_pack_mxfp4(_ptr(src), rows, d, _ptr(codes), _ptr(exps)), "pack_mxfp4")
    return codes, exps


def unpack_mxfp4(codes: np.ndarray, exps: np.ndarray, d: int) -> np.ndarray:
    codes = _c(codes, np.uint8).reshape(-1, d // 2)
    exps = _c(exps, np.uint8).reshape(-1, d // 32)
    out = np.empty((codes.shape[0], d), np.float32)
    _check(_load().orc_unpack_mxfp4(_ptr(codes), _ptr(exps), codes.shape[0], d, _ptr(out)),
           "unpack_mxfp4")
    return out


def index_score_fp4k_row(q, w, codes, exps) -> np.ndarray:
    """q int8 [H_I, d_I], w fp32 [H_I], codes u8 [N, d_I/2], exps u8 [N, d_I/32] -> fp32 [N]."""
    q, w = _c(q, np.int8), _c(w, np.float32)
    codes, exps = _c(codes, np.uint8), _c(exps, np.uint8)
    H_I, d_I = q.shape
    N = codes.shape[0]
    out = np.empty(N, np.float32)
    _load().orc_index_score_fp4k_row(_ptr(q), _ptr(w), _ptr(codes), _ptr(exps), H_I, d_I, N,
                                     _ptr(out))
    return out


def index_topk_fp4k(q_idx, w, codes, exps, topk, want_scores=False):
    """Decode rows over FP4 keys: q_idx int8 [B,H_I,d_I] (or [B,1,H_I,d_I]),
    w fp32 [B,H_I], codes u8 [B,N,d_I/2], exps u8 [B,N,d_I/32] -> idx int32
    [B, topk] (and scores fp32 [B, N])."""
    q_idx = _c(q_idx, np.int8)
    B = q_idx.shape[0]
    H_I, d_I = q_idx.shape[-2:]
    q_idx = q_idx.reshape(B, H_I, d_I)
    w = _c(w, np.float32).reshape(B, H_I)
    codes, exps = _c(codes, np.uint8), _c(exps, np.uint8)
    N = codes.shape[1]
    idx = np.empty((B, topk), np.int32)
    scores = np.empty((B, N), np.float32) if want_scores else None
    _check(_load().orc_index_topk_fp4k(_ptr(q_idx), _ptr(w), _ptr(codes), _ptr(exps), B, H_I, d_I,
                                       N, topk, _ptr(idx), _ptr(scores)), "index_topk_fp4k")
    return (idx, scores) if want_scores else idx


# --- hierarchical indexer (candidate pool of a Full layer) ---------------------

def block_pool(scores: np.ndarray, block: int, n_blocks: int) -> np.ndarray:
    """A Full layer's visible scores fp32 [V] -> the pool's positions int32,
    ascending: every visible position of the n_blocks best blocks of `block`
    consecutive positions (block score = its largest score; ties to the
    lower block)."""
    scores = _c(scores, np.float32)
    out = np.empty(block * n_blocks, np.int32)
    n = np.zeros(1, np.int64)
    _check(_load().orc_block_pool(_ptr(scores), scores.shape[0], block, n_blocks, _ptr(out),
                                  _ptr(n)), "block_pool")
    return out[: int(n[0])].copy()


def pool_topk(q: np.ndarray, w: np.ndarray, keys: np.ndarray, pool: np.ndarray, k: int) -> np.ndarray:
    """One query row (q int8 [H_I, d_I], w fp32 [H_I]) over the pool's
    positions of keys int8 [N, d_I]: top-k positions, ascending, -1 padded."""
    q, w, keys, pool = _c(q, np.int8), _c(w, np.float32), _c(keys, np.int8), _c(pool, np.int32)
    H_I, d_I = q.shape
    out = np.empty(k, np.int32)
    _check(_load().orc_pool_topk(_ptr(q), _ptr(w), _ptr(keys), H_I, d_I, keys.shape[0],
                                 _ptr(pool), pool.shape[0], k, _ptr(out)), "pool_topk")
    return out


# --- attention --------------------------------------------------------------

def sparse_attn(q, codes, scales, idx, win_k, win_v, sm_scale=None, rows=None):
    """q bf16-bits uint16 [B,T,H,D]; codes u8 [B,N,D/2]; scales fp32 [B,N,D/16];
    idx int32 [B,T,topk]; win_k/win_v bf16-bits uint16 [B,W-1+T,D] or None.

    Returns (out float64 [nrows,H,D], lse float64 [nrows,H]).
    """
    q = _c(q, np.uint16)
    B, T, H, D = q.shape
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.float32)
    N = codes.shape[1]
    idx = _c(idx, np.int32)
    topk = idx.shape[-1]
    if win_k is None:
        W = 0
    else:
        win_k, win_v = _c(win_k, np.uint16), _c(win_v, np.uint16)
        W = win_k.shape[1] - T + 1
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(D)
    rows_arr = None if rows is None else _c(rows, np.int64)
    nrows = B * T if rows is None else rows_arr.shape[0]
    out = np.empty((nrows, H, D), np.float64)
    lse = np.empty((nrows, H), np.float64)
    _check(_load().orc_sparse_attn(_ptr(q), _ptr(codes), _ptr(scales), _ptr(idx), _ptr(win_k),
                                   _ptr(win_v), B, T, H, D, N, topk, W, float(sm_scale),
                                   _ptr(rows_arr), nrows, _ptr(out), _ptr(lse)),
           "sparse_attn")
    return out, lse


# --- cross-layer modes ------------------------------------------------------

def validate_modes(modes) -> bool:
    m = _c(modes, np.int32).reshape(-1, 3)
    return _load().orc_validate_modes(_ptr(m), m.shape[0]) == OK


def group_cache_bytes(modes, entries, numbers_per_entry, bits_per_number) -> int:
    m = _c(modes, np.int32).reshape(-1, 3)
    out = np.zeros(1, np.uint64)
    _check(_load().orc_group_cache_bytes(_ptr(m), m.shape[0], entries, numbers_per_entry,
                                         bits_per_number, _ptr(out)), "group_cache_bytes")
    return int(out[0])


def layer_group(modes, layers, topk, n_prior=-1, ratio=4, sm_scale=None, rows=None,
                pool=None):
    """Walk a mode table in layer order.

    ``layers[l]`` is a dict with the layer's own ``q``, ``q_idx``, ``w``,
    ``win_k``, ``win_v`` and, for a layer that keeps its own entries (Full),
    ``codes``, ``scales``, ``k_idx``.  Per layer the entry store is that of
    layer kv_src and the selection is computed (Full, Reindex: own index
    query over the store's index keys) or taken from layer idx_src (Reuse).
    A REINDEX_POOL layer (decode rows only; ``pool`` = (block, n_blocks))
    scores only the candidate pool of its kv_src Full layer -- the n_blocks
    best blocks of `block` positions by the Full layer's own index scores
    (``block_pool``) -- with its own index query and keeps their top-k
    (``pool_topk``).
    Returns a list of dicts with ``idx``, ``out``, ``lse`` and ``store`` (the
    layer id whose entries were read).
    """
    m = _c(modes, np.int32).reshape(-1, 3)
    checked = m.copy()
    checked[checked[:, 0] == REINDEX_POOL, 0] = REINDEX  # the same table rules
    if not validate_modes(checked):
        raise OracleError("invalid mode table")
    results = []
    for l, (mode, kv_src, idx_src) in enumerate(m.tolist()):
        lay = layers[l]
        store = layers[kv_src]
        B, T = lay["q"].shape[:2]
        if mode == REINDEX_POOL:
            if pool is None or n_prior >= 0 or T != 1 or rows is not None:
                raise OracleError("a pool layer needs pool=(block, n_blocks) and decode rows")
            block, n_blocks = pool
            idx = np.empty((B, 1, topk), np.int32)
            for b in range(B):
                full = index_score_row(store["q_idx"][b, 0], store["w"][b, 0], store["k_idx"][b])
                cand = block_pool(full, block, n_blocks)
                idx[b, 0] = pool_topk(lay["q_idx"][b, 0], lay["w"][b, 0], store["k_idx"][b],
                                      cand, topk)
        elif mode in (FULL, REINDEX):
            sel = index_topk(lay["q_idx"], lay["w"], store["k_idx"], topk, n_prior, ratio,
                             rows=rows)
            if rows is None:
                idx = sel.reshape(B, T, topk)
            else:  # only the sampled rows are computed; the rest stay -1
                idx = np.full((B * T, topk), -1, np.int32)
                idx[np.asarray(rows)] = sel
                idx = idx.reshape(B, T, topk)
        else:
            idx = results[idx_src]["idx"]
        out, lse = sparse_attn(lay["q"], store["codes"], store["scales"], idx, lay["win_k"],
                               lay["win_v"], sm_scale, rows)
        results.append({"idx": idx, "out": out, "lse": lse, "store": kv_src})
    return results
