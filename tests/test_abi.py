"""The C ABI loads and exports what include/csa2.h declares; host-side logic
(validation, mode tables, cache accounting, status strings) works without a
GPU.  No call here launches a kernel."""
import ctypes
import json
import os
import re

import pytest

import compressed_sparse_attention_topk_b200 as csa2
from compressed_sparse_attention_topk_b200 import build as csa2_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa2.h")


@pytest.fixture(scope="module")
def lib():
    csa2_build.build()
    return csa2.lib()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(csa2_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_functions()
    assert len(declared) >= 14
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(declared) == sorted(csa2.EXPORTED)


def test_status_strings_and_version(lib):
    for code in range(6):
        assert lib.csa2_status_string(code).startswith(b"CSA2_")
    assert lib.csa2_status_string(99) == b"unknown csa2 status"
    assert lib.csa2_version() >= 10000


def test_cache_accounting_matches_worked_example(lib):
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "cache_sharing_example.json")))
    args = (g["entries"], g["numbers_per_entry"], g["bits_per_number"])
    all_full = [(0, l, l) for l in range(g["layers"])]
    grouped = []
    for f in range(0, g["layers"], 4):
        grouped += [(0, f, f), (1, f, f + 1), (2, f, f + 1), (2, f, f + 1)]
    assert csa2.group_cache_bytes(all_full, *args) == g["bytes_every_layer_own_copy"]
    assert csa2.group_cache_bytes(grouped, *args) == g["bytes_one_copy_per_group_of_four"]


@pytest.mark.parametrize("table,ok", [
    ([(0, 0, 0)], True),
    ([(0, 0, 0), (1, 0, 1), (2, 0, 1), (2, 0, 1)], True),
    ([(0, 0, 0), (2, 0, 0)], True),
    ([(1, 0, 0)], False),
    ([(0, 0, 0), (0, 0, 1)], False),
    ([(0, 0, 0), (2, 0, 1)], False),
    ([(0, 0, 0), (1, 0, 1), (1, 1, 2)], False),
    ([(0, 0, 0), (0, 1, 1), (2, 0, 1)], False),
    ([(0, 0, 0), (2, 0, 0), (2, 0, 1)], False),
    ([(0, 0, 0), (3, 0, 0)], False),
])
def test_mode_validation_agrees_with_rules(lib, table, ok):
    assert csa2.validate_modes(table) is ok


def test_workspace_queries(lib):
    assert csa2.index_topk_workspace_size(4, 1, 4, 64, 262144, 2048) > 4 * 262144 * 12
    assert csa2.index_topk_workspace_size(4, 1, 3, 64, 262144, 2048) == 0   # H_I unsupported
    assert csa2.index_topk_workspace_size(4, 1, 4, 48, 262144, 2048) == 0   # d_I unsupported
    assert csa2.index_topk_workspace_size(4, 1, 4, 64, 1024, 0) == 0        # topk < 1


def test_invalid_arguments_rejected_before_any_launch(lib):
    P = ctypes.c_void_p
    fake = P(256)  # never dereferenced: validation fails first
    # null q_idx
    rc = lib.csa2_index_topk(None, fake, fake, 1, 1, 4, 64, 100, -1, 4, 8, fake, None, fake,
                             1 << 20, None)
    assert rc == csa2.CSA2_ERR_INVALID_ARG
    # d_I not a multiple of 16
    rc = lib.csa2_index_topk(fake, fake, fake, 1, 1, 4, 40, 100, -1, 4, 8, fake, None, fake,
                             1 << 20, None)
    assert rc == csa2.CSA2_ERR_INVALID_ARG
    # topk < 1
    rc = lib.csa2_index_topk(fake, fake, fake, 1, 1, 4, 64, 100, -1, 4, 0, fake, None, fake,
                             1 << 20, None)
    assert rc == csa2.CSA2_ERR_INVALID_ARG
    # misaligned key pointer
    rc = lib.csa2_index_topk(fake, fake, P(258), 1, 1, 4, 64, 100, -1, 4, 8, fake, None, fake,
                             1 << 20, None)
    assert rc == csa2.CSA2_ERR_INVALID_ARG
    # prefill without a ratio
    rc = lib.csa2_index_topk(fake, fake, fake, 1, 4, 4, 64, 100, 10, 0, 8, fake, None, fake,
                             1 << 20, None)
    assert rc == csa2.CSA2_ERR_INVALID_ARG
    # unsupported entry dim
    rc = lib.csa2_sparse_attn_decode(fake, fake, fake, fake, fake, fake, 1, 8, 96, 100, 8, 4,
                                     0.1, fake, fake, fake, 1 << 20, None)
    assert rc == csa2.CSA2_ERR_UNSUPPORTED
    # window requested without window pointers
    rc = lib.csa2_sparse_attn_decode(fake, fake, fake, fake, None, None, 1, 8, 128, 100, 8, 4,
                                     0.1, fake, fake, fake, 1 << 20, None)
    assert rc == csa2.CSA2_ERR_INVALID_ARG
    # pack: D not a multiple of 16
    assert lib.csa2_pack_fp4(fake, 4, 24, fake, fake, None) == csa2.CSA2_ERR_INVALID_ARG
    # empty work is a no-op
    assert lib.csa2_pack_fp4(None, 0, 64, None, None, None) == csa2.CSA2_OK
    assert lib.csa2_index_topk(None, None, None, 0, 1, 4, 64, 100, -1, 4, 8, None, None, None, 0,
                               None) == csa2.CSA2_OK


def test_group_run_rejects_bad_table_before_launch(lib):
    modes = csa2._modes_array([(0, 0, 0), (2, 0, 1)])
    io = (csa2.LayerIO * 2)()
    dims = csa2.make_dims(1, 1, 16, 128, 100, 4, 64, 8, 4)
    rc = lib.csa2_layer_group_run(modes, io, 2, ctypes.byref(dims), None, 0, None)
    assert rc == csa2.CSA2_ERR_INVALID_ARG


def test_pool_calls_validate_before_any_launch(lib):
    P = ctypes.c_void_p
    fake = P(256)
    # workspace queries: supported sizes > 0, unsupported or invalid sizes 0
    assert lib.csa2_index_pool_workspace_size(4, 4, 64, 262144, 8, 2048) > 4 * 262144 * 12
    assert lib.csa2_index_pool_workspace_size(4, 4, 64, 262144, 65, 16) == 0    # block > 64
    assert lib.csa2_index_pool_workspace_size(4, 4, 64, 262144, 8, 8193) == 0   # pool > 65,536
    assert lib.csa2_index_pool_workspace_size(4, 3, 64, 262144, 8, 2048) == 0   # H_I unsupported
    assert lib.csa2_pool_topk_workspace_size(4, 16384, 2048) > 4 * 16384 * 12
    assert lib.csa2_pool_topk_workspace_size(4, 70000, 2048) == 0
    assert lib.csa2_pool_topk_workspace_size(4, 16384, 0) == 0
    # argument checks
    rc = lib.csa2_index_pool(fake, fake, fake, 1, 4, 64, 100, 0, 4, fake, fake, 1 << 20, None)
    assert rc == csa2.CSA2_ERR_INVALID_ARG
    rc = lib.csa2_index_pool(fake, fake, fake, 1, 4, 64, 100, 128, 4, fake, fake, 1 << 20, None)
    assert rc == csa2.CSA2_ERR_UNSUPPORTED
    rc = lib.csa2_index_pool(fake, fake, P(258), 1, 4, 64, 100, 8, 4, fake, fake, 1 << 20, None)
    assert rc == csa2.CSA2_ERR_INVALID_ARG                      # misaligned keys
    rc = lib.csa2_pool_topk(fake, fake, fake, 1, 4, 64, 100, fake, 16, 0, fake, fake, 1 << 20,
                            None)
    assert rc == csa2.CSA2_ERR_INVALID_ARG                      # topk < 1
    rc = lib.csa2_pool_topk(fake, fake, fake, 1, 4, 64, 100, None, 16, 8, fake, fake, 1 << 20,
                            None)
    assert rc == csa2.CSA2_ERR_INVALID_ARG                      # no pool
    # no sequences: nothing to do
    assert lib.csa2_index_pool(None, None, None, 0, 4, 64, 100, 8, 4, None, None, 0,
                               None) == csa2.CSA2_OK
    assert lib.csa2_pool_topk(None, None, None, 0, 4, 64, 100, None, 16, 8, None, None, 0,
                              None) == csa2.CSA2_OK


def test_noalloc_refuses_by_the_documented_workspace_size(lib):
    """The allocation-free index + top-k refuses, before any launch, every
    size whose csa2_index_topk_workspace_size exceeds its 16 MiB scratch --
    including many-query shapes where only the tensor-core path's scratch
    is too large."""
    fake = ctypes.c_void_p(256)
    limit = 16 << 20
    # 512 queries over 1,000 entries: the per-row scan would need ~10 MB,
    # the tensor-core path ~17 MB
    assert csa2.index_topk_workspace_size(1, 512, 4, 64, 1000, 256) > limit
    rc = lib.csa2_index_topk_noalloc(fake, fake, fake, 1, 512, 4, 64, 1000, -1, 4, 256, fake,
                                     None, None)
    assert rc == csa2.CSA2_ERR_UNSUPPORTED
    # 4 x 1,000,000 decode entries: ~48 MB
    rc = lib.csa2_index_topk_noalloc(fake, fake, fake, 4, 1, 4, 64, 1_000_000, -1, 4, 2048,
                                     fake, None, None)
    assert rc == csa2.CSA2_ERR_UNSUPPORTED


def test_stage_copies_validate_before_any_query(lib):
    """csa2_stage_copies refuses bad counts, sizes, strides and alignment
    before it asks where a pointer lives or launches anything."""
    C = csa2.Copy2D
    ok = C(256, 512, 2, 32, 32, 64)

    def run(*copies, n=None):
        arr = (C * max(len(copies), 1))(*copies)
        return lib.csa2_stage_copies(arr, len(copies) if n is None else n, None)

    assert lib.csa2_stage_copies(None, 0, None) == csa2.CSA2_OK
    assert run(C(None, None, 0, 16, 16, 16)) == csa2.CSA2_OK          # no rows: skipped
    assert run(C(None, None, 4, 0, 16, 16)) == csa2.CSA2_OK           # empty rows: skipped
    assert lib.csa2_stage_copies(None, 1, None) == csa2.CSA2_ERR_INVALID_ARG
    assert run(ok, n=-1) == csa2.CSA2_ERR_INVALID_ARG
    assert run(*([ok] * 17)) == csa2.CSA2_ERR_INVALID_ARG             # > CSA2_MAX_STAGE_COPIES
    assert run(C(None, 512, 1, 16, 16, 16)) == csa2.CSA2_ERR_INVALID_ARG
    assert run(C(256, None, 1, 16, 16, 16)) == csa2.CSA2_ERR_INVALID_ARG
    assert run(C(264, 512, 1, 16, 16, 16)) == csa2.CSA2_ERR_INVALID_ARG  # src misaligned
    assert run(C(256, 520, 1, 16, 16, 16)) == csa2.CSA2_ERR_INVALID_ARG  # dst misaligned
    assert run(C(256, 512, 1, 24, 32, 32)) == csa2.CSA2_ERR_INVALID_ARG  # row bytes % 16
    assert run(C(256, 512, 2, 32, 40, 64)) == csa2.CSA2_ERR_INVALID_ARG  # src stride % 16
    assert run(C(256, 512, 2, 32, 32, 16)) == csa2.CSA2_ERR_INVALID_ARG  # rows overlap in dst
    assert run(C(256, 512, 2, 32, -32, 64)) == csa2.CSA2_ERR_INVALID_ARG
    assert run(C(256, 512, -1, 32, 32, 64)) == csa2.CSA2_ERR_INVALID_ARG
    assert run(ok, C(256, 512, 1, 8, 16, 16)) == csa2.CSA2_ERR_INVALID_ARG  # second copy bad


def test_stage_copies_binding_collapses_rows():
    """The binding's row view: leading dims that collapse to one stride, a
    strided slot per row, and views it must refuse."""
    import torch
    w = torch.zeros(6, 4, 128, 64, dtype=torch.bfloat16)
    assert csa2._rows_of(w[:, :, -1], "x") == (24, 128, 128 * 64 * 2)
    assert csa2._rows_of(w[2], "x") == (512, 128, 128)
    assert csa2._rows_of(torch.zeros(100, dtype=torch.uint8), "x") == (1, 100, 100)
    with pytest.raises(ValueError):
        csa2._rows_of(w[:, 1:3, -1], "x")       # dims 0 and 1 do not collapse
    with pytest.raises(ValueError):
        csa2._rows_of(w[..., ::2], "x")         # last dim not contiguous
    with pytest.raises(TypeError):
        csa2.stage_copies([(torch.zeros(16), torch.zeros(16))])  # pageable CPU tensors
