"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching a device. These
run without a GPU (no kernel is launched)."""
import ctypes
import os
import re

import pytest

import sparse_attention_long_fp8_b200 as dsa
from sparse_attention_long_fp8_b200 import build as dsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


@pytest.fixture(scope="module")
def lib():
    dsa_build.build()
    return dsa.load_library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_]+)\s*\(", text)))


def test_header_declares_the_path_calls():
    names = _declared_functions()
    for n in ("dsa_indexer_scores", "dsa_indexer_topk", "dsa_topk", "dsa_sparse_attn", "dsa_forward",
              "dsa_workspace_size", "dsa_check", "dsa_status_string", "dsa_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def _shape(**kw):
    cfg = dsa.custom_config("prefill_4k", **kw) if kw else dsa.CONFIGS["prefill_4k"]
    return dsa.shape_of(cfg)


FAKE = 0x100000  # never dereferenced: validation fails before any launch


def _call_indexer(lib, shape, rb=0, re_=16, ptrs=None, flags=0):
    p = ptrs or [FAKE] * 5
    return lib.dsa_indexer_scores(ctypes.byref(shape) if shape is not None else None,
                                  p[0], p[1], p[2], p[3], p[4], None, None, rb, re_, flags,
                                  FAKE, None)


def test_indexer_topk_rejects_unsupported_shapes_before_launch(lib):
    tiny = dsa.shape_of(dsa.CONFIGS["tiny"])
    st = lib.dsa_indexer_topk(ctypes.byref(tiny), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 0, 16,
                              FAKE, None)
    assert st == dsa.DSA_ERR_UNSUPPORTED
    big_k = _shape(topk=4096)
    st = lib.dsa_indexer_topk(ctypes.byref(big_k), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 0, 16,
                              FAKE, None)
    assert st == dsa.DSA_ERR_UNSUPPORTED
    ok_shape = _shape()
    st = lib.dsa_indexer_topk(ctypes.byref(ok_shape), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 5, 5,
                              FAKE, None)
    assert st == dsa.DSA_ERR_INVALID_ARG


def test_selftest_rejects_bad_limit_before_launch(lib):
    assert lib.dsa_selftest_wait_timeout(0, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_selftest_wait_timeout(10001, None) == dsa.DSA_ERR_INVALID_ARG


def test_quantiser_argument_checks(lib):
    assert lib.dsa_quantize_e4m3(16, 96, FAKE, FAKE, FAKE, None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_quantize_e4m3(-1, 128, FAKE, FAKE, FAKE, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_quantize_e4m3(16, 128, None, FAKE, FAKE, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_quantize_e4m3(16, 128, FAKE + 2, FAKE, FAKE, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_quantize_e4m3(0, 128, FAKE, FAKE, FAKE, None) == dsa.DSA_OK


def test_status_strings(lib):
    for st in range(7):
        assert lib.dsa_status_string(st)
    assert lib.dsa_version().decode().count(".") == 2


def test_null_shape_is_invalid(lib):
    assert _call_indexer(lib, None) == dsa.DSA_ERR_INVALID_ARG
    assert b"shape" in lib.dsa_last_error()


def test_null_pointer_is_invalid(lib):
    st = _call_indexer(lib, _shape(), ptrs=[FAKE, None, FAKE, FAKE, FAKE])
    assert st == dsa.DSA_ERR_INVALID_ARG


@pytest.mark.parametrize("rb,re_", [(-1, 4), (5, 5), (10, 4), (0, 4097)])
def test_bad_row_range(lib, rb, re_):
    assert _call_indexer(lib, _shape(), rb, re_) == dsa.DSA_ERR_INVALID_ARG


def test_unknown_flags(lib):
    assert _call_indexer(lib, _shape(), flags=2) == dsa.DSA_ERR_INVALID_ARG


def test_misaligned_fp8_pointer(lib):
    st = _call_indexer(lib, _shape(), ptrs=[FAKE + 8, FAKE, FAKE, FAKE, FAKE])
    assert st == dsa.DSA_ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [dict(idx_heads=32), dict(idx_dim=64), dict(idx_heads=4)])
def test_unsupported_indexer_shape(lib, kw):
    assert _call_indexer(lib, _shape(**kw)) == dsa.DSA_ERR_UNSUPPORTED


@pytest.mark.parametrize("kw,status", [
    (dict(topk=0), dsa.DSA_ERR_INVALID_ARG),
    (dict(heads=129), dsa.DSA_ERR_UNSUPPORTED),
    (dict(qk_dim=128), dsa.DSA_ERR_UNSUPPORTED),
    (dict(v_dim=256), dsa.DSA_ERR_UNSUPPORTED),
    (dict(n_q=0), dsa.DSA_ERR_INVALID_ARG),
    (dict(batch=0), dsa.DSA_ERR_INVALID_ARG),
])
def test_attention_shape_checks(lib, kw, status):
    shape = _shape(**kw)
    n = ctypes.c_size_t(0)
    assert lib.dsa_workspace_size(ctypes.byref(shape), dsa.DSA_OP_SPARSE_ATTN, ctypes.byref(n)) == status
    st = lib.dsa_sparse_attn(ctypes.byref(shape), FAKE, FAKE, FAKE, FAKE, 0, None, None, 0, None)
    assert st == status


def test_bad_out_dtype_and_workspace(lib):
    shape = _shape()
    assert lib.dsa_sparse_attn(ctypes.byref(shape), FAKE, FAKE, FAKE, FAKE, 7, None, None, 0,
                               None) == dsa.DSA_ERR_INVALID_ARG
    dec = dsa.shape_of(dsa.CONFIGS["decode_32k"])   # the two-pass plan needs a score buffer
    st = lib.dsa_forward(ctypes.byref(dec), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE,
                         FAKE, FAKE, FAKE, 0, None, None, 0, None)
    assert st == dsa.DSA_ERR_WORKSPACE


def test_workspace_sizes(lib):
    # prefill: scores and selection are fused, so no score buffer and no
    # split-K partials
    assert dsa.workspace_size(_shape(), dsa.DSA_OP_FORWARD) == 0
    assert dsa.workspace_size(_shape(), dsa.DSA_OP_SPARSE_ATTN) == 0
    assert dsa.workspace_size(_shape(), dsa.DSA_OP_TOPK) == 0
    big = dsa.shape_of(dsa.CONFIGS["prefill_64k"])
    assert dsa.workspace_size(big, dsa.DSA_OP_FORWARD) == 0
    assert dsa.forward_chunk_rows(big) == 65536
    # decode (64 query groups < SMs): the split score kernel writes one chunk
    # of 64 x 32768 fp32 scores, then the separate selection runs
    dec = dsa.shape_of(dsa.CONFIGS["decode_32k"])
    assert dsa.workspace_size(dec, dsa.DSA_OP_FORWARD) >= 64 * 32768 * 4
    # the tiny shape is not supported by the fused kernel: two passes
    tiny = dsa.shape_of(dsa.CONFIGS["tiny"])
    assert dsa.workspace_size(tiny, dsa.DSA_OP_FORWARD) == 256 * 256 * 4
    # a handful of rows: split-K partials are needed
    few = _shape(n_q=4)
    assert dsa.workspace_size(few, dsa.DSA_OP_SPARSE_ATTN) > 0
    with pytest.raises(dsa.DsaError):
        dsa.workspace_size(_shape(), 9)


def test_valid_call_without_device_reports_no_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = _call_indexer(lib, _shape())
    assert st == dsa.DSA_ERR_NO_DEVICE


def _layout(page, max_pages, pool_rows, table=FAKE, row_pos=None):
    lay = dsa.DsaLayout()
    lay.row_pos = row_pos
    lay.block_table = table
    lay.max_pages = max_pages
    lay.page_size = page
    lay.pool_rows = pool_rows
    return lay


@pytest.mark.parametrize("page,max_pages,pool_rows,table", [
    (100, 64, 64 * 100, FAKE),          # not a power of two
    (64, 128, 64 * 128, FAKE),          # below one indexer tile
    (256, 15, 256 * 64, FAKE),          # 4096 keys need 16 pages
    (256, 16, 256 * 64 + 3, FAKE),      # pool not a whole number of pages
    (256, 16, 1 << 31, FAKE),           # pool past the 32-bit TMA coordinate
    (256, 16, 256 * 64, FAKE + 2),      # misaligned table
])
def test_paged_layout_checks_before_launch(lib, page, max_pages, pool_rows, table):
    lay = _layout(page, max_pages, pool_rows, table)
    st = lib.dsa_forward_ex(ctypes.byref(_shape()), ctypes.byref(lay), FAKE, FAKE, FAKE, FAKE,
                            FAKE, None, None, FAKE, FAKE, FAKE, FAKE, 0, None, None, 0, None)
    assert st == dsa.DSA_ERR_INVALID_ARG
    st = lib.dsa_sparse_attn_ex(ctypes.byref(_shape()), ctypes.byref(lay), FAKE, FAKE, FAKE, FAKE,
                                0, None, None, 0, None)
    assert st == dsa.DSA_ERR_INVALID_ARG


def test_row_pos_alignment_checked(lib):
    lay = _layout(0, 0, 0, table=None, row_pos=FAKE + 2)
    st = lib.dsa_indexer_scores_ex(ctypes.byref(_shape()), ctypes.byref(lay), FAKE, FAKE, FAKE,
                                   FAKE, FAKE, None, None, 0, 16, 0, FAKE, None)
    assert st == dsa.DSA_ERR_INVALID_ARG


def test_forward_plan_query(lib):
    assert dsa.forward_plan(_shape()) == {"fused": True, "chunk_rows": 4096, "attn_splits": 1}
    dec = dsa.forward_plan(dsa.shape_of(dsa.CONFIGS["decode_32k"]))
    assert dec["fused"] is False and dec["chunk_rows"] == 1
