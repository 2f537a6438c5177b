"""dsa_sparse_attn_noalloc: the attention entry point for callers that cannot
call cudaMalloc (their device memory belongs to another framework's
allocator, or an allocation is not acceptable inside their decode loop), so
they cannot hand in the split-K workspace dsa_sparse_attn asks for. It must
give what the workspace entry point gives, call after call, even though
every call reuses the same static scratch array inside the library.

Both entry points run the same kernels with the same split plan, so their
results must be identical bit for bit.

This file is collected last on purpose: a run that stops at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import sparse_attention_long_fp8_b200 as dsa
from sparse_attention_long_fp8_b200 import inputs as dsa_inputs

pytestmark = pytest.mark.gpu

NOALLOC_SCRATCH_BYTES = 16 << 20


def _case(seed, n_rows):
    cfg = dsa_inputs.custom_config("prefill_4k", n_q=n_rows, name=f"noalloc{n_rows}")
    inp = dsa_inputs.make_inputs(cfg, seed=seed)
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, cfg.n_kv, size=(n_rows, cfg.topk)).astype(np.int32)
    idx[rng.random(idx.shape) < 0.1] = -1
    return cfg, inp["q"].cuda(), inp["kv"].cuda(), torch.from_numpy(idx)[None].cuda()


def _noalloc_via_abi(shape, q, kv, idx, out, lse):
    lib = dsa.load_library()
    out_dtype = dsa.DSA_OUT_BF16 if out.dtype == torch.bfloat16 else dsa.DSA_OUT_F32
    return lib.dsa_sparse_attn_noalloc(ctypes.byref(shape), q.data_ptr(), kv.data_ptr(),
                                       idx.data_ptr(), out.data_ptr(), out_dtype,
                                       lse.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _compare(seed, n_rows, out_dtype):
    cfg, q, kv, idx = _case(seed, n_rows)
    shape = dsa.shape_of(cfg)
    ws, n = dsa.alloc_workspace(shape, dsa.DSA_OP_SPARSE_ATTN)
    shp = (1, cfg.n_q, cfg.heads)
    ref_o = torch.empty(*shp, cfg.v_dim, device="cuda", dtype=out_dtype)
    ref_l = torch.empty(*shp, device="cuda")
    dsa.dsa_sparse_attn(shape, q, kv, idx, ref_o, ref_l, ws, n)
    got_o = torch.full_like(ref_o, float("nan"))
    got_l = torch.full_like(ref_l, float("nan"))
    st = _noalloc_via_abi(shape, q, kv, idx, got_o, got_l)
    assert st == dsa.DSA_OK, dsa.load_library().dsa_last_error().decode()
    dsa.dsa_check()
    assert torch.equal(got_o, ref_o), "out differs from dsa_sparse_attn"
    assert torch.equal(got_l, ref_l), "lse differs from dsa_sparse_attn"
    return n


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    # Two calls in a row: the second finds the first call's partials in the
    # shared scratch array and must not read any of them.
    for seed in (11, 12):
        need = _compare(seed, 3, torch.float32)
        assert 0 < need <= NOALLOC_SCRATCH_BYTES   # split-K: the scratch array is used


def test_noalloc_bf16_output_and_no_split_plan():
    need = _compare(13, 3, torch.bfloat16)
    assert need > 0
    # enough rows that the plan needs no split-K partials: no scratch at all
    need = _compare(14, 300, torch.float32)
    assert need == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # the fewest query rows whose split-K partials exceed the 16 MiB array
    n_rows = next(n for n in range(1, 148)
                  if dsa.workspace_size(dsa.shape_of(dsa_inputs.custom_config(
                      "prefill_4k", n_q=n, name="nb")), dsa.DSA_OP_SPARSE_ATTN)
                  > NOALLOC_SCRATCH_BYTES)
    cfg, q, kv, idx = _case(15, n_rows)
    shape = dsa.shape_of(cfg)
    out = torch.zeros(1, n_rows, cfg.heads, cfg.v_dim, device="cuda")
    lse = torch.zeros(1, n_rows, cfg.heads, device="cuda")
    st = _noalloc_via_abi(shape, q, kv, idx, out, lse)
    assert st == dsa.DSA_ERR_WORKSPACE
    assert b"16777216" in dsa.load_library().dsa_last_error()
    torch.cuda.synchronize()
    assert (out == 0).all() and (lse == 0).all(), "nothing may be launched"
