"""dsa_sparse_attn_noalloc: the attention entry point for callers that cannot
call cudaMalloc (their device memory belongs to another framework's
allocator, or an allocation is not acceptable inside their decode loop), so
they cannot hand in the split-K workspace dsa_sparse_attn asks for. It must
give what the workspace entry point gives, call after call, even though
every call reuses the same static scratch array inside the library.

This file is collected last on purpose: a run that stops at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import sparse_attention_long_fp8_b200 as dsa
from sparse_attention_long_fp8_b200 import inputs as dsa_inputs

from parity import check_attn

pytestmark = pytest.mark.gpu

NOALLOC_SCRATCH_BYTES = 16 << 20


def _case(seed, n_rows=3):
    cfg = dsa_inputs.custom_config("prefill_4k", n_q=n_rows, name=f"noalloc{n_rows}")
    inp = dsa_inputs.make_inputs(cfg, seed=seed)
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, cfg.n_kv, size=(n_rows, cfg.topk)).astype(np.int32)
    idx[rng.random(idx.shape) < 0.1] = -1
    return cfg, inp["q"].cuda(), inp["kv"].cuda(), torch.from_numpy(idx)[None].cuda()


def _noalloc_via_abi(shape, q, kv, idx, out, lse):
    lib = dsa.load_library()
    st = lib.dsa_sparse_attn_noalloc(ctypes.byref(shape), q.data_ptr(), kv.data_ptr(),
                                     idx.data_ptr(), out.data_ptr(), dsa.DSA_OUT_F32,
                                     lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == dsa.DSA_OK, lib.dsa_last_error().decode()


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    for seed in (11, 12):   # two calls in a row: the second sees the first's scratch contents
        cfg, q, kv, idx = _case(seed)
        shape = dsa.shape_of(cfg)
        need = dsa.workspace_size(shape, dsa.DSA_OP_SPARSE_ATTN)
        assert 0 < need <= NOALLOC_SCRATCH_BYTES   # the split-K path, i.e. the scratch is used
        ws, n = dsa.alloc_workspace(shape, dsa.DSA_OP_SPARSE_ATTN)
        shp = (1, cfg.n_q, cfg.heads)
        ref_o = torch.empty(*shp, cfg.v_dim, device="cuda")
        ref_l = torch.empty(*shp, device="cuda")
        dsa.dsa_sparse_attn(shape, q, kv, idx, ref_o, ref_l, ws, n)
        got_o = torch.full_like(ref_o, float("nan"))
        got_l = torch.full_like(ref_l, float("nan"))
        _noalloc_via_abi(shape, q, kv, idx, got_o, got_l)
        dsa.dsa_check()
        check_attn(got_o.cpu().numpy(), ref_o.cpu().double().numpy(),
                   got_l.cpu().numpy(), ref_l.cpu().double().numpy())


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # enough query rows to need split-K partials beyond the 16 MiB array
    cfg = dsa_inputs.custom_config("prefill_4k", n_q=36, name="noalloc_big")
    shape = dsa.shape_of(cfg)
    assert dsa.workspace_size(shape, dsa.DSA_OP_SPARSE_ATTN) > NOALLOC_SCRATCH_BYTES
    fake = 0x100000
    lib = dsa.load_library()
    st = lib.dsa_sparse_attn_noalloc(ctypes.byref(shape), fake, fake, fake, fake,
                                     dsa.DSA_OUT_F32, None, None)
    assert st == dsa.DSA_ERR_WORKSPACE
    assert b"16777216" in lib.dsa_last_error()
