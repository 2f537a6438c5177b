"""dsa_layout on the GPU, through the C ABI:

* explicit query positions (row_pos): one prefill's rows split into shards
  (the query-sharded prefill's partition) give exactly the selections and,
  on the same index order, bit-for-bit the outputs of the unsplit call;
* a paged key cache (block_table over shared pools, the PagedAttention
  layout of page "DeepSeek-V3 MoE blog", section 4.1): the same selections
  as the contiguous cache and bit-for-bit the same attention, and at the
  64 x 32768 decode size with ragged lengths the oracle's band rule and
  attention tolerance;
* a page outside the pool is skipped and reported by dsa_check.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_long_fp8_b200 as dsa
from sparse_attention_long_fp8_b200 import inputs as dsa_inputs
from sparse_attention_long_fp8_b200 import shard

from parity import check_attn, check_topk_band

pytestmark = pytest.mark.gpu


def _gpu_inputs(cfg, seed):
    return dsa_inputs.make_inputs(cfg, seed=seed, device="cuda")


def _sets(a):
    return np.sort(a.cpu().numpy(), axis=-1)


def _attn(cfg, q, kv, idx, layout=None):
    shape = dsa.shape_of(cfg)
    ws, n = dsa.alloc_workspace(shape, dsa.DSA_OP_SPARSE_ATTN)
    out = torch.empty(cfg.batch, cfg.n_q, cfg.heads, cfg.v_dim, device="cuda")
    lse = torch.empty(cfg.batch, cfg.n_q, cfg.heads, device="cuda")
    dsa.dsa_sparse_attn(shape, q, kv, idx, out, lse, ws, n, layout=layout)
    dsa.dsa_check()
    return out, lse


# ------------------------------------------------------------------ row positions

@pytest.mark.parametrize("base,n,R", [("prefill_4k", 2600, 3), ("tiny", 256, 2)])
def test_row_pos_shards_reproduce_the_full_prefill(base, n, R):
    cfg = dsa_inputs.custom_config(base, n_q=n, n_kv=n, name=f"shard{n}")
    g = _gpu_inputs(cfg, 31)
    full = dsa.forward(g, cfg)
    dsa.dsa_check()
    for r in range(R):
        rows = shard.shard_rows(n, R, r)
        sh = shard.shard_inputs(g, rows)
        scfg = dsa_inputs.custom_config(base, n_q=len(rows), n_kv=n, name=f"s{r}")
        lay = dsa.make_layout(row_pos=sh["row_pos"])
        res = dsa.forward(sh, scfg, layout=lay)
        dsa.dsa_check()
        assert np.array_equal(_sets(res["indices"][0]), _sets(full["indices"][0][rows]))
        # the attention over the same index order is the same computation
        o, l = _attn(scfg, sh["q"], g["kv"], full["indices"][:, rows].contiguous())
        assert torch.equal(o, full["out"][:, rows]) and torch.equal(l, full["lse"][:, rows])


# ------------------------------------------------------------------ paged caches

def _paged(g, cfg, page, seed, spare=5):
    """The contiguous key tensors copied into pools of pages in a random
    physical order; returns (pools dict, block_table, pool_rows)."""
    B, S = cfg.batch, cfg.n_kv
    per_seq = math.ceil(S / page)
    n_pages = B * per_seq + spare
    gen = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n_pages, generator=gen)[: B * per_seq]
    table = perm.view(B, per_seq).to(torch.int32).cuda()
    s = torch.arange(S, device="cuda")
    phys = (table[:, s // page].long() * page + (s % page)[None, :]).reshape(-1)
    pools = {}
    for k in ("k_fp8", "k_scale", "kv"):
        t = g[k]
        pool = torch.zeros((n_pages * page,) + tuple(t.shape[2:]), dtype=t.dtype, device="cuda")
        pool[phys] = t.reshape((B * S,) + tuple(t.shape[2:]))
        pools[k] = pool
    return pools, table, n_pages * page


def _ragged_decode(cfg, seed):
    g = _gpu_inputs(cfg, seed)
    gen = torch.Generator().manual_seed(seed)
    kvl = torch.randint(cfg.n_kv // 2, cfg.n_kv + 1, (cfg.batch,), generator=gen, dtype=torch.int32)
    kvl[0] = cfg.n_kv
    kvl[-1] = min(cfg.n_kv, 1000)       # shorter than a selection plus one page
    g["kv_len"] = kvl.cuda()
    g["q_pos0"] = (kvl - 1).cuda()
    return g


@pytest.mark.parametrize("page", [128, 1024])
def test_paged_decode_equals_contiguous(page):
    cfg = dsa_inputs.custom_config("decode_32k", batch=8, n_kv=8192, name="pdec")
    g = _ragged_decode(cfg, 41)
    ref = dsa.forward(g, cfg)
    dsa.dsa_check()
    pools, table, rows = _paged(g, cfg, page, seed=page)
    lay = dsa.make_layout(block_table=table, page_size=page, pool_rows=rows)
    gp = dict(g, **pools)
    res = dsa.forward(gp, cfg, layout=lay)
    dsa.dsa_check()
    assert np.array_equal(_sets(res["indices"]), _sets(ref["indices"]))
    o, l = _attn(cfg, g["q"], pools["kv"], ref["indices"], layout=lay)
    assert torch.equal(o, ref["out"]) and torch.equal(l, ref["lse"])


def test_paged_prefill_fused_equals_contiguous():
    cfg = dsa_inputs.custom_config("prefill_4k", n_q=1500, n_kv=1500, name="ppre")
    g = _gpu_inputs(cfg, 43)
    assert dsa.forward_plan(dsa.shape_of(cfg))["fused"]
    ref = dsa.forward(g, cfg)
    dsa.dsa_check()
    pools, table, rows = _paged(g, cfg, 512, seed=3)
    lay = dsa.make_layout(block_table=table, page_size=512, pool_rows=rows)
    res = dsa.forward(dict(g, **pools), cfg, layout=lay)
    dsa.dsa_check()
    assert np.array_equal(_sets(res["indices"]), _sets(ref["indices"]))
    o, l = _attn(cfg, g["q"], pools["kv"], ref["indices"], layout=lay)
    assert torch.equal(o, ref["out"]) and torch.equal(l, ref["lse"])


def test_paged_decode_64x32768_ragged_against_oracle():
    cfg = dsa_inputs.CONFIGS["decode_32k"]
    g = _ragged_decode(cfg, 47)
    pools, table, rows = _paged(g, cfg, 256, seed=9)
    lay = dsa.make_layout(block_table=table, page_size=256, pool_rows=rows)
    res = dsa.forward(dict(g, **pools), cfg, layout=lay)
    dsa.dsa_check()
    for b in (0, 5, 40, 63):
        kvl = int(g["kv_len"][b])
        pos = np.array([kvl - 1], dtype=np.int32)
        ref_s = oracle.indexer_scores(g["q_fp8"][b], g["q_scale"][b], g["w"][b], g["k_fp8"][b],
                                      g["k_scale"][b], pos, kvl)
        gidx = res["indices"][b].cpu().numpy()
        check_topk_band(gidx, ref_s, cfg.topk)
        o_ref, l_ref = oracle.sparse_attn(g["q"][b], g["kv"][b], gidx, cfg.softmax_scale, cfg.v_dim)
        check_attn(res["out"][b].cpu().numpy(), o_ref, res["lse"][b].cpu().numpy(), l_ref)


def test_page_outside_the_pool_is_skipped_and_reported():
    cfg = dsa_inputs.custom_config("decode_32k", batch=2, n_kv=1024, name="pbad")
    g = _gpu_inputs(cfg, 53)
    pools, table, rows = _paged(g, cfg, 256, seed=1)
    table[1, 2] = rows // 256 + 7           # a page past the end of the pool
    lay = dsa.make_layout(block_table=table, page_size=256, pool_rows=rows)
    dsa.forward(dict(g, **pools), cfg, layout=lay)
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_check()
    assert e.value.status == dsa.DSA_ERR_INVALID_ARG
    dsa.forward(g, cfg)                       # the context is still usable
    dsa.dsa_check()
