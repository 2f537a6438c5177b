"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs. Acceptance rules are in tests/parity.py."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_long_fp8_b200 as dsa
from sparse_attention_long_fp8_b200 import inputs as dsa_inputs

from parity import check_attn, check_scores, check_topk_band, score_magnitude

pytestmark = pytest.mark.gpu

_CACHE = {}


def _inputs(name, device="cpu", cfg=None, seed=0):
    key = (name, device, seed, cfg)
    if key not in _CACHE:
        c = cfg or dsa_inputs.CONFIGS[name]
        inp = dsa_inputs.make_inputs(c, seed=seed, device=device)
        gpu = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
        _CACHE.clear()
        _CACHE[key] = (c, inp, gpu)
    return _CACHE[key]


def _gpu_scores(cfg, g, row_begin=0, row_end=None):
    row_end = cfg.n_q if row_end is None else row_end
    sc = torch.empty(cfg.batch, row_end - row_begin, cfg.n_kv, device="cuda")
    dsa.dsa_indexer_scores(dsa.shape_of(cfg), g["q_fp8"], g["q_scale"], g["w"], g["k_fp8"],
                           g["k_scale"], g["q_pos0"], g["kv_len"], row_begin, row_end, sc)
    dsa.dsa_check()
    return sc


def _oracle_scores(cfg, inp, b, rows):
    rows = np.asarray(rows)
    pos = (rows + int(inp["q_pos0"][b])).astype(np.int32)
    sel = torch.as_tensor(rows, device=inp["q_fp8"].device)
    return oracle.indexer_scores(inp["q_fp8"][b].index_select(0, sel),
                                 inp["q_scale"][b].index_select(0, sel),
                                 inp["w"][b].index_select(0, sel), inp["k_fp8"][b],
                                 inp["k_scale"][b], pos, int(inp["kv_len"][b]))


def _magnitude(inp, b, rows):
    sel = torch.as_tensor(np.asarray(rows), device=inp["q_fp8"].device)
    return score_magnitude(inp["q_fp8"][b].index_select(0, sel), inp["q_scale"][b].index_select(0, sel),
                           inp["w"][b].index_select(0, sel), inp["k_fp8"][b], inp["k_scale"][b])


def _oracle_attn(cfg, inp, b, rows, idx):
    sel = torch.as_tensor(np.asarray(rows), device=inp["q"].device)
    return oracle.sparse_attn(inp["q"][b].index_select(0, sel), inp["kv"][b], idx,
                              cfg.softmax_scale, cfg.v_dim)


SAMPLE_4K = [0, 1, 2, 127, 128, 129, 1000, 2046, 2047, 2048, 2049, 3071, 4000, 4095]


# ------------------------------------------------------------------ indexer

def test_indexer_tiny_all_rows():
    cfg, inp, g = _inputs("tiny")
    sc = _gpu_scores(cfg, g).cpu().numpy()[0]
    rows = np.arange(cfg.n_q)
    check_scores(sc, _oracle_scores(cfg, inp, 0, rows), _magnitude(inp, 0, rows))


def test_indexer_4k_sampled_rows():
    cfg, inp, g = _inputs("prefill_4k")
    sc = _gpu_scores(cfg, g).cpu().numpy()[0]
    check_scores(sc[SAMPLE_4K], _oracle_scores(cfg, inp, 0, SAMPLE_4K), _magnitude(inp, 0, SAMPLE_4K))


def test_indexer_row_range_matches_full():
    cfg, inp, g = _inputs("prefill_4k")
    full = _gpu_scores(cfg, g)
    part = _gpu_scores(cfg, g, 1001, 1100)
    assert torch.equal(part[0], full[0, 1001:1100])


@pytest.mark.parametrize("n,kvl,pos0", [(300, 300, 0), (300, 257, 0), (200, 200, 37), (5, 130, 120)])
def test_indexer_ragged_masks(n, kvl, pos0):
    cfg = dsa_inputs.custom_config("prefill_4k", n_q=n, n_kv=max(n, kvl), name=f"rag{n}")
    inp = dsa_inputs.make_inputs(cfg, seed=3)
    inp["kv_len"][:] = kvl
    inp["q_pos0"][:] = pos0
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    sc = _gpu_scores(cfg, g).cpu().numpy()[0]
    rows = np.arange(n)
    check_scores(sc, _oracle_scores(cfg, inp, 0, rows), _magnitude(inp, 0, rows))


# ------------------------------------------------------------------ top-k

def _random_scores(rows, n_kv, seed, ties=True):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal((rows, n_kv)).astype(np.float32)
    if ties:
        s[:, ::7] = np.round(s[:, ::7], 1)        # many exact ties
        s[0, :] = 0.5                               # a row of all-equal scores
        s[1, : n_kv // 2] = -0.0                    # signed zeros tie with +0
        s[1, n_kv // 2:] = 0.0
    return s


@pytest.mark.parametrize("n_kv,k,pos0", [(300, 64, 0), (300, 64, 200), (4096, 2048, 4090),
                                           (5000, 2048, 2044), (50000, 2048, 49994),
                                           (70000, 100, 69994), (40001, 2048, 39995)])
def test_topk_exact_on_given_scores(n_kv, k, pos0):
    """Integer work: on the same fp32 scores the selection must equal the
    oracle's (ties to the lower index) exactly. With an odd n_kv every row
    but the first starts off a 16-byte boundary and takes the scalar scan;
    the all-equal row overflows the candidate buffers (the fallback)."""
    rows = 6
    cfg = dsa_inputs.custom_config("prefill_4k", n_q=pos0 + rows, n_kv=n_kv, topk=k, name="tk")
    s32 = _random_scores(rows, n_kv, seed=n_kv)
    shape = dsa.shape_of(cfg)
    scores = torch.from_numpy(s32).cuda()[None]
    idx = torch.empty(1, rows, k, dtype=torch.int32, device="cuda")
    q_pos0 = torch.tensor([0], dtype=torch.int32, device="cuda")
    dsa.dsa_topk(shape, scores, pos0, pos0 + rows, q_pos0, None, idx)
    dsa.dsa_check()
    ref_s = s32.astype(np.float64)
    for r in range(rows):
        ref_s[r, pos0 + r + 1:] = -np.inf
    want = oracle.topk(ref_s, k)
    got = idx.cpu().numpy()[0]
    for r in range(rows):
        assert sorted(got[r].tolist()) == sorted(want[r].tolist()), f"row {r}"


def test_topk_band_on_gpu_scores_4k():
    cfg, inp, g = _inputs("prefill_4k")
    sc = _gpu_scores(cfg, g)
    idx = torch.empty(1, cfg.n_q, cfg.topk, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(dsa.shape_of(cfg), sc, 0, cfg.n_q, g["q_pos0"], g["kv_len"], idx)
    dsa.dsa_check()
    got = idx.cpu().numpy()[0]
    check_topk_band(got[SAMPLE_4K], _oracle_scores(cfg, inp, 0, SAMPLE_4K), cfg.topk)


# ------------------------------------------------------------------ fused indexer + top-k

def _two_pass(cfg, g, rb, re_):
    sc = _gpu_scores(cfg, g, rb, re_)
    idx = torch.empty(cfg.batch, re_ - rb, cfg.topk, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(dsa.shape_of(cfg), sc, rb, re_, g["q_pos0"], g["kv_len"], idx)
    dsa.dsa_check()
    return idx


def _fused(cfg, g, rb, re_):
    idx = torch.full((cfg.batch, re_ - rb, cfg.topk), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_indexer_topk(dsa.shape_of(cfg), g["q_fp8"], g["q_scale"], g["w"], g["k_fp8"],
                         g["k_scale"], g["q_pos0"], g["kv_len"], rb, re_, idx)
    dsa.dsa_check()
    return idx


def _assert_same_sets(a, b):
    """Both kernels form each score with the same fp32 operations, so the
    selected sets must be identical (integer work: bit-exact)."""
    a = np.sort(a.cpu().numpy() if torch.is_tensor(a) else np.asarray(a), axis=-1)
    b = np.sort(b.cpu().numpy() if torch.is_tensor(b) else np.asarray(b), axis=-1)
    bad = np.nonzero((a != b).any(axis=-1))
    assert a.shape == b.shape and len(bad[0]) == 0, f"rows differ: {list(zip(*bad))[:8]}"


def _check_fused_against_oracle(cfg, inp, g, rb, re_, fused, band_rows):
    """The fused selection against the oracle directly:
    * exact: the oracle's top-k (full sort, ties to the lower index) of the
      GPU's own fp32 scores of every tested row gives the same sets;
    * band: on sampled rows, against the oracle's fp64 scores."""
    sc = _gpu_scores(cfg, g, rb, re_).double().cpu().numpy()
    got = fused.cpu().numpy()
    for b in range(cfg.batch):
        _assert_same_sets(got[b], oracle.topk(sc[b], cfg.topk))
        rows = [r for r in band_rows if rb <= r < re_]
        ref = _oracle_scores(cfg, inp, b, rows)
        check_topk_band(got[b][np.asarray(rows) - rb], ref, cfg.topk)


def test_indexer_topk_equals_two_pass_4k():
    cfg, inp, g = _inputs("prefill_4k")
    fused = _fused(cfg, g, 0, cfg.n_q)
    _assert_same_sets(fused, _two_pass(cfg, g, 0, cfg.n_q))
    check_topk_band(fused.cpu().numpy()[0][SAMPLE_4K], _oracle_scores(cfg, inp, 0, SAMPLE_4K),
                    cfg.topk)


@pytest.mark.parametrize("n,kvl,pos0,rb,re_", [(300, 300, 0, 0, 300), (301, 257, 0, 3, 298),
                                                (200, 200, 37, 0, 199), (5, 130, 120, 1, 5),
                                                (2600, 2600, 0, 2045, 2600)])
def test_indexer_topk_ragged(n, kvl, pos0, rb, re_):
    cfg = dsa_inputs.custom_config("prefill_4k", n_q=n, n_kv=max(n, kvl), topk=min(2048, 64 + n // 2),
                                   batch=2, name=f"frag{n}")
    inp = dsa_inputs.make_inputs(cfg, seed=5)
    inp["kv_len"][:] = torch.tensor([kvl, max(1, kvl - 9)], dtype=torch.int32)
    inp["q_pos0"][:] = torch.tensor([pos0, pos0 + 1], dtype=torch.int32)
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    fused = _fused(cfg, g, rb, re_)
    _assert_same_sets(fused, _two_pass(cfg, g, rb, re_))
    _check_fused_against_oracle(cfg, inp, g, rb, re_, fused, [rb, rb + 1, (rb + re_) // 2, re_ - 1])


def test_indexer_topk_all_ties_take_lowest_indices():
    """w = 0 makes every visible score exactly 0: the k lowest key indices win."""
    cfg = dsa_inputs.custom_config("prefill_4k", n_q=3000, n_kv=3000, topk=2048, name="ties")
    inp = dsa_inputs.make_inputs(cfg, seed=7)
    inp["w"][:, 2500:] = 0.0
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    fused = _fused(cfg, g, 2400, 3000)
    _assert_same_sets(fused, _two_pass(cfg, g, 2400, 3000))
    got = np.sort(fused.cpu().numpy()[0][100:], axis=-1)
    assert np.array_equal(got, np.broadcast_to(np.arange(2048, dtype=np.int32), got.shape))
    _check_fused_against_oracle(cfg, inp, g, 2400, 3000, fused, [2400, 2499, 2500, 2999])


def test_indexer_topk_rising_scores_force_compactions():
    """Positive codes and a key scale that grows with the key index make
    nearly every new key enter the candidate set: each row's buffer is
    compacted many times before the end."""
    cfg = dsa_inputs.custom_config("prefill_4k", n_q=16384, n_kv=16384, topk=2048, name="rise")
    inp = dsa_inputs.make_inputs(cfg, seed=11)
    inp["q_fp8"] = inp["q_fp8"] & 0x7F                      # clear the e4m3 sign bit
    inp["k_fp8"] = inp["k_fp8"] & 0x7F
    inp["q_fp8"][inp["q_fp8"] == 0x7F] = 0x7E                # no NaN codes
    inp["k_fp8"][inp["k_fp8"] == 0x7F] = 0x7E
    inp["w"] = inp["w"].abs()
    inp["k_scale"] = inp["k_scale"] * (1.0 + torch.arange(cfg.n_kv, dtype=torch.float32) / 64.0)
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    rb, re_ = cfg.n_q - 256, cfg.n_q
    fused = _fused(cfg, g, rb, re_)
    _assert_same_sets(fused, _two_pass(cfg, g, rb, re_))
    _check_fused_against_oracle(cfg, inp, g, rb, re_, fused, [rb, rb + 127, re_ - 1])


# ------------------------------------------------------------------ attention

def _rand_indices(n_rows, k, n_kv, seed, empty_frac=0.1):
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, n_kv, size=(n_rows, k)).astype(np.int32)
    idx[rng.random((n_rows, k)) < empty_frac] = -1
    return idx


@pytest.mark.parametrize("name,n_rows", [("tiny", 40), ("prefill_4k", 300), ("prefill_4k", 3)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_sparse_attn_random_sets(name, n_rows, out_dtype):
    """Random selections (with empty slots and repeats); n_rows = 3 runs the
    split-K + combine path."""
    base = dsa_inputs.CONFIGS[name]
    cfg = dsa_inputs.custom_config(name, n_q=n_rows, n_kv=base.n_kv, name=f"{name}_{n_rows}")
    inp = dsa_inputs.make_inputs(cfg, seed=5)
    idx = _rand_indices(n_rows, cfg.topk, cfg.n_kv, seed=n_rows)
    idx[0, :] = -1                                    # a row with no valid slot
    shape = dsa.shape_of(cfg)
    ws, n = dsa.alloc_workspace(shape, dsa.DSA_OP_SPARSE_ATTN)
    out = torch.empty(1, n_rows, cfg.heads, cfg.v_dim, dtype=out_dtype, device="cuda")
    lse = torch.empty(1, n_rows, cfg.heads, device="cuda")
    dsa.dsa_sparse_attn(shape, inp["q"].cuda(), inp["kv"].cuda(), torch.from_numpy(idx)[None].cuda(),
                        out, lse, ws, n)
    dsa.dsa_check()
    ref_o, ref_l = oracle.sparse_attn(inp["q"][0], inp["kv"][0], idx, cfg.softmax_scale, cfg.v_dim)
    got = out.float().cpu().numpy()[0]
    if out_dtype == torch.bfloat16:
        # bf16 rounding of the output adds up to 2^-9 relative
        ref_o = ref_o.astype(np.float32).astype(np.float64)
        d = np.abs(got - ref_o)
        assert (d <= 1e-2 + 2.0 ** -8 * np.abs(ref_o)).all()
    else:
        check_attn(got, ref_o, lse.cpu().numpy()[0], ref_l)
    assert (got[0] == 0).all() and np.isneginf(lse.cpu().numpy()[0, 0]).all()


# ------------------------------------------------------------------ whole path

def _check_forward(cfg, inp, g, b, rows):
    res = dsa.forward(g, cfg)
    dsa.dsa_check()
    ref_s = _oracle_scores(cfg, inp, b, rows)
    gidx = res["indices"][b].cpu().numpy()[rows]
    check_topk_band(gidx, ref_s, cfg.topk)
    o_ref, l_ref = _oracle_attn(cfg, inp, b, rows, gidx)
    o = res["out"][b].cpu().numpy()[rows]
    l = res["lse"][b].cpu().numpy()[rows]
    return check_attn(o, o_ref, l, l_ref)


def test_forward_tiny():
    cfg, inp, g = _inputs("tiny")
    _check_forward(cfg, inp, g, 0, np.arange(cfg.n_q))


def test_forward_4k_sampled():
    cfg, inp, g = _inputs("prefill_4k")
    _check_forward(cfg, inp, g, 0, np.array(SAMPLE_4K))


def test_forward_decode_32k_sampled_sequences():
    cfg, inp, g = _inputs("decode_32k", device="cuda")
    res = dsa.forward(g, cfg)
    dsa.dsa_check()
    for b in (0, 21, 63):
        ref_s = _oracle_scores(cfg, inp, b, [0])
        gidx = res["indices"][b].cpu().numpy()
        check_topk_band(gidx, ref_s, cfg.topk)
        o_ref, l_ref = _oracle_attn(cfg, inp, b, [0], gidx)
        check_attn(res["out"][b].cpu().numpy(), o_ref, res["lse"][b].cpu().numpy(), l_ref)


# rows of the k boundary, 128-row tile edges, mid-sequence and the last row
SAMPLE_16K = [0, 1, 127, 128, 2046, 2047, 2048, 2049, 4095, 4096, 8191, 8192, 12345, 16256,
              16383]


def test_forward_16k_sampled_rows():
    """Prefill at L = 16384 through dsa_forward (the fused indexer + top-k,
    then the attention), the launches the bench times."""
    cfg, inp, g = _inputs("prefill_16k", device="cuda")
    _check_forward(cfg, inp, g, 0, np.array(SAMPLE_16K))


def test_forward_decode_64k_sampled_sequences():
    """Batch decode, 64 sequences x 65536 cached tokens, through dsa_forward."""
    cfg, inp, g = _inputs("decode_64k", device="cuda")
    res = dsa.forward(g, cfg)
    dsa.dsa_check()
    for b in (0, 1, 31, 62, 63):
        ref_s = _oracle_scores(cfg, inp, b, [0])
        gidx = res["indices"][b].cpu().numpy()
        check_topk_band(gidx, ref_s, cfg.topk)
        o_ref, l_ref = _oracle_attn(cfg, inp, b, [0], gidx)
        check_attn(res["out"][b].cpu().numpy(), o_ref, res["lse"][b].cpu().numpy(), l_ref)


@pytest.mark.slow
def test_forward_64k_sampled_rows():
    """Full-size prefill in the launch configuration the bench times."""
    cfg, inp, g = _inputs("prefill_64k", device="cuda")
    rows = np.array([0, 2047, 2048, 30000, 65407, 65535])
    _check_forward(cfg, inp, g, 0, rows)
