"""Pins for the fp64 CPU oracle, independent of the oracle's own code.

Each test checks the oracle against something fixed outside it: the OCP E4M3
definition and torch's float8 cast, closed-form identities of ReLU, library
routines (torch matmul / scaled_dot_product_attention / logsumexp) on special
cases, brute-force rank counting, and invariants the method implies (page
"DeepseekV3.2 拆解", section "核心组件": the indexer equation I_{t,s} and the
selection equation u_t = Attn(h_t, {c_s | I_{t,s} in Top-k(I_{t,:})})).
A plausible slip in the oracle (dropped term, wrong sign, wrong index,
transposed operand, wrong tie rule) fails at least one test here.
"""
import math
import os

import numpy as np
import pytest
import torch

from sparse_attention_long_fp8_b200 import inputs as dsa_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _decode_fp8_torch(codes_u8):
    return codes_u8.view(torch.float8_e4m3fn).to(torch.float64)


def _bf16_to_f64(x):
    return x.to(torch.float64)


def _small_indexer(seed, n, S, HI, DI, w_pos=False):
    g = torch.Generator().manual_seed(seed)
    q8, qs = dsa_inputs.quantize_e4m3_rows(torch.randn(n, HI, DI, generator=g))
    k8, ks = dsa_inputs.quantize_e4m3_rows(torch.randn(S, DI, generator=g))
    w = torch.randn(n, HI, generator=g)
    if w_pos:
        w = w.abs()
    return q8, qs, w, k8, ks


# ---------------------------------------------------------------- e4m3 decode

def test_e4m3_golden_points(oracle_lib):
    path = os.path.join(GOLDEN, "e4m3_ocp_points.txt")
    n = 0
    for line in open(path, encoding="utf-8"):
        if not line.strip() or line.startswith("#"):
            continue
        code, val = line.split()
        got = oracle_lib.e4m3_value(int(code, 16))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))
        n += 1
    assert n >= 10


def test_e4m3_exhaustive_vs_torch(oracle_lib):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle_lib.e4m3_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(got), c
        else:
            assert got == ref[c], (c, got, ref[c])


# ---------------------------------------------------------------- indexer

def _finite_codes():
    return [c for c in range(256) if (c & 0x7F) != 0x7F]


def test_e4m3_encode_round_trips_every_finite_code(oracle_lib):
    """Encoding a code's own value gives the code back (sign of zero kept)."""
    for c in _finite_codes():
        v = oracle_lib.e4m3_value(c)
        assert oracle_lib.e4m3_encode(v if c != 0x80 else -0.0) == c


def test_e4m3_encode_ties_go_to_even_mantissa(oracle_lib):
    """Exactly half-way between two adjacent codes (exact in fp32) the code
    with the even mantissa wins; a hair either side picks the nearer one."""
    for c in range(0x00, 0x7E):
        lo, hi = oracle_lib.e4m3_value(c), oracle_lib.e4m3_value(c + 1)
        mid = np.float32((lo + hi) / 2)
        assert float(mid) == (lo + hi) / 2
        even = c if c % 2 == 0 else c + 1
        assert oracle_lib.e4m3_encode(float(mid)) == even
        assert oracle_lib.e4m3_encode(-float(mid)) == (0x80 | even)
        below = np.nextafter(mid, np.float32(-np.inf), dtype=np.float32)
        above = np.nextafter(mid, np.float32(np.inf), dtype=np.float32)
        assert oracle_lib.e4m3_encode(float(below)) == c
        assert oracle_lib.e4m3_encode(float(above)) == c + 1


def test_e4m3_encode_saturates(oracle_lib):
    for v, want in [(448.0, 0x7E), (460.0, 0x7E), (1e30, 0x7E), (-449.0, 0xFE), (-1e30, 0xFE)]:
        assert oracle_lib.e4m3_encode(v) == want


def test_e4m3_encode_matches_library_cast(oracle_lib):
    """Library special case: torch's round-to-nearest-even float8_e4m3fn cast,
    after clamping to the finite range, on a dense sweep of fp32 values."""
    g = torch.Generator().manual_seed(3)
    v = torch.cat([torch.randn(20000, generator=g) * 100,
                   torch.randn(5000, generator=g) * 1e-2,
                   torch.linspace(-460, 460, 9201)]).float()
    ref = v.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle_lib.e4m3_encode(float(x)) for x in v.numpy()], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_quantize_rows_scale_and_extremes(oracle_lib):
    """Per row: scale = amax / 448 in fp32, the amax element encodes to the
    extreme code, a zero row gets scale 1 and zero codes, and decoding
    (code value * scale) is within half an E4M3 step of x."""
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(6, 128, generator=g) * torch.tensor([1, 1e-3, 50, 1, 1, 0]).view(6, 1))
    x = x.to(torch.bfloat16)
    codes, scales = oracle_lib.quantize_rows(x)
    xf = x.float().numpy()
    for r in range(6):
        amax = np.float32(np.abs(xf[r]).max())
        if amax == 0:
            assert scales[r] == 1.0 and ((codes[r] & 0x7F) == 0).all()   # +-0 keep their sign
            continue
        assert scales[r] == np.float32(amax / np.float32(448.0))
        j = int(np.abs(xf[r]).argmax())
        assert codes[r, j] in (0x7E, 0xFE)
        dec = np.array([oracle_lib.e4m3_value(int(c)) for c in codes[r]]) * scales[r]
        # relative E4M3 step is 2^-3 for normals; absolute floor at the subnormal step
        tol = np.maximum(np.abs(xf[r]) * 2.0 ** -4, 2.0 ** -10 * scales[r]) * 1.0001
        assert (np.abs(dec - xf[r]) <= tol).all()


def test_quantize_rows_matches_library_encoding(oracle_lib):
    """Library special case: torch's amax / 448, fp32 division and RNE cast."""
    g = torch.Generator().manual_seed(7)
    x = (torch.randn(64, 128, generator=g) * torch.rand(64, 1, generator=g) * 10).to(torch.bfloat16)
    codes, scales = oracle_lib.quantize_rows(x)
    tc, ts = dsa_inputs.quantize_e4m3_rows(x)
    assert np.array_equal(codes, tc.numpy()) and np.array_equal(scales, ts.numpy())


def test_indexer_single_head_is_relu_matmul(oracle_lib):
    """H^I = 1, w = 1, unit scales: I[t,s] = ReLU(q_t . k_s), a plain matmul."""
    n, S, DI = 9, 13, 32
    q8, _, _, k8, _ = _small_indexer(1, n, S, 1, DI)
    qs = torch.ones(n, 1); ks = torch.ones(S); w = torch.ones(n, 1)
    pos = np.arange(n, dtype=np.int32) + 3
    got = oracle_lib.indexer_scores(q8, qs, w, k8, ks, pos, kv_len=S)
    dots = _decode_fp8_torch(q8[:, 0, :]) @ _decode_fp8_torch(k8).T
    ref = torch.relu(dots).numpy()
    for t in range(n):
        for s in range(S):
            if s <= pos[t]:
                assert got[t, s] == pytest.approx(ref[t, s], rel=1e-12, abs=1e-9)
            else:
                assert got[t, s] == -np.inf


def _flip_sign(codes):
    return codes ^ torch.tensor(0x80, dtype=torch.uint8)


@pytest.mark.parametrize("HI,DI", [(4, 32), (64, 128)])
def test_indexer_relu_identities(oracle_lib, HI, DI):
    """ReLU(x) - ReLU(-x) = x and ReLU(x) + ReLU(-x) = |x| give two closed
    forms: I(q) - I(-q) = sum_j w_j x_j and I(q) + I(-q) = sum_j w_j |x_j|,
    with x_j = (qs_j q_j) . (ks_s k_s) computed by a library matmul."""
    n, S = 6, 20
    q8, qs, w, k8, ks = _small_indexer(2, n, S, HI, DI)
    pos = np.full(n, S - 1, dtype=np.int32)
    i_pos = oracle_lib.indexer_scores(q8, qs, w, k8, ks, pos, S)
    i_neg = oracle_lib.indexer_scores(_flip_sign(q8), qs, w, k8, ks, pos, S)
    qhat = _decode_fp8_torch(q8) * qs.double()[..., None]          # [n, HI, DI]
    khat = _decode_fp8_torch(k8) * ks.double()[:, None]            # [S, DI]
    x = torch.einsum("njd,sd->njs", qhat, khat)                    # [n, HI, S]
    lin = (w.double()[..., None] * x).sum(1).numpy()
    absum = (w.double()[..., None] * x.abs()).sum(1).numpy()
    scale = np.abs(absum).max()
    np.testing.assert_allclose(i_pos - i_neg, lin, rtol=0, atol=1e-12 * scale)
    np.testing.assert_allclose(i_pos + i_neg, absum, rtol=0, atol=1e-12 * scale)


def test_indexer_head_terms_nonnegative(oracle_lib):
    """Every head term w_j * ReLU(.) has the sign of w_j: w >= 0 gives I >= 0,
    w <= 0 gives I <= 0, and a single head with w = 1 is >= 0."""
    n, S, HI, DI = 5, 16, 4, 32
    q8, qs, w, k8, ks = _small_indexer(3, n, S, HI, DI, w_pos=True)
    pos = np.full(n, S - 1, dtype=np.int32)
    assert (oracle_lib.indexer_scores(q8, qs, w, k8, ks, pos, S) >= 0).all()
    assert (oracle_lib.indexer_scores(q8, qs, -w, k8, ks, pos, S) <= 0).all()


def test_indexer_head_permutation_invariance(oracle_lib):
    n, S, HI, DI = 4, 24, 64, 128
    q8, qs, w, k8, ks = _small_indexer(4, n, S, HI, DI)
    pos = np.arange(n, dtype=np.int32) * 5
    perm = torch.randperm(HI, generator=torch.Generator().manual_seed(9))
    a = oracle_lib.indexer_scores(q8, qs, w, k8, ks, pos, S)
    b = oracle_lib.indexer_scores(q8[:, perm], qs[:, perm], w[:, perm], k8, ks, pos, S)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_indexer_linear_in_w_and_homogeneous_in_scales(oracle_lib):
    n, S, HI, DI = 4, 18, 4, 32
    q8, qs, _, k8, ks = _small_indexer(5, n, S, HI, DI)
    # dyadic weights keep w + w2 exact in fp32
    gw = torch.Generator().manual_seed(6)
    w = torch.randint(-8, 9, (n, HI), generator=gw).float() / 8
    w2 = torch.randint(-8, 9, (n, HI), generator=gw).float() / 8
    pos = np.full(n, S - 1, dtype=np.int32)
    f = lambda **kw: oracle_lib.indexer_scores(kw.get("q8", q8), kw.get("qs", qs),
                                               kw.get("w", w), k8, kw.get("ks", ks), pos, S)
    base = f()
    tol = 1e-12 * np.abs(base).max()
    np.testing.assert_allclose(f(w=w + w2), base + f(w=w2), rtol=0, atol=10 * tol)
    np.testing.assert_allclose(f(qs=qs * 4.0), 4.0 * base, rtol=0, atol=10 * tol)
    np.testing.assert_allclose(f(ks=ks * 0.25), 0.25 * base, rtol=0, atol=10 * tol)
    # scaling one head's q-scale scales only that head's term
    qs1 = qs.clone(); qs1[:, 2] *= 2.0
    w_only2 = torch.zeros_like(w); w_only2[:, 2] = w[:, 2]
    np.testing.assert_allclose(f(qs=qs1) - base, f(w=w_only2), rtol=0, atol=10 * tol)


def test_indexer_mask_causal_and_kv_len(oracle_lib):
    n, S, HI, DI = 6, 30, 4, 32
    q8, qs, w, k8, ks = _small_indexer(7, n, S, HI, DI)
    pos = np.array([0, 3, 10, 25, 29, 40], dtype=np.int32)
    kv_len = 27
    sc = oracle_lib.indexer_scores(q8, qs, w, k8, ks, pos, kv_len)
    for t in range(n):
        for s in range(S):
            assert np.isfinite(sc[t, s]) == (s <= pos[t] and s < kv_len)


# ---------------------------------------------------------------- top-k

def _rank_count_topk(row, k):
    """s is selected iff fewer than k valid keys beat it, where s' beats s when
    its score is higher, or equal with a lower index."""
    valid = [s for s in range(len(row)) if np.isfinite(row[s])]
    sel = set()
    for s in valid:
        beats = sum(1 for s2 in valid if row[s2] > row[s] or (row[s2] == row[s] and s2 < s))
        if beats < k:
            sel.add(s)
    return sel


@pytest.mark.parametrize("seed", range(12))
def test_topk_brute_force_rank_count(oracle_lib, seed):
    rng = np.random.default_rng(seed)
    L = int(rng.integers(1, 13))
    k = int(rng.integers(1, 15))
    # coarse values force ties; some -inf entries are invalid keys
    scores = rng.integers(-3, 4, size=(4, L)).astype(np.float64)
    scores[rng.random((4, L)) < 0.2] = -np.inf
    got = oracle_lib.topk(scores, k)
    for r in range(4):
        want = _rank_count_topk(scores[r], k)
        sel = [int(i) for i in got[r] if i >= 0]
        assert len(sel) == len(set(sel)) == len(want)
        assert set(sel) == want
        # the -1 pads come last
        assert all(i == -1 for i in got[r][len(sel):])


def test_topk_all_ties_take_lowest_indices(oracle_lib):
    scores = np.zeros((2, 50))
    got = oracle_lib.topk(scores, 7)
    assert sorted(got[0].tolist()) == list(range(7))


# ---------------------------------------------------------------- attention

def _attn_case(seed, n, S, H, Dqk):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(n, H, Dqk, generator=g).to(torch.bfloat16)
    kv = torch.randn(S, Dqk, generator=g).to(torch.bfloat16)
    return q, kv


@pytest.mark.parametrize("Dqk,Dv", [(64, 64), (64, 48)])
def test_attn_full_set_equals_dense_causal_sdpa(oracle_lib, Dqk, Dv):
    """k >= t+1: the selection keeps every causal key, so the result is dense
    causal attention (torch SDPA in float64 as the textbook reference)."""
    T, H = 12, 8
    q, kv = _attn_case(11, T, T, H, Dqk)
    scale = 0.125
    idx = np.full((T, T + 3), -1, dtype=np.int32)
    rng = np.random.default_rng(0)
    for t in range(T):
        idx[t, : t + 1] = rng.permutation(t + 1)
    o, lse = oracle_lib.sparse_attn(q, kv, idx, scale, Dv)
    qd = _bf16_to_f64(q).permute(1, 0, 2)[None]                       # [1, H, T, D]
    kd = _bf16_to_f64(kv)[None, None].expand(1, H, T, Dqk)
    vd = _bf16_to_f64(kv)[:, :Dv][None, None].expand(1, H, T, Dv)
    ref = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, is_causal=True, scale=scale)
    np.testing.assert_allclose(o, ref[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
    z = (qd @ kd.transpose(-1, -2)) * scale
    z = z.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(z, -1)[0].T.numpy(), rtol=0, atol=1e-12)


def test_attn_zero_scale_is_mean_of_rows(oracle_lib):
    q, kv = _attn_case(12, 3, 40, 4, 64)
    idx = np.array([[5, 1, 9, -1], [0, -1, -1, -1], [39, 38, 2, 17]], dtype=np.int32)
    o, lse = oracle_lib.sparse_attn(q, kv, idx, 0.0, 64)
    kvd = _bf16_to_f64(kv).numpy()
    for r in range(3):
        rows = [i for i in idx[r] if i >= 0]
        for h in range(4):
            np.testing.assert_allclose(o[r, h], kvd[rows].mean(0), rtol=0, atol=1e-12)
            assert lse[r, h] == pytest.approx(math.log(len(rows)), abs=1e-12)


def test_attn_single_key_and_empty_set(oracle_lib):
    q, kv = _attn_case(13, 2, 10, 3, 64)
    idx = np.array([[4, -1], [-1, -1]], dtype=np.int32)
    o, lse = oracle_lib.sparse_attn(q, kv, idx, 0.3, 32)
    kvd = _bf16_to_f64(kv).numpy(); qd = _bf16_to_f64(q).numpy()
    for h in range(3):
        np.testing.assert_allclose(o[0, h], kvd[4, :32], rtol=0, atol=0)
        assert lse[0, h] == pytest.approx(0.3 * float(qd[0, h] @ kvd[4]), rel=1e-12)
        assert (o[1, h] == 0).all() and lse[1, h] == -np.inf


def test_attn_slot_order_irrelevant(oracle_lib):
    q, kv = _attn_case(14, 2, 64, 8, 64)
    idx = np.stack([np.arange(0, 64, 3)[:16], np.arange(1, 64, 4)[:16]]).astype(np.int32)
    o1, l1 = oracle_lib.sparse_attn(q, kv, idx, 0.125, 64)
    o2, l2 = oracle_lib.sparse_attn(q, kv, idx[:, ::-1].copy(), 0.125, 64)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- full path

def test_forward_tiny_invariants(oracle_lib):
    """Tiny config: selections are causal, sized min(k, t+1), and the first k
    rows (where k >= t+1) equal dense causal attention."""
    cfg = dsa_inputs.CONFIGS["tiny"]
    inp = dsa_inputs.make_inputs(cfg, seed=0)
    rows = np.array([0, 1, 2, 30, 62, 63, 64, 65, 130, 255])
    res = oracle_lib.forward(inp, cfg, rows=rows)
    for r, t in enumerate(rows):
        sel = res["indices"][r]
        valid = sel[sel >= 0]
        assert len(valid) == min(cfg.topk, t + 1)
        assert (valid <= t).all() and len(set(valid.tolist())) == len(valid)
    dense_rows = rows[rows + 1 <= cfg.topk]
    q = inp["q"][0]; kv = inp["kv"][0]
    H, D = cfg.heads, cfg.qk_dim
    for r, t in enumerate(rows):
        if t + 1 > cfg.topk:
            continue
        qd = _bf16_to_f64(q[t])                                      # [H, D]
        kd = _bf16_to_f64(kv[: t + 1])                               # [t+1, D]
        p = torch.softmax(qd @ kd.T * cfg.softmax_scale, -1)
        np.testing.assert_allclose(res["o"][r], (p @ kd[:, : cfg.v_dim]).numpy(), rtol=0, atol=1e-12)
    assert len(dense_rows) > 0


# ---------------------------------------------------------------- warm-up loss
# Page "DeepseekV3.2 拆解", section "预训练策略 / 密集预热阶段": the indexer
# is trained against the dense attention distribution with
# L^I = sum_t KL(p_{t,:} || Softmax(I_{t,:})).

def _bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)


def test_kl_two_key_case_by_hand(oracle_lib):
    """Two query rows over two keys, one main head, one indexer head of one
    dim, every value exact in bf16 / e4m3. Row 0 sees only key 0: both
    distributions are [1], so its loss and gradient vanish. Row 1: the main
    logits are (0, a) and the indexer scores (0, b) with b = w q^ k^_1, so
    p = (1, e^a) / (1 + e^a), r = (1, e^b) / (1 + e^b); x_0 = 0 contributes
    neither to I nor to the gradient (ReLU and its mask are both zero)."""
    scale, wv, qsv, ks1 = 0.75, 1.5, 2.0, 0.5
    q = _bf16_bits([[[1.0, 0.0]], [[1.0, 0.0]]])              # [2 rows, 1 head, 2]
    kv = _bf16_bits([[0.0, 0.0], [1.0, 0.0]])                 # c_0 = 0, c_1 = e_0
    one = 0x38                                                # e4m3 code of 1.0
    q8 = torch.tensor([[[one]], [[one]]], dtype=torch.uint8)  # [2, 1, 1]
    k8 = torch.tensor([[0x00], [one]], dtype=torch.uint8)     # k^_0 = 0, k^_1 = ks1
    qs = torch.full((2, 1), qsv)
    w = torch.full((2, 1), wv)
    ks = torch.tensor([1.0, ks1])
    res = oracle_lib.indexer_kl(q8, qs, w, k8, ks, np.array([0, 1], np.int32), 2, q, kv, scale)
    a = scale * 1.0
    xq = qsv * ks1                                            # x[1, 0, 1] = q^ . k^_1
    b = wv * xq
    p1 = math.exp(a) / (1 + math.exp(a))
    r1 = math.exp(b) / (1 + math.exp(b))
    p0, r0 = 1 - p1, 1 - r1
    want = p0 * math.log(p0 / r0) + p1 * math.log(p1 / r1)
    g1 = r1 - p1
    assert res["loss"][0] == 0.0 and (res["dw"][0] == 0).all() and (res["dq"][0] == 0).all()
    assert abs(res["loss"][1] - want) < 1e-14
    assert abs(res["dw"][1, 0] - g1 * xq) < 1e-14
    assert abs(res["dq"][1, 0, 0] - g1 * wv * ks1) < 1e-14
    assert abs(res["dk"][1, 0] - g1 * wv * qsv) < 1e-14
    assert res["dk"][0, 0] == 0.0


def _kl_case(seed, n=20, HI=4, DI=32, H=8, Dqk=64, kv_len=None, w_scale=0.5):
    q8, qs, w, k8, ks = _small_indexer(seed, n, n, HI, DI)
    g = torch.Generator().manual_seed(seed + 1)
    q = (torch.randn(n, H, Dqk, generator=g) * 0.5).to(torch.bfloat16)
    kv = torch.randn(n, Dqk, generator=g).to(torch.bfloat16)
    return dict(q8=q8, qs=qs, w=w * w_scale, k8=k8, ks=ks, pos=np.arange(n, dtype=np.int32),
                kv_len=n if kv_len is None else kv_len, q=q, kv=kv, scale=0.125)


def _kl(oracle_lib, c, **over):
    d = dict(c, **over)
    return oracle_lib.indexer_kl(d["q8"], d["qs"], d["w"], d["k8"], d["ks"], d["pos"],
                                 d["kv_len"], d["q"], d["kv"], d["scale"])


def test_kl_matches_library_kl_div_and_is_nonnegative(oracle_lib):
    """Given the (separately pinned) indexer scores, the loss is torch's
    kl_div of log_softmax(I) against the head-averaged causal softmax of the
    main logits (torch softmax over masked float64 logits)."""
    c = _kl_case(3)
    res = _kl(oracle_lib, c)
    n = len(c["pos"])
    sc = oracle_lib.indexer_scores(c["q8"], c["qs"], c["w"], c["k8"], c["ks"], c["pos"], n)
    I = torch.from_numpy(sc)
    qd, kd = c["q"].double(), c["kv"].double()
    z = torch.einsum("thd,sd->ths", qd, kd) * c["scale"]
    mask = torch.triu(torch.ones(n, n, dtype=torch.bool), 1)
    p = torch.softmax(z.masked_fill(mask[:, None, :], -math.inf), -1).mean(1)
    for t in range(n):
        want = torch.nn.functional.kl_div(torch.log_softmax(I[t, : t + 1], -1), p[t, : t + 1],
                                          reduction="sum").item()
        assert abs(res["loss"][t] - want) < 1e-12
    assert (res["loss"] >= -1e-15).all() and res["loss"][1:].max() > 1e-3


def test_kl_vanishes_when_both_distributions_are_uniform(oracle_lib):
    """w = 0 makes every indexer score 0 and q = 0 every main logit 0: both
    distributions are uniform over the visible keys, loss and gradient 0."""
    c = _kl_case(4)
    res = _kl(oracle_lib, c, w=torch.zeros_like(c["w"]), q=torch.zeros_like(c["q"]))
    # zero up to the rounding of 1/n against the mean of H equal 1/n values
    assert np.abs(res["loss"]).max() < 1e-14
    assert np.abs(res["dw"]).max() < 1e-12 and np.abs(res["dq"]).max() < 1e-12
    assert np.abs(res["dk"]).max() < 1e-12


def test_kl_gradient_of_w_by_central_differences(oracle_lib):
    c = _kl_case(5)
    res = _kl(oracle_lib, c)
    eps = 1e-6
    for (t, j) in [(1, 0), (7, 3), (19, 2), (12, 1)]:
        wp, wm = c["w"].clone(), c["w"].clone()
        wp[t, j] += eps
        wm[t, j] -= eps
        # the fp32 w cannot hold w +- 1e-6 exactly: difference by the actual step
        h = float(wp[t, j]) - float(wm[t, j])
        fd = (_kl(oracle_lib, c, w=wp)["loss"].sum() - _kl(oracle_lib, c, w=wm)["loss"].sum()) / h
        assert abs(fd - res["dw"][t, j]) <= 1e-6 * max(1.0, abs(res["dw"][t, j])), (t, j)


def test_kl_gradient_along_the_scales_by_central_differences(oracle_lib):
    """q^[t,j] = code * q_scale[t,j]: d loss / d q_scale[t,j] = dq[t,j] . code;
    likewise for k_scale[s] and dk[s]."""
    c = _kl_case(6)
    res = _kl(oracle_lib, c)
    dec_q = _decode_fp8_torch(c["q8"]).numpy()
    dec_k = _decode_fp8_torch(c["k8"]).numpy()
    rel = 2e-6
    for (t, j) in [(3, 1), (15, 0), (19, 3)]:
        qp, qm = c["qs"].clone(), c["qs"].clone()
        qp[t, j] *= 1 + rel
        qm[t, j] *= 1 - rel
        h = float(qp[t, j]) - float(qm[t, j])
        fd = (_kl(oracle_lib, c, qs=qp)["loss"].sum() - _kl(oracle_lib, c, qs=qm)["loss"].sum()) / h
        want = float(res["dq"][t, j] @ dec_q[t, j])
        assert abs(fd - want) <= 1e-5 * max(1.0, abs(want)), (t, j)
    for s in [0, 4, 11, 19]:
        kp, km = c["ks"].clone(), c["ks"].clone()
        kp[s] *= 1 + rel
        km[s] *= 1 - rel
        h = float(kp[s]) - float(km[s])
        fd = (_kl(oracle_lib, c, ks=kp)["loss"].sum() - _kl(oracle_lib, c, ks=km)["loss"].sum()) / h
        want = float(res["dk"][s] @ dec_k[s])
        assert abs(fd - want) <= 1e-5 * max(1.0, abs(want)), s


def test_kl_gradients_match_autograd(oracle_lib):
    """Element-wise dq^ and dk^ (and dw) against torch autograd of the loss
    written with library ops on the dequantised vectors, with a kv_len cut."""
    n, HI = 20, 4
    c = _kl_case(7, n=n, HI=HI, kv_len=16)
    res = _kl(oracle_lib, c)
    qh = (_decode_fp8_torch(c["q8"]) * c["qs"].double()[..., None]).requires_grad_()
    kh = (_decode_fp8_torch(c["k8"]) * c["ks"].double()[:, None]).requires_grad_()
    w = c["w"].double().requires_grad_()
    x = torch.einsum("tjd,sd->tjs", qh, kh)
    I = torch.einsum("tj,tjs->ts", w, torch.relu(x))
    z = torch.einsum("thd,sd->ths", c["q"].double(), c["kv"].double()) * c["scale"]
    s_idx = torch.arange(n)
    vis = (s_idx[None, :] <= s_idx[:, None]) & (s_idx[None, :] < c["kv_len"])
    p = torch.softmax(z.masked_fill(~vis[:, None, :], -math.inf), -1).mean(1)
    logr = torch.log_softmax(I.masked_fill(~vis, -math.inf), -1)
    terms = torch.where(vis & (p > 0), p * (torch.log(p) - logr), torch.zeros_like(p))
    terms.sum().backward()
    np.testing.assert_allclose(res["loss"], terms.sum(-1).detach().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["dw"], w.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["dq"], qh.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(res["dk"], kh.grad.numpy(), rtol=0, atol=1e-11)
    assert (res["dk"][16:] == 0).all()      # keys past kv_len see no row
