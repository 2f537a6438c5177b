"""The indexer warm-up loss and its gradient (dsa_indexer_kl, through the C
ABI) against the fp64 oracle (page "DeepseekV3.2 拆解", section
"预训练策略 / 密集预热阶段": L^I = sum_t KL(p_{t,:} || Softmax(I_{t,:}))).

Tolerances follow from the arithmetic:
* the GPU scores carry |dI| <= 1.2e-5 A[t,s] (the score bound of
  tests/parity.py), so log Softmax(I) moves by at most 2 max_s |dI|; p comes
  from fp32 exponentials of fp32-accumulated logits (relative ~1e-5). So
  |dg[t,s]| <= r (2.4e-5 max_s A[t,s] + 1e-5) + 1e-5 p, and the loss moves by
  at most 2.4e-5 max_s A + 2e-5 (p sums to one);
* the gradient sums add n_vis * 2^-24 relative (fp32 accumulation);
* the ReLU mask [x > 0] is decided on the GPU by the sign of an fp32 sum of
  128 exact products: where |x| is within 2^-17 sum |products| of zero the
  mask may differ from the exact one, and those terms' full size is allowed.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_long_fp8_b200 as dsa
from sparse_attention_long_fp8_b200 import inputs as dsa_inputs

from parity import score_magnitude

pytestmark = pytest.mark.gpu


def _f8(t):
    return t.cpu().view(torch.float8_e4m3fn).double().numpy()


def _bounds(cfg, inp):
    """Per-element error bounds for loss, dw, dq, dk (float64 numpy)."""
    T, S = cfg.n_q, cfg.n_kv
    q8, k8 = _f8(inp["q_fp8"][0]), _f8(inp["k_fp8"][0])          # codes as values
    qs = inp["q_scale"][0].double().numpy()
    ks = inp["k_scale"][0].double().numpy()
    w = inp["w"][0].double().numpy()
    qh = q8 * qs[..., None]                                        # [T, HI, DI]
    kh = k8 * ks[:, None]                                          # [S, DI]
    code_dot = q8 @ k8.T                                           # [T, HI, S], exact in fp64
    code_abs = np.abs(q8) @ np.abs(k8).T
    ambiguous = np.abs(code_dot) <= 2.0 ** -17 * code_abs          # GPU mask may differ
    pos = np.arange(T)[:, None]
    vis = np.arange(S)[None, :] <= pos                              # [T, S]
    I = oracle.indexer_scores(inp["q_fp8"][0], inp["q_scale"][0], inp["w"][0], inp["k_fp8"][0],
                              inp["k_scale"][0], np.arange(T, dtype=np.int32), S)
    Iv = np.where(vis, I, -np.inf)
    r = np.exp(Iv - Iv.max(1, keepdims=True))
    r /= r.sum(1, keepdims=True)
    qd = inp["q"][0].double()
    z = torch.einsum("thd,sd->ths", qd, inp["kv"][0].double()) * cfg.softmax_scale
    z = z.masked_fill(~torch.from_numpy(vis)[:, None, :], -math.inf)
    p = torch.softmax(z, -1).mean(1).numpy()
    A = score_magnitude(inp["q_fp8"][0], inp["q_scale"][0], inp["w"][0], inp["k_fp8"][0],
                        inp["k_scale"][0])
    amax = np.where(vis, A, 0.0).max(1)                             # [T]
    n_vis = vis.sum(1)
    dg = r * (2.4e-5 * amax + 1e-5)[:, None] + 1e-5 * p             # |error of g|
    acc = (n_vis * 2.0 ** -24)[:, None] * (r + p)                   # fp32 summation
    e = np.where(vis, dg + acc, 0.0)                                # [T, S]
    gabs = np.where(vis, np.abs(r - p), 0.0)
    amb = ambiguous * gabs[:, None, :]                              # [T, HI, S]
    # the loss: the bound on log Softmax(I) plus fp32 exp / log / summation
    loss_b = 2.4e-5 * amax + 1e-4
    aw = np.abs(w)
    HI, DI = qh.shape[1], qh.shape[2]
    akh = np.abs(kh)
    # dq = w U, U = sum_s g [x > 0] k^
    dq_b = aw[..., None] * ((e @ akh)[:, None, :]
                            + (amb.reshape(T * HI, S) @ akh).reshape(T, HI, DI))
    # dw = U . q^ = sum_s g ReLU(x^): x^ = code_dot qs ks
    xabs = np.abs(code_dot) * qs[..., None] * ks[None, None, :]
    dw_b = (e[:, None, :] * xabs).sum(-1) + (amb * xabs).sum(-1)
    # dk = sum_t sum_j g w [x > 0] q^
    wq = (aw[..., None] * np.abs(qh))                               # [T, HI, DI]
    dk_b = e.T @ wq.sum(1) + amb.transpose(2, 0, 1).reshape(S, T * HI) @ wq.reshape(T * HI, DI)
    return loss_b, dw_b, dq_b, dk_b


def _check(got, want, bound, what):
    err = np.abs(np.asarray(got, dtype=np.float64) - want)
    ratio = float((err / (bound + 1e-30)).max())
    assert ratio <= 1.0, f"{what}: error {ratio:.3f} x bound (max-abs {err.max():.3e})"
    return ratio


@pytest.mark.parametrize("base,L", [("tiny", 256), ("prefill_4k", 384)])
def test_warmup_loss_and_gradient_match_oracle(base, L):
    cfg = dsa_inputs.custom_config(base, n_q=L, n_kv=L, name=f"kl{L}")
    inp = dsa_inputs.make_inputs(cfg, seed=17)
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    res = dsa.indexer_kl(g, cfg)
    dsa.dsa_check()
    ref = oracle.indexer_kl(inp["q_fp8"][0], inp["q_scale"][0], inp["w"][0], inp["k_fp8"][0],
                            inp["k_scale"][0], np.arange(L, dtype=np.int32), L, inp["q"][0],
                            inp["kv"][0], cfg.softmax_scale)
    loss_b, dw_b, dq_b, dk_b = _bounds(cfg, inp)
    _check(res["loss"][0].cpu().numpy(), ref["loss"], loss_b, "loss")
    _check(res["dw"][0].cpu().numpy(), ref["dw"], dw_b, "dw")
    _check(res["dq"][0].cpu().numpy(), ref["dq"], dq_b, "dq")
    _check(res["dk"][0].cpu().numpy(), ref["dk"], dk_b, "dk")
    assert res["loss"][0, 0].item() == 0.0 and ref["loss"][1:].max() > 1e-3


def test_warmup_loss_calls_are_repeatable():
    """Two calls on the same inputs give the same bits (dk is cleared by the
    call and summed in a fixed order; nothing is accumulated across calls)."""
    cfg = dsa_inputs.custom_config("prefill_4k", n_q=300, n_kv=300, name="kl_rep")
    g = dsa_inputs.make_inputs(cfg, seed=19, device="cuda")
    a = dsa.indexer_kl(g, cfg)
    b = dsa.indexer_kl(g, cfg)
    dsa.dsa_check()
    for k in ("loss", "dw", "dq", "dk"):
        assert torch.equal(a[k], b[k]), k
