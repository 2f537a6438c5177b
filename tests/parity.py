"""Acceptance rules for GPU-vs-oracle comparisons.

* Scores: |I_gpu - I_oracle| <= SCORE_RTOL * A[t,s], where
  A[t,s] = k_scale[s] * sum_j |c_j| * sum_d |q8_jd| |k8_sd| is the magnitude
  the fp32 sums run over; (d^I + H^I) * 2^-24 bounds the relative rounding of
  an fp32 accumulation of that many terms, and 1.2e-5 covers d^I + H^I <= 192.
* Top-k index sets: per row, every key in the symmetric difference between
  the GPU set and the oracle set must have an oracle score within 1e-4
  relative of that row's k-th oracle score; both sets have min(k, visible)
  distinct visible keys and the GPU pads with -1 after them.
* Attention: against fp64 attention over the GPU-chosen set: max-abs <= 1e-2
  and mean-abs <= 1e-3 (unit-scale inputs), LSE within 1e-3.
"""
import numpy as np
import torch

SCORE_RTOL = 1.2e-5
BAND_RTOL = 1e-4
ATTN_MAX_ABS = 1e-2
ATTN_MEAN_ABS = 1e-3
LSE_ABS = 1e-3


def score_magnitude(q8, qs, w, k8, ks):
    """A[t,s] for rows q8 [n, HI, DI] against keys k8 [S, DI] (float64)."""
    qa = q8.cpu().view(torch.float8_e4m3fn).double().abs()
    ka = k8.cpu().view(torch.float8_e4m3fn).double().abs()
    c = (w.cpu().double() * qs.cpu().double()).abs()                  # [n, HI]
    dots = torch.einsum("njd,sd->njs", qa, ka)                         # [n, HI, S]
    return (torch.einsum("nj,njs->ns", c, dots) * ks.cpu().double()[None, :]).numpy()


def check_scores(gpu, ref, mag):
    gpu = np.asarray(gpu, dtype=np.float64)
    inv_ref = ~np.isfinite(ref)
    assert (np.isneginf(gpu) == inv_ref).all(), "visibility mask differs"
    fin = ~inv_ref
    err = np.abs(gpu[fin] - ref[fin])
    bound = SCORE_RTOL * mag[fin] + 1e-30
    worst = float((err / bound).max()) if err.size else 0.0
    assert worst <= 1.0, f"score error {worst:.3f} x bound"
    return worst


def check_topk_band(gpu_idx, ref_scores, k):
    """gpu_idx [n, k] int32, ref_scores [n, S] float64 (oracle). Returns the
    number of keys that differ (all inside the band)."""
    gpu_idx = np.asarray(gpu_idx)
    n_diff = 0
    for r in range(gpu_idx.shape[0]):
        row = ref_scores[r]
        visible = np.flatnonzero(np.isfinite(row))
        m = min(k, len(visible))
        sel = gpu_idx[r]
        g = sel[:m]
        assert (sel[m:] == -1).all(), f"row {r}: padding"
        assert len(set(g.tolist())) == m, f"row {r}: duplicates or pads inside"
        assert np.isfinite(row[g]).all(), f"row {r}: invisible key selected"
        if m == len(visible):
            assert set(g.tolist()) == set(visible.tolist())
            continue
        order = np.lexsort((visible, -row[visible]))
        ref_set = set(visible[order[:m]].tolist())
        kth = row[visible[order[m - 1]]]
        diff = ref_set.symmetric_difference(g.tolist())
        for s in diff:
            assert abs(row[s] - kth) <= BAND_RTOL * abs(kth), (
                f"row {r}: key {s} score {row[s]!r} outside band of k-th {kth!r}")
        n_diff += len(diff)
    return n_diff


def check_attn(gpu_o, ref_o, gpu_lse=None, ref_lse=None):
    d = np.abs(np.asarray(gpu_o, dtype=np.float64) - ref_o)
    assert d.max() <= ATTN_MAX_ABS, f"max-abs {d.max():.3e}"
    assert d.mean() <= ATTN_MEAN_ABS, f"mean-abs {d.mean():.3e}"
    if gpu_lse is not None:
        g = np.asarray(gpu_lse, dtype=np.float64)
        both_inf = np.isneginf(g) & np.isneginf(ref_lse)
        assert (np.isneginf(g) == np.isneginf(ref_lse)).all()
        dl = np.abs(g[~both_inf] - ref_lse[~both_inf])
        assert dl.size == 0 or dl.max() <= LSE_ABS, f"lse max-abs {dl.max():.3e}"
    return float(d.max()), float(d.mean())
