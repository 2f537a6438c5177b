"""Python access to the fp64 CPU oracle (oracle.cpp).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the library under
``sparse_attention_long_fp8_b200`` never does.

Each wrapper takes numpy arrays (or CPU torch tensors), works on ONE
sequence, and returns numpy float64 / int32 arrays. See oracle.cpp for the
definitions and the page passages they follow.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so next to it (plain g++, no CUDA)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
                        "-ffp-contract=off", "-o", tmp, _SRC], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.oracle_hardware_threads.restype = I
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_quantize_rows.argtypes = [ctypes.c_longlong, I, P, P, P]
        lib.oracle_indexer_scores.argtypes = [I, I, I, I, P, P, P, P, P, P, I, P, I]
        lib.oracle_topk.argtypes = [I, I, I, P, P, I]
        lib.oracle_sparse_attn.argtypes = [I, I, I, I, I, I, ctypes.c_double,
                                           P, P, P, P, P, I]
        lib.oracle_indexer_kl.argtypes = [I, I, I, I, P, P, P, P, P, P, I, I, I,
                                          ctypes.c_double, P, P, P, P, P, P, I]
        _lib = lib
    return _lib


def _np(x, dtype):
    """numpy copy of x in ``dtype``; fp8 / bf16 tensors give their raw bits."""
    import torch
    if isinstance(x, torch.Tensor):
        x = x.detach().contiguous().cpu()
        if x.dtype == torch.float8_e4m3fn:
            x = x.view(torch.uint8)
        elif x.dtype == torch.bfloat16:
            x = x.view(torch.int16)
        x = x.numpy()
    x = np.asarray(x)
    dt = np.dtype(dtype)
    if x.dtype.kind in "iu" and dt.kind in "iu" and x.dtype.itemsize == dt.itemsize:
        return np.ascontiguousarray(x).view(dt)
    return np.ascontiguousarray(x, dtype=dt)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def hardware_threads() -> int:
    return int(_load().oracle_hardware_threads())


def e4m3_value(code: int) -> float:
    return float(_load().oracle_e4m3_value(int(code)))


def e4m3_encode(v: float) -> int:
    return int(_load().oracle_e4m3_encode(float(v)))


def quantize_rows(x):
    """Per-row E4M3 encoding of bf16 rows x [rows, dim] (torch bf16 or raw
    uint16 bits): returns (codes uint8 [rows, dim], scales float32 [rows])."""
    xb = _np(x, np.uint16)
    rows, dim = xb.shape
    codes = np.zeros((rows, dim), dtype=np.uint8)
    scales = np.zeros(rows, dtype=np.float32)
    _load().oracle_quantize_rows(rows, dim, _ptr(xb), _ptr(codes), _ptr(scales))
    return codes, scales


def indexer_scores(q8, qs, w, k8, ks, pos, kv_len, n_threads=0):
    """I[t,s] for rows given by q8 [n, HI, DI], qs/w [n, HI], pos [n].

    k8 [S, DI], ks [S]. Invalid pairs are -inf. Returns float64 [n, S].
    """
    q8 = _np(q8, np.uint8); k8 = _np(k8, np.uint8)
    qs = _np(qs, np.float32); w = _np(w, np.float32); ks = _np(ks, np.float32)
    pos = _np(pos, np.int32)
    n, HI, DI = q8.shape
    S = k8.shape[0]
    assert k8.shape == (S, DI) and qs.shape == (n, HI) and w.shape == (n, HI)
    assert ks.shape == (S,) and pos.shape == (n,)
    out = np.empty((n, S), dtype=np.float64)
    _load().oracle_indexer_scores(n, S, HI, DI, _ptr(q8), _ptr(qs), _ptr(w),
                                  _ptr(k8), _ptr(ks), _ptr(pos), int(kv_len),
                                  _ptr(out), int(n_threads))
    return out


def topk(scores, k, n_threads=0):
    """Top-k key indices per row of float64 scores [n, S] (-inf = invalid)."""
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    n, S = scores.shape
    out = np.empty((n, k), dtype=np.int32)
    _load().oracle_topk(n, S, int(k), _ptr(scores), _ptr(out), int(n_threads))
    return out


def sparse_attn(q, kv, idx, scale, v_dim, n_threads=0):
    """Attention of q [n, H, Dqk] (bf16) over kv rows idx [n, k] of kv [S, Dqk].

    Returns (o float64 [n, H, v_dim], lse float64 [n, H]).
    """
    q = _np(q, np.uint16); kv = _np(kv, np.uint16); idx = _np(idx, np.int32)
    n, H, Dqk = q.shape
    S = kv.shape[0]
    k = idx.shape[1]
    assert kv.shape == (S, Dqk) and idx.shape[0] == n
    o = np.empty((n, H, v_dim), dtype=np.float64)
    lse = np.empty((n, H), dtype=np.float64)
    _load().oracle_sparse_attn(n, S, H, Dqk, int(v_dim), k, float(scale), _ptr(q),
                               _ptr(kv), _ptr(idx), _ptr(o), _ptr(lse), int(n_threads))
    return o, lse


def indexer_kl(q8, qs, w, k8, ks, pos, kv_len, q, kv, scale, n_threads=0):
    """Indexer warm-up loss and gradient (see oracle.cpp, oracle_indexer_kl)
    for rows q8 [n, HI, DI], qs/w [n, HI], pos [n], main queries q [n, H, Dqk]
    (bf16) against keys k8 [S, DI], ks [S] and latent rows kv [S, Dqk].

    Returns dict(loss [n], dw [n, HI], dq [n, HI, DI], dk [S, DI]), float64;
    dq / dk are gradients with respect to the dequantised indexer vectors.
    """
    q8 = _np(q8, np.uint8); k8 = _np(k8, np.uint8)
    qs = _np(qs, np.float32); w = _np(w, np.float32); ks = _np(ks, np.float32)
    pos = _np(pos, np.int32); q = _np(q, np.uint16); kv = _np(kv, np.uint16)
    n, HI, DI = q8.shape
    S = k8.shape[0]
    _, H, Dqk = q.shape
    assert k8.shape == (S, DI) and qs.shape == (n, HI) and w.shape == (n, HI)
    assert ks.shape == (S,) and pos.shape == (n,) and q.shape[0] == n and kv.shape == (S, Dqk)
    loss = np.empty(n, dtype=np.float64)
    dw = np.empty((n, HI), dtype=np.float64)
    dq = np.empty((n, HI, DI), dtype=np.float64)
    dk = np.empty((S, DI), dtype=np.float64)
    _load().oracle_indexer_kl(n, S, HI, DI, _ptr(q8), _ptr(qs), _ptr(w), _ptr(k8), _ptr(ks),
                              _ptr(pos), int(kv_len), H, Dqk, float(scale), _ptr(q), _ptr(kv),
                              _ptr(loss), _ptr(dw), _ptr(dq), _ptr(dk), int(n_threads))
    return {"loss": loss, "dw": dw, "dq": dq, "dk": dk}


def forward(inp, cfg, b=0, rows=None, n_threads=0):
    """Full path (scores -> top-k -> attention) for rows of sequence b.

    ``inp`` is a dict from ``inputs.make_inputs`` (CPU or GPU tensors);
    ``rows`` are query-row indices within the sequence (default: all).
    Returns dict(scores, indices, o, lse).
    """
    import torch
    T = cfg.n_q
    rows = np.arange(T) if rows is None else np.asarray(rows)
    rt = torch.as_tensor(rows, dtype=torch.long)
    dev_rows = rt.to(inp["q_fp8"].device)
    q_pos0 = int(inp["q_pos0"][b])
    kv_len = int(inp["kv_len"][b])
    pos = (rows + q_pos0).astype(np.int32)
    sc = indexer_scores(inp["q_fp8"][b].index_select(0, dev_rows),
                        inp["q_scale"][b].index_select(0, dev_rows),
                        inp["w"][b].index_select(0, dev_rows),
                        inp["k_fp8"][b], inp["k_scale"][b], pos, kv_len, n_threads)
    idx = topk(sc, cfg.topk, n_threads)
    o, lse = sparse_attn(inp["q"][b].index_select(0, dev_rows), inp["kv"][b], idx,
                         cfg.softmax_scale, cfg.v_dim, n_threads)
    return {"scores": sc, "indices": idx, "o": o, "lse": lse}
