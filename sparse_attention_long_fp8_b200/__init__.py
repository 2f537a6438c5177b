"""DeepSeek Sparse Attention forward path on B200 (sm_100a).

Thin ctypes binding over the C ABI in ``include/dsa.h`` (libdsa.so). Every
step of the path runs in the library's CUDA kernels; this module only checks
tensor dtypes/devices, passes raw pointers and turns status codes into
exceptions. There is no CPU fallback: if the library is missing, importing a
call raises.
"""
from __future__ import annotations

import ctypes
import os

from .inputs import CONFIGS, DsaConfig, custom_config, make_inputs  # noqa: F401

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa.so")

DSA_OK = 0
DSA_ERR_INVALID_ARG = 1
DSA_ERR_UNSUPPORTED = 2
DSA_ERR_WORKSPACE = 3
DSA_ERR_CUDA = 4
DSA_ERR_TIMEOUT = 5
DSA_ERR_NO_DEVICE = 6

DSA_OUT_F32 = 0
DSA_OUT_BF16 = 1

DSA_SCORES_ALL = 0
DSA_SCORES_VISIBLE_ONLY = 1

DSA_OP_INDEXER = 0
DSA_OP_TOPK = 1
DSA_OP_SPARSE_ATTN = 2
DSA_OP_FORWARD = 3
DSA_OP_INDEXER_KL = 4


class DsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"[{status}] {message}")
        self.status = status


class DsaShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q", ctypes.c_int32), ("n_kv", ctypes.c_int32),
                ("idx_heads", ctypes.c_int32), ("idx_dim", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("qk_dim", ctypes.c_int32), ("v_dim", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float)]


class DsaLayout(ctypes.Structure):
    """dsa_layout: explicit query positions and / or a paged key cache."""
    _fields_ = [("row_pos", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("max_pages", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("pool_rows", ctypes.c_int64)]


def make_layout(row_pos=None, block_table=None, page_size=0, pool_rows=0):
    """A DsaLayout from CUDA tensors: row_pos [B, n_q] int32 and/or
    block_table [B, max_pages] int32 with the pool geometry. The tensors must
    outlive every call that uses the layout."""
    lay = DsaLayout()
    lay.row_pos = _ptr(row_pos, _dt()["i32"], "row_pos")
    if block_table is not None:
        lay.block_table = _ptr(block_table, _dt()["i32"], "block_table")
        lay.max_pages = int(block_table.shape[-1])
        lay.page_size = int(page_size)
        lay.pool_rows = int(pool_rows)
    return lay


_lib = None


def load_library(path: str | None = None):
    """Load libdsa.so (built by ``python -m sparse_attention_long_fp8_b200.build``)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m sparse_attention_long_fp8_b200.build`")
    try:  # share torch's CUDA runtime when torch is present
        import torch  # noqa: F401
    except ImportError:
        pass
    lib = ctypes.CDLL(path)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    SP = ctypes.POINTER(DsaShape)
    lib.dsa_indexer_scores.argtypes = [SP, P, P, P, P, P, P, P, I32, I32, I32, P, P]
    lib.dsa_indexer_topk.argtypes = [SP, P, P, P, P, P, P, P, I32, I32, P, P]
    lib.dsa_topk.argtypes = [SP, P, I32, I32, P, P, P, P, SZ, P]
    lib.dsa_sparse_attn.argtypes = [SP, P, P, P, P, I32, P, P, SZ, P]
    lib.dsa_sparse_attn_noalloc.argtypes = [SP, P, P, P, P, I32, P, P]
    lib.dsa_forward.argtypes = [SP, P, P, P, P, P, P, P, P, P, P, P, I32, P, P, SZ, P]
    lib.dsa_workspace_size.argtypes = [SP, I32, ctypes.POINTER(SZ)]
    lib.dsa_indexer_kl.argtypes = [SP, P, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
    lib.dsa_check.argtypes = [P]
    lib.dsa_quantize_e4m3.argtypes = [ctypes.c_int64, I32, P, P, P, P]
    lib.dsa_quantize_e4m3.restype = ctypes.c_int
    lib.dsa_selftest_wait_timeout.argtypes = [ctypes.c_uint32, P]
    lib.dsa_selftest_wait_timeout.restype = ctypes.c_int
    lib.dsa_forward_chunk_rows.argtypes = [SP, ctypes.POINTER(I32)]
    lib.dsa_forward_plan.argtypes = [SP, ctypes.POINTER(I32), ctypes.POINTER(I32),
                                     ctypes.POINTER(I32)]
    LP = ctypes.POINTER(DsaLayout)
    lib.dsa_indexer_scores_ex.argtypes = [SP, LP, P, P, P, P, P, P, P, I32, I32, I32, P, P]
    lib.dsa_indexer_topk_ex.argtypes = [SP, LP, P, P, P, P, P, P, P, I32, I32, P, P]
    lib.dsa_topk_ex.argtypes = [SP, LP, P, I32, I32, P, P, P, P, SZ, P]
    lib.dsa_sparse_attn_ex.argtypes = [SP, LP, P, P, P, P, I32, P, P, SZ, P]
    lib.dsa_forward_ex.argtypes = [SP, LP, P, P, P, P, P, P, P, P, P, P, P, I32, P, P, SZ, P]
    lib.dsa_status_string.argtypes = [ctypes.c_int]
    lib.dsa_status_string.restype = ctypes.c_char_p
    lib.dsa_last_error.restype = ctypes.c_char_p
    lib.dsa_version.restype = ctypes.c_char_p
    for fn in ("dsa_indexer_scores", "dsa_indexer_topk", "dsa_topk", "dsa_sparse_attn", "dsa_forward",
               "dsa_workspace_size", "dsa_check", "dsa_forward_chunk_rows",
               "dsa_sparse_attn_noalloc", "dsa_forward_plan", "dsa_indexer_scores_ex",
               "dsa_indexer_topk_ex", "dsa_topk_ex", "dsa_sparse_attn_ex", "dsa_forward_ex",
               "dsa_indexer_kl"):
        getattr(lib, fn).restype = ctypes.c_int
    if path == LIB_PATH:
        _lib = lib
    return lib


def _raise(status: int):
    if status != DSA_OK:
        lib = load_library()
        msg = lib.dsa_last_error().decode() or lib.dsa_status_string(status).decode()
        raise DsaError(status, msg)


def shape_of(cfg: DsaConfig) -> DsaShape:
    return DsaShape(cfg.batch, cfg.n_q, cfg.n_kv, cfg.idx_heads, cfg.idx_dim, cfg.topk,
                    cfg.heads, cfg.qk_dim, cfg.v_dim, cfg.softmax_scale)


def _ptr(t, dtype=None, what="tensor"):
    """Raw device pointer of a contiguous CUDA tensor (or None -> NULL)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if dtype is not None and t.dtype not in dtype:
        raise ValueError(f"{what} has dtype {t.dtype}, expected one of {dtype}")
    return t.data_ptr()


def _lay(layout):
    return ctypes.byref(layout) if layout is not None else None


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _dt():
    import torch
    return {
        "u8": (torch.uint8, torch.float8_e4m3fn), "f32": (torch.float32,),
        "i32": (torch.int32,), "bf16": (torch.bfloat16, torch.int16),
    }


def workspace_size(shape: DsaShape, op: int) -> int:
    n = ctypes.c_size_t(0)
    _raise(load_library().dsa_workspace_size(ctypes.byref(shape), op, ctypes.byref(n)))
    return n.value


def forward_chunk_rows(shape: DsaShape) -> int:
    n = ctypes.c_int32(0)
    _raise(load_library().dsa_forward_chunk_rows(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def forward_plan(shape: DsaShape) -> dict:
    """dsa_forward's plan for this shape: fused (bool), chunk_rows, attn_splits."""
    f, c, sp = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_int32(0)
    _raise(load_library().dsa_forward_plan(ctypes.byref(shape), ctypes.byref(f), ctypes.byref(c),
                                           ctypes.byref(sp)))
    return {"fused": bool(f.value), "chunk_rows": c.value, "attn_splits": sp.value}


def dsa_indexer_scores(shape, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0, kv_len,
                       row_begin, row_end, scores, stream=None, flags=DSA_SCORES_ALL,
                       layout=None):
    d = _dt()
    _raise(load_library().dsa_indexer_scores_ex(
        ctypes.byref(shape), _lay(layout), _ptr(q_fp8, d["u8"], "q_fp8"), _ptr(q_scale, d["f32"], "q_scale"),
        _ptr(w, d["f32"], "w"), _ptr(k_fp8, d["u8"], "k_fp8"), _ptr(k_scale, d["f32"], "k_scale"),
        _ptr(q_pos0, d["i32"], "q_pos0"), _ptr(kv_len, d["i32"], "kv_len"),
        int(row_begin), int(row_end), int(flags), _ptr(scores, d["f32"], "scores"),
        _stream(stream)))


def dsa_indexer_topk(shape, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0, kv_len,
                     row_begin, row_end, indices, stream=None, layout=None):
    d = _dt()
    _raise(load_library().dsa_indexer_topk_ex(
        ctypes.byref(shape), _lay(layout), _ptr(q_fp8, d["u8"], "q_fp8"), _ptr(q_scale, d["f32"], "q_scale"),
        _ptr(w, d["f32"], "w"), _ptr(k_fp8, d["u8"], "k_fp8"), _ptr(k_scale, d["f32"], "k_scale"),
        _ptr(q_pos0, d["i32"], "q_pos0"), _ptr(kv_len, d["i32"], "kv_len"),
        int(row_begin), int(row_end), _ptr(indices, d["i32"], "indices"), _stream(stream)))


def dsa_quantize_e4m3(x, codes, scales, stream=None):
    """Per-row E4M3 quantisation of a bf16 tensor x [..., dim] into codes
    (uint8, same shape) and scales (fp32, x.shape[:-1])."""
    import torch
    d = _dt()
    rows = x.numel() // x.shape[-1] if x.numel() else 0
    if codes.shape != x.shape or tuple(scales.shape) != tuple(x.shape[:-1]):
        raise ValueError("codes must match x and scales must be x.shape[:-1]")
    for t, name in ((x, "x"), (codes, "codes"), (scales, "scales")):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    _raise(load_library().dsa_quantize_e4m3(
        int(rows), int(x.shape[-1]), _ptr(x, d["bf16"], "x"),
        _ptr(codes, (torch.uint8, torch.float8_e4m3fn), "codes"), _ptr(scales, d["f32"], "scales"),
        _stream(stream)))


def dsa_selftest_wait_timeout(limit_ms=100, stream=None):
    """Launch the bounded-wait self-test; the next dsa_check() raises a
    DsaError with status DSA_ERR_TIMEOUT."""
    _raise(load_library().dsa_selftest_wait_timeout(int(limit_ms), _stream(stream)))


def dsa_topk(shape, scores, row_begin, row_end, q_pos0, kv_len, indices, ws=None,
             ws_bytes=0, stream=None, layout=None):
    d = _dt()
    _raise(load_library().dsa_topk_ex(
        ctypes.byref(shape), _lay(layout), _ptr(scores, d["f32"], "scores"), int(row_begin), int(row_end),
        _ptr(q_pos0, d["i32"], "q_pos0"), _ptr(kv_len, d["i32"], "kv_len"),
        _ptr(indices, d["i32"], "indices"), _ptr(ws, None, "ws"), int(ws_bytes),
        _stream(stream)))


def dsa_sparse_attn(shape, q, kv, indices, out, lse=None, ws=None, ws_bytes=0, stream=None,
                    layout=None):
    import torch
    d = _dt()
    out_dtype = DSA_OUT_BF16 if out.dtype == torch.bfloat16 else DSA_OUT_F32
    _raise(load_library().dsa_sparse_attn_ex(
        ctypes.byref(shape), _lay(layout), _ptr(q, d["bf16"], "q"), _ptr(kv, d["bf16"], "kv"),
        _ptr(indices, d["i32"], "indices"), _ptr(out, (torch.float32, torch.bfloat16), "out"),
        out_dtype, _ptr(lse, d["f32"], "lse"), _ptr(ws, None, "ws"), int(ws_bytes),
        _stream(stream)))


def dsa_sparse_attn_noalloc(shape, q, kv, indices, out, lse=None, stream=None):
    """dsa_sparse_attn for callers that cannot allocate: the split-K scratch
    is a 16 MiB array inside the library (see include/dsa.h)."""
    import torch
    d = _dt()
    out_dtype = DSA_OUT_BF16 if out.dtype == torch.bfloat16 else DSA_OUT_F32
    _raise(load_library().dsa_sparse_attn_noalloc(
        ctypes.byref(shape), _ptr(q, d["bf16"], "q"), _ptr(kv, d["bf16"], "kv"),
        _ptr(indices, d["i32"], "indices"), _ptr(out, (torch.float32, torch.bfloat16), "out"),
        out_dtype, _ptr(lse, d["f32"], "lse"), _stream(stream)))


def dsa_forward(shape, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0, kv_len, q, kv,
                indices_out, out, lse=None, ws=None, ws_bytes=0, stream=None, layout=None):
    import torch
    d = _dt()
    out_dtype = DSA_OUT_BF16 if out.dtype == torch.bfloat16 else DSA_OUT_F32
    _raise(load_library().dsa_forward_ex(
        ctypes.byref(shape), _lay(layout), _ptr(q_fp8, d["u8"], "q_fp8"), _ptr(q_scale, d["f32"], "q_scale"),
        _ptr(w, d["f32"], "w"), _ptr(k_fp8, d["u8"], "k_fp8"), _ptr(k_scale, d["f32"], "k_scale"),
        _ptr(q_pos0, d["i32"], "q_pos0"), _ptr(kv_len, d["i32"], "kv_len"),
        _ptr(q, d["bf16"], "q"), _ptr(kv, d["bf16"], "kv"),
        _ptr(indices_out, d["i32"], "indices_out"),
        _ptr(out, (torch.float32, torch.bfloat16), "out"), out_dtype,
        _ptr(lse, d["f32"], "lse"), _ptr(ws, None, "ws"), int(ws_bytes), _stream(stream)))


def dsa_indexer_kl(shape, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0, kv_len, q, kv,
                   loss, dw, dq, dk, ws=None, ws_bytes=0, stream=None):
    d = _dt()
    _raise(load_library().dsa_indexer_kl(
        ctypes.byref(shape), _ptr(q_fp8, d["u8"], "q_fp8"), _ptr(q_scale, d["f32"], "q_scale"),
        _ptr(w, d["f32"], "w"), _ptr(k_fp8, d["u8"], "k_fp8"), _ptr(k_scale, d["f32"], "k_scale"),
        _ptr(q_pos0, d["i32"], "q_pos0"), _ptr(kv_len, d["i32"], "kv_len"),
        _ptr(q, d["bf16"], "q"), _ptr(kv, d["bf16"], "kv"), _ptr(loss, d["f32"], "loss"),
        _ptr(dw, d["f32"], "dw"), _ptr(dq, d["f32"], "dq"), _ptr(dk, d["f32"], "dk"),
        _ptr(ws, None, "ws"), int(ws_bytes), _stream(stream)))


def indexer_kl(inp: dict, cfg: DsaConfig, stream=None):
    """The warm-up loss and gradient on CUDA tensors from ``make_inputs``;
    returns dict(loss, dw, dq, dk). Buffers are allocated with torch."""
    import torch
    shape = shape_of(cfg)
    dev = inp["q"].device
    B, T, S = cfg.batch, cfg.n_q, cfg.n_kv
    loss = torch.empty(B, T, device=dev)
    dw = torch.empty(B, T, cfg.idx_heads, device=dev)
    dq = torch.empty(B, T, cfg.idx_heads, cfg.idx_dim, device=dev)
    dk = torch.empty(B, S, cfg.idx_dim, device=dev)
    ws, n = alloc_workspace(shape, DSA_OP_INDEXER_KL, dev)
    dsa_indexer_kl(shape, inp["q_fp8"], inp["q_scale"], inp["w"], inp["k_fp8"], inp["k_scale"],
                   inp["q_pos0"], inp["kv_len"], inp["q"], inp["kv"], loss, dw, dq, dk, ws, n,
                   stream)
    return {"loss": loss, "dw": dw, "dq": dq, "dk": dk}


def dsa_check(stream=None):
    _raise(load_library().dsa_check(_stream(stream)))


# ------------------------------------------------------------------ conveniences

def alloc_workspace(shape: DsaShape, op: int, device="cuda"):
    """A 256-byte aligned uint8 workspace tensor of the size ``op`` needs."""
    import torch
    n = workspace_size(shape, op)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device), n


def forward(inp: dict, cfg: DsaConfig, out_dtype=None, ws=None, stream=None, layout=None):
    """Run the whole path on CUDA tensors from ``make_inputs``; returns
    dict(indices, out, lse). Output buffers are allocated with torch."""
    import torch
    shape = shape_of(cfg)
    dev = inp["q"].device
    B, T = cfg.batch, cfg.n_q
    out = torch.empty(B, T, cfg.heads, cfg.v_dim, device=dev,
                      dtype=out_dtype or torch.float32)
    lse = torch.empty(B, T, cfg.heads, device=dev, dtype=torch.float32)
    idx = torch.empty(B, T, cfg.topk, device=dev, dtype=torch.int32)
    if ws is None:
        ws, n = alloc_workspace(shape, DSA_OP_FORWARD, dev)
    else:
        n = ws.numel()
    dsa_forward(shape, inp["q_fp8"], inp["q_scale"], inp["w"], inp["k_fp8"], inp["k_scale"],
                inp["q_pos0"], inp["kv_len"], inp["q"], inp["kv"], idx, out, lse, ws, n, stream,
                layout=layout)
    return {"indices": idx, "out": out, "lse": lse}
