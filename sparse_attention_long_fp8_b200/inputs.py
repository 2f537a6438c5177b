"""Seeded synthetic inputs for the DSA forward path.

This module only draws random numbers and packs them into the layouts the
library and the oracle both read. It holds none of the method's arithmetic:
no score, no selection, no attention. The FP8 encoding step is the upstream
quantiser that produces the path's inputs (page "DeepseekV3.2 拆解", section
"核心组件 / 闪电索引器": the indexer consumes FP8 q and k).

Input recipe (all tensors contiguous):

* indexer query  ``q_fp8``  [B, T, HI, DI] uint8 (e4m3fn bit patterns),
  per (token, head) row scale ``q_scale`` [B, T, HI] fp32 = amax/448
  (amax == 0 gives scale 1);
* head weights   ``w``      [B, T, HI] fp32 ~ N(0, 1) * w_std;
* indexer key    ``k_fp8``  [B, S, DI] uint8, per-token ``k_scale`` [B, S];
* main query     ``q``      [B, T, H, Dqk] bf16 ~ N(0, 1);
* latent rows    ``kv``     [B, S, Dqk] bf16 ~ N(0, 1); V is kv[..., :Dv];
* hot keys: round(hot_frac * S) positions per sequence, drawn without
  replacement, get ``hot_mag * u`` added to the indexer key (before
  quantisation) and to the latent row, with one shared direction u per
  sequence and per tensor, scaled to per-element RMS 1.
"""
from __future__ import annotations

import dataclasses
import math

import torch

FP8_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class DsaConfig:
    """Shape of one DSA workload."""

    name: str
    batch: int
    n_q: int          # query rows per sequence (T)
    n_kv: int         # key rows per sequence (S)
    idx_heads: int    # H^I
    idx_dim: int      # d^I
    topk: int         # k
    heads: int        # H (main attention query heads)
    qk_dim: int       # D_qk
    v_dim: int        # D_v
    softmax_scale: float
    w_std: float
    hot_frac: float
    hot_mag: float = 3.0
    decode: bool = False   # one query per sequence at position kv_len-1


def _cfg_prefill(name, L, seed_dims="full"):
    if seed_dims == "tiny":
        return DsaConfig(name, 1, L, L, 4, 32, 64, 8, 64, 64, 1.0 / 8.0,
                         1.0 / 2.0, 0.0)
    return DsaConfig(name, 1, L, L, 64, 128, 2048, 128, 576, 512,
                     1.0 / math.sqrt(576.0), 1.0 / 8.0, 0.05)


CONFIGS = {
    "tiny": _cfg_prefill("tiny", 256, "tiny"),
    "prefill_4k": _cfg_prefill("prefill_4k", 4096),
    "prefill_16k": _cfg_prefill("prefill_16k", 16384),
    "prefill_64k": _cfg_prefill("prefill_64k", 65536),
    "decode_32k": DsaConfig("decode_32k", 64, 1, 32768, 64, 128, 2048, 128,
                            576, 512, 1.0 / math.sqrt(576.0), 1.0 / 8.0,
                            0.05, decode=True),
    "decode_64k": DsaConfig("decode_64k", 64, 1, 65536, 64, 128, 2048, 128,
                            576, 512, 1.0 / math.sqrt(576.0), 1.0 / 8.0,
                            0.05, decode=True),
}


def custom_config(base: str = "tiny", **changes) -> DsaConfig:
    """A named config with some fields replaced (for edge-case tests)."""
    return dataclasses.replace(CONFIGS[base], **changes)


def quantize_e4m3_rows(x: torch.Tensor):
    """Per-row (last dim) e4m3fn encoding with scale amax/448.

    Returns (codes uint8 with the same shape, scales fp32 with the last dim
    dropped). Rounding is torch's round-to-nearest-even cast after clamping to
    the finite range.
    """
    x = x.float()
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax))
    y = (x / scale.unsqueeze(-1)).clamp(-FP8_MAX, FP8_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()


def _unit_rms_direction(dim, gen, device):
    g = torch.randn(dim, generator=gen, device=device, dtype=torch.float32)
    return g * (math.sqrt(dim) / g.norm())


def make_inputs(cfg: DsaConfig, seed: int = 0, device="cpu"):
    """Draw every input of one DSA forward call for ``cfg``.

    Deterministic for a given (cfg, seed, device type). Large configs should
    be drawn on the GPU (``device='cuda'``); the oracle then reads host copies
    of the rows it checks.
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    B, T, S = cfg.batch, cfg.n_q, cfg.n_kv
    HI, DI, H, Dqk = cfg.idx_heads, cfg.idx_dim, cfg.heads, cfg.qk_dim

    q_idx = torch.randn(B, T, HI, DI, generator=gen, device=device)
    k_idx = torch.randn(B, S, DI, generator=gen, device=device)
    w = torch.randn(B, T, HI, generator=gen, device=device) * cfg.w_std
    q = torch.randn(B, T, H, Dqk, generator=gen, device=device,
                    dtype=torch.bfloat16)
    kv = torch.randn(B, S, Dqk, generator=gen, device=device)

    n_hot = int(round(cfg.hot_frac * S))
    hot_pos = []
    if n_hot > 0:
        for b in range(B):
            pos = torch.randperm(S, generator=gen, device=device)[:n_hot]
            u_k = _unit_rms_direction(DI, gen, device)
            u_c = _unit_rms_direction(Dqk, gen, device)
            k_idx[b, pos] += cfg.hot_mag * u_k
            kv[b, pos] += cfg.hot_mag * u_c
            hot_pos.append(pos)

    q_fp8, q_scale = quantize_e4m3_rows(q_idx)
    k_fp8, k_scale = quantize_e4m3_rows(k_idx)
    del q_idx, k_idx

    if cfg.decode:
        kv_len = torch.full((B,), S, dtype=torch.int32, device=device)
        q_pos0 = kv_len - 1
    else:
        kv_len = torch.full((B,), S, dtype=torch.int32, device=device)
        q_pos0 = torch.zeros(B, dtype=torch.int32, device=device)

    return {
        "q_fp8": q_fp8, "q_scale": q_scale, "w": w.contiguous(),
        "k_fp8": k_fp8, "k_scale": k_scale,
        "q": q.contiguous(), "kv": kv.to(torch.bfloat16).contiguous(),
        "q_pos0": q_pos0, "kv_len": kv_len,
        "hot_pos": hot_pos,
    }
