"""Query-sharded prefill: one DSA prefill split over several GPUs.

The path shards with one exchange (page "DeepseekV3.2 拆解", complexity
table: the indexer search grows as L^2 and the core attention as L*k, so a
long prefill is worth spreading). Query rows are independent once every GPU
holds all keys: the FP8 indexer keys with their scales and the latent rows
(132 + 1152 bytes per token, 84 MB at L = 65536). So:

* the 4-row query groups the fused indexer works on are dealt to the ranks
  longest-first, round-robin: rank r takes groups G-1-r, G-1-r-R, ... of the
  G = ceil(L / 4) groups. Group g costs about g key tiles in the indexer and
  4 rows in the attention, so every rank gets the same number of rows and
  indexer work within one group;
* each rank runs dsa_forward_ex on its rows only, compacted, with their
  absolute positions in a dsa_layout (row_pos), so the causal masks are
  those of the whole sequence;
* when the keys were produced sequence-sharded (rank r holds keys
  [r S / R, (r + 1) S / R)), one all-gather per key tensor brings them into
  every GPU's own memory first. No kernel reads another GPU's memory.

This module is host plumbing: the partition, the row gathers (torch index
ops) and the collective. Every step of the method runs in the library's
kernels.
"""
from __future__ import annotations

import numpy as np

GROUP = 4   # query rows per fused-indexer tile group


def shard_groups(n_q: int, n_shards: int, shard: int) -> np.ndarray:
    """The 4-row groups of one shard, in increasing order (the fused kernel
    runs the last, longest group of a call first)."""
    if not (0 <= shard < n_shards):
        raise ValueError(f"shard {shard} outside [0, {n_shards})")
    n_groups = (n_q + GROUP - 1) // GROUP
    return np.arange(n_groups - 1 - shard, -1, -n_shards, dtype=np.int64)[::-1].copy()


def shard_rows(n_q: int, n_shards: int, shard: int) -> np.ndarray:
    """Query rows of one shard, in increasing order: whole 4-row groups, the
    last group cut at n_q."""
    g = shard_groups(n_q, n_shards, shard)
    rows = (g[:, None] * GROUP + np.arange(GROUP)[None, :]).reshape(-1)
    return rows[rows < n_q]


def shard_cost(n_q: int, n_kv: int, n_shards: int, shard: int, topk: int):
    """(indexer visible pairs, attention selected pairs) of a shard's rows in
    a causal prefill from position 0: the work the partition balances."""
    rows = shard_rows(n_q, n_shards, shard)
    vis = np.minimum(rows + 1, n_kv)
    return int(vis.sum()), int(np.minimum(vis, topk).sum())


def key_slice(n_kv: int, n_shards: int, shard: int):
    """[begin, end) of the keys a rank holds when they are produced
    sequence-sharded (equal slices; the last one takes the remainder)."""
    per = (n_kv + n_shards - 1) // n_shards
    return min(n_kv, shard * per), min(n_kv, (shard + 1) * per)


def all_gather_keys(local, n_kv, dist, group=None):
    """Every rank's slice of a key tensor [B, slice, ...] -> the full tensor
    [B, n_kv, ...] in this rank's memory (one all-gather along the key axis;
    slices are padded to equal length for the collective)."""
    import torch
    dtype = local.dtype
    if local.dim() >= 3 and (local.shape[-1] * local.element_size()) % 4 == 0 and dtype != torch.int32:
        # moved as 32-bit words: every backend gathers int32 (gloo has no
        # uint8 / bf16 collectives), and the bytes are what matter
        return all_gather_keys(local.contiguous().view(torch.int32), n_kv, dist, group).view(dtype)
    world = dist.get_world_size(group)
    per = (n_kv + world - 1) // world
    B = local.shape[0]
    pad = torch.zeros((B, per) + tuple(local.shape[2:]), dtype=local.dtype, device=local.device)
    pad[:, : local.shape[1]] = local
    out = torch.empty((world * B, per) + tuple(local.shape[2:]), dtype=local.dtype,
                      device=local.device)
    dist.all_gather_into_tensor(out, pad.contiguous(), group=group)
    full = out.view((world, B, per) + tuple(local.shape[2:])).transpose(0, 1)
    return full.reshape((B, world * per) + tuple(local.shape[2:]))[:, :n_kv].contiguous()


def shard_inputs(inp: dict, rows: np.ndarray) -> dict:
    """The query-side inputs of one shard's rows, compacted, with their
    absolute positions (row_pos) for a dsa_layout; key-side inputs are
    passed through."""
    import torch
    dev = inp["q"].device
    sel = torch.as_tensor(rows, device=dev)
    out = dict(inp)
    for k in ("q_fp8", "q_scale", "w", "q"):
        out[k] = inp[k].index_select(1, sel).contiguous()
    out["row_pos"] = (inp["q_pos0"][:, None] + sel.to(torch.int32)[None, :]).to(torch.int32)
    out["row_pos"] = out["row_pos"].contiguous()
    return out
