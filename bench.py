#!/usr/bin/env python
"""Benchmark of the DSA forward path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one call of the public ``dsa_forward`` over one batch of synthetic
input: the lightning indexer with its top-k selection (one fused kernel for
prefill; a score kernel and a selection kernel per row chunk for decode),
then the sparse attention over all rows. The headline workload is DSA
prefill at L = 65536 (batch 1, H^I = 64, d^I = 128, k = 2048, 128-head MQA
over the 576-d latent); prefill at L = 16384 and batch decode (64 x 32768
and 64 x 65536 cached tokens) are measured after it.

The step time is K timed dsa_forward calls between CUDA events. A second,
eager pass runs the same launches through the library's stage calls with
events around each kernel: it gives the per-kernel times the rooflines use.

Rank 0 prints ONE JSON line on stdout; everything else goes to stderr.
Under torchrun every rank runs its own independent problem (weak scaling,
no data-path collective); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DSA prefill tokens/s at L=64K (indexer FP8 TFLOP/s); decode HBM GB/s"
HEADLINE = "prefill_64k"


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--shard", action="store_true",
                    help="run the query-sharded prefill path even on one rank")
    ap.add_argument("--only-warmup-loss", action="store_true",
                    help="time only the indexer warm-up loss + gradient on --workload")
    return ap.parse_args()


# ---------------------------------------------------------------- algorithmic work

def visible_pairs(cfg):
    """sum over query rows of visible keys (causal prefill or decode)."""
    if cfg.decode:
        return cfg.batch * cfg.n_kv
    L = cfg.n_q
    return cfg.batch * L * (L + 1) // 2


def selected_rows(cfg):
    if cfg.decode:
        return cfg.batch * min(cfg.topk, cfg.n_kv)
    L, k = cfg.n_q, cfg.topk
    m = min(L, k)
    return cfg.batch * (m * (m + 1) // 2 + (L - m) * k)


def indexer_flops(cfg):
    return 2.0 * cfg.idx_heads * cfg.idx_dim * visible_pairs(cfg)


def attn_flops(cfg):
    return 2.0 * cfg.heads * (cfg.qk_dim + cfg.v_dim) * selected_rows(cfg)


def decode_bytes(cfg):
    """Algorithmic HBM bytes of one decode step, the bytes the path must move
    once: the indexer key cache (fp8 codes + scale), the query-side indexer
    inputs (codes, scale, weight), the selected indices, the gathered latent
    rows, bf16 q, and the fp32 output with its LSE. Scores are not counted:
    storing them is a choice of the implementation, not part of the path."""
    B, S, k = cfg.batch, cfg.n_kv, min(cfg.topk, cfg.n_kv)
    kcache = B * S * (cfg.idx_dim + 4)
    qside = B * cfg.idx_heads * (cfg.idx_dim + 8)
    idx = B * k * 4
    gather = B * k * cfg.qk_dim * 2
    q = B * cfg.heads * cfg.qk_dim * 2
    out = B * cfg.heads * (cfg.v_dim * 4 + 4)
    return {"total": kcache + qside + idx + gather + q + out,
            "attention": gather + q + out + idx,
            "indexer": kcache + qside}


# ---------------------------------------------------------------- clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"dsa_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = list(csv.reader(io.StringIO(open(self.path).read())))
        os.unlink(self.path)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = max(mx, float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- peaks

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------- the step

class Step:
    """The path for one workload: the public dsa_forward call (the timed
    step) and the same launches through the stage calls (the per-kernel
    breakdown), following the plan dsa_forward_plan reports."""

    def __init__(self, cfg, seed, device, dist=None, shard=None):
        """shard = (rank, ranks): this rank's 4-row query groups of the one
        prefill all ranks share (same seed everywhere), with the keys held
        sequence-sharded and all-gathered each step; None: the whole
        workload on this GPU."""
        import torch
        import sparse_attention_long_fp8_b200 as dsa
        from sparse_attention_long_fp8_b200 import inputs, shard as shard_mod
        self.dsa, self.torch, self.dist = dsa, torch, dist
        self.full_cfg = cfg
        inp = dsa.make_inputs(cfg, seed=seed, device=device)
        self.layout, self.key_local = None, None
        if shard is not None:
            rank, ranks = shard
            rows = shard_mod.shard_rows(cfg.n_q, ranks, rank)
            inp = shard_mod.shard_inputs(inp, rows)
            cfg = inputs.custom_config(cfg.name, n_q=len(rows), name=f"{cfg.name}_shard{rank}")
            self.layout = dsa.make_layout(row_pos=inp["row_pos"])
            if dist is not None:
                # this rank's slice of the keys; the full tensors are refilled
                # by the all-gather of every step
                k0, k1 = shard_mod.key_slice(cfg.n_kv, ranks, rank)
                self.key_local = {k: inp[k][:, k0:k1].clone() for k in ("k_fp8", "k_scale", "kv")}
        self.cfg, self.inp = cfg, inp
        self.shard_mod = shard_mod
        self.shape = dsa.shape_of(cfg)
        B, T = cfg.batch, cfg.n_q
        plan = dsa.forward_plan(self.shape)
        self.fused, self.chunk = plan["fused"], plan["chunk_rows"]
        self.attn_splits = plan["attn_splits"]
        self.attn_ws_bytes = dsa.workspace_size(self.shape, dsa.DSA_OP_SPARSE_ATTN)
        self.fwd_ws, self.fwd_ws_bytes = dsa.alloc_workspace(self.shape, dsa.DSA_OP_FORWARD, device)
        self.attn_ws = torch.empty(max(self.attn_ws_bytes, 256), dtype=torch.uint8, device=device)
        self.idx = torch.empty(B, T, cfg.topk, dtype=torch.int32, device=device)
        self.out = torch.empty(B, T, cfg.heads, cfg.v_dim, device=device)
        self.lse = torch.empty(B, T, cfg.heads, device=device)
        self.chunks = [(r0, min(T, r0 + self.chunk)) for r0 in range(0, T, self.chunk)]
        if B > 1 and len(self.chunks) > 1:
            raise ValueError("stage composition needs one chunk when batch > 1")
        self.scores = None if self.fused else torch.empty(B, min(self.chunk, T), cfg.n_kv,
                                                          device=device)
        per_chunk = 1 if self.fused else 2
        self.launches = per_chunk * len(self.chunks) + 1 + (1 if self.attn_splits > 1 else 0)

    def gather_keys(self):
        """Sharded prefill: every rank's key slices into this GPU's full key
        tensors (NCCL all-gather)."""
        if self.key_local is None:
            return
        for k, loc in self.key_local.items():
            self.inp[k].copy_(self.shard_mod.all_gather_keys(loc, self.cfg.n_kv, self.dist))

    def run_forward(self):
        """One step through the public call."""
        self.gather_keys()
        x = self.inp
        self.dsa.dsa_forward(self.shape, x["q_fp8"], x["q_scale"], x["w"], x["k_fp8"],
                             x["k_scale"], x["q_pos0"], x["kv_len"], x["q"], x["kv"], self.idx,
                             self.out, self.lse, self.fwd_ws, self.fwd_ws_bytes,
                             layout=self.layout)

    def run(self, ev=None):
        """The same launches through the stage calls; with ev (a dict of event
        lists per stage) each launch is bracketed by events on the current
        stream."""
        dsa, x, cfg = self.dsa, self.inp, self.cfg
        rec = (lambda name: ev[name].append(self.torch.cuda.Event(enable_timing=True)) or
               ev[name][-1].record()) if ev is not None else (lambda name: None)
        lay = self.layout
        if self.key_local is not None:
            rec("gather")
            self.gather_keys()
            rec("gather")
        if self.fused:
            rec("indexer")
            dsa.dsa_indexer_topk(self.shape, x["q_fp8"], x["q_scale"], x["w"], x["k_fp8"],
                                 x["k_scale"], x["q_pos0"], x["kv_len"], 0, cfg.n_q, self.idx,
                                 layout=lay)
            rec("indexer")
        for r0, r1 in ([] if self.fused else self.chunks):
            rec("indexer")
            dsa.dsa_indexer_scores(self.shape, x["q_fp8"], x["q_scale"], x["w"], x["k_fp8"],
                                   x["k_scale"], x["q_pos0"], x["kv_len"], r0, r1, self.scores,
                                   flags=dsa.DSA_SCORES_VISIBLE_ONLY, layout=lay)
            rec("indexer")
            rec("topk")
            dsa.dsa_topk(self.shape, self.scores, r0, r1, x["q_pos0"], x["kv_len"],
                         self.idx[:, r0:r1] if cfg.batch == 1 else self.idx, layout=lay)
            rec("topk")
        rec("attn")
        dsa.dsa_sparse_attn(self.shape, x["q"], x["kv"], self.idx, self.out, self.lse,
                            self.attn_ws, self.attn_ws_bytes, layout=lay)
        rec("attn")


def max_over_ranks(x, dist, device="cuda"):
    """The max of x over all ranks (x itself without a process group)."""
    if not dist:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def all_ranks(flag, dist, device="cuda"):
    """True iff flag holds on every rank: a decision every rank then takes
    the same way, so that all ranks run the same collectives."""
    if not dist:
        return bool(flag)
    import torch
    t = torch.tensor([1 if flag else 0], dtype=torch.int32, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MIN)
    return bool(t.item())


def quantiser_bench(cfg, peaks, reps=10):
    """The per-row FP8 quantiser on the workload's indexer inputs (bf16
    q [T, H^I, d^I] and k [S, d^I]); HBM-bound: 3 bytes per element plus a
    scale per row. Inputs (2.2 GB at 64K) exceed L2."""
    import torch
    import sparse_attention_long_fp8_b200 as dsa
    g = torch.Generator(device="cuda").manual_seed(5)
    xs = [torch.randn(cfg.batch * cfg.n_q, cfg.idx_heads, cfg.idx_dim, device="cuda", generator=g,
                      dtype=torch.bfloat16),
          torch.randn(cfg.batch * cfg.n_kv, cfg.idx_dim, device="cuda", generator=g,
                      dtype=torch.bfloat16)]
    outs = [(torch.empty(x.shape, dtype=torch.uint8, device="cuda"),
             torch.empty(x.shape[:-1], device="cuda")) for x in xs]
    nbytes = sum(x.numel() * 3 + x.numel() // x.shape[-1] * 4 for x in xs)

    def run():
        for x, (c, sc) in zip(xs, outs):
            dsa.dsa_quantize_e4m3(x, c, sc)

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    dsa.dsa_check()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(reps):
        run()
    e.record()
    torch.cuda.synchronize()
    dsa.dsa_check()
    ms = s.elapsed_time(e) / reps
    gbs = nbytes / (ms / 1e3) / 1e9
    del xs, outs
    torch.cuda.empty_cache()
    return {"ms_per_step": ms, "GB_per_s": gbs, "frac_hbm": gbs / peaks["hbm"],
            "algorithmic_bytes": nbytes, "launches": 2,
            "what": "q [T*H^I, d^I] and k [S, d^I] bf16 -> e4m3 codes + fp32 row scales"}


def stage_ms(ev):
    """Average per-launch milliseconds and total per stage from event pairs."""
    res = {}
    for name, lst in ev.items():
        d = [lst[i].elapsed_time(lst[i + 1]) for i in range(0, len(lst), 2)]
        res[name] = {"launches": len(d), "total_ms": sum(d), "avg_ms": sum(d) / max(1, len(d))}
    return res


def timed(step, steps, warmup, dist, graph=False):
    """W untimed steps, then K timed dsa_forward calls between barriers and
    CUDA events; returns ms per step as the max over ranks.

    With graph=True (short, launch-bound steps: decode) the step is captured
    once into a CUDA graph and the K timed steps are graph replays."""
    import torch
    for _ in range(warmup):
        step.run_forward()
    torch.cuda.synchronize()
    step.dsa.dsa_check()
    g = None
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step.run_forward()
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        step.dsa.dsa_check()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        if g is not None:
            g.replay()
        else:
            step.run_forward()
    end.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    step.dsa.dsa_check()
    ms = max_over_ranks(start.elapsed_time(end) / steps, dist)
    del g
    return ms


def breakdown(step, steps):
    """K eager steps through the stage calls, each launch between CUDA events
    on the launching stream: per-kernel times for the rooflines."""
    import torch
    ev = {"gather": [], "indexer": [], "topk": [], "attn": []}
    step.run()
    torch.cuda.synchronize()
    for _ in range(steps):
        step.run(ev)
    torch.cuda.synchronize()
    step.dsa.dsa_check()
    return stage_ms(ev)


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# sparse_attn_vh_kernel over the 4096-row prefill, from one ncu capture, and
# the SHA-256 of the kernel source that capture ran. The kernel's traffic is
# q read once plus out and lse written once (the latent gathers hit L2), so it
# grows in proportion to the rows and is scaled by them. When the source no
# longer matches, the figure is stale and the line reports null.
ATTN_TRAFFIC_4K = {"bytes": 642.458624e6 + 1022.275e6, "rows": 4096,
                   "source_sha256": "576884927b8853594d6ee7f667b2a6e341b0b8ebaa4b53573f4b85f8bb4a35f6"}


def kernel_source_sha256(name):
    import hashlib
    path = os.path.join(ROOT, "sparse_attention_long_fp8_b200", "csrc", name)
    return hashlib.sha256(open(path, "rb").read()).hexdigest()


def attn_traffic(cfg):
    """Per-launch DRAM bytes of the attention kernel at cfg, or None when the
    captured figure does not belong to the current kernel source."""
    cap = ATTN_TRAFFIC_4K
    if cap["source_sha256"] != kernel_source_sha256("sparse_attn_vh.cuh"):
        return None
    return cap["bytes"] / cap["rows"] * cfg.batch * cfg.n_q


def prefill_leg(cfg, seed, steps, warmup, dist, peaks, shard=None):
    """dsa_forward over one prefill workload: tokens/s from the timed calls,
    per-kernel TFLOP/s from the breakdown pass. With shard = (rank, ranks)
    this rank runs its share of the one prefill all ranks split; the flop
    rates are then this rank's share of the work over its kernel times."""
    import torch
    step = Step(cfg, seed, "cuda", dist=dist, shard=shard)
    log(f"[bench] {cfg.name}: fused {step.fused}, chunk rows {step.chunk}, "
        f"{step.launches} launches/step")
    ms = timed(step, steps, warmup, dist)
    stages = breakdown(step, steps)
    launches = step.launches
    fused = step.fused
    rows = step.cfg.n_q
    if shard is not None:
        from sparse_attention_long_fp8_b200 import shard as shard_mod
        vis, sel = shard_mod.shard_cost(cfg.n_q, cfg.n_kv, shard[1], shard[0], cfg.topk)
        ix_f = 2.0 * cfg.idx_heads * cfg.idx_dim * vis
        at_f = 2.0 * cfg.heads * (cfg.qk_dim + cfg.v_dim) * sel
    else:
        ix_f, at_f = indexer_flops(cfg), attn_flops(cfg)
    del step
    torch.cuda.empty_cache()
    per = {k: v["total_ms"] / steps for k, v in stages.items()}
    fp8_peak = 2.0 * peaks["bf16_sustained"]
    ix_ms = per["indexer"] + (0.0 if fused else per["topk"])
    stage_names = ({"indexer_topk_fused": per["indexer"], "attention": per["attn"]}
                   if fused else {"indexer": per["indexer"], "topk": per["topk"],
                                  "attention": per["attn"]})
    if shard is not None and stages["gather"]["launches"]:
        stage_names["key_all_gather"] = per["gather"]
    res = {"ms_per_step": ms, "tokens_per_s": cfg.batch * cfg.n_q / (ms / 1e3),
           "rows_this_rank": rows,
           "stages_ms": stage_names,
           "stage_sum_ms": sum(per.values()),
           "indexer_tflops_fp8": ix_f / (ix_ms / 1e3) / 1e12,
           "attention_tflops_bf16": at_f / (per["attn"] / 1e3) / 1e12,
           "launches_per_step": launches}
    res["indexer_frac_fp8"] = res["indexer_tflops_fp8"] / fp8_peak
    res["attention_frac_bf16"] = res["attention_tflops_bf16"] / peaks["bf16_sustained"]
    return res, stages, fused


def warmup_loss_flops(cfg):
    """Algorithmic flops of one indexer warm-up loss step (dsa_indexer_kl)
    over a causal prefill: the dense attention logits that give p
    (2 H D_qk per visible pair), the indexer scores (2 H^I d^I per pair) and
    the two gradient contractions U and dk (2 H^I d^I per pair each)."""
    pairs = visible_pairs(cfg)
    return {"probs_bf16": 2.0 * cfg.heads * cfg.qk_dim * pairs,
            "scores_fp8": 2.0 * cfg.idx_heads * cfg.idx_dim * pairs,
            "grads_fp32": 4.0 * cfg.idx_heads * cfg.idx_dim * pairs}


def warmup_loss_leg(cfg, seed, steps, warmup):
    """dsa_indexer_kl (loss + dL/dw, dL/dq^, dL/dk^) over one prefill."""
    import torch
    import sparse_attention_long_fp8_b200 as dsa
    g = dsa.make_inputs(cfg, seed=seed, device="cuda")
    shape = dsa.shape_of(cfg)
    B, T, S = cfg.batch, cfg.n_q, cfg.n_kv
    loss = torch.empty(B, T, device="cuda")
    dw = torch.empty(B, T, cfg.idx_heads, device="cuda")
    dq = torch.empty(B, T, cfg.idx_heads, cfg.idx_dim, device="cuda")
    dk = torch.empty(B, S, cfg.idx_dim, device="cuda")
    ws, n = dsa.alloc_workspace(shape, dsa.DSA_OP_INDEXER_KL)

    def run():
        dsa.dsa_indexer_kl(shape, g["q_fp8"], g["q_scale"], g["w"], g["k_fp8"], g["k_scale"],
                           g["q_pos0"], g["kv_len"], g["q"], g["kv"], loss, dw, dq, dk, ws, n)

    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    dsa.dsa_check()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        run()
    e.record()
    torch.cuda.synchronize()
    dsa.dsa_check()
    ms = s.elapsed_time(e) / steps
    fl = warmup_loss_flops(cfg)
    del g, loss, dw, dq, dk, ws
    torch.cuda.empty_cache()
    return {"ms_per_step": ms, "tokens_per_s": B * T / (ms / 1e3),
            "algorithmic_tflop": {k: v / 1e12 for k, v in fl.items()},
            "what": "loss and gradient w.r.t. w, q^, k^ of sum_t KL(p_t || Softmax(I_t))"}


def decode_leg(cfg, seed, steps, warmup, dist, peaks):
    """Batch decode: dsa_forward captured in a CUDA graph (a step is ~0.2 ms
    of a few launches), bytes per step as decode_bytes counts them."""
    import torch
    step = Step(cfg, seed, "cuda")
    ms = timed(step, steps, warmup, dist, graph=True)
    stages = breakdown(step, steps)
    launches = step.launches
    del step
    torch.cuda.empty_cache()
    nb = decode_bytes(cfg)
    per = {k: v["total_ms"] / steps for k, v in stages.items()}
    gbs = nb["total"] / (ms / 1e3) / 1e9
    return {"ms_per_step": ms, "GB_per_s": gbs, "frac_hbm": gbs / peaks["hbm"],
            "attention_ms": per["attn"],
            "attention_GB_per_s": nb["attention"] / (per["attn"] / 1e3) / 1e9,
            "indexer_GB_per_s": nb["indexer"] / (per["indexer"] / 1e3) / 1e9,
            "stages_ms": per, "launches_per_step": launches,
            "timing": "CUDA graph replays of dsa_forward; stages from an eager pass",
            "algorithmic_bytes": nb["total"]}


# ---------------------------------------------------------------- e2e

def e2e(cfg, seed, steps, dist, shard=None, n_chunks=8):
    """The same path through the public dsa_forward_ex call with HOST
    buffers: every step copies the inputs host->device from pinned memory,
    runs the forward and reads the results (out, lse, indices) back.

    The copies are pipelined against the compute: the rows (this rank's rows
    when sharded) are cut into n_chunks runs of consecutive 4-row groups;
    chunk c's query inputs go up on a copy stream, its forward runs on a
    compute stream (dsa_forward_ex with the chunk's absolute row positions,
    against all keys, which go up first), and its results come down on a
    third stream, so the host link in both directions overlaps the kernels.
    Sharded: each rank uploads its slice of the keys and all-gathers them."""
    import torch
    import sparse_attention_long_fp8_b200 as dsa
    from sparse_attention_long_fp8_b200 import inputs, shard as shard_mod
    dev_inp = dsa.make_inputs(cfg, seed=seed, device="cuda")
    full_n_kv = cfg.n_kv
    if cfg.batch != 1:
        raise ValueError("the pipelined e2e splits the rows of one sequence")
    rows_all = (shard_mod.shard_rows(cfg.n_q, shard[1], shard[0]) if shard is not None
                else None)
    kslice = None
    if shard is not None:
        dev_inp = shard_mod.shard_inputs(dev_inp, rows_all)
        if dist is not None:
            kslice = shard_mod.key_slice(full_n_kv, shard[1], shard[0])
    else:
        dev_inp["row_pos"] = (dev_inp["q_pos0"][:, None] +
                              torch.arange(cfg.n_q, device="cuda", dtype=torch.int32)[None, :])
    T = dev_inp["q"].shape[1]
    qkeys = ["q_fp8", "q_scale", "w", "q", "row_pos"]
    kkeys = ["k_fp8", "k_scale", "kv"]
    host, dev = {}, {}
    for k in qkeys + kkeys + ["kv_len", "q_pos0"]:
        t = dev_inp[k]
        if kslice is not None and k in kkeys:
            t = t[:, kslice[0]:kslice[1]]
        host[k] = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        host[k].copy_(t)
        dev[k] = torch.empty_like(dev_inp[k])
    dev_local = ({k: torch.empty(host[k].shape, dtype=host[k].dtype, device="cuda") for k in kkeys}
                 if kslice is not None else None)
    del dev_inp
    # chunks: runs of whole 4-row groups
    groups = (T + 3) // 4
    bounds = [min(T, 4 * ((groups * c) // n_chunks)) for c in range(n_chunks + 1)]
    chunks = [(bounds[c], bounds[c + 1]) for c in range(n_chunks) if bounds[c + 1] > bounds[c]]
    out = torch.empty(1, T, cfg.heads, cfg.v_dim, device="cuda")
    lse = torch.empty(1, T, cfg.heads, device="cuda")
    idx = torch.empty(1, T, cfg.topk, dtype=torch.int32, device="cuda")
    h_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h_lse = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    h_idx = torch.empty(idx.shape, dtype=idx.dtype, pin_memory=True)
    plans = []
    for r0, r1 in chunks:
        ccfg = inputs.custom_config(cfg.name, n_q=r1 - r0, n_kv=full_n_kv, name="e2e_chunk")
        shape = dsa.shape_of(ccfg)
        ws, n = dsa.alloc_workspace(shape, dsa.DSA_OP_FORWARD)
        lay = dsa.make_layout(row_pos=dev["row_pos"][:, r0:r1])
        plans.append((r0, r1, shape, ws, n, lay))
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in (h_out, h_lse, h_idx))
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def one():
        cur = torch.cuda.current_stream()
        s_in.wait_stream(cur)
        with torch.cuda.stream(s_in):
            for k in kkeys + ["kv_len", "q_pos0"]:
                (dev_local[k] if dev_local is not None and k in kkeys else dev[k]).copy_(
                    host[k], non_blocking=True)
            keys_in = torch.cuda.Event()
            keys_in.record(s_in)
        s_comp.wait_event(keys_in)
        if dev_local is not None:
            with torch.cuda.stream(s_comp):
                for k in kkeys:
                    dev[k].copy_(shard_mod.all_gather_keys(dev_local[k], full_n_kv, dist))
        for r0, r1, shape, ws, n, lay in plans:
            with torch.cuda.stream(s_in):
                for k in qkeys:
                    dev[k][:, r0:r1].copy_(host[k][:, r0:r1], non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(s_in)
            s_comp.wait_event(ready)
            with torch.cuda.stream(s_comp):
                dsa.dsa_forward(shape, dev["q_fp8"][:, r0:r1], dev["q_scale"][:, r0:r1],
                                dev["w"][:, r0:r1], dev["k_fp8"], dev["k_scale"], dev["q_pos0"],
                                dev["kv_len"], dev["q"][:, r0:r1], dev["kv"], idx[:, r0:r1],
                                out[:, r0:r1], lse[:, r0:r1], ws, n, stream=s_comp, layout=lay)
                done = torch.cuda.Event()
                done.record(s_comp)
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                h_out[:, r0:r1].copy_(out[:, r0:r1], non_blocking=True)
                h_lse[:, r0:r1].copy_(lse[:, r0:r1], non_blocking=True)
                h_idx[:, r0:r1].copy_(idx[:, r0:r1], non_blocking=True)
        cur.wait_stream(s_out)
        cur.wait_stream(s_comp)
        cur.wait_stream(s_in)

    one()
    torch.cuda.synchronize()
    dsa.dsa_check()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        one()
    e.record()
    torch.cuda.synchronize()
    dsa.dsa_check()
    ms = max_over_ranks(s.elapsed_time(e) / steps, dist)
    del host, dev, out, lse, idx, h_out, h_lse, h_idx, plans, dev_local
    torch.cuda.empty_cache()
    return ms, h2d, d2h


def e2e_host_bytes(cfg):
    B, T, S = cfg.batch, cfg.n_q, cfg.n_kv
    inputs = B * T * cfg.idx_heads * (cfg.idx_dim + 8) + B * S * (cfg.idx_dim + 4) + \
        B * T * cfg.heads * cfg.qk_dim * 2 + B * S * cfg.qk_dim * 2
    outputs = B * T * cfg.heads * (cfg.v_dim + 1) * 4 + B * T * cfg.topk * 4
    return inputs + outputs


def host_available_bytes():
    try:
        for line in open("/proc/meminfo"):
            if line.startswith("MemAvailable:"):
                return int(line.split()[1]) * 1024
    except OSError:
        return None
    return None


# ---------------------------------------------------------------- CPU oracle

def oracle_sample_rows(cfg, n_rows, offset=0.5):
    """n_rows evenly spaced query rows of the workload (offset in [0, 1)
    shifts them within their spacing); evenly spaced rows have the
    workload's average per-row cost, so rows/s extrapolates to the whole
    config."""
    import numpy as np
    T = cfg.n_q
    return np.unique(((np.arange(n_rows) + offset) * T / n_rows).astype(np.int64))


def oracle_inputs(cfg, seed):
    """The workload's inputs, drawn once (on the GPU when there is one: the
    drawing is not timed)."""
    import torch
    from sparse_attention_long_fp8_b200 import inputs
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    return inputs.make_inputs(cfg, seed=seed, device=dev)


def oracle_rows_per_s(cfg, inp, rows):
    """The fp64 oracle (as it stands) over the given query rows of sequence
    0 on this host's cores: (rows/s, seconds, threads used, rows)."""
    import numpy as np
    import torch
    import oracle
    sel = torch.as_tensor(rows, device=inp["q_fp8"].device)
    small = {"q_fp8": inp["q_fp8"][:, sel].cpu(), "q_scale": inp["q_scale"][:, sel].cpu(),
             "w": inp["w"][:, sel].cpu(), "k_fp8": inp["k_fp8"].cpu(),
             "k_scale": inp["k_scale"].cpu(), "q": inp["q"][:, sel].cpu(),
             "kv": inp["kv"].cpu(), "q_pos0": inp["q_pos0"].cpu(), "kv_len": inp["kv_len"].cpu()}
    b = 0
    pos = (np.asarray(rows) + int(small["q_pos0"][b])).astype(np.int32)
    t0 = time.perf_counter()
    sc = oracle.indexer_scores(small["q_fp8"][b], small["q_scale"][b], small["w"][b],
                               small["k_fp8"][b], small["k_scale"][b], pos,
                               int(small["kv_len"][b]))
    idx = oracle.topk(sc, cfg.topk)
    oracle.sparse_attn(small["q"][b], small["kv"][b], idx, cfg.softmax_scale, cfg.v_dim)
    dt = time.perf_counter() - t0
    cores = min(oracle.hardware_threads(), len(rows))
    return len(rows) / dt, dt, cores, len(rows)


# ---------------------------------------------------------------- main

def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return main_reference(args, world, rank)

    import torch
    from sparse_attention_long_fp8_b200 import inputs
    import sparse_attention_long_fp8_b200 as dsa
    dsa.load_library()
    torch.cuda.set_device(local)
    dist = None
    if world > 1 or (args.shard and "MASTER_ADDR" in os.environ):
        # (a one-rank group under torchrun with --shard runs the all-gather too)
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    peaks = measured_peaks()
    cfg = inputs.CONFIGS[args.workload]
    if args.only_warmup_loss:
        leg = warmup_loss_leg(cfg, 1000 + rank, args.steps, args.warmup)
        if rank == 0:
            print(json.dumps({"workload": cfg.name, "warmup_loss": leg}), flush=True)
        if dist:
            dist.destroy_process_group()
        return
    # Several GPUs split ONE prefill by query rows (strong scaling): every
    # rank draws the same inputs and takes its share of the rows. --shard
    # runs that path on a single rank too.
    sharded = (world > 1 or args.shard) and not cfg.decode
    shard = (rank, world) if sharded else None
    seed = 1000 if sharded else 1000 + rank

    clocks = ClockSampler(local)
    clocks.start()
    head, stages, fused = prefill_leg(cfg, seed, args.steps, args.warmup, dist, peaks, shard)
    clock_info = clocks.stop()
    ms = head["ms_per_step"]
    tokens = cfg.batch * cfg.n_q
    # sharded: the ranks together finish one prefill per step
    value = (1 if sharded else world) * tokens / (ms / 1e3)

    per = {k: v["total_ms"] / args.steps for k, v in stages.items()}
    at_ms, ix_ms = per["attn"], per["indexer"]
    dominant = max(("indexer", ix_ms), ("attn", at_ms), ("topk", per["topk"]),
                   key=lambda x: x[1])[0]
    if dominant == "attn":
        traffic = attn_traffic(cfg)
        roof = {"kernel": "sparse_attn_vh_kernel", "bound": "tensor",
                "achieved": head["attention_tflops_bf16"], "peak": peaks["bf16_sustained"],
                "unit": "TFLOP/s", "traffic": traffic,
                "traffic_source": ("ncu DRAM bytes of one 4096-row launch of the same kernel "
                                   "source, scaled by rows") if traffic else
                                  "null: no capture of the current kernel source"}
    elif dominant == "indexer":
        kern = "indexer_topk_kernel<64,128,4>" if fused else "indexer_scores_kernel<64,128,4>"
        roof = {"kernel": kern, "bound": "tensor",
                "achieved": indexer_flops(cfg) / (ix_ms / 1e3) / 1e12,
                "peak": 2.0 * peaks["bf16_sustained"], "unit": "TFLOP/s", "traffic": None}
    else:
        roof = {"kernel": "topk_kernel", "bound": "hbm", "achieved": None,
                "peak": peaks["hbm"], "unit": "GB/s", "traffic": None}
    if roof["achieved"] is not None:
        roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = f"{peaks['source']} ({'bf16 sustained' if roof['unit'] == 'TFLOP/s' else 'hbm copy'}" + \
        (", x2 for fp8" if roof.get("kernel", "").startswith("indexer") else "") + ")"
    roof["launches_timed"] = stages[dominant]["launches"]

    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong" if sharded else "weak",
        "vs_baseline": None,
        "dtype": "fp8e4m3 indexer, bf16 attention, fp32 accumulate",
        "data": "synthetic (seeded; page-shaped workloads)",
        "config": bench_config(cfg, world, sharded),
        "stages_ms": head["stages_ms"], "stage_sum_ms": head["stage_sum_ms"],
        "indexer_tflops_fp8": head["indexer_tflops_fp8"],
        "indexer_frac_fp8": head["indexer_frac_fp8"],
        "attention_tflops_bf16": head["attention_tflops_bf16"],
        "attention_frac_bf16": head["attention_frac_bf16"],
        "roofline": roof, "gpu_launches": head["launches_per_step"] * args.steps,
        "clocks": clock_info,
    }

    if not args.no_decode and args.workload == HEADLINE:
        pcfg = inputs.CONFIGS["prefill_16k"]
        leg, _, _ = prefill_leg(pcfg, seed, args.steps, args.warmup, dist, peaks, shard)
        leg["tokens_per_s"] = pcfg.n_q * (1 if sharded else world) / (leg["ms_per_step"] / 1e3)
        result["prefill_16k"] = leg
        result["quantiser"] = quantiser_bench(cfg, peaks)
        result["warmup_loss_4k"] = warmup_loss_leg(inputs.CONFIGS["prefill_4k"], seed,
                                                   max(3, args.steps // 4), args.warmup)
        result["decode"] = {}
        for name in ("decode_32k", "decode_64k"):
            # decode steps are ~0.2 ms: many of them, after a longer warm-up;
            # under several ranks each rank decodes its own batch (weak)
            result["decode"][name] = decode_leg(inputs.CONFIGS[name], 1000 + rank,
                                                max(args.steps, 100), max(args.warmup, 20),
                                                dist, peaks)
            result["decode"][name]["scaling"] = "weak"
            torch.cuda.empty_cache()

    # The ranks of a node share its host RAM: every rank needs its own pinned
    # copy, and all ranks must agree before any of them enters e2e().
    need = e2e_host_bytes(cfg) // (world if sharded else 1)
    avail = host_available_bytes()
    fits = avail is None or avail >= 2 * need * world
    fits = all_ranks(fits, dist)
    if not args.no_e2e and not fits:
        result["e2e"] = {"value": None, "unit": "tokens/s",
                         "skipped": "host RAM: " + ("unknown" if avail is None else
                                                    f"{avail / 2**30:.0f} GiB") +
                                    f" available, {world * need / 2**30:.0f} GiB pinned needed"}
    elif not args.no_e2e:
        e_ms, h2d, d2h = e2e(cfg, seed, max(2, min(args.steps, 3)), dist, shard)
        result["e2e"] = {"value": (1 if sharded else world) * tokens / (e_ms / 1e3),
                         "unit": "tokens/s",
                         "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                         "ms_per_step": e_ms}

    if not args.no_cpu and world == 1 and rank == 0:
        # A calibration sample of one row per host thread, then a sample
        # sized for about 12 s of oracle work, on every host thread.
        import oracle
        threads = max(1, oracle.hardware_threads())
        oinp = oracle_inputs(cfg, seed)
        _, dt0, _, nr0 = oracle_rows_per_s(cfg, oinp, oracle_sample_rows(cfg, threads))
        reps = max(1, min(32, int(12.0 / max(dt0, 1e-3))))
        n_rows = min(cfg.n_q, nr0 * reps)
        rps, dt, cores, nr = oracle_rows_per_s(cfg, oinp, oracle_sample_rows(cfg, n_rows))
        del oinp
        result["cpu_baseline"] = {"value": rps * cfg.batch, "unit": "tokens/s", "cores": cores,
                                  "kind": "oracle",
                                  "sample": f"{nr} evenly spaced query rows of {cfg.name} "
                                            f"(indexer + top-k + attention, fp64), {dt:.1f} s"}

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def bench_config(cfg, world, sharded=False):
    """The workload description both arms print."""
    return {"workload": cfg.name, "batch": cfg.batch, "seq_len": cfg.n_q,
            "idx_heads": cfg.idx_heads, "idx_dim": cfg.idx_dim, "topk": cfg.topk,
            "heads": cfg.heads, "qk_dim": cfg.qk_dim, "v_dim": cfg.v_dim,
            "parallelism": (f"query-sharded x{world} (one prefill; keys all-gathered)"
                            if sharded else f"replicas x{world}"),
            "l2": "inputs larger than L2 (q is 9.7 GB per step)"}


def main_reference(args, world, rank):
    """The reference arm: the fp64 oracle as it stands on this host's cores,
    same workload, metric and unit; each step is a bounded sample of rows."""
    if rank != 0:
        return
    from sparse_attention_long_fp8_b200 import inputs
    import oracle
    cfg = inputs.CONFIGS[args.workload]
    # One sampled row per host thread and step, so every thread works; the
    # steps take differently offset evenly spaced rows of one drawn input.
    n_rows = min(cfg.n_q, max(1, oracle.hardware_threads()))
    inp = oracle_inputs(cfg, 1000)
    total = args.warmup + args.steps
    secs, cores, done = [], 1, 0
    for i in range(total):
        rows = oracle_sample_rows(cfg, n_rows, offset=(i + 0.5) / total)
        _, dt, cores, nr = oracle_rows_per_s(cfg, inp, rows)
        if i >= args.warmup:
            secs.append(dt)
            done += nr
    value = done / sum(secs)
    sample = (f"{n_rows} evenly spaced query rows of {cfg.name} per step on {cores} threads "
              f"(fp64 oracle: indexer + top-k + attention)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(secs) / len(secs), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(cfg, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


if __name__ == "__main__":
    main()
