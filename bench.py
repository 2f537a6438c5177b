#!/usr/bin/env python
"""Benchmark of the DSA forward path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole path over one batch of synthetic input: the
lightning indexer with its top-k selection (one fused kernel for prefill; a
score kernel and a selection kernel per row chunk for decode), then the
sparse attention over all rows, composed from the library's stage calls
exactly as dsa_forward launches them, so each kernel can be timed with CUDA
events on its stream. The headline workload is DSA prefill at L = 65536 (batch 1,
H^I = 64, d^I = 128, k = 2048, 128-head MQA over the 576-d latent); batch
decode (64 x 32768 and 64 x 65536 cached tokens) is measured after it.

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
    """Algorithmic HBM bytes of one decode step (each byte the path must move
    once): indexer key cache (fp8 + scale), query-side indexer inputs, the
    fp32 score row written and read once by top-k, the selected indices, the
    gathered latent rows, q, and the fp32 output."""
    B, S, k = cfg.batch, cfg.n_kv, min(cfg.topk, cfg.n_kv)
    kcache = B * S * (cfg.idx_dim + 4)
    qside = B * cfg.idx_heads * (cfg.idx_dim + 8)
    scores = 2 * B * S * 4
    idx = 2 * B * k * 4
    gather = B * k * cfg.qk_dim * 2
    q = B * cfg.heads * cfg.qk_dim * 2
    out = B * cfg.heads * (cfg.v_dim * 4 + 4)
    return {"total": kcache + qside + scores + idx + gather + q + out,
            "attention": gather + q + out + B * k * 4}


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
    """The path for one workload, composed from the library's stage calls."""

    def __init__(self, cfg, seed, device):
        import torch
        import sparse_attention_long_fp8_b200 as dsa
        self.dsa, self.torch, self.cfg = dsa, torch, cfg
        self.inp = dsa.make_inputs(cfg, seed=seed, device=device)
        self.shape = dsa.shape_of(cfg)
        B, T = cfg.batch, cfg.n_q
        self.chunk = dsa.forward_chunk_rows(self.shape)
        self.attn_ws_bytes = dsa.workspace_size(self.shape, dsa.DSA_OP_SPARSE_ATTN)
        self.fwd_ws_bytes = dsa.workspace_size(self.shape, dsa.DSA_OP_FORWARD)
        self.attn_ws = torch.empty(max(self.attn_ws_bytes, 256), dtype=torch.uint8, device=device)
        self.idx = torch.empty(B, T, cfg.topk, dtype=torch.int32, device=device)
        self.out = torch.empty(B, T, cfg.heads, cfg.v_dim, device=device)
        self.lse = torch.empty(B, T, cfg.heads, device=device)
        self.chunks = [(r0, min(T, r0 + self.chunk)) for r0 in range(0, T, self.chunk)]
        if B > 1 and len(self.chunks) > 1:
            raise ValueError("stage composition needs one chunk when batch > 1")
        # dsa_forward's plan: the fused indexer + selection needs no score
        # buffer, so its forward workspace is the attention's alone.
        self.fused = self.fwd_ws_bytes == self.attn_ws_bytes
        self.scores = None if self.fused else torch.empty(B, min(self.chunk, T), cfg.n_kv,
                                                          device=device)
        per_chunk = 1 if self.fused else 2
        self.launches = per_chunk * len(self.chunks) + 1 + (1 if self.attn_ws_bytes > 0 else 0)

    def run(self, ev=None):
        """One step; with ev = (list of (start, end) event pairs per stage) the
        stage boundaries are recorded on the current stream."""
        dsa, x, cfg = self.dsa, self.inp, self.cfg
        rec = (lambda name: ev[name].append(self.torch.cuda.Event(enable_timing=True)) or
               ev[name][-1].record()) if ev is not None else (lambda name: None)
        if self.fused:
            rec("indexer")
            dsa.dsa_indexer_topk(self.shape, x["q_fp8"], x["q_scale"], x["w"], x["k_fp8"],
                                 x["k_scale"], x["q_pos0"], x["kv_len"], 0, cfg.n_q, self.idx)
            rec("indexer")
        for r0, r1 in ([] if self.fused else self.chunks):
            rec("indexer")
            dsa.dsa_indexer_scores(self.shape, x["q_fp8"], x["q_scale"], x["w"], x["k_fp8"],
                                   x["k_scale"], x["q_pos0"], x["kv_len"], r0, r1, self.scores,
                                   flags=dsa.DSA_SCORES_VISIBLE_ONLY)
            rec("indexer")
            rec("topk")
            dsa.dsa_topk(self.shape, self.scores, r0, r1, x["q_pos0"], x["kv_len"],
                         self.idx[:, r0:r1] if cfg.batch == 1 else self.idx)
            rec("topk")
        rec("attn")
        dsa.dsa_sparse_attn(self.shape, x["q"], x["kv"], self.idx, self.out, self.lse,
                            self.attn_ws, self.attn_ws_bytes)
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
    """W untimed steps, then K timed steps between barriers; returns
    (ms per step as max over ranks, per-stage event timings).

    With graph=True (short, launch-bound steps: decode) the step is captured
    once into a CUDA graph and the K timed steps are graph replays; the
    per-stage times then come from a separate eager pass with events."""
    import torch
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    step.dsa.dsa_check()
    ev = {"indexer": [], "topk": [], "attn": []}
    g = None
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step.run()
        for _ in range(warmup):
            g.replay()
        for _ in range(steps):      # the eager pass for the stage breakdown
            step.run(ev)
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
            step.run(ev)
    end.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    step.dsa.dsa_check()
    ms = max_over_ranks(start.elapsed_time(end) / steps, dist)
    del g
    return ms, stage_ms(ev)


# ---------------------------------------------------------------- e2e

def e2e(cfg, seed, steps, dist):
    """Same path through the public dsa_forward call with HOST buffers:
    every step copies the inputs host->device from pinned memory, runs the
    forward and reads the result (out, lse, indices) back."""
    import torch
    import sparse_attention_long_fp8_b200 as dsa
    dev_inp = dsa.make_inputs(cfg, seed=seed, device="cuda")
    keys = ["q_fp8", "q_scale", "w", "k_fp8", "k_scale", "q_pos0", "kv_len", "q", "kv"]
    host = {k: torch.empty(dev_inp[k].shape, dtype=dev_inp[k].dtype, pin_memory=True) for k in keys}
    for k in keys:
        host[k].copy_(dev_inp[k])
    dev = {k: torch.empty_like(dev_inp[k]) for k in keys}
    del dev_inp
    shape = dsa.shape_of(cfg)
    B, T = cfg.batch, cfg.n_q
    out = torch.empty(B, T, cfg.heads, cfg.v_dim, device="cuda")
    lse = torch.empty(B, T, cfg.heads, device="cuda")
    idx = torch.empty(B, T, cfg.topk, dtype=torch.int32, device="cuda")
    h_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h_lse = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    h_idx = torch.empty(idx.shape, dtype=idx.dtype, pin_memory=True)
    ws, n = dsa.alloc_workspace(shape, dsa.DSA_OP_FORWARD)
    h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
    d2h = sum(t.numel() * t.element_size() for t in (h_out, h_lse, h_idx))

    def one():
        for k in keys:
            dev[k].copy_(host[k], non_blocking=True)
        dsa.dsa_forward(shape, dev["q_fp8"], dev["q_scale"], dev["w"], dev["k_fp8"],
                        dev["k_scale"], dev["q_pos0"], dev["kv_len"], dev["q"], dev["kv"], idx,
                        out, lse, ws, n)
        h_out.copy_(out, non_blocking=True)
        h_lse.copy_(lse, non_blocking=True)
        h_idx.copy_(idx, non_blocking=True)

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
    del host, dev, out, lse, idx, h_out, h_lse, h_idx, ws
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

def oracle_rows_per_s(cfg, seed, n_rows):
    """The fp64 oracle (as it stands) over n_rows evenly spaced query rows of
    the workload on this host's cores; evenly spaced rows have the workload's
    average per-row cost, so rows/s extrapolates to the whole config."""
    import numpy as np
    import torch
    import oracle
    from sparse_attention_long_fp8_b200 import inputs
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = inputs.make_inputs(cfg, seed=seed, device=dev)
    T = cfg.n_q
    rows = np.unique(((np.arange(n_rows) + 0.5) * T / n_rows).astype(np.int64))
    sel = torch.as_tensor(rows, device=inp["q_fp8"].device)
    small = {"q_fp8": inp["q_fp8"][:, sel].cpu(), "q_scale": inp["q_scale"][:, sel].cpu(),
             "w": inp["w"][:, sel].cpu(), "k_fp8": inp["k_fp8"].cpu(),
             "k_scale": inp["k_scale"].cpu(), "q": inp["q"][:, sel].cpu(),
             "kv": inp["kv"].cpu(), "q_pos0": inp["q_pos0"].cpu(), "kv_len": inp["kv_len"].cpu()}
    del inp
    b = 0
    pos = (rows + int(small["q_pos0"][b])).astype(np.int32)
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
    if world > 1:
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    peaks = measured_peaks()
    cfg = inputs.CONFIGS[args.workload]
    seed = 1000 + rank

    clocks = ClockSampler(local)
    step = Step(cfg, seed, "cuda")
    log(f"[bench] {cfg.name}: chunk rows {step.chunk}, {len(step.chunks)} chunks, "
        f"{step.launches} launches/step")
    clocks.start()
    ms, stages = timed(step, args.steps, args.warmup, dist)
    clock_info = clocks.stop()
    fused = step.fused
    del step
    torch.cuda.empty_cache()

    tokens = cfg.batch * cfg.n_q
    value = world * tokens / (ms / 1e3)
    ix_f, at_f = indexer_flops(cfg), attn_flops(cfg)
    ix_ms = stages["indexer"]["total_ms"] / args.steps
    at_ms = stages["attn"]["total_ms"] / args.steps
    tk_ms = stages["topk"]["total_ms"] / args.steps
    fp8_peak = 2.0 * peaks["bf16_sustained"]
    ix_tf = ix_f / (ix_ms / 1e3) / 1e12
    at_tf = at_f / (at_ms / 1e3) / 1e12
    dominant = max(("indexer", ix_ms), ("attn", at_ms), ("topk", tk_ms), key=lambda x: x[1])[0]
    ix_kernel = "indexer_topk_kernel<64,128,4>" if fused else "indexer_scores_kernel<64,128,4>"
    if dominant == "attn":
        # DRAM bytes of sparse_attn_vh_kernel from one ncu capture at L = 4096
        # (dram__bytes_read.sum + dram__bytes_write.sum = 642.5 MB + 1022.6 MB,
        # profiles/ncu_full_prefill_4k.md); its traffic grows in proportion to
        # the query rows, so it is scaled by rows. Re-capture when the kernel
        # changes.
        traffic = (642.484736e6 + 1022.602e6) / 4096 * cfg.batch * cfg.n_q
        roof = {"kernel": "sparse_attn_vh_kernel", "bound": "tensor",
                "achieved": at_f / (at_ms / 1e3) / 1e12, "peak": peaks["bf16_sustained"],
                "unit": "TFLOP/s", "traffic": traffic,
                "traffic_source": "ncu DRAM bytes of one 4096-row launch, scaled by rows"}
    elif dominant == "indexer":
        roof = {"kernel": ix_kernel, "bound": "tensor",
                "achieved": ix_tf, "peak": fp8_peak, "unit": "TFLOP/s", "traffic": None}
    else:
        roof = {"kernel": "topk_kernel", "bound": "hbm", "achieved": None,
                "peak": peaks["hbm"], "unit": "GB/s", "traffic": None}
    if roof["achieved"] is not None:
        roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = f"{peaks['source']} ({'bf16 sustained' if roof['unit'] == 'TFLOP/s' else 'hbm copy'}" + \
        (", x2 for fp8" if roof.get("kernel", "").startswith("indexer") else "") + ")"

    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8e4m3 indexer, bf16 attention, fp32 accumulate",
        "data": "synthetic (seeded; page-shaped workloads)",
        "config": bench_config(cfg, world),
        "stages_ms": ({"indexer_topk_fused": ix_ms, "attention": at_ms} if fused else
                      {"indexer": ix_ms, "topk": tk_ms, "attention": at_ms}),
        "indexer_tflops_fp8": ix_tf, "indexer_frac_fp8": ix_tf / fp8_peak,
        "attention_tflops_bf16": at_tf, "attention_frac_bf16": at_tf / peaks["bf16_sustained"],
        "roofline": roof, "gpu_launches": step_launches_total(stages),
        "clocks": clock_info,
    }

    if not args.no_decode:
        result["quantiser"] = quantiser_bench(cfg, peaks)

    if not args.no_decode:
        result["decode"] = {}
        for name in ("decode_32k", "decode_64k"):
            dcfg = inputs.CONFIGS[name]
            dstep = Step(dcfg, seed, "cuda")
            # decode steps are ~0.2 ms: many of them, after a longer warm-up,
            # replayed from a CUDA graph
            dsteps = max(args.steps, 100)
            dms, dst = timed(dstep, dsteps, max(args.warmup, 20), dist, graph=True)
            nb = decode_bytes(dcfg)
            at = dst["attn"]["total_ms"] / dsteps
            result["decode"][name] = {
                "ms_per_step": dms, "GB_per_s": nb["total"] / (dms / 1e3) / 1e9,
                "frac_hbm": nb["total"] / (dms / 1e3) / 1e9 / peaks["hbm"],
                "attention_ms": at,
                "attention_GB_per_s": nb["attention"] / (at / 1e3) / 1e9,
                "stages_ms": {k: v["total_ms"] / dsteps for k, v in dst.items()},
                "timing": "CUDA graph replays of the step; stages from an eager pass",
                "algorithmic_bytes": nb["total"]}
            del dstep
            torch.cuda.empty_cache()

    # The ranks of a node share its host RAM: every rank needs its own pinned
    # copy, and all ranks must agree before any of them enters e2e().
    need = e2e_host_bytes(cfg)
    avail = host_available_bytes()
    fits = avail is None or avail >= 2 * need * world
    fits = all_ranks(fits, dist)
    if not args.no_e2e and not fits:
        result["e2e"] = {"value": None, "unit": "tokens/s",
                         "skipped": "host RAM: " + ("unknown" if avail is None else
                                                    f"{avail / 2**30:.0f} GiB") +
                                    f" available, {world * need / 2**30:.0f} GiB pinned needed"}
    elif not args.no_e2e:
        e_ms, h2d, d2h = e2e(cfg, seed, max(2, min(args.steps, 3)), dist)
        result["e2e"] = {"value": world * tokens / (e_ms / 1e3), "unit": "tokens/s",
                         "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                         "ms_per_step": e_ms}

    if not args.no_cpu and world == 1 and rank == 0:
        # A calibration sample of one row per host thread, then a sample
        # sized for about 12 s of oracle work.
        import oracle
        threads = max(1, oracle.hardware_threads())
        _, dt0, _, nr0 = oracle_rows_per_s(cfg, seed, threads)
        reps = max(1, min(32, int(12.0 / max(dt0, 1e-3))))
        n_rows = min(cfg.n_q, nr0 * reps)
        rps, dt, cores, nr = oracle_rows_per_s(cfg, seed, n_rows)
        result["cpu_baseline"] = {"value": rps * cfg.batch, "unit": "tokens/s", "cores": cores,
                                  "kind": "oracle",
                                  "sample": f"{nr} evenly spaced query rows of {cfg.name} "
                                            f"(indexer + top-k + attention, fp64), {dt:.1f} s"}

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def bench_config(cfg, world):
    """The workload description both arms print."""
    return {"workload": cfg.name, "batch": cfg.batch, "seq_len": cfg.n_q,
            "idx_heads": cfg.idx_heads, "idx_dim": cfg.idx_dim, "topk": cfg.topk,
            "heads": cfg.heads, "qk_dim": cfg.qk_dim, "v_dim": cfg.v_dim,
            "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (q is 9.7 GB per step)"}


def step_launches_total(stages):
    return sum(v["launches"] for v in stages.values())


def main_reference(args, world, rank):
    """The reference arm: the fp64 oracle as it stands on this host's cores,
    same workload, metric and unit; each step is a bounded sample of rows."""
    if rank != 0:
        return
    from sparse_attention_long_fp8_b200 import inputs
    cfg = inputs.CONFIGS[args.workload]
    n_rows = 8
    for _ in range(args.warmup):
        oracle_rows_per_s(cfg, 7, 2)
    rates, secs, cores = [], [], 1
    for i in range(args.steps):
        rps, dt, cores, nr = oracle_rows_per_s(cfg, 1000 + i, n_rows)
        rates.append(rps)
        secs.append(dt)
    value = len(rates) * n_rows / sum(secs)
    sample = f"{n_rows} evenly spaced query rows of {cfg.name} per step (fp64 oracle)"
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
