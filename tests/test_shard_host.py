"""Query-sharded prefill, host side, on CPU: the partition of one prefill's
query rows over ranks and the all-gather of sequence-sharded keys, with two
gloo ranks. Each rank's oracle rows (computed with the rows' absolute
positions against the gathered keys) must equal the unsharded oracle's."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_attention_long_fp8_b200 import inputs as dsa_inputs
from sparse_attention_long_fp8_b200 import shard


@pytest.mark.parametrize("L,R", [(1, 1), (5, 2), (256, 2), (4096, 8), (4097, 3), (65536, 8),
                                 (13, 8)])
def test_partition_is_exact_and_balanced(L, R):
    parts = [shard.shard_rows(L, R, r) for r in range(R)]
    allrows = np.concatenate(parts)
    assert len(allrows) == L and np.array_equal(np.sort(allrows), np.arange(L))
    for p in parts:
        assert (np.diff(p) > 0).all()                     # increasing within a shard
        assert len(p) % 4 == 0 or (L - 1) in p            # whole groups but the cut last one
    sizes = [len(p) for p in parts]
    assert max(sizes) - min(sizes) <= 4
    cost = [shard.shard_cost(L, L, R, r, 2048)[0] for r in range(R)]
    assert max(cost) - min(cost) <= 4 * L                 # within one group's indexer work


def test_key_slices_tile_the_sequence():
    for n_kv, R in [(256, 2), (1000, 3), (7, 8)]:
        sl = [shard.key_slice(n_kv, R, r) for r in range(R)]
        assert sl[0][0] == 0 and sl[-1][1] == n_kv
        assert all(a[1] == b[0] for a, b in zip(sl, sl[1:]))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        cfg = dsa_inputs.CONFIGS["tiny"]
        inp = dsa_inputs.make_inputs(cfg, seed=21)       # every rank draws the same inputs
        k0, k1 = shard.key_slice(cfg.n_kv, world, rank)
        # this rank's slice of the keys, as a sequence-sharded upstream would hold it
        full = {}
        for key in ("k_fp8", "k_scale", "kv"):
            t = inp[key]
            loc = t[:, k0:k1]
            g = shard.all_gather_keys(loc, cfg.n_kv, dist)
            full[key] = g
            assert torch.equal(g, t), key
        rows = shard.shard_rows(cfg.n_q, world, rank)
        sh = shard.shard_inputs(inp, rows)
        pos = sh["row_pos"][0].numpy()
        assert np.array_equal(pos, rows)
        sc = oracle.indexer_scores(sh["q_fp8"][0], sh["q_scale"][0], sh["w"][0], full["k_fp8"][0],
                                   full["k_scale"][0], pos, cfg.n_kv)
        idx = oracle.topk(sc, cfg.topk)
        o, lse = oracle.sparse_attn(sh["q"][0], full["kv"][0], idx, cfg.softmax_scale, cfg.v_dim)
        queue.put((rank, rows, idx, o, lse))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_the_unsharded_oracle(oracle_lib):
    world = 2
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    res = []
    import queue as _q
    while len(res) < world:          # fail fast if a rank dies
        try:
            res.append(queue.get(timeout=2))
        except _q.Empty:
            assert all(p.is_alive() or p.exitcode == 0 for p in procs), "a rank failed"
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    cfg = dsa_inputs.CONFIGS["tiny"]
    inp = dsa_inputs.make_inputs(cfg, seed=21)
    ref = oracle_lib.forward(inp, cfg)
    seen = np.zeros(cfg.n_q, dtype=int)
    for _, rows, idx, o, lse in res:
        seen[rows] += 1
        assert np.array_equal(idx, ref["indices"][rows])
        np.testing.assert_array_equal(o, ref["o"][rows])
        np.testing.assert_array_equal(lse, ref["lse"][rows])
    assert (seen == 1).all()
