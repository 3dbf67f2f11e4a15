"""Multi-rank host logic on CPU with the gloo backend (world size 2): token
shards cover every token once, each rank's shard of the forward equals the
same tokens of the whole batch (tokens are independent), and timing takes the
max over ranks.  The per-rank compute here is the oracle; on GPUs it is the
CUDA path with the same sharding and no collective on the data path."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from ternary_butterfly_experts_b200.shard import max_over_ranks, token_range


def test_token_range_partitions():
    for T in (0, 1, 7, 16, 1001):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                a, b = token_range(T, r, world)
                assert 0 <= a <= b <= T
                seen.extend(range(a, b))
            assert seen == list(range(T))
    with pytest.raises(ValueError):
        token_range(10, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import workloads as W
        from oracle import bfmoe_oracle as O

        wl = W.custom("mr", d=16, n_experts=5, k=2, tokens=11, dtype="f32", bias_var=0.5)
        inp = W.generate(wl, seed=4)
        a, b = token_range(wl.tokens, rank, world)
        x = inp.x_f64()[a:b]
        idx, g, _, _ = O.route(x, inp.w_gate, inp.bias, wl.k)
        y = O.forward(x, inp.w_base, inp.alpha, inp.theta, inp.phi, idx, g)
        # gather only to check the result; the data path itself has no collective
        sizes = [None] * world
        dist.all_gather_object(sizes, y.tolist())
        t_max = max_over_ranks(1.0 + rank)
        if rank == 0:
            full = np.concatenate([np.array(s).reshape(-1, wl.d) for s in sizes])
            idx_f, g_f, _, _ = O.route(inp.x_f64(), inp.w_gate, inp.bias, wl.k)
            ref = O.forward(inp.x_f64(), inp.w_base, inp.alpha, inp.theta, inp.phi, idx_f, g_f)
            np.save(os.path.join(out_dir, "diff.npy"), np.array([np.abs(full - ref).max(), t_max]))
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_match_whole_batch(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    diff, t_max = np.load(os.path.join(tmp_path, "diff.npy"))
    assert diff < 1e-12
    assert t_max == 2.0


def test_max_over_ranks_without_group():
    assert max_over_ranks(3.5) == 3.5
