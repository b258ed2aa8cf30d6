"""The data-parallel path's host logic on two CPU ranks (gloo): each rank draws its own batch (seed =
rank, weak scaling), the flat gradient buffer is all-reduced once per step, device times are the max
over ranks and tokens the sum over ranks. The same helpers bench.py uses under torchrun with NCCL."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from hstu_sequential_transduction_causal_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = W.make_workload("c3", seed=rank, lengths=None)
        D, L = 64, 32
        flat, views = bench.grad_buffer(D, L, "cpu")
        # a per-rank stand-in for the gradients: deterministic values from the rank's own batch
        rng = np.random.default_rng(int(wl.T) + rank)
        for v in views:
            v.copy_(torch.from_numpy(rng.standard_normal(v.numel()).astype(np.float32)))
        local = flat.clone()
        dist.all_reduce(flat)
        t_ms, a_ms, tokens = bench.reduce_over_ranks(1.0 + rank, 0.5 * (2 - rank), wl.T, world, "cpu")
        q.put((rank, int(wl.T), local.numpy(), flat.numpy(), t_ms, a_ms, tokens,
               [int(v.data_ptr() - flat.data_ptr()) for v in views]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_and_gradient_allreduce():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in range(world)], key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, T0, loc0, red0, t0, a0, n0, offs), (_, T1, loc1, red1, t1, a1, n1, _) = res
    assert T0 != T1                                   # each rank has its own batch
    assert np.allclose(red0, loc0 + loc1) and np.array_equal(red0, red1)
    assert t0 == t1 == 2.0 and a0 == a1 == 1.0          # max over ranks
    assert n0 == n1 == float(T0 + T1)                   # tokens summed
    assert all(o % 16 == 0 for o in offs)               # every gradient view 16-byte aligned
