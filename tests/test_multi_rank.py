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


def _rank_dp_oracle(rank, world, port, q):
    """One rank of a data-parallel step on CPU: the library's split of one global batch, the oracle's
    layer forward+backward on this rank's shard, and the gradient sum over ranks (gloo)."""
    from oracle import hstu_oracle as O
    from hstu_sequential_transduction_causal_b200 import hstu as H
    from hstu_sequential_transduction_causal_b200.runtime import shard_rows
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = _dp_batch()
        rank_of, cost = H.hstu_dp_partition(np.diff(wl.offsets), wl.D, world)
        off, rows = shard_rows(wl.offsets, rank_of, rank)
        thr = O.time_bucket_thresholds(128)
        p = wl.layers[0]
        args = (off, wl.timestamps[rows], wl.H, 1.0 / wl.N, wl.pos_max_len, thr)
        y, sv = O.layer_fwd(wl.x[rows], p, *args)
        g = O.layer_bwd(wl.dy[rows], p, sv, *args)
        flat = torch.from_numpy(np.concatenate([np.ravel(g[k]) for k in GRAD_NAMES]))
        dist.all_reduce(flat)
        q.put((rank, rank_of, cost, rows, y, g["dx"], flat.numpy()))
    finally:
        dist.destroy_process_group()


GRAD_NAMES = ("dW1", "db1", "dW2", "db2", "dgamma", "dbeta", "drab_pos", "drab_time")


def _dp_batch():
    lengths = [37, 5, 130, 0, 64, 1, 90, 257, 12, 70, 3]
    return W.make_workload("c3", seed=11, lengths=lengths, D=32, H=2, N=300, pos_max_len=300, backward=True)


def test_two_ranks_cost_balanced_split_sums_to_the_single_rank_gradients():
    """Two gloo ranks split one global batch with hstu_dp_partition: the shards cover every sequence
    exactly once, both ranks compute the same split, its largest load is within the 4/3 bound of the
    greedy rule, each rank's outputs equal the single-rank outputs of its rows, and the all-reduced
    gradients equal the gradients of the whole batch on one rank."""
    from oracle import hstu_oracle as O
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_dp_oracle, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=180) for _ in range(world)], key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = _dp_batch()
    (_, ro0, c0, rows0, y0, dx0, red0), (_, ro1, c1, rows1, y1, dx1, red1) = res
    assert np.array_equal(ro0, ro1) and np.array_equal(c0, c1)
    both = np.concatenate([rows0, rows1])
    assert np.array_equal(np.sort(both), np.arange(wl.T))        # every row exactly once
    lens = np.diff(wl.offsets)
    from hstu_sequential_transduction_causal_b200 import hstu as H
    costs = np.array([H.lib().hstu_dp_sequence_cost(int(n), wl.D) for n in lens])
    assert np.isclose(c0.sum(), costs.sum())
    assert c0.max() <= 4.0 / 3.0 * max(costs.sum() / world, costs.max()) + 1e-9
    thr = O.time_bucket_thresholds(128)
    p = wl.layers[0]
    args = (wl.offsets, wl.timestamps, wl.H, 1.0 / wl.N, wl.pos_max_len, thr)
    y, sv = O.layer_fwd(wl.x, p, *args)
    g = O.layer_bwd(wl.dy, p, sv, *args)
    for rows, yr, dxr in ((rows0, y0, dx0), (rows1, y1, dx1)):
        assert np.allclose(yr, y[rows], rtol=1e-12, atol=1e-12)
        assert np.allclose(dxr, g["dx"][rows], rtol=1e-12, atol=1e-12)
    ref = np.concatenate([np.ravel(g[k]) for k in GRAD_NAMES])
    assert np.array_equal(red0, red1)
    assert np.allclose(red0, ref, rtol=1e-10, atol=1e-10)
