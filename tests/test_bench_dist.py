"""CPU (gloo, world size 2) checks of bench.py's multi-rank logic: each rank
draws its own batch, the step time reported is the max over ranks, and the
batch-summed parameter gradients are summed over ranks, as a data-parallel
training step needs.  No GPU: the CUDA kernels are not involved."""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import bench
    from semi_markov_crf_b200 import synth
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        seed = bench.shard_seed(synth.WORKLOADS["speech"].seed, rank)
        w = synth.make("speech", B=2, T=50, seed=seed)
        t = bench.reduce_max(float(rank + 1) * 1.5)
        g1 = torch.full((3, 3), float(rank + 1))
        g2 = torch.arange(4, dtype=torch.float32) * (rank + 1)
        bench.allreduce_param_grads([g1, g2])
        out[rank] = (seed, float(w["em"].sum()), t, g1.tolist(), g2.tolist())
    finally:
        dist.destroy_process_group()


def test_two_rank_sharding_timing_and_gradient_sum():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    s0, e0, t0, g10, g20 = res[0]
    s1, e1, t1, g11, g21 = res[1]
    assert s0 != s1 and e0 != e1           # different batches per rank
    assert t0 == t1 == 3.0                 # max over ranks
    assert g10 == g11 == [[3.0] * 3] * 3   # 1 + 2
    assert g20 == g21 == [0.0, 3.0, 6.0, 9.0]


def test_single_process_helpers_are_identities():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(2.5) == 2.5
    t = torch.ones(2)
    bench.allreduce_param_grads([t])
    assert t.tolist() == [1.0, 1.0]
    assert bench.edges_of([10, 5], 3, 2) == 15 * 3 * 4
    assert bench.algorithmic_ops_per_position("chain_kernel", 30, 39) == (2 * 30 * 39, "mufu")
