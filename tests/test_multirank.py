"""Multi-process host logic of the benchmark (world size 2, gloo, CPU):
weak-scaling workloads per rank, max-over-ranks timing, aggregate value."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from block_sparse_attention_sbsa_b200 import workloads as W
    w = bench.rank_workload(W.CONFIGS["rbs128k"], rank)
    got = bench.reduce_max([10.0 + rank, 5.0 - rank, float(w.seed)])
    out[rank] = got
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_distinct_sequences():
    world, port = 2, _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    from block_sparse_attention_sbsa_b200 import workloads as W
    base = W.CONFIGS["rbs128k"].seed
    for r in range(world):
        assert out[r][:2] == [11.0, 5.0]
        assert out[r][2] == float(base + 1000)       # max of the per-rank seeds
    import bench
    # 2 ranks x 3 steps x 131072 tokens over the slowest 30 ms
    assert bench.weak_throughput(131072, 2, 3, 30.0) == pytest.approx(131072 * 6 / 0.03)


def test_single_process_reduce_is_identity():
    import bench
    assert bench.reduce_max([1.5, 2.5]) == [1.5, 2.5]
