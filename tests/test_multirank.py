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


# ------------------------------------------------ head-sharded prefill

@pytest.mark.parametrize("hkv,world", [(8, 1), (8, 2), (8, 3), (8, 8), (2, 2), (1, 1)])
def test_head_shards_partition_the_kv_heads(hkv, world):
    import bench
    ranges = [bench.head_shard(hkv, r, world) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == hkv
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0
    sizes = [g1 - g0 for g0, g1 in ranges]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_more_ranks_than_kv_heads_is_refused():
    import bench
    with pytest.raises(ValueError):
        bench.head_shard(2, 0, 3)


@pytest.mark.parametrize("name", ["gqa_small", "msa_small", "quest_gate_small"])
def test_the_method_decomposes_by_kv_head(name):
    """Head sharding is exact: the oracle on each rank's kv heads (and the
    query heads reading them) reproduces the full problem's lists and output
    rows of those heads."""
    import numpy as np
    import bench
    import oracle as O
    from block_sparse_attention_sbsa_b200 import workloads as W
    w = W.SMALL[name].scaled(seq_len=1024 + 37)
    data = W.generate(w, "cpu")

    def run(wk, d):
        return O.prefill(d["q"], d["k"], d["v"], block=wk.block_size, mode=wk.select_mode,
                         top_k_=wk.top_k, mass=wk.mass_threshold, margin=wk.gate_margin,
                         tau=wk.rescue_tau, group_shared=wk.group_shared, q_idx=d["q_idx"],
                         k_idx=d["k_idx"], max_blocks=wk.max_blocks, backbone=wk.backbone)
    full = run(w, data)
    for rank in range(2):
        ws, (g0, g1) = bench.shard_workload(w, rank, 2)
        part = run(ws, bench.shard_tensors(data, w, g0, g1))
        hs0, hs1 = (g0, g1) if w.group_shared else (g0 * w.group, g1 * w.group)
        assert np.array_equal(part["idx"], full["idx"][hs0:hs1])
        assert np.array_equal(part["o"], full["o"][g0 * w.group:g1 * w.group])


def _shard_worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from block_sparse_attention_sbsa_b200 import workloads as W
    ws, (g0, g1) = bench.shard_workload(W.CONFIGS["rbs128k"], rank, world)
    got = bench.reduce_max([float(ws.n_kv_heads), float(g1)])
    out[rank] = (g0, g1, ws.n_q_heads, got)
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_split_one_sequence_by_kv_head():
    world, port = 2, _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
    assert (out[0][0], out[0][1]) == (0, 4) and (out[1][0], out[1][1]) == (4, 8)
    assert out[0][2] == out[1][2] == 16
    assert out[0][3] == out[1][3] == [4.0, 8.0]
    import bench
    # one sequence of 131072 tokens, 3 steps, slowest rank 30 ms
    assert bench.weak_throughput(131072, 1, 3, 30.0) == pytest.approx(131072 * 3 / 0.03)


# ------------------------------------------------ self-launching ranks

def _bench(*args, timeout=240):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args], cwd=root, env=env,
                       capture_output=True, text=True, timeout=timeout)
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return r.returncode, (json.loads(lines[-1]) if lines else None), r.stderr


def test_gpus_two_starts_two_ranks_itself():
    """`bench.py --gpus 2` outside torchrun starts both ranks on this node (gloo
    here, no GPU); rank 0 reports a world of two."""
    rc, line, err = _bench("--gpus", "2", "--launch-check")
    assert rc == 0, err
    assert line["n_gpus"] == 2 and sorted(line["ranks"]) == [0, 1]


def test_gpus_beyond_the_visible_devices_fails_loudly():
    rc, line, err = _bench("--gpus", "4096", "--launch-check")
    assert rc != 0 and line is None
    assert "visible" in err


# ------------------------------------- percentile gate across head shards

def _gate_shard_worker(rank, world, port, name, out):
    """One rank of a sequence sharded by kv head under the percentile gate:
    the oracle's cut margins of this rank's selection heads, summed per tile,
    all-reduced over the ranks, then the tile decisions and this rank's lists."""
    import math
    import numpy as np
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    import oracle as O
    from block_sparse_attention_sbsa_b200 import workloads as W
    w = W.SMALL[name]
    data = W.generate(w, "cpu")
    ws, (g0, g1) = bench.shard_workload(w, rank, world)
    d = bench.shard_tensors(data, w, g0, g1)
    ks = d["k_idx"] if ws.index_dim else d["k"]
    qs = d["q_idx"] if ws.index_dim else d["q"]
    c, r = O.pool_keys(ks, ws.block_size, with_radius=False)
    r = np.zeros(c.shape[:2])
    mm = O.pool_keys_minmax(ks, ws.block_size) if ws.backbone == "minmax" else None
    qbar = O.pool_queries(qs, ws.block_size, group=1)
    scale = 1.0 / math.sqrt(ws.score_dim)
    kv = lambda hs: hs // ws.group
    nb, k = ws.n_blocks, ws.top_k

    def scores(h, i):
        if mm is None:
            return O.block_scores(qbar[h, i], c[kv(h)], i, scale)
        return O.block_bounds_minmax(qbar[h, i], mm[0][kv(h)], mm[1][kv(h)], i, scale)
    sums = torch.zeros(nb, dtype=torch.float64)
    for i in range(k + 1, nb):
        tot = 0.0
        for h in range(ws.n_sel_heads):            # this rank's heads, head order
            tot += O.cut_margin(scores(h, i), k)
        sums[i] = tot
    dist.all_reduce(sums)                          # the one exchange of the path
    total = w.n_sel_heads
    sbar = {i: float(sums[i]) / total for i in range(k + 1, nb)}
    q = float(np.float32(w.gate_quantile))
    fired = O.percentile_fire(sbar, q)
    idx, cnt, _ = O.select(qbar, c, r, block_count=nb, mode=ws.select_mode, top_k_=k,
                           scale=scale, kv_of_sel=kv, max_blocks=ws.max_blocks, minmax=mm,
                           sigma_gate=(q, w.gate_rho), fired=fired)
    out[rank] = (g0, g1, sorted(fired), sbar, idx, cnt)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("name", ["sigma_small", "sigma_quest_small"])
def test_percentile_gate_decomposes_over_head_shards_with_one_all_reduce(name):
    """The percentile gate couples heads (a tile's mean margin over all
    selection heads).  Two ranks, each holding half the kv heads, reproduce the
    unsharded oracle's fired tiles and lists after one all-reduce of their
    per-tile margin sums."""
    import numpy as np
    import oracle as O
    import parity as PT
    from block_sparse_attention_sbsa_b200 import workloads as W
    world, port = 2, _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_gate_shard_worker, args=(world, port, name, out), nprocs=world, join=True)
    w = W.SMALL[name]
    data = W.generate(w, "cpu")
    q = float(np.float32(w.gate_quantile))
    full = O.prefill(data["q"], data["k"], data["v"], block=w.block_size, mode=w.select_mode,
                     top_k_=w.top_k, max_blocks=w.max_blocks, backbone=w.backbone,
                     sigma_gate=(q, w.gate_rho))
    fired0, fired1 = out[0][2], out[1][2]
    assert fired0 == fired1                          # both ranks decided alike
    # the ranks' sums add in another order than one head-order sum: every
    # tile's decision agrees with the unsharded one outside SIGMA_BAND
    budgets = PT.percentile_budgets(full["sbar"], full["fired"], w.top_k, w.gate_rho)
    for i, b in budgets.items():
        took = w.gate_rho * w.top_k if i in fired0 else w.top_k
        assert took in b, i
        assert abs(out[0][3][i] - full["sbar"][i]) < 1e-12
    for rank in range(world):
        g0, g1 = out[rank][0], out[rank][1]
        hs0, hs1 = g0 * w.group, g1 * w.group
        if set(fired0) == set(full["fired"]):
            assert np.array_equal(out[rank][4], full["idx"][hs0:hs1])
            assert np.array_equal(out[rank][5], full["cnt"][hs0:hs1])
