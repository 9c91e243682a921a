#!/usr/bin/env python
"""Sparse-prefill benchmark on B200: tokens/s of one block-sparse attention
prefill (pool -> select -> attend) at 128k tokens, the RBS dual-branch
workload (32 query / 8 kv heads, d = 128, B = 128, bf16, cumulative score
mass 0.9 united with the radius rescue branch).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sbsa|reference]

One process per GPU.  With --gpus N > 1 and no torchrun environment the
script starts the N ranks itself (torch.distributed.run on this node) and
refuses N above the visible device count.  By default every rank runs its
own independent sequence (weak scaling); with --shard heads the ranks split
one sequence by kv head, each prefilling its kv heads and their query heads
(strong scaling).  The selection and the attention of a kv head need
nothing from another, with one exception: the percentile gate averages a
tile's cut margins over every head, so under --shard heads its per-tile
margin sums are all-reduced (NCCL) between its two halves.  The reported
time is the maximum over ranks.  Rank 0 prints one JSON line.
`--impl reference` times the CPU oracle on a bounded sample of the same
workload instead.
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse prefill tokens/s and attended TFLOP/s at 128k; % of bf16 TC / HBM roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
# dram__bytes_read.sum + dram__bytes_write.sum of one attention launch, from the
# ncu capture summarised in profiles/, keyed by workload and by the hash of the
# kernel source it was taken on: once that source changes the figure no longer
# describes the kernel and the line reports null.
NCU_ATTEND_TRAFFIC = {
    # profiles/attend_ps_kernel_dram_rbs.md: 2.35 GB read + 1.05 GB written
    "rbs128k": {"bytes": 3.40e9, "source": "block_sparse_attention_sbsa_b200/csrc/attend_persist.cu",
                "sha": "2772f1140986d557"},
}


def selection_stats(w, p, st, meta) -> dict:
    """What the selection produced: rows whose gap gate fired, rows the
    radius rescue added blocks to, planted needles found, and the attention
    stage's algorithmic bytes (Q + O + each distinct K/V block once)."""
    import torch
    from block_sparse_attention_sbsa_b200 import sbsa
    flags = st.flags.to(torch.int32)
    out = {
        "rows": int(flags.numel()),
        "gate_fired_fraction": float(((flags & sbsa.FLAG_GATE) != 0).float().mean()),
        "rescued_rows_fraction": float(((flags & sbsa.FLAG_RESCUE) != 0).float().mean()),
    }
    nb, kmax = w.n_blocks, st.idx.shape[-1]
    valid = torch.arange(kmax, device=st.idx.device).view(1, 1, -1) < st.cnt.unsqueeze(-1)
    ids = torch.where(valid, st.idx, torch.full_like(st.idx, -1)).to(torch.int64)
    # distinct (kv head, key block) pairs named by any list
    grp = 1 if w.group_shared else w.n_q_heads // w.n_kv_heads
    kvh = (torch.arange(ids.shape[0], device=ids.device) // grp).view(-1, 1, 1).expand_as(ids)
    used = torch.zeros(w.n_kv_heads * nb, dtype=torch.bool, device=ids.device)
    sel = ids >= 0
    used[(kvh[sel] * nb + ids[sel]).unique()] = True
    es = 2 if w.dtype == "bf16" else 4
    blk = w.block_size * w.head_dim * es
    out["distinct_kv_blocks"] = int(used.sum())
    out["attend_algorithmic_bytes"] = int(2 * w.n_q_heads * w.seq_len * w.head_dim * es
                                          + 2 * int(used.sum()) * blk)
    needles = meta.get("needles", [])
    if needles and w.group_shared:
        hits = 0
        idx_cpu, cnt_cpu = st.idx.cpu(), st.cnt.cpu()
        for (g, pos, qb) in needles:
            row = idx_cpu[g, qb, :int(cnt_cpu[g, qb])]
            hits += int((row == pos // w.block_size).any())
        out["needle_hit_rate"] = hits / len(needles)
    return out


def source_hash(rel: str) -> str:
    import hashlib
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def attend_kernel_source(w) -> str:
    """The source file of the attention kernel that workload w dispatches to."""
    name = attend_kernel_name(w)
    base = "block_sparse_attention_sbsa_b200/csrc/"
    for key, f in (("attend_pair", "attend_pair.cu"), ("attend_duo", "attend_duo.cu"),
                   ("attend_ps64", "attend_ps64.cu"), ("attend_ps", "attend_persist.cu")):
        if name.startswith(key):
            return base + f
    return base + "attend.cu"


def measured_traffic(w):
    """ncu DRAM bytes of one attention launch for w, or None when none was
    captured on the current kernel source."""
    rec = NCU_ATTEND_TRAFFIC.get(w.name)
    if not rec:
        return None
    src = attend_kernel_source(w)
    return rec["bytes"] if rec.get("source") == src and rec.get("sha") == source_hash(src) else None


def spread(xs):
    """Median and 10th / 90th percentiles of per-step times (ms)."""
    ys = sorted(xs)
    if not ys:
        return {}

    def q(f):
        k = f * (len(ys) - 1)
        lo = int(math.floor(k))
        hi = min(lo + 1, len(ys) - 1)
        return ys[lo] + (ys[hi] - ys[lo]) * (k - lo)
    return {"median": q(0.5), "p10": q(0.1), "p90": q(0.9), "mean": statistics.mean(ys)}


def attend_kernel_name(w) -> str:
    """The attention kernel sbsa_attend dispatches to for workload w (the rule
    of launch_attend in csrc/attend.cu)."""
    big = w.dtype == "bf16" and w.block_size == 128 and w.head_dim in (64, 128)
    pairable = big and w.group_shared and (w.n_q_heads // w.n_kv_heads) % 2 == 0
    shape = f"{w.dtype}, B={w.block_size}, d={w.head_dim}"
    if w.dtype == "bf16" and w.block_size == 64:
        return (f"attend_ps64_kernel<{w.head_dim}> (persistent, tiles of two 64-token query "
                f"blocks, tcgen05, {shape})")
    if pairable:
        return f"attend_pair_kernel<{w.head_dim}> (two query heads share K/V, tcgen05, {shape})"
    if big:
        return f"attend_ps_kernel<{w.head_dim}> (persistent, tcgen05, {shape})"
    return f"attend_kernel (one CTA per query block, tcgen05, {shape})"


def launches_per_step(w) -> int:
    """Kernels one staged prefill step launches (the calls of sbsa.Staged):
    key pooling; query pooling, or the three-part centroid split and the
    row-max scores; with the mean backbone and mean tile scores the tf32 split
    and the tensor-core centroid scores; the selection (four launches under
    the percentile gate: first pass, per-tile sums, tile decisions, second
    pass); the attention."""
    rowmax = w.tile_score == "rowmax"
    n = 1 + (2 if rowmax else 1)
    if w.backbone == "mean" and not rowmax and w.n_blocks >= 2:
        n += 2
    n += 4 if w.gate_quantile is not None else 1
    return n + 1


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="sbsa", choices=["sbsa", "reference"])
    ap.add_argument("--workload", default="rbs128k")
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--cpu-blocks", type=int, default=6,
                    help="query blocks (all heads) in the CPU-oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", default="sequences", choices=["sequences", "heads"],
                    help="N > 1: independent sequences per rank (weak scaling) or one "
                         "sequence split by kv head (strong scaling)")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override the workload length (small cases for profiling)")
    ap.add_argument("--launch-check", action="store_true",
                    help="only start the ranks, join the process group and report the world")
    return ap.parse_args(argv)


def pick_workload(args):
    from block_sparse_attention_sbsa_b200 import workloads as W
    w = W.CONFIGS[args.workload]
    if args.seq_len:
        w = w.scaled(name=f"{w.name}@{args.seq_len}", seq_len=args.seq_len)
    return w


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = None

    def start(self):
        """Start sampling every 20 ms and return once the first sample is in,
        so that even a timed region of a few tens of milliseconds is sampled
        (the first sample, taken just before the region, is dropped when
        later ones exist)."""
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        deadline = time.time() + 3.0
        while time.time() < deadline and self.proc.poll() is None:
            if os.path.getsize(self.tmp.name) > 0:
                break
            time.sleep(0.005)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = list(csv.reader(io.StringIO(self.tmp.read())))
        os.unlink(self.tmp.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = [r for r in rows if len(r) >= 9]
        if len(rows) > 1:
            rows = rows[1:]  # the first sample precedes the timed region
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for nm, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------- CPU oracle leg
def oracle_sample(w, data_cpu, blocks):
    """Oracle work for the full key pooling plus selection and attention of
    the given query blocks (all heads).  Returns the two timings and what the
    oracle computed (lists, tables, outputs of the sampled blocks) so that the
    GPU's results can be compared with it afterwards."""
    import numpy as np
    import oracle as O
    t0 = time.perf_counter()
    ks = data_cpu["k_idx"] if w.index_dim else data_cpu["k"]
    c, r = O.pool_keys(ks, w.block_size, with_radius=w.rescue_tau is not None)
    if r is None:
        r = np.zeros(c.shape[:2])
    minmax = O.pool_keys_minmax(ks, w.block_size) if w.backbone == "minmax" else None
    nb, b = w.n_blocks, w.block_size
    grp = w.group if w.group_shared else 1
    qbar = np.zeros((w.n_sel_heads, nb, w.score_dim))
    sigma_gate, fired, sbar = None, None, None
    kv_of = (lambda hs: hs) if w.group_shared else (lambda hs: hs // w.group)
    if w.gate_quantile is not None:
        # the gate's global part (every tile's margin and the tile decisions)
        # is per prefill, not per block
        qbar = O.pool_queries(data_cpu["q_all"], b, group=grp)
        sigma_gate = (w.gate_quantile, w.gate_rho)
        info = {}
        O.select(qbar, c, r, block_count=nb, mode=w.select_mode, top_k_=w.top_k,
                 scale=1.0 / math.sqrt(w.score_dim), kv_of_sel=kv_of, max_blocks=w.max_blocks,
                 rows=[], minmax=minmax, sigma_gate=sigma_gate, info=info)
        fired, sbar = info["fired"], info["sbar"]
    t_pool = time.perf_counter() - t0
    t1 = time.perf_counter()
    qsrc = data_cpu["q_rows_idx"] if w.index_dim else data_cpu["q_rows"]
    for bi, i in enumerate(blocks):
        qbar[:, i] = O.pool_queries(qsrc[:, bi * b:(bi + 1) * b], b, group=grp)[:, 0]
    rows = [(hs, i) for hs in range(w.n_sel_heads) for i in blocks]
    row_scores = None
    if w.tile_score == "rowmax":
        where = {i: bi for bi, i in enumerate(blocks)}

        def row_scores(hs, i):
            heads = range(hs * grp, (hs + 1) * grp) if w.group_shared else [hs]
            bi = where[i]
            tile = np.concatenate([np.asarray(qsrc[h, bi * b:(bi + 1) * b].double())
                                   for h in heads])
            return O.block_scores_rowmax(tile, c[kv_of(hs)], i, 1.0 / math.sqrt(w.score_dim))
    idx, cnt, _ = O.select(qbar, c, r, block_count=nb, mode=w.select_mode, top_k_=w.top_k,
                           mass=w.mass_threshold, margin=w.gate_margin, tau=w.rescue_tau,
                           scale=1.0 / math.sqrt(w.score_dim), kv_of_sel=kv_of,
                           max_blocks=w.max_blocks, rows=rows, minmax=minmax,
                           sigma_gate=sigma_gate, row_scores=row_scores, fired=fired)
    scale = 1.0 / math.sqrt(w.head_dim)
    outs = {}
    for bi, i in enumerate(blocks):
        for h in range(w.n_q_heads):
            hs = h // w.group if w.group_shared else h
            ids = [int(x) for x in idx[hs, i, :cnt[hs, i]]]
            outs[(h, i)] = O.attend_block(data_cpu["q_rows"][h, bi * b:(bi + 1) * b],
                                          data_cpu["k"][h // w.group], data_cpu["v"][h // w.group],
                                          ids, i, b, scale)
    t_rows = time.perf_counter() - t1
    return dict(t_pool=t_pool, t_rows=t_rows, idx=idx, cnt=cnt, rows=rows, qbar=qbar, c=c, r=r,
                minmax=minmax, row_scores=row_scores, fired=fired, sbar=sbar, outs=outs,
                kv_of=kv_of)


def cpu_copy_for_oracle(w, data, blocks):
    import torch
    b = w.block_size
    out = {"k": data["k"].cpu(), "v": data["v"].cpu(),
           "k_idx": data["k_idx"].cpu() if data["k_idx"] is not None else None}
    out["q_rows"] = torch.cat([data["q"][:, i * b:(i + 1) * b] for i in blocks], dim=1).cpu()
    if data["q_idx"] is not None:
        out["q_rows_idx"] = torch.cat([data["q_idx"][:, i * b:(i + 1) * b] for i in blocks],
                                      dim=1).cpu()
    if w.gate_quantile is not None:
        # the percentile gate ranks every tile: the oracle needs every query block
        out["q_all"] = (data["q_idx"] if data["q_idx"] is not None else data["q"]).cpu()
    return out


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max((d.get("num_threads", 1) for d in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


class CpuMeter:
    """Wall and process CPU time of a region: their ratio is the number of
    host cores the region kept busy on average."""

    def __enter__(self):
        self.w0, self.c0 = time.perf_counter(), time.process_time()
        return self

    def __exit__(self, *exc):
        self.wall = time.perf_counter() - self.w0
        self.cpu = time.process_time() - self.c0
        return False

    @property
    def cores(self) -> float:
        return round(self.cpu / self.wall, 2) if self.wall > 0 else 0.0


def sample_blocks(w, count, salt=0):
    import torch
    g = torch.Generator().manual_seed(w.seed + 101 + salt)
    picks = set()
    while len(picks) < min(count, w.n_blocks):
        picks.add(int(torch.randint(0, w.n_blocks, (1,), generator=g)))
    return sorted(picks)


def parity_on_sample(w, res, gpu_idx, gpu_cnt, gpu_o, blocks):
    """The GPU's lists and outputs of the sampled query blocks against the
    oracle's: rows equal to the oracle's, rows that differ only inside the fp32
    tie band, and output errors over the rows whose lists are equal."""
    import numpy as np
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import parity as PT
    nb = w.n_blocks
    gi = np.full((w.n_sel_heads, nb, w.max_blocks), -1, dtype=np.int32)
    gc = np.zeros((w.n_sel_heads, nb), dtype=np.int32)
    gi[:, blocks] = gpu_idx[:, blocks].cpu().numpy()
    gc[:, blocks] = gpu_cnt[:, blocks].cpu().numpy()
    budgets = None
    if w.gate_quantile is not None:
        budgets = PT.percentile_budgets(res["sbar"], res["fired"], w.top_k, w.gate_rho)
    exact, tie = PT.compare_lists(gi, gc, res["idx"], res["cnt"], res["rows"], res["qbar"],
                                  res["c"], res["r"], w, res["kv_of"], minmax=res["minmax"],
                                  budgets=budgets, score_fn=res["row_scores"])
    errs = []
    b = w.block_size
    for (h, i), ref in res["outs"].items():
        hs = h // w.group if w.group_shared else h
        if not np.array_equal(gi[hs, i], res["idx"][hs, i]):
            continue
        got = gpu_o[h, i * b:min(w.seq_len, (i + 1) * b)].float().cpu().numpy()
        errs.append(PT.output_errors(got, ref))
    return {"rows": exact + tie, "exact": exact, "tie": tie,
            "sigma_band_tiles": PT.sigma_band_tiles(budgets),
            "max_abs": max(e[0] for e in errs) if errs else None,
            "mean_abs": float(np.mean([e[1] for e in errs])) if errs else None,
            "bounds": {"max_abs": PT.MAX_ABS, "mean_abs": PT.MEAN_ABS, "tie_band": PT.BAND},
            "sample": f"{len(blocks)} query blocks x {w.n_sel_heads} selection heads "
                      f"(outputs of all {w.n_q_heads} query heads)"}


def cpu_baseline_and_parity(w, data, nblocks, gpu_idx, gpu_cnt, gpu_o):
    blocks = sample_blocks(w, nblocks)
    cdata = cpu_copy_for_oracle(w, data, blocks)
    with CpuMeter() as m:
        res = oracle_sample(w, cdata, blocks)
    t_pool, t_rows = res["t_pool"], res["t_rows"]
    full = t_pool + t_rows * w.n_blocks / len(blocks)
    base = {
        "value": w.seq_len / full, "unit": UNIT, "cores": m.cores, "kind": "oracle",
        "threads_available": blas_threads(),
        "sample": (f"numpy float64 oracle: key pooling of all {w.n_blocks} blocks "
                   f"({t_pool:.1f}s) + selection and attention of {len(blocks)} query blocks x "
                   f"{w.n_q_heads} heads ({t_rows:.1f}s), extrapolated per query block to the "
                   f"full {w.seq_len}-token prefill ({full:.0f}s); cores = process CPU time / "
                   f"wall time of the sample"),
    }
    return base, parity_on_sample(w, res, gpu_idx, gpu_cnt, gpu_o, blocks)


# ------------------------------------------------------------ reference arm
def run_reference(args):
    """The oracle as it stands, on the host cores: each step is a bounded
    sample of the workload (key pooling of all blocks, selection and
    attention of one query block in all heads); ms_per_step is the measured
    time of that sample and the value extrapolates it per query block to the
    full prefill."""
    import torch
    from block_sparse_attention_sbsa_b200 import workloads as W
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = pick_workload(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    data = W.generate(w, dev)
    sample_s, full_s, cpu_s = 0.0, 0.0, 0.0
    for s in range(args.warmup + args.steps):
        blocks = sample_blocks(w, 1, salt=s)
        cdata = cpu_copy_for_oracle(w, data, blocks)
        with CpuMeter() as m:
            res = oracle_sample(w, cdata, blocks)
        if s >= args.warmup:
            sample_s += m.wall
            cpu_s += m.cpu
            full_s += res["t_pool"] + res["t_rows"] * w.n_blocks / len(blocks)
    value = w.seq_len * args.steps / full_s
    cores = round(cpu_s / sample_s, 2) if sample_s > 0 else 0.0
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * sample_s / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "extrapolated": {"ms_per_full_prefill": 1000.0 * full_s / max(1, args.steps),
                         "note": "value = tokens of a full prefill / the sampled step's time "
                                 "scaled per query block; ms_per_step is the sample as timed"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "threads_available": blas_threads(),
                         "sample": ("per step: key pooling of all blocks + selection and "
                                    "attention of 1 query block x all heads, extrapolated per "
                                    "query block to the full prefill; cores = process CPU time "
                                    "/ wall time")},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def workload_config(w, world: int = 1, heads: bool = False):
    if w.select_mode == "cummass":
        sel = f"cumulative mass {w.mass_threshold} + rescue tau {w.rescue_tau}"
    else:
        sel = f"top-{w.top_k}"
        if w.gate_margin is not None:
            sel += f" gated x2 margin {w.gate_margin}"
        if w.gate_quantile is not None:
            sel += f" percentile gate q {w.gate_quantile} rho {w.gate_rho}"
        if w.group_shared:
            sel += " per GQA group"
    if w.backbone != "mean":
        sel += ", K-min/K-max upper-bound scores"
    if w.tile_score != "mean":
        sel += ", row-max tile scores"
    return {"workload": w.name, "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads,
            "seq_len": w.seq_len, "head_dim": w.head_dim, "block_size": w.block_size,
            "select": sel, "global_batch": 1, "seq": w.seq_len,
            "l2": "inputs larger than L2 (Q, K, V each exceed 126 MB); no flush between steps",
            "parallelism": (f"kv heads split over {world} GPUs" if heads else
                            f"{world} independent sequence(s), one per GPU")}


# ------------------------------------------------------- rank bookkeeping
def rank_workload(base, rank: int):
    """Weak scaling: every rank prefills its own sequence of the same shape."""
    return base.scaled(seed=base.seed + 1000 * rank)


def head_shard(n_kv_heads: int, rank: int, world: int):
    """Contiguous kv-head range [g0, g1) of a rank when one sequence is split
    by kv head: as even as possible, the first ranks take one more."""
    if world > n_kv_heads:
        raise ValueError(f"{world} ranks cannot split {n_kv_heads} kv heads")
    base, rem = divmod(n_kv_heads, world)
    g0 = rank * base + min(rank, rem)
    return g0, g0 + base + (1 if rank < rem else 0)


def shard_workload(w, rank: int, world: int):
    """The sub-problem of one rank under head sharding: its kv heads and the
    query heads that read them, same sequence and seed."""
    g0, g1 = head_shard(w.n_kv_heads, rank, world)
    return w.scaled(n_q_heads=(g1 - g0) * w.group, n_kv_heads=g1 - g0), (g0, g1)


def shard_tensors(data: dict, w_full, g0: int, g1: int) -> dict:
    """Head slices of a generated workload (head-major layout: contiguous)."""
    grp = w_full.group
    out = dict(data)
    out["q"] = data["q"][g0 * grp:g1 * grp]
    out["k"], out["v"] = data["k"][g0:g1], data["v"][g0:g1]
    if data.get("q_idx") is not None:
        out["q_idx"] = data["q_idx"][g0 * grp:g1 * grp]
        out["k_idx"] = data["k_idx"][g0:g1]
    return out


def reduce_max(values, device="cpu"):
    """Element-wise maximum over ranks (identity on one process)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def weak_throughput(seq_len: int, world: int, steps: int, max_ms: float) -> float:
    """Tokens of all ranks' sequences over the slowest rank's time."""
    return seq_len * world * steps / (max_ms / 1000.0)


# ------------------------------------------------------------- launching
def free_port() -> int:
    import socket
    so = socket.socket()
    so.bind(("127.0.0.1", 0))
    port = so.getsockname()[1]
    so.close()
    return port


def visible_devices() -> int:
    import torch
    return torch.cuda.device_count()


def relaunch(args, argv) -> int:
    """--gpus N > 1 without a torchrun environment: start the N ranks on this
    node (one process per GPU) and return their exit status."""
    n = visible_devices() if not args.launch_check else (visible_devices() or os.cpu_count())
    if args.gpus > n:
        raise SystemExit(f"--gpus {args.gpus}: only {n} device(s) visible")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
           "--master-port", str(free_port()), os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd)


def launch_check(args) -> int:
    """Each rank joins the process group (NCCL on GPUs, gloo on CPU) and
    reports itself; rank 0 prints the world it saw."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    dev = "cpu"
    if backend == "nccl":
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dev = "cuda"
    if world > 1:
        from datetime import timedelta
        dist.init_process_group(backend, timeout=timedelta(seconds=60))
    ranks = [rank]
    if world > 1:
        got = [None] * world
        dist.all_gather_object(got, rank)
        ranks = got
    if rank == 0:
        print(json.dumps({"n_gpus": world, "ranks": ranks, "backend": backend, "device": dev}))
    if world > 1:
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------ GPU arm
def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    args = parse_args(argv)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and args.impl != "reference":
        return relaunch(args, argv)
    if args.launch_check:
        return launch_check(args)
    if args.impl == "reference":
        return run_reference(args)
    import torch
    import torch.distributed as dist
    from block_sparse_attention_sbsa_b200 import sbsa
    from block_sparse_attention_sbsa_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))

    heads = args.shard == "heads" and world > 1
    exchange = None
    if heads:
        # every rank draws the same sequence and keeps its kv heads
        w_full = pick_workload(args)
        if w_full.gate_quantile is not None:
            # the percentile gate averages a tile's margins over every head:
            # one all-reduce of the per-tile sums between its two halves
            exchange = lambda t: dist.all_reduce(t)
        w, (g0, g1) = shard_workload(w_full, rank, world)
        data = shard_tensors(W.generate(w_full, "cuda"), w_full, g0, g1)
    else:
        w_full = w = rank_workload(pick_workload(args), rank)
        data = W.generate(w, "cuda")
    p = sbsa.params_for(w)
    st = sbsa.Staged(p)
    q, k, v = data["q"], data["k"], data["v"]
    qs = data["q_idx"] if w.index_dim else q
    ks = data["k_idx"] if w.index_dim else k
    o = torch.empty_like(q)
    stream = torch.cuda.current_stream()

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        st.pool(qs, ks)
        if evs:
            evs[1].record(stream)
        st.select(exchange=exchange, total_heads=w_full.n_sel_heads)
        if evs:
            evs[2].record(stream)
        st.attend(q, k, v, o)
        if evs:
            evs[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    stat = sbsa.get_status()
    if stat != sbsa.OK:
        raise RuntimeError(f"device status after warm-up: {sbsa.status_string(stat)}")
    pairs = sbsa.attended_pairs(p, st.cnt)
    attend_flops = 4.0 * w.head_dim * pairs
    mean_cnt = float(st.cnt.float().mean())
    valid_entries = int(st.cnt.to(torch.int64).sum())
    # planted needles are indexed by the full problem's kv heads
    sel_stats = selection_stats(w, p, st, {} if heads else data.get("meta", {}))

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start.record(stream)
    for s in range(args.steps):
        step(evs[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    pool_t = [e[0].elapsed_time(e[1]) for e in evs]
    sel_t = [e[1].elapsed_time(e[2]) for e in evs]
    att_t = [e[2].elapsed_time(e[3]) for e in evs]
    step_t = [e[0].elapsed_time(e[3]) for e in evs]
    pool_ms, sel_ms, att_ms = (statistics.mean(x) for x in (pool_t, sel_t, att_t))
    stat = sbsa.get_status()
    if stat != sbsa.OK:
        raise RuntimeError(f"device status after timing: {sbsa.status_string(stat)}")

    # ---- end to end through the C ABI with host buffers ----
    # Every request is one sbsa_prefill_host call on pinned host tensors: the
    # library copies each chunk of kv heads in, prefills it and copies its O
    # out, the three overlapped across chunks.  Two requests are in flight:
    # they alternate between two streams (each with its own workspace and
    # output buffer), so one request's input copies follow the other's
    # without waiting for its output copies; the host -> device link stays busy.
    pin = {name: t.cpu().pin_memory() for name, t in
           (("q", q), ("k", k), ("v", v), ("q_idx", data["q_idx"]), ("k_idx", data["k_idx"]))
           if t is not None}
    o_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
    host_calls = [sbsa.PrefillHost(p) for _ in range(2)]
    streams = [stream, torch.cuda.Stream()]
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = o_host[0].numel() * o_host[0].element_size()

    def request(r):
        host_calls[r % 2](pin["q"], pin["k"], pin["v"], o_host[r % 2], pin.get("q_idx"),
                          pin.get("k_idx"), stream=streams[r % 2])
    request(0)
    request(1)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(streams[0])
    streams[1].wait_event(e0)
    for r in range(args.e2e_steps):
        request(r)
    streams[0].wait_stream(streams[1])
    e1.record(streams[0])
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    stat = sbsa.get_status()
    if stat != sbsa.OK:
        raise RuntimeError(f"device status after e2e: {sbsa.status_string(stat)}")
    e2e_ok = all(torch.equal(oh.to(o.device), o) for oh in o_host)

    # ---- max over ranks ----
    elapsed_ms, e2e_ms, att_ms, pool_ms, sel_ms = reduce_max(
        [elapsed_ms, e2e_ms, att_ms, pool_ms, sel_ms], device="cuda")
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    peaks, src = load_peaks()
    value = weak_throughput(w.seq_len, 1 if heads else world, args.steps, elapsed_ms)
    ms_per_step = elapsed_ms / args.steps
    att_tflops = attend_flops / (att_ms / 1000.0) / 1e12
    peak_tf = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_bw = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    # algorithmic bytes of pooling + selection: read Q and K (or the index
    # tensors) once, write the fp32 tables and read them back, write the valid
    # list entries, the counts and the flags; the -1 padding of the fixed-width
    # lists is reported beside it
    es = q.element_size()
    nb, hs, ds = w.n_blocks, w.n_sel_heads, w.score_dim
    tables = 4 * (hs * nb * ds + w.n_kv_heads * nb * ds + (w.n_kv_heads * nb if w.rescue_tau else 0))
    lists = 4 * valid_entries + hs * nb * (4 + 1)
    padding = 4 * (hs * nb * w.max_blocks - valid_entries)
    sel_bytes = (qs.numel() + ks.numel()) * es + 2 * tables + lists
    sel_gbs = sel_bytes / ((pool_ms + sel_ms) / 1000.0) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong" if heads else "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "fp32",
        "data": "synthetic (seeded generator, RBS-style clustered keys with outliers)",
        "config": workload_config(w_full, world, heads),
        "attended_tflops": att_tflops,
        "roofline": {
            "bound": "tensor", "achieved": att_tflops, "peak": peak_tf, "unit": "TFLOP/s",
            "frac": att_tflops / peak_tf,
            "traffic": measured_traffic(w),
            "kernel": attend_kernel_name(w),
            "note": (f"peak = bf16_tflops burst, of {src}; achieved = 4*d*unmasked pairs / mean "
                     f"launch time (CUDA events on the launching stream); traffic = ncu "
                     f"dram bytes of one launch on the current kernel source, else null"),
        },
        "selection_roofline": {
            "bound": "hbm", "achieved": sel_gbs, "peak": peak_bw, "unit": "GB/s",
            "frac": sel_gbs / peak_bw, "bytes": sel_bytes, "list_padding_bytes": padding,
            "note": (f"pool + select kernels; bytes count valid list entries only (the -1 "
                     f"padding is list_padding_bytes); peak = hbm_gbs copy, of {src}"),
        },
        "stages_ms": {"pool": pool_ms, "select": sel_ms, "attend": att_ms},
        "stages_ms_spread": {"pool": spread(pool_t), "select": spread(sel_t),
                             "attend": spread(att_t), "step": spread(step_t)},
        "selected_blocks_per_row": mean_cnt,
        "selection_stats": sel_stats,
        "attend_bytes": {
            "algorithmic": sel_stats["attend_algorithmic_bytes"],
            "gbs": sel_stats["attend_algorithmic_bytes"] / (att_ms / 1000.0) / 1e9,
            "note": "Q + O + every distinct (kv head, block) of K and V a list names, once each; "
                    "far below the HBM peak: attention is not bound by DRAM",
        },
        "attended_pairs": pairs,
        "gpu_launches": launches_per_step(w) * args.steps,
        "clocks": clk,
        "e2e": {"value": weak_throughput(w.seq_len, world, args.e2e_steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": ("per request one sbsa_prefill_host call on pinned host tensors: "
                         "host -> device copies, prefill and device -> host copy of O, "
                         "pipelined over chunks of kv heads inside the call; two requests "
                         "in flight on two streams"),
                "output_matches_device_run": e2e_ok},
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"], line["parity"] = cpu_baseline_and_parity(
            w, data, args.cpu_blocks, st.idx, st.cnt, o)
    print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
