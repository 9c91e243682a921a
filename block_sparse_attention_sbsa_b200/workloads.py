"""Seeded synthetic workloads for block-sparse attention prefill.

This module only draws random tensors with the shapes, distributions and
planted structure of the workloads; it holds none of the method's arithmetic
(no pooling, scoring, selection or attention).  Both the CUDA path and the
CPU oracle consume the tensors it returns, so it is the one piece of code
they share.

Five workload families, one per configuration of the benchmark suite:

* ``tiny``    1 head, N=1024, d=64, B=64, fp32, top-4.  Q, K, V ~ N(0,1); one
              key row of block 5 is replaced by 4*q_dir and the queries of
              block 12 get +q_dir (a needle the selection should find).
* ``gqa32k``  32/8 heads, d=128, N=32768, B=128, bf16, top-16 per query head.
              K = N(0,1) + m[g, block], m ~ N(0, 0.5^2) per (kv head, block).
* ``rbs128k`` 32/8 heads, d=128, N=131072, B=128, bf16, cumulative mass 0.9
              united with the radius rescue branch (tau = 60).  Clustered keys
              (block mean mu ~ N(0, I), rows mu + 0.25*eps), 8 outlier keys of
              per-coordinate scale 6 per kv head, queries biased towards the
              means of 4 seeded past blocks.
* ``gate64k`` 32/8 heads, d=128, N=65536, B=64, bf16, top-8 with the gap
              gate (margin 0.05).  Block means are designed along orthonormal
              directions so that about 30% of query blocks have a tied pair of
              key blocks at ranks 8/9 (see ``_gen_gate``).
* ``msa512k`` 64/8 heads, d=128, N=524288, B=128, bf16, top-32 shared per GQA
              group on index tensors of width 64 (Q_idx = Q P, K_idx = K P for
              a seeded matrix P with orthonormal columns), 256 needles.
* ``quest32k`` 32/8 heads, d=128, N=32768, B=128, bf16, top-16 per query head
              scored by the K-min/K-max upper bound; the RBS recipe's clustered
              keys with outliers, whose blocks the bound is designed to catch.
* ``rowmax32k`` the GQA-32k recipe (32/8 heads, top-16 per query head) with
              the page's tile score: the largest q_t . c_j over the tile's
              query rows (a tensor-core contraction) instead of the pooled query.
* ``sigma64k`` the gate recipe at 64k (32/8 heads, B=64, top-8) with the
              page's own gate instead of the gap test: tiles whose head-averaged
              normalised cut margin is in the lowest 30% take the top 16.

The pages behind the method (RBS-Attention, "Uncertainty-gated selection for
block-sparse attention", MiniMax Sparse Attention) evaluate on long-context
suites with trained models; these tensors stand in for them.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    family: str
    n_q_heads: int
    n_kv_heads: int
    seq_len: int
    head_dim: int
    block_size: int
    dtype: str                      # "bf16" | "fp32"
    select_mode: str                # "topk" | "cummass"
    top_k: int = 0
    mass_threshold: float = 0.0
    rescue_tau: Optional[float] = None
    gate_margin: Optional[float] = None
    group_shared: bool = False
    index_dim: int = 0
    seed: int = 0
    backbone: str = "mean"          # "mean" (centroids) | "minmax" (K-min/K-max bound)
    gate_quantile: Optional[float] = None  # the page's percentile gate: q ...
    gate_rho: int = 2                      # ... and the expansion factor rho
    tile_score: str = "mean"               # "mean" (pooled query) | "rowmax" (max over rows)

    @property
    def n_blocks(self) -> int:
        return (self.seq_len + self.block_size - 1) // self.block_size

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def score_dim(self) -> int:
        return self.index_dim if self.index_dim else self.head_dim

    @property
    def n_sel_heads(self) -> int:
        return self.n_kv_heads if self.group_shared else self.n_q_heads

    @property
    def max_blocks(self) -> int:
        """Smallest list width that can hold every row's selection."""
        if self.select_mode == "cummass" or self.rescue_tau is not None:
            return self.n_blocks
        if self.gate_margin is not None:
            return min(2 * self.top_k, self.n_blocks - 1) + 1
        if self.gate_quantile is not None:
            return min(self.gate_rho * self.top_k, self.n_blocks - 1) + 1
        return min(self.top_k, self.n_blocks - 1) + 1

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": Workload("tiny", "tiny", 1, 1, 1024, 64, 64, "fp32", "topk",
                     top_k=4, seed=1001),
    "gqa32k": Workload("gqa32k", "gqa", 32, 8, 32768, 128, 128, "bf16", "topk",
                       top_k=16, seed=1002),
    "rbs128k": Workload("rbs128k", "rbs", 32, 8, 131072, 128, 128, "bf16",
                        "cummass", mass_threshold=0.9, rescue_tau=60.0,
                        seed=1003),
    "gate64k": Workload("gate64k", "gate", 32, 8, 65536, 128, 64, "bf16",
                        "topk", top_k=8, gate_margin=0.05, seed=1004),
    "msa512k": Workload("msa512k", "msa", 64, 8, 524288, 128, 128, "bf16",
                        "topk", top_k=32, group_shared=True, index_dim=64,
                        seed=1005),
    "quest32k": Workload("quest32k", "rbs", 32, 8, 32768, 128, 128, "bf16", "topk",
                         top_k=16, seed=1006, backbone="minmax"),
    "sigma64k": Workload("sigma64k", "gate", 32, 8, 65536, 128, 64, "bf16", "topk",
                         top_k=8, seed=1004, gate_quantile=0.3, gate_rho=2),
    "rowmax32k": Workload("rowmax32k", "gqa", 32, 8, 32768, 128, 128, "bf16", "topk",
                          top_k=16, seed=1002, tile_score="rowmax"),
}

# Reduced shapes of the same recipes, small enough for the CPU oracle to
# finish in seconds while still spanning several tiles (and, where the
# recipe allows it, a ragged last block).
SMALL = {
    "tiny": CONFIGS["tiny"],
    "gqa_small": CONFIGS["gqa32k"].scaled(name="gqa_small", n_q_heads=4,
                                          n_kv_heads=2, seq_len=4096 + 77,
                                          top_k=8),
    "rbs_small": CONFIGS["rbs128k"].scaled(name="rbs_small", n_q_heads=4,
                                           n_kv_heads=2, seq_len=8192 + 50),
    "gate_small": CONFIGS["gate64k"].scaled(name="gate_small", n_q_heads=4,
                                            n_kv_heads=2, seq_len=8192),
    "msa_small": CONFIGS["msa512k"].scaled(name="msa_small", n_q_heads=8,
                                           n_kv_heads=2, seq_len=8192 + 100,
                                           top_k=8),
    "quest_small": CONFIGS["quest32k"].scaled(name="quest_small", n_q_heads=4,
                                              n_kv_heads=2, seq_len=8192 + 50, top_k=8),
    "quest_gate_small": CONFIGS["quest32k"].scaled(name="quest_gate_small", n_q_heads=4,
                                                   n_kv_heads=2, seq_len=8192 + 50, top_k=8,
                                                   gate_margin=0.05),
    "sigma_small": CONFIGS["sigma64k"].scaled(name="sigma_small", n_q_heads=4, n_kv_heads=2,
                                              seq_len=8192),
    "rowmax_small": CONFIGS["rowmax32k"].scaled(name="rowmax_small", n_q_heads=4,
                                                n_kv_heads=2, seq_len=4096 + 77, top_k=8),
    "rowmax_msa_small": CONFIGS["msa512k"].scaled(name="rowmax_msa_small", n_q_heads=8,
                                                  n_kv_heads=2, seq_len=8192 + 100, top_k=8,
                                                  tile_score="rowmax"),
    "sigma_quest_small": CONFIGS["quest32k"].scaled(name="sigma_quest_small", n_q_heads=4,
                                                    n_kv_heads=2, seq_len=8192 + 50, top_k=8,
                                                    gate_quantile=0.5, gate_rho=3),
}

TORCH_DTYPE = {"bf16": torch.bfloat16, "fp32": torch.float32}

RUN = 16            # key blocks per designed run in the gate recipe
TIED_FRACTION = 0.3


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(gen, shape, device, scale=1.0):
    x = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x


def _orthonormal(gen, rows, cols, device):
    """Seeded matrix with orthonormal columns (QR of a Gaussian matrix)."""
    a = torch.randn(rows, cols, generator=gen, device=device, dtype=torch.float64)
    qm, r = torch.linalg.qr(a)
    # fix the sign convention so the result depends only on the draw
    qm = qm * torch.sign(torch.diagonal(r)).unsqueeze(0)
    return qm.to(torch.float32)


def _block_expand(per_block: torch.Tensor, seq_len: int, block: int):
    """[H, NB, d] -> [H, N, d] by repeating each block vector over its rows."""
    h, nb, d = per_block.shape
    full = per_block.repeat_interleave(block, dim=1)
    return full[:, :seq_len]


def generate(w: Workload, device="cpu") -> dict:
    """Draw the inputs of workload ``w`` on ``device``.

    Returns a dict with ``q`` [Hq, N, d], ``k`` and ``v`` [Hkv, N, d] in the
    workload dtype, ``q_idx``/``k_idx`` (index tensors, MSA family only, else
    None) and ``meta`` (planted structure the tests use as expectations).
    The stream of random numbers depends on the seed and on the device type.
    """
    fam = {"tiny": _gen_tiny, "gqa": _gen_gqa, "rbs": _gen_rbs,
           "gate": _gen_gate, "msa": _gen_msa}[w.family]
    with torch.no_grad():
        out = fam(w, device)
    out.setdefault("q_idx", None)
    out.setdefault("k_idx", None)
    out.setdefault("meta", {})
    return out


def _cast(x, w):
    return x.to(TORCH_DTYPE[w.dtype])


def _gen_tiny(w, device):
    g = _gen(w.seed, device)
    hq, hk, n, d, b = w.n_q_heads, w.n_kv_heads, w.seq_len, w.head_dim, w.block_size
    q = _randn(g, (hq, n, d), device)
    k = _randn(g, (hk, n, d), device)
    v = _randn(g, (hk, n, d), device)
    q_dir = _randn(g, (d,), device)
    needle_block, query_block = 5, 12
    r = int(torch.randint(0, b, (1,), generator=g, device=device).item())
    needle_row = needle_block * b + r
    k[:, needle_row] = 4.0 * q_dir
    q[:, query_block * b:(query_block + 1) * b] += q_dir
    return dict(q=_cast(q, w), k=_cast(k, w), v=_cast(v, w),
                meta=dict(needle_row=needle_row, needle_block=needle_block,
                          query_block=query_block))


def _gen_gqa(w, device):
    g = _gen(w.seed, device)
    hq, hk, n, d, b = w.n_q_heads, w.n_kv_heads, w.seq_len, w.head_dim, w.block_size
    nb = w.n_blocks
    dt = TORCH_DTYPE[w.dtype]
    m = _randn(g, (hk, nb, d), device, 0.5)
    k = torch.empty(hk, n, d, dtype=dt, device=device)
    for h in range(hk):
        kh = _randn(g, (1, n, d), device)
        kh += _block_expand(m[h:h + 1], n, b)
        k[h] = kh[0].to(dt)
    v = torch.empty(hk, n, d, dtype=dt, device=device)
    for h in range(hk):
        v[h] = _randn(g, (n, d), device).to(dt)
    q = torch.empty(hq, n, d, dtype=dt, device=device)
    for h in range(hq):
        q[h] = _randn(g, (n, d), device).to(dt)
    return dict(q=q, k=k, v=v, meta={})


def _gen_rbs(w, device, n_outliers_per_kv=8, n_targets=4):
    g = _gen(w.seed, device)
    hq, hk, n, d, b = w.n_q_heads, w.n_kv_heads, w.seq_len, w.head_dim, w.block_size
    nb, grp = w.n_blocks, w.group
    dt = TORCH_DTYPE[w.dtype]
    mu = _randn(g, (hk, nb, d), device)
    k = torch.empty(hk, n, d, dtype=dt, device=device)
    outliers = []
    for h in range(hk):
        kh = _randn(g, (1, n, d), device, 0.25)
        kh += _block_expand(mu[h:h + 1], n, b)
        pos = torch.randperm(n, generator=g, device=device)[:n_outliers_per_kv]
        z = _randn(g, (n_outliers_per_kv, d), device, 6.0)
        kh[0, pos] = z
        k[h] = kh[0].to(dt)
        outliers.extend((h, int(p)) for p in pos.tolist())
    v = torch.empty(hk, n, d, dtype=dt, device=device)
    for h in range(hk):
        v[h] = _randn(g, (n, d), device).to(dt)
    # per (q head, query block i >= 1): n_targets past blocks drawn uniformly
    # from [0, i) with replacement; their cluster means are added to every
    # query row of block i.
    i_idx = torch.arange(nb, device=device, dtype=torch.float64)
    u = torch.rand(hq, nb, n_targets, generator=g, device=device, dtype=torch.float64)
    targets = torch.floor(u * i_idx.view(1, nb, 1)).to(torch.int64)   # in [0, i)
    q = torch.empty(hq, n, d, dtype=dt, device=device)
    for h in range(hq):
        qh = _randn(g, (n, d), device)
        bias = mu[h // grp][targets[h]].sum(dim=1)      # [nb, d]
        bias[0] = 0.0                                   # block 0 has no past
        qh += bias.repeat_interleave(b, dim=0)[:n]
        q[h] = qh.to(dt)
    return dict(q=q, k=k, v=v,
                meta=dict(outliers=outliers, targets=targets.cpu()))


def _gen_gate(w, device):
    """Designed block means for the uncertainty gate.

    Per kv head g an orthonormal basis E_g of R^d is drawn.  Key block j
    belongs to run j // 16; the run's 16 blocks share the direction
    E_g[:, run] and carry the magnitudes 2, 4, ..., 32 in a seeded order.
    In a seeded ~30% of the runs (never run 0) the 9th-largest magnitude is
    raised to equal the 8th-largest and both blocks get an extra N(0, 0.01^2)
    per-coordinate offset: a near-tied pair exactly at the top-8 cut.
    Query block i of head h points along the direction of one run whose 16
    blocks all precede i (run 0 for i < 32); with probability 0.3 a tied run
    is chosen when one is available.  Key and query rows are the designed
    block vector plus antithetic N(0,1) noise (rows come in +eps/-eps pairs),
    so each block's mean equals its designed vector up to the dtype rounding.
    ``meta['tied_rows']`` marks the (q head, query block) rows that point at
    a tied run: these are the rows where the top-8 cut is ambiguous.
    """
    g = _gen(w.seed, device)
    hq, hk, n, d, b = w.n_q_heads, w.n_kv_heads, w.seq_len, w.head_dim, w.block_size
    nb, grp = w.n_blocks, w.group
    assert n % b == 0 and b % 2 == 0 and nb % RUN == 0
    n_runs = nb // RUN
    assert n_runs <= d, "one direction per run"
    dt = TORCH_DTYPE[w.dtype]
    mags_sorted = torch.arange(RUN, 0, -1, device=device, dtype=torch.float32) * 2.0
    k = torch.empty(hk, n, d, dtype=dt, device=device)
    bases, tied_runs = [], []
    for h in range(hk):
        E = _orthonormal(g, d, d, device)                     # columns e_r
        bases.append(E)
        tied = torch.rand(n_runs, generator=g, device=device) < TIED_FRACTION
        tied[0] = False
        tied_runs.append(tied)
        cent = torch.empty(nb, d, device=device)
        for r in range(n_runs):
            mags = mags_sorted.clone()
            if bool(tied[r]):
                mags[8] = mags[7]            # ranks 8 and 9 (1-based) tie
            perm = torch.randperm(RUN, generator=g, device=device)
            lam = mags[perm]
            cent[r * RUN:(r + 1) * RUN] = lam.view(RUN, 1) * E[:, r].view(1, d)
            if bool(tied[r]):
                # blocks of the run holding sorted ranks 8 and 9
                pos7 = int((perm == 7).nonzero()[0])
                pos8 = int((perm == 8).nonzero()[0])
                cent[r * RUN + pos7] += _randn(g, (d,), device, 0.01)
                cent[r * RUN + pos8] += _randn(g, (d,), device, 0.01)
        eps = _randn(g, (nb, b // 2, d), device)
        rows = torch.cat([cent.view(nb, 1, d) + eps, cent.view(nb, 1, d) - eps], dim=1)
        k[h] = rows.reshape(n, d).to(dt)
    v = torch.empty(hk, n, d, dtype=dt, device=device)
    for h in range(hk):
        v[h] = _randn(g, (n, d), device).to(dt)
    q = torch.empty(hq, n, d, dtype=dt, device=device)
    tied_rows = torch.zeros(hq, nb, dtype=torch.bool)
    chosen = torch.zeros(hq, nb, dtype=torch.int64)
    for h in range(hq):
        kv = h // grp
        tied = tied_runs[kv].cpu().tolist()
        tied_lists = [[x for x in range(a) if tied[x]] for a in range(n_runs + 1)]
        untied_lists = [[x for x in range(a) if not tied[x]] for a in range(n_runs + 1)]
        u_pick = torch.rand(nb, generator=g, device=device).cpu()
        u_run = torch.rand(nb, generator=g, device=device).cpu()
        for i in range(nb):
            avail = i // RUN                  # runs whose blocks all precede i
            if avail == 0:
                r = 0
            else:
                t_list = tied_lists[avail]
                u_list = untied_lists[avail]
                use_tied = bool(u_pick[i] < TIED_FRACTION) and len(t_list) > 0
                pool = t_list if use_tied else u_list
                r = pool[min(int(u_run[i] * len(pool)), len(pool) - 1)]
                tied_rows[h, i] = use_tied
            chosen[h, i] = r
        E = bases[kv]
        qbar = E[:, chosen[h].to(device)].T                  # [nb, d]
        eps = _randn(g, (nb, b // 2, d), device)
        rows = torch.cat([qbar.view(nb, 1, d) + eps, qbar.view(nb, 1, d) - eps], dim=1)
        q[h] = rows.reshape(n, d).to(dt)
    return dict(q=q, k=k, v=v,
                meta=dict(tied_rows=tied_rows, chosen_run=chosen,
                          tied_runs=torch.stack([t.cpu() for t in tied_runs])))


def _gen_msa(w, device, n_needles=256):
    g = _gen(w.seed, device)
    hq, hk, n, d, b = w.n_q_heads, w.n_kv_heads, w.seq_len, w.head_dim, w.block_size
    nb, grp, di = w.n_blocks, w.group, w.index_dim
    dt = TORCH_DTYPE[w.dtype]
    P = _orthonormal(g, d, di, device)                     # d x d_idx
    # needles: kv head, key position, later query block, direction
    nd_head = torch.randint(0, hk, (n_needles,), generator=g, device=device).cpu()
    nd_pos = torch.randint(0, max(1, (nb - 1) * b), (n_needles,), generator=g,
                           device=device).cpu()
    u = torch.rand(n_needles, generator=g, device=device, dtype=torch.float64).cpu()
    nd_blk = nd_pos // b
    nd_qblk = nd_blk + 1 + torch.floor(u * (nb - 1 - nd_blk).to(torch.float64)).to(torch.int64)
    nd_dir = _randn(g, (n_needles, d), device)
    k = torch.empty(hk, n, d, dtype=dt, device=device)
    k_idx = torch.empty(hk, n, di, dtype=dt, device=device)
    for h in range(hk):
        kh = _randn(g, (n, d), device)
        sel = (nd_head == h).nonzero().flatten()
        for s in sel.tolist():
            kh[int(nd_pos[s])] = 4.0 * nd_dir[s]
        k[h] = kh.to(dt)
        k_idx[h] = (kh @ P).to(dt)
    v = torch.empty(hk, n, d, dtype=dt, device=device)
    for h in range(hk):
        v[h] = _randn(g, (n, d), device).to(dt)
    q = torch.empty(hq, n, d, dtype=dt, device=device)
    q_idx = torch.empty(hq, n, di, dtype=dt, device=device)
    for h in range(hq):
        qh = _randn(g, (n, d), device)
        sel = (nd_head == h // grp).nonzero().flatten()
        for s in sel.tolist():
            i = int(nd_qblk[s])
            qh[i * b:min(n, (i + 1) * b)] += nd_dir[s]
        q[h] = qh.to(dt)
        q_idx[h] = (qh @ P).to(dt)
    needles = [(int(nd_head[s]), int(nd_pos[s]), int(nd_qblk[s])) for s in range(n_needles)]
    return dict(q=q, k=k, v=v, q_idx=q_idx, k_idx=k_idx,
                meta=dict(needles=needles))


def sample_query_blocks(w: Workload, meta: dict, count: int = 64) -> list:
    """Query blocks on which the full-size MSA workload is checked: the last
    block, up to half of ``count`` needle query blocks, the rest seeded."""
    nb = w.n_blocks
    picked = [nb - 1]
    for (_, _, qb) in meta.get("needles", []):
        if len(picked) >= 1 + count // 2:
            break
        if qb not in picked:
            picked.append(qb)
    g = _gen(w.seed + 7, "cpu")
    while len(picked) < count:
        i = int(torch.randint(0, nb, (1,), generator=g).item())
        if i not in picked:
            picked.append(i)
    return sorted(picked)
