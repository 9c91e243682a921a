"""Comparison helpers for GPU-vs-oracle parity.

Block lists must match the oracle exactly, except where a selection decision
lies inside the fp32 tie band: a block whose decision quantity (its score
against the k-th score, the cumulative mass against the threshold, its rescue
bound against tau, the gate gap against margin*std) is within
1e-5 * max(1, |value|) of the cut may be decided either way.  Such rows are
counted and reported; any other difference fails.
"""
from __future__ import annotations

import math

import numpy as np

import oracle as O

BAND = 1e-5
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
# A tile's head-averaged cut margin is a ratio of score differences; one fp32
# ulp in a score near a tie moves it by far more than the score band, so the
# percentile gate's decision is free within this absolute band of the cut.
SIGMA_BAND = 1e-4


def percentile_budgets(sbar: dict, fired: set, k: int, rho: int) -> dict:
    """Budgets each tile may take under the percentile gate: rho*k when it
    fired, k when it did not, either when its mean margin lies within
    SIGMA_BAND of the cut between the last fired and the first kept tile."""
    order = sorted(sbar, key=lambda i: (sbar[i], i))
    n_fire = len(fired)
    lo = sbar[order[n_fire - 1]] if n_fire > 0 else -math.inf
    hi = sbar[order[n_fire]] if n_fire < len(order) else math.inf
    out = {}
    for i, v in sbar.items():
        b = {rho * k} if i in fired else {k}
        if abs(v - lo) <= SIGMA_BAND or abs(v - hi) <= SIGMA_BAND:
            b = {k, rho * k}
        out[i] = b
    return out


# Counts each parity test reports (printed in the session summary, see
# conftest.py): exact and tie-band rows, tiles inside SIGMA_BAND, output errors.
REPORT: list = []


def record(test: str, workload: str, **counts) -> None:
    REPORT.append(dict(test=test, workload=workload, **counts))


def sigma_band_tiles(budgets) -> int:
    """Tiles whose percentile-gate decision lies inside SIGMA_BAND of the cut
    (either budget accepted)."""
    return 0 if budgets is None else sum(1 for b in budgets.values() if len(b) > 1)


def band(x: float) -> float:
    return BAND * max(1.0, abs(x))


def near(a: float, b: float) -> bool:
    return abs(a - b) <= band(max(abs(a), abs(b)))


def _base_alternatives(s, i, w, budgets_i=None):
    """Base-branch sets the oracle's decisions allow within the tie band,
    as (must_have, may_have, sizes) triples."""
    s64 = np.asarray(s, dtype=np.float64)
    n = len(s64)
    order = O.ranked(s64)
    alts = []
    if w.select_mode == "topk":
        budgets = [w.top_k]
        if budgets_i is not None:
            budgets = sorted(budgets_i)
        elif w.gate_margin is not None and n > w.top_k:
            fired, gap, thr = O.gate(s, w.top_k, w.gate_margin)
            if abs(gap - thr) <= band(thr):
                budgets = [w.top_k, 2 * w.top_k]
            elif fired:
                budgets = [2 * w.top_k]
        for kk in budgets:
            if n <= kk:
                alts.append((set(range(n)), set(), {n}))
                continue
            cut = s64[order[kk - 1]]
            must = {j for j in range(n) if s64[j] > cut + band(cut)}
            may = {j for j in range(n) if abs(s64[j] - cut) <= band(cut)}
            alts.append((must, may, {kk}))
    else:
        kept, cum = O.cumulative_mass(s, w.mass_threshold)
        m = len(kept)
        if n == 0:
            return [(set(), set(), {0})]
        sizes = {m}
        # the mass boundary may move by one block either way
        if m >= 2 and abs(cum[m - 2] - w.mass_threshold) <= band(w.mass_threshold):
            sizes.add(m - 1)
        if abs(cum[m - 1] - w.mass_threshold) <= band(w.mass_threshold) and m < n:
            sizes.add(m + 1)
        for size in sizes:
            cut = s64[order[size - 1]]
            must = {j for j in range(n) if s64[j] > cut + band(cut)}
            may = {j for j in range(n) if abs(s64[j] - cut) <= band(cut)}
            alts.append((must, may, {size}))
    return alts


def row_matches(gpu_ids, s, ub, i, w, budgets_i=None):
    """True when the GPU list of query block i is allowed by the oracle's
    decisions (exact or within the tie band)."""
    g = set(int(x) for x in gpu_ids)
    if i not in g or any(x > i or x < 0 for x in g):
        return False
    body = g - {i}
    n = i
    rescue_must, rescue_may = set(), set()
    if w.rescue_tau is not None:
        ub64 = np.asarray(ub, dtype=np.float64)
        for j in range(n):
            if abs(ub64[j] - w.rescue_tau) <= band(w.rescue_tau):
                rescue_may.add(j)
            elif ub64[j] > w.rescue_tau:
                rescue_must.add(j)
    # body = B | R with must <= B <= must | may (|B| one of sizes) and
    # rescue_must <= R <= rescue_must | rescue_may
    if not rescue_must <= body:
        return False
    r_range = rescue_must | rescue_may
    x = body - r_range                      # blocks only the base branch can explain
    for must, may, sizes in _base_alternatives(s, i, w, budgets_i):
        if not must <= body or not x <= (must | may):
            continue
        lo = len(must | x)
        hi = len((must | may) & body)
        if any(lo <= sz <= hi for sz in sizes):
            return True
    return False


def compare_lists(gpu_idx, gpu_cnt, oracle_idx, oracle_cnt, rows, qbar, c, r, w, kv_of_sel,
                  minmax=None, budgets=None, score_fn=None):
    """Returns (exact, tie) counts over ``rows``; raises AssertionError on a
    difference the tie band does not explain.  ``minmax`` = (kmin, kmax)
    selects the upper-bound backbone's scores instead of the centroids';
    ``budgets`` (tile -> allowed top-k budgets) carries the percentile gate's
    decisions; ``score_fn(hs, i)`` gives the oracle's scores of a row
    directly (row-max tile scores)."""
    exact = tie = 0
    scale = 1.0 / math.sqrt(w.score_dim)
    for (hs, i) in rows:
        gi = gpu_idx[hs, i, :gpu_cnt[hs, i]].tolist()
        oi = oracle_idx[hs, i, :oracle_cnt[hs, i]].tolist()
        if gi == oi:
            exact += 1
            continue
        g = kv_of_sel(hs)
        if score_fn is not None:
            s = score_fn(hs, i)
        elif minmax is None:
            s = O.block_scores(qbar[hs, i], c[g], i, scale)
        else:
            s = O.block_bounds_minmax(qbar[hs, i], minmax[0][g], minmax[1][g], i, scale)
        ub = O.rescue_bounds(qbar[hs, i], c[g], r[g], i, scale) if w.rescue_tau is not None else None
        if not row_matches(gi, s, ub, i, w, None if budgets is None else budgets.get(i)):
            raise AssertionError(f"row (head {hs}, block {i}): gpu {gi} vs oracle {oi}")
        tie += 1
    return exact, tie


def output_errors(gpu_o, oracle_o):
    d = np.abs(np.asarray(gpu_o, dtype=np.float64) - np.asarray(oracle_o, dtype=np.float64))
    return float(d.max()) if d.size else 0.0, float(d.mean()) if d.size else 0.0
