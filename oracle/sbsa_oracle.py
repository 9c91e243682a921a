"""CPU oracle for block-sparse attention prefill.

TEST INFRASTRUCTURE ONLY.  This module is the slow, plain reference that the
CUDA path is checked against.  Only the test suite, the smoke check of the
package entry file and the CPU-baseline / reference legs of the benchmark may
import it; the library itself never does, and it never imports the library.

Everything is computed in float64 with numpy (matrix products and sorts are
library primitives used as single steps).  Where floating point decides an
integer -- which blocks are selected -- the decision is taken on scores
rounded to float32, the precision the kernels decide in.

Sources (web pages; cited by title and section):

* "RBS-Attention: un metodo de prefill disperso ..." (iaonda.com), the
  method paragraph: keys are grouped into blocks that are summarised by a
  centroid; a base branch keeps blocks by centroid relevance, a rescue branch
  keeps blocks at risk of being underestimated through a dynamic key-block
  radius; each branch has its own threshold and the two masks are united; the
  attention itself stays compatible with sparse FlashAttention.
* "Uncertainty-gated selection for block-sparse attention" (gist.science,
  paper 2607.07724), technical summary, Metodologia steps 1-5: mean-pooled
  block scores (SSA-style K-mean), selection per query tile, top-k block
  lists kv_idx, expansion of ambiguous tiles from k to rho*k (rho = 2) with
  sentinel padding; the lay explainer's 9.9 / 9.8 example of a near tie.
* "MiniMax presenta MSA ..." (iaonda.com), section "Que es MSA y como
  funciona?": one top-k block selection per GQA group by a light index
  branch, full attention over the selected blocks only.
* The uncertainty-gated page, Metodologia step 1 and Contribuciones
  (Componibilidad): the block-scoring backbone is interchangeable; besides
  SSA-style mean pooling it names Quest's per-coordinate upper bounds from
  the block's K-min / K-max.

Readings where the pages are silent (each one also listed in the design
notes): the radius is the largest l2 distance of a block's keys from its
centroid; the query side of a pair score is the mean of the query block's
rows (per head, or additionally averaged over the heads of a GQA group);
scores are scaled by 1/sqrt(d_s); ties rank the lower block id first; the
diagonal block is always kept and is not a candidate; the gate fires when
the k-th minus (k+1)-th largest score is below margin * (population std of
the row's candidate scores); cumulative mass uses a softmax over the
candidates and keeps the shortest prefix of the ranked order whose mass
reaches the threshold; the rescue test is (q.c + |q| r) * scale > tau.
The K-min/K-max backbone bounds q.k over the block's keys coordinate by
coordinate: sum_d max(q_d * min_d, q_d * max_d), scaled like the mean score.
Row-max tile scores (Metodologia step 2: the tile score is the largest
score among the tile's query rows): s_ij = max_t (q_t . c_j) * scale over
the rows t of query block i (and, in group mode, over the heads of the
group); the kernels take this contraction on bf16 tensor cores, so the
decision precision is theirs: centroids rounded to bf16, products exact,
the sum and the maximum in float64, the result rounded to float32.
The page's own gate (Metodologia steps 3-5): the normalised cut margin
sigma = (s_(k-1) - s_(k)) / (s_(0) - s_(k)) on the descending 0-based order
(0 when s_(0) = s_(k)), defined for rows with more than k candidates; its
mean over the selection heads gives one value per query tile; the floor(q T)
eligible tiles with the smallest mean (lower tile first on equal means; T
eligible tiles) fire -- the empirical percentile q of the layer -- and take
the top rho*k blocks in every head, the others the top k.
"""
from __future__ import annotations

import math

import numpy as np

FLAG_GATE = 1      # the uncertainty gate doubled this row's budget
FLAG_RESCUE = 2    # the rescue branch added a block the base branch missed


def n_blocks(seq_len: int, block: int) -> int:
    """Token t lies in block t // B; the last block may be partial."""
    return (seq_len + block - 1) // block


def block_rows(j: int, seq_len: int, block: int) -> range:
    return range(j * block, min(seq_len, (j + 1) * block))


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):            # torch tensor (any dtype, CPU)
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def _take(x, rows) -> np.ndarray:
    """Rows ``rows`` of a [N, d] array or CPU torch tensor, as float64."""
    if hasattr(x, "detach"):
        import torch
        return _f64(x[torch.as_tensor(np.asarray(rows, dtype=np.int64))])
    return _f64(np.asarray(x)[rows])


# --------------------------------------------------------------------------
# Pooling (RBS-Attention method paragraph: centroid and dynamic radius;
# Uncertainty-gated selection, Metodologia step 1: mean pooling of key blocks)
# --------------------------------------------------------------------------

def pool_keys(k, block: int, with_radius: bool = True, heads=None):
    """Centroid c[g, j] = mean of the keys of block j; radius r[g, j] = the
    largest l2 distance of those keys from c[g, j] (direct difference)."""
    k = k if heads is None else k[heads]
    hk, n, d = k.shape
    nb = n_blocks(n, block)
    c = np.zeros((hk, nb, d))
    r = np.zeros((hk, nb))
    for g in range(hk):
        kg = _f64(k[g])
        for j in range(nb):
            rows = kg[j * block:min(n, (j + 1) * block)]
            c[g, j] = rows.sum(axis=0) / rows.shape[0]
            if with_radius:
                r[g, j] = np.sqrt(((rows - c[g, j]) ** 2).sum(axis=1)).max()
    return c, (r if with_radius else None)


def pool_keys_minmax(k, block: int):
    """Per-coordinate minimum and maximum of the keys of each block (the
    K-min / K-max table of the upper-bound backbone).  Returns (kmin, kmax),
    each [Hkv, NB, d]."""
    hk, n, d = k.shape
    nb = n_blocks(n, block)
    kmin = np.zeros((hk, nb, d))
    kmax = np.zeros((hk, nb, d))
    for g in range(hk):
        kg = _f64(k[g])
        for j in range(nb):
            rows = kg[j * block:min(n, (j + 1) * block)]
            kmin[g, j] = rows.min(axis=0)
            kmax[g, j] = rows.max(axis=0)
    return kmin, kmax


def pool_queries(q, block: int, group: int = 1, blocks=None):
    """Pooled query of block i: the mean of the block's query rows (one query
    tile per block).  With ``group`` > 1 (one selection per GQA group), the
    per-head pooled queries of the group's heads are averaged as well.
    Returns [Hq / group, NB, d]; with ``blocks`` only those blocks are
    computed and the others stay zero."""
    hq, n, d = q.shape
    nb = n_blocks(n, block)
    blist = list(range(nb)) if blocks is None else list(blocks)
    out = np.zeros((hq // group, nb, d))
    for hs in range(hq // group):
        for i in blist:
            acc = np.zeros(d)
            for h in range(hs * group, (hs + 1) * group):
                rows = _f64(q[h, i * block:min(n, (i + 1) * block)])
                acc += rows.sum(axis=0) / rows.shape[0]
            out[hs, i] = acc / group
    return out


# --------------------------------------------------------------------------
# Scoring (Uncertainty-gated selection, Metodologia step 1; RBS base branch)
# --------------------------------------------------------------------------

def block_scores(qbar_i, c_g, i: int, scale: float):
    """s_j = (qbar_i . c_j) * scale for the candidate blocks j < i, rounded to
    float32 (the precision the selection decision is taken in)."""
    s = (c_g[:i] @ qbar_i) * scale
    return s.astype(np.float32)


def block_bounds_minmax(qbar_i, kmin_g, kmax_g, i: int, scale: float):
    """Upper-bound backbone: s_j = sum_d max(qbar_d * min_jd, qbar_d * max_jd)
    * scale for the candidates j < i -- the largest q.k over any key inside
    the block's coordinate box -- rounded to float32."""
    lo = kmin_g[:i] * qbar_i
    hi = kmax_g[:i] * qbar_i
    return (np.maximum(lo, hi).sum(axis=1) * scale).astype(np.float32)


def block_scores_rowmax(q_rows, c_g, i: int, scale: float):
    """Tile score of query block i against candidates j < i: the largest
    q_t . c_j over the tile's query rows t (all rows given, e.g. the rows of
    every head of a group), times scale, in float64 from the centroids as
    given, rounded to float32 once at the end (the precision the selection
    decision is taken in).  The page defines the tile score as the largest
    row score; nothing in it rounds the operands."""
    q = _f64(q_rows)
    c = _f64(c_g[:i])
    if i == 0:
        return np.zeros(0, dtype=np.float32)
    return ((q @ c.T).max(axis=0) * scale).astype(np.float32)


def rescue_bounds(qbar_i, c_g, r_g, i: int, scale: float):
    """Upper bound of q.k over block j when k lies within r_j of c_j
    (Cauchy-Schwarz): (qbar . c_j + |qbar| r_j) * scale, rounded to float32."""
    ub = (c_g[:i] @ qbar_i + np.linalg.norm(qbar_i) * r_g[:i]) * scale
    return ub.astype(np.float32)


# --------------------------------------------------------------------------
# Selection (Uncertainty-gated selection steps 2-5; RBS two branches + union)
# --------------------------------------------------------------------------

def ranked(s) -> np.ndarray:
    """Candidate ids ordered by score descending, lower id first on ties."""
    s = np.asarray(s, dtype=np.float64)
    ids = np.arange(len(s))
    return np.lexsort((ids, -s))


def top_k(s, k: int) -> np.ndarray:
    """The min(k, |C|) best-ranked candidates."""
    return np.sort(ranked(s)[:min(k, len(s))])


def gate(s, k: int, margin: float):
    """Gap test of the uncertainty gate: with s_(m) the m-th largest score
    (1-based), fire when s_(k) - s_(k+1) < margin * std(s) (population std
    over all candidates).  Only defined when there are more than k
    candidates.  Returns (fired, gap, threshold)."""
    s64 = np.asarray(s, dtype=np.float64)
    if len(s64) <= k:
        return False, math.inf, 0.0
    order = ranked(s64)
    gap = s64[order[k - 1]] - s64[order[k]]
    thr = margin * s64.std()
    return bool(gap < thr), float(gap), float(thr)


def cut_margin(s, k: int) -> float:
    """Normalised cut margin of a row with more than k candidates:
    (s_(k-1) - s_(k)) / (s_(0) - s_(k)) with s_(m) the m-th largest (0-based),
    in float64 from the row's (float32) scores; 0 when s_(0) = s_(k)."""
    s64 = np.asarray(s, dtype=np.float64)
    if len(s64) <= k:
        raise ValueError("cut margin needs more than k candidates")
    order = ranked(s64)
    top, last, first_out = s64[order[0]], s64[order[k - 1]], s64[order[k]]
    if top == first_out:
        return 0.0
    return float((last - first_out) / (top - first_out))


def percentile_fire(sbar: dict, q: float) -> set:
    """Tiles that fire: the floor(q T) tiles with the smallest head-averaged
    margin among the T eligible ones (lower tile index first on ties)."""
    order = sorted(sbar, key=lambda i: (sbar[i], i))
    return set(order[:int(math.floor(q * len(order)))])


def cumulative_mass(s, mass: float):
    """Base branch with its own threshold: p = softmax over the candidates;
    keep the shortest prefix of the ranked order whose mass reaches ``mass``.
    Returns (kept ids ascending, cumulative masses along the ranked order)."""
    s64 = np.asarray(s, dtype=np.float64)
    if len(s64) == 0:
        return np.zeros(0, dtype=np.int64), np.zeros(0)
    p = np.exp(s64 - s64.max())
    p /= p.sum()
    order = ranked(s64)
    cum = np.cumsum(p[order])
    reach = np.nonzero(cum >= mass)[0]
    m = (reach[0] + 1) if len(reach) else len(order)
    return np.sort(order[:m]), cum


def select_row(s, i: int, *, mode: str, top_k_: int = 0, mass: float = 0.0,
               margin=None, ub=None, tau=None, budget=None):
    """Block list of query block i: base branch (top-k, gated top-k or
    cumulative mass), united with the rescue branch, plus the diagonal block
    i, ascending.  ``budget`` overrides k (the percentile gate's rho*k for a
    fired tile).  Returns (ids, flags)."""
    flags = 0
    n = i
    if mode == "topk" and budget is not None:
        base = set(top_k(s, budget).tolist())
        if budget > top_k_:
            flags |= FLAG_GATE
    elif mode == "topk":
        kk = top_k_
        if margin is not None and n > top_k_:
            fired, _, _ = gate(s, top_k_, margin)
            if fired:
                kk = 2 * top_k_
                flags |= FLAG_GATE
        base = set(top_k(s, kk).tolist())
    elif mode == "cummass":
        base = set(cumulative_mass(s, mass)[0].tolist())
    else:
        raise ValueError(mode)
    sel = set(base)
    if tau is not None:
        rescue = set(np.nonzero(np.asarray(ub, dtype=np.float64) > tau)[0].tolist())
        if rescue - base:
            flags |= FLAG_RESCUE
        sel |= rescue
    sel.add(i)
    return np.array(sorted(sel), dtype=np.int64), flags


def select(qbar, c, r, *, block_count: int, mode: str, top_k_: int = 0,
           mass: float = 0.0, margin=None, tau=None, scale: float,
           kv_of_sel=None, max_blocks: int, rows=None, minmax=None, sigma_gate=None,
           info=None, row_scores=None, fired=None):
    """Lists for every selection head hs and query block i (or the (hs, i)
    pairs in ``rows``).  ``qbar`` is [Hs, NB, d_s] and ``c``/``r`` are the key
    tables [Hkv, NB, ...]; ``kv_of_sel(hs)`` gives the kv head whose key table
    a selection head scores against.  Returns idx [Hs, NB, Kmax] (-1 padded),
    cnt [Hs, NB] and flags [Hs, NB]."""
    hs_n = qbar.shape[0]
    nb = block_count
    idx = np.full((hs_n, nb, max_blocks), -1, dtype=np.int32)
    cnt = np.zeros((hs_n, nb), dtype=np.int32)
    flags = np.zeros((hs_n, nb), dtype=np.uint8)
    pairs = rows if rows is not None else [(h, i) for h in range(hs_n) for i in range(nb)]

    def scores(h, i):
        g = kv_of_sel(h)
        if row_scores is not None:
            return row_scores(h, i)
        if minmax is None:
            return block_scores(qbar[h, i], c[g], i, scale)
        return block_bounds_minmax(qbar[h, i], minmax[0][g], minmax[1][g], i, scale)

    given_fired = fired is not None
    fired = set(fired) if given_fired else set()  # the gate's tiles, when decided earlier
    if sigma_gate is not None and not given_fired:
        if mode != "topk" or margin is not None:
            raise ValueError("the percentile gate applies to plain top-k")
        q, rho = sigma_gate
        sbar = {}
        for i in range(top_k_ + 1, nb):          # tiles with more than k candidates
            tot = 0.0
            for h in range(hs_n):                 # head order, one sum
                tot += cut_margin(scores(h, i), top_k_)
            sbar[i] = tot / hs_n
        fired = percentile_fire(sbar, q)
        if info is not None:
            info["sbar"], info["fired"] = sbar, fired
    for (h, i) in pairs:
        g = kv_of_sel(h)
        s = scores(h, i)
        ub = rescue_bounds(qbar[h, i], c[g], r[g], i, scale) if tau is not None else None
        budget = sigma_gate[1] * top_k_ if i in fired else None
        ids, fl = select_row(s, i, mode=mode, top_k_=top_k_, mass=mass,
                             margin=margin, ub=ub, tau=tau, budget=budget)
        if len(ids) > max_blocks:
            raise ValueError("selection wider than max_blocks")
        idx[h, i, :len(ids)] = ids
        cnt[h, i] = len(ids)
        flags[h, i] = fl
    return idx, cnt, flags


# --------------------------------------------------------------------------
# Attention over the selected blocks (RBS: sparse FlashAttention-compatible
# prefill; MSA: full attention over the preselected blocks)
# --------------------------------------------------------------------------

def attend_block(q_rows, k, v, blocks, i: int, block: int, scale: float):
    """Output rows of query block i for one head: for each query t, softmax
    over the keys u of the listed blocks with u <= t of (q_t . k_u) * scale,
    weighting v_u.  Rows that see no key return zeros.  q_rows holds the
    query rows of block i, k and v are [N, d] of the head's kv head."""
    n = k.shape[0]
    t_rows = np.arange(i * block, min(n, (i + 1) * block))
    u = np.concatenate([np.arange(j * block, min(n, (j + 1) * block))
                        for j in blocks]) if len(blocks) else np.zeros(0, np.int64)
    qt = _f64(q_rows)
    out = np.zeros((len(t_rows), v.shape[1]))
    if len(u) == 0:
        return out
    ku = _take(k, u)
    vu = _take(v, u)
    logits = (qt @ ku.T) * scale
    visible = u[None, :] <= t_rows[:, None]
    logits = np.where(visible, logits, -np.inf)
    seen = visible.any(axis=1)
    if not seen.any():
        return out
    rows = np.nonzero(seen)[0]
    z = logits[rows] - logits[rows].max(axis=1, keepdims=True)
    p = np.exp(z)                              # exp(-inf) = 0 off the mask
    p /= p.sum(axis=1, keepdims=True)
    out[rows] = p @ vu
    return out


def attend(q, k, v, idx, cnt, *, block: int, scale: float, group_shared: bool,
           rows=None):
    """O[h, t] for every query head h and token t (or only the (h, i) query
    blocks in ``rows``; other rows stay zero).  Query head h reads kv head
    h // G; its list is idx[h] (per head) or idx[h // G] (group shared)."""
    hq, n, d = q.shape
    hk = k.shape[0]
    grp = hq // hk
    nb = n_blocks(n, block)
    out = np.zeros((hq, n, v.shape[2]))
    pairs = rows if rows is not None else [(h, i) for h in range(hq) for i in range(nb)]
    for (h, i) in pairs:
        g = h // grp
        hs = g if group_shared else h
        blocks = [int(x) for x in idx[hs, i, :cnt[hs, i]]]
        lo, hi = i * block, min(n, (i + 1) * block)
        out[h, lo:hi] = attend_block(q[h, lo:hi], k[g], v[g], blocks, i, block, scale)
    return out


def attend_dense_masked(q, k, v, idx, cnt, *, block: int, scale: float,
                        group_shared: bool):
    """The same output written as dense masked attention: softmax over all N
    keys of (q_t . k_u) * scale with -inf wherever u > t or block(u) is not
    in the list of (h, block(t)).  Only for small N."""
    hq, n, d = q.shape
    hk = k.shape[0]
    grp = hq // hk
    out = np.zeros((hq, n, v.shape[2]))
    for h in range(hq):
        g = h // grp
        hs = g if group_shared else h
        qh, kh, vh = _f64(q[h]), _f64(k[g]), _f64(v[g])
        logits = (qh @ kh.T) * scale
        mask = np.zeros((n, n), dtype=bool)
        for t in range(n):
            allowed = set(int(x) for x in idx[hs, t // block, :cnt[hs, t // block]])
            for uu in range(t + 1):
                mask[t, uu] = (uu // block) in allowed
        logits = np.where(mask, logits, -np.inf)
        for t in range(n):
            if mask[t].any():
                z = logits[t] - logits[t][mask[t]].max()
                p = np.exp(z)
                out[h, t] = (p / p.sum()) @ vh
    return out


# --------------------------------------------------------------------------
# The whole prefill: pool -> score/select -> attend
# --------------------------------------------------------------------------

def prefill(q, k, v, *, block: int, mode: str, top_k_: int = 0,
            mass: float = 0.0, margin=None, tau=None, group_shared: bool = False,
            q_idx=None, k_idx=None, max_blocks: int, scale=None,
            score_scale=None, sel_rows=None, attend_rows=None, backbone: str = "mean",
            sigma_gate=None, tile_score: str = "mean"):
    """Selection tables and lists from the index tensors (q_idx/k_idx when
    given, else q/k), then attention over the lists.  ``sel_rows`` restricts
    selection to (hs, i) pairs, ``attend_rows`` restricts attention to
    (h, i) query blocks (for large workloads)."""
    hq, n, d = q.shape
    hk = k.shape[0]
    grp = hq // hk
    qs = q if q_idx is None else q_idx
    ks = k if k_idx is None else k_idx
    d_s = qs.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    score_scale = 1.0 / math.sqrt(d_s) if score_scale is None else score_scale
    nb = n_blocks(n, block)
    c, r = pool_keys(ks, block, with_radius=tau is not None)
    if r is None:
        r = np.zeros(c.shape[:2])
    if backbone == "minmax":
        if tau is not None:
            raise ValueError("the rescue branch needs the mean backbone")
        minmax = pool_keys_minmax(ks, block)
    elif backbone == "mean":
        minmax = None
    else:
        raise ValueError(backbone)
    if group_shared:
        qbar = pool_queries(qs, block, group=grp)
        kv_of_sel = lambda hs: hs
    else:
        qbar = pool_queries(qs, block, group=1)
        kv_of_sel = lambda hs: hs // grp
    row_scores = None
    if tile_score == "rowmax":
        if backbone != "mean" or tau is not None:
            raise ValueError("row-max tile scores use the centroids, without the rescue branch")

        def row_scores(h, i):
            heads = range(h * grp, (h + 1) * grp) if group_shared else [h]
            rows = np.concatenate([_f64(qs[hh, i * block:min(n, (i + 1) * block)])
                                   for hh in heads])
            return block_scores_rowmax(rows, c[h if group_shared else h // grp], i,
                                       score_scale)
    elif tile_score != "mean":
        raise ValueError(tile_score)
    info = {}
    idx, cnt, flags = select(qbar, c, r, block_count=nb, mode=mode, top_k_=top_k_,
                             mass=mass, margin=margin, tau=tau, scale=score_scale,
                             kv_of_sel=kv_of_sel, max_blocks=max_blocks,
                             rows=sel_rows, minmax=minmax, sigma_gate=sigma_gate, info=info,
                             row_scores=row_scores)
    out = attend(q, k, v, idx, cnt, block=block, scale=scale,
                 group_shared=group_shared, rows=attend_rows)
    return dict(c=c, r=r, qbar=qbar, idx=idx, cnt=cnt, flags=flags, o=out,
                minmax=minmax, sbar=info.get("sbar"), fired=info.get("fired"))
