"""Pins of the CPU oracle against facts fixed outside of it.

Each test checks the oracle against something other than its own formulas:
a library routine (torch's causal SDPA, scipy's softmax, statistics.pstdev),
a closed form, brute force on tiny inputs, an invariant of the definitions,
the pages' own worked example, or structure the workload generator planted.
"""
import json
import math
import os
import statistics
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy.special import softmax as scipy_softmax

import oracle as O
from block_sparse_attention_sbsa_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(12345)


def _all_lists(hs, nb):
    """Lists that hold every causal block: i -> [0..i]."""
    idx = np.full((hs, nb, nb), -1, dtype=np.int32)
    cnt = np.zeros((hs, nb), dtype=np.int32)
    for h in range(hs):
        for i in range(nb):
            idx[h, i, :i + 1] = np.arange(i + 1)
            cnt[h, i] = i + 1
    return idx, cnt


# ---------------------------------------------------------------- attention

@pytest.mark.parametrize("n,b,hq,hk,d", [(200, 64, 4, 2, 16), (96, 32, 2, 2, 8), (64, 64, 1, 1, 8)])
def test_all_blocks_equals_torch_causal_sdpa(n, b, hq, hk, d):
    """k >= NB keeps every past block: the method reduces to dense causal
    attention, computed here by torch's SDPA in float64 (library routine)."""
    g = torch.Generator().manual_seed(n + d)
    q = torch.randn(hq, n, d, generator=g, dtype=torch.float64)
    k = torch.randn(hk, n, d, generator=g, dtype=torch.float64)
    v = torch.randn(hk, n, d, generator=g, dtype=torch.float64)
    nb = O.n_blocks(n, b)
    idx, cnt = _all_lists(hq, nb)
    got = O.attend(q, k, v, idx, cnt, block=b, scale=1 / math.sqrt(d), group_shared=False)
    rep = hq // hk
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.unsqueeze(0), k.repeat_interleave(rep, 0).unsqueeze(0),
        v.repeat_interleave(rep, 0).unsqueeze(0), is_causal=True)[0]
    np.testing.assert_allclose(got, ref.numpy(), atol=1e-12, rtol=1e-10)


def test_prefill_with_k_at_least_all_blocks_is_dense():
    """Through the whole prefill path (pool, score, top-k, attend)."""
    n, b, hq, hk, d = 300, 64, 4, 2, 16
    g = torch.Generator().manual_seed(7)
    q = torch.randn(hq, n, d, generator=g, dtype=torch.float64)
    k = torch.randn(hk, n, d, generator=g, dtype=torch.float64)
    v = torch.randn(hk, n, d, generator=g, dtype=torch.float64)
    nb = O.n_blocks(n, b)
    res = O.prefill(q, k, v, block=b, mode="topk", top_k_=nb, max_blocks=nb)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.unsqueeze(0), k.repeat_interleave(2, 0).unsqueeze(0),
        v.repeat_interleave(2, 0).unsqueeze(0), is_causal=True)[0]
    np.testing.assert_allclose(res["o"], ref.numpy(), atol=1e-12, rtol=1e-10)


def test_closed_form_golden():
    spec = json.load(open(os.path.join(GOLDEN, "closed_form_attention.json")))
    q = np.array(spec["q"]).reshape(1, 4, 1)
    k = np.array(spec["k"]).reshape(1, 4, 1)
    v = np.array(spec["v"]).reshape(1, 4, 1)
    for case in spec["cases"]:
        lists = case["lists"]
        idx = np.full((1, 2, 2), -1, dtype=np.int32)
        cnt = np.zeros((1, 2), dtype=np.int32)
        for i, lst in enumerate(lists):
            idx[0, i, :len(lst)] = lst
            cnt[0, i] = len(lst)
        got = O.attend(q, k, v, idx, cnt, block=spec["block"], scale=1.0, group_shared=False)
        want = [float(Fraction(x)) for x in case["expected_o"]]
        np.testing.assert_allclose(got[0, :, 0], want, atol=1e-12)


def test_value_ones_gives_ones():
    n, b, d = 160, 32, 8
    q = RNG.standard_normal((2, n, d))
    k = RNG.standard_normal((1, n, d))
    v = np.ones((1, n, d))
    res = O.prefill(q, k, v, block=b, mode="topk", top_k_=2, max_blocks=3)
    np.testing.assert_allclose(res["o"], 1.0, atol=1e-12)


def test_one_hot_values_expose_the_mask_and_probabilities():
    """V = one-hot token ids: output row t is the probability vector over
    keys; it must vanish outside the listed blocks and above the diagonal,
    sum to one, and have ratios exp((q.k_u - q.k_u') * scale)."""
    n, b, d = 96, 16, 4
    q = RNG.standard_normal((1, n, d))
    k = RNG.standard_normal((1, n, d))
    v = np.eye(n).reshape(1, n, n)
    nb = O.n_blocks(n, b)
    res = O.prefill(q, k, v, block=b, mode="topk", top_k_=2, max_blocks=3)
    P = res["o"][0]
    scale = 1 / math.sqrt(d)
    for t in range(n):
        i = t // b
        allowed = set(res["idx"][0, i, :res["cnt"][0, i]].tolist())
        vis = [u for u in range(n) if u <= t and u // b in allowed]
        off = [u for u in range(n) if u not in vis]
        assert np.all(P[t, off] == 0.0)
        assert abs(P[t].sum() - 1.0) < 1e-12
        u0 = vis[0]
        for u in vis[1:]:
            want = math.exp((q[0, t] @ k[0, u] - q[0, t] @ k[0, u0]) * scale)
            assert abs(P[t, u] / P[t, u0] - want) < 1e-9 * max(1.0, want)


def test_block_form_equals_dense_masked_form_on_tiny():
    w = W.CONFIGS["tiny"]
    data = W.generate(w)
    res = O.prefill(data["q"], data["k"], data["v"], block=w.block_size, mode="topk",
                    top_k_=w.top_k, max_blocks=w.max_blocks)
    dense = O.attend_dense_masked(data["q"], data["k"], data["v"], res["idx"], res["cnt"],
                                  block=w.block_size, scale=1 / math.sqrt(w.head_dim),
                                  group_shared=False)
    np.testing.assert_allclose(res["o"], dense, atol=1e-12)


# ------------------------------------------------------------------ pooling

def test_pooling_is_invariant_to_row_order_within_blocks():
    n, b, d = 100, 16, 6
    k = RNG.standard_normal((2, n, d))
    c0, r0 = O.pool_keys(k, b)
    kp = k.copy()
    for j in range(O.n_blocks(n, b)):
        rows = np.arange(j * b, min(n, (j + 1) * b))
        kp[:, rows] = k[:, RNG.permutation(rows)]
    c1, r1 = O.pool_keys(kp, b)
    np.testing.assert_allclose(c0, c1, atol=1e-13)
    np.testing.assert_allclose(r0, r1, atol=1e-13)


@pytest.mark.parametrize("group", [1, 3])
def test_pair_score_is_mean_of_dense_subblock(group):
    """Brute force: the pair score times sqrt(d_s) equals the mean over the
    group's heads h, the query rows t of block i and the key rows u of block j
    of q_t . k_u (bilinearity of the dot product), ragged last block too."""
    n, b, d = 45, 8, 5
    hq = group
    q = RNG.standard_normal((hq, n, d))
    k = RNG.standard_normal((1, n, d))
    c, _ = O.pool_keys(k, b, with_radius=False)
    qbar = O.pool_queries(q, b, group=group)
    nb = O.n_blocks(n, b)
    for i in range(nb):
        s = O.block_scores(qbar[0, i], c[0], i, 1.0)
        for j in range(i):
            tot, cntp = 0.0, 0
            for h in range(hq):
                mean_h = 0.0
                ti = list(range(i * b, min(n, (i + 1) * b)))
                uj = list(range(j * b, min(n, (j + 1) * b)))
                for t in ti:
                    for u in uj:
                        mean_h += sum(q[h, t, x] * k[0, u, x] for x in range(d))
                tot += mean_h / (len(ti) * len(uj))
            want = tot / hq
            assert abs(float(s[j]) - want) <= 1e-6 * max(1.0, abs(want))


def test_radius_bounds_every_key_and_is_tight():
    n, b, d = 128, 32, 8
    k = RNG.standard_normal((1, n, d)) * RNG.uniform(0.2, 3.0, size=(1, n, 1))
    c, r = O.pool_keys(k, b)
    for j in range(O.n_blocks(n, b)):
        rows = k[0, j * b:(j + 1) * b]
        for _ in range(20):
            qv = RNG.standard_normal(d)
            ub = qv @ c[0, j] + np.linalg.norm(qv) * r[0, j]
            assert np.all(rows @ qv <= ub + 1e-12)
        far = rows[np.argmax(np.linalg.norm(rows - c[0, j], axis=1))]
        qv = far - c[0, j]
        ub = qv @ c[0, j] + np.linalg.norm(qv) * r[0, j]
        assert abs(far @ qv - ub) < 1e-10 * max(1.0, abs(ub))


# ---------------------------------------------------------------- selection

def _brute_rank(s):
    """rank(j) = #{l : s_l > s_j or (s_l == s_j and l < j)}."""
    n = len(s)
    return [sum(1 for l in range(n) if s[l] > s[j] or (s[l] == s[j] and l < j)) for j in range(n)]


def test_top_k_matches_brute_force_ranks_with_ties():
    for trial in range(200):
        n = int(RNG.integers(0, 12))
        s = RNG.integers(-3, 4, size=n).astype(np.float32)     # many ties
        k = int(RNG.integers(1, 6))
        got = set(O.top_k(s, k).tolist())
        ranks = _brute_rank(s.tolist())
        want = {j for j in range(n) if ranks[j] < k}
        assert got == want


def test_near_tie_golden_from_the_page():
    spec = json.load(open(os.path.join(GOLDEN, "toy_near_tie.json")))
    s = np.array(spec["scores"], dtype=np.float32)
    assert O.top_k(s, spec["top_k"]).tolist() == spec["expected_top_k"]
    for case in spec["gate_cases"]:
        fired, _, _ = O.gate(s, spec["top_k"], case["margin"])
        assert fired == case["fires"], case


def test_gate_fires_exactly_when_gap_below_margin_std():
    for trial in range(300):
        n = int(RNG.integers(2, 40))
        k = int(RNG.integers(1, n))
        s = (RNG.standard_normal(n) * RNG.uniform(0.1, 5)).astype(np.float32)
        if trial % 3 == 0:                        # plant a near tie at the cut
            order = sorted(range(n), key=lambda j: (-float(s[j]), j))
            s[order[k]] = np.float32(float(s[order[k - 1]]) - 1e-3)
        margin = float(RNG.uniform(0.0, 0.5))
        vals = sorted((float(x) for x in s), reverse=True)
        gap = vals[k - 1] - vals[k]
        thr = margin * statistics.pstdev(float(x) for x in s)
        if abs(gap - thr) < 1e-9:
            continue
        fired, _, _ = O.gate(s, k, margin)
        assert fired == (gap < thr)


def test_gated_selection_supersets_and_sizes():
    for trial in range(200):
        i = int(RNG.integers(0, 30))
        k = int(RNG.integers(1, 8))
        s = RNG.standard_normal(i).astype(np.float32)
        base = set(O.top_k(s, k).tolist())
        double = set(O.top_k(s, 2 * k).tolist())
        assert base <= double
        ids, fl = O.select_row(s, i, mode="topk", top_k_=k, margin=0.3)
        body = set(ids.tolist()) - {i}
        assert len(body) in {min(k, i), min(2 * k, i)}
        assert base <= body
        if fl & O.FLAG_GATE:
            assert body == double
        else:
            assert body == base


def test_cumulative_mass_is_the_shortest_reaching_prefix():
    for trial in range(200):
        n = int(RNG.integers(1, 60))
        s = (RNG.standard_normal(n) * RNG.uniform(0.2, 6)).astype(np.float32)
        tau = float(RNG.uniform(0.05, 0.99))
        kept, _ = O.cumulative_mass(s, tau)
        p = scipy_softmax(s.astype(np.float64))
        kept_l = kept.tolist()
        assert math.fsum(p[kept_l]) >= tau - 1e-12
        unkept = [j for j in range(n) if j not in kept_l]
        if unkept:
            assert min(float(s[j]) for j in kept_l) >= max(float(s[j]) for j in unkept)
        # dropping the weakest kept block (last in rank order) falls short
        order = sorted(kept_l, key=lambda j: (-float(s[j]), j))
        assert math.fsum(p[order[:-1]]) < tau + 1e-12


def test_rescue_union_and_infinite_threshold():
    for trial in range(100):
        i = int(RNG.integers(1, 40))
        s = RNG.standard_normal(i).astype(np.float32)
        ub = (s + np.abs(RNG.standard_normal(i)) * 3).astype(np.float32)
        tau = float(RNG.uniform(-1, 4))
        base = set(O.cumulative_mass(s, 0.9)[0].tolist())
        rescue = {j for j in range(i) if float(ub[j]) > tau}
        ids, fl = O.select_row(s, i, mode="cummass", mass=0.9, ub=ub, tau=tau)
        got = set(ids.tolist()) - {i}
        assert got == base | rescue
        assert bool(fl & O.FLAG_RESCUE) == bool(rescue - base)
        ids_inf, _ = O.select_row(s, i, mode="cummass", mass=0.9, ub=ub, tau=math.inf)
        assert set(ids_inf.tolist()) - {i} == base


def test_group_mode_with_one_head_per_group_equals_per_head_mode():
    n, b, d = 256, 32, 8
    q = RNG.standard_normal((3, n, d))
    k = RNG.standard_normal((3, n, d))
    v = RNG.standard_normal((3, n, d))
    a = O.prefill(q, k, v, block=b, mode="topk", top_k_=2, max_blocks=3, group_shared=True)
    p = O.prefill(q, k, v, block=b, mode="topk", top_k_=2, max_blocks=3, group_shared=False)
    np.testing.assert_array_equal(a["idx"], p["idx"])
    np.testing.assert_allclose(a["o"], p["o"], atol=0)


def _check_lists(idx, cnt, nb):
    for h in range(idx.shape[0]):
        for i in range(nb):
            c = int(cnt[h, i])
            ids = idx[h, i, :c].tolist()
            assert ids == sorted(set(ids))
            assert ids[-1] == i and all(0 <= x <= i for x in ids)
            assert np.all(idx[h, i, c:] == -1)


@pytest.mark.parametrize("name", ["tiny", "gqa_small", "rbs_small", "gate_small", "msa_small",
                                  "quest_small", "quest_gate_small"])
def test_small_workload_lists_are_causal_sorted_padded(name):
    w = W.SMALL[name]
    data = W.generate(w)
    res = O.prefill(data["q"], data["k"], data["v"], block=w.block_size, mode=w.select_mode,
                    top_k_=w.top_k, mass=w.mass_threshold, margin=w.gate_margin,
                    tau=w.rescue_tau, group_shared=w.group_shared, q_idx=data["q_idx"],
                    k_idx=data["k_idx"], max_blocks=w.max_blocks,
                    attend_rows=[(0, w.n_blocks - 1)], backbone=w.backbone)
    _check_lists(res["idx"], res["cnt"], w.n_blocks)


# ------------------------------------------------ planted workload structure

def test_tiny_needle_block_is_selected():
    w = W.CONFIGS["tiny"]
    data = W.generate(w)
    meta = data["meta"]
    res = O.prefill(data["q"], data["k"], data["v"], block=w.block_size, mode="topk",
                    top_k_=w.top_k, max_blocks=w.max_blocks)
    qb = meta["query_block"]
    assert meta["needle_block"] in res["idx"][0, qb, :res["cnt"][0, qb]].tolist()


def test_gate_fires_on_exactly_the_planted_tied_rows():
    w = W.SMALL["gate_small"]
    data = W.generate(w)
    res = O.prefill(data["q"], data["k"], data["v"], block=w.block_size, mode="topk",
                    top_k_=w.top_k, margin=w.gate_margin, max_blocks=w.max_blocks,
                    attend_rows=[])
    fired = (res["flags"] & O.FLAG_GATE) != 0
    planted = data["meta"]["tied_rows"].numpy()
    assert planted.sum() > 0
    np.testing.assert_array_equal(fired, planted)


def test_rbs_rescue_adds_the_past_outlier_blocks():
    w = W.SMALL["rbs_small"]
    data = W.generate(w)
    res = O.prefill(data["q"], data["k"], data["v"], block=w.block_size, mode="cummass",
                    mass=w.mass_threshold, tau=w.rescue_tau, max_blocks=w.max_blocks,
                    attend_rows=[])
    grp = w.group
    outl = {}
    for (g, p) in data["meta"]["outliers"]:
        outl.setdefault(g, set()).add(p // w.block_size)
    for h in range(w.n_q_heads):
        for i in range(w.n_blocks):
            ids = set(res["idx"][h, i, :res["cnt"][h, i]].tolist())
            past = {j for j in outl[h // grp] if j < i}
            assert past <= ids
    # the base branch stays sparse: on average a handful of blocks per row
    assert res["cnt"].mean() < 16


# --------------------------------------------------------------------------
# K-min / K-max upper-bound backbone (uncertainty-gated page, Metodologia
# step 1 and Componibilidad: per-coordinate bounds from K-min / K-max)
# --------------------------------------------------------------------------

def test_minmax_table_is_the_tightest_box_around_each_block():
    rng = np.random.default_rng(21)
    k = rng.standard_normal((2, 203, 8)).astype(np.float32)  # ragged last block
    kmin, kmax = O.pool_keys_minmax(k, 64)
    for g in range(2):
        for j in range(O.n_blocks(203, 64)):
            rows = k[g, j * 64:min(203, (j + 1) * 64)].astype(np.float64)
            # every key inside the box ...
            assert (rows >= kmin[g, j] - 0).all() and (rows <= kmax[g, j] + 0).all()
            # ... and every face touched by some key
            for c in range(8):
                assert (rows[:, c] == kmin[g, j, c]).any()
                assert (rows[:, c] == kmax[g, j, c]).any()


def test_minmax_bound_is_the_maximum_over_the_box_corners():
    """q.x over the box [lo, hi] is linear, so its maximum sits at a corner:
    brute force over all 2^d corners must give the same value."""
    import itertools
    rng = np.random.default_rng(22)
    d = 5
    for trial in range(20):
        lo = rng.standard_normal((3, d))
        hi = lo + rng.random((3, d)) * 2
        q = rng.standard_normal(d)
        got = O.block_bounds_minmax(q, lo, hi, 3, 1.0).astype(np.float64)
        for j in range(3):
            best = max(float(np.dot(q, np.where(np.array(corner), hi[j], lo[j])))
                       for corner in itertools.product([0, 1], repeat=d))
            assert got[j] == pytest.approx(best, rel=1e-6, abs=1e-6)


def test_minmax_bound_dominates_every_key_and_is_exact_for_a_point_block():
    rng = np.random.default_rng(23)
    k = rng.standard_normal((1, 256, 16))
    k[0, 128:192] = k[0, 128]  # block 2: one key repeated
    kmin, kmax = O.pool_keys_minmax(k, 64)
    q = rng.standard_normal(16)
    ub = O.block_bounds_minmax(q, kmin[0], kmax[0], 4, 1.0).astype(np.float64)
    for j in range(4):
        dots = k[0, j * 64:(j + 1) * 64] @ q
        assert ub[j] >= dots.max() - 1e-5
    assert ub[2] == pytest.approx(float(k[0, 128] @ q), rel=1e-6)
    # sign-definite queries pick one face: q >= 0 -> q.max, q <= 0 -> q.min
    qp = np.abs(q)
    assert O.block_bounds_minmax(qp, kmin[0], kmax[0], 4, 1.0) == pytest.approx(
        (kmax[0] @ qp).astype(np.float32), rel=1e-6)
    assert O.block_bounds_minmax(-qp, kmin[0], kmax[0], 4, 1.0) == pytest.approx(
        (kmin[0] @ -qp).astype(np.float32), rel=1e-6)


def test_minmax_backbone_finds_the_spread_out_block_the_mean_misses():
    """A block whose keys swing to +-10 along the query direction has a mean
    near 0 (invisible to the centroid score) but the largest bound."""
    rng = np.random.default_rng(24)
    n, b, d = 8 * 32, 32, 16
    q = rng.standard_normal((1, n, d)) * 0.1
    k = rng.standard_normal((1, n, d)) * 0.1
    v = rng.standard_normal((1, n, d))
    u = np.zeros(d)
    u[0] = 1.0
    q[0, 7 * b:] += 2.0 * u                     # the last query block looks along e_0
    k[0, 3 * b:4 * b:2, 0] += 10.0              # block 3: alternate keys at +10 ...
    k[0, 3 * b + 1:4 * b:2, 0] -= 10.0          # ... and -10 (mean unchanged)
    k[0, 5 * b:6 * b, 0] += 0.5                 # block 5: a modest shift of the mean
    common = dict(block=b, mode="topk", top_k_=1, max_blocks=2)
    mean = O.prefill(q, k, v, backbone="mean", **common)
    mm = O.prefill(q, k, v, backbone="minmax", **common)
    assert mean["idx"][0, 7, :2].tolist() == [5, 7]
    assert mm["idx"][0, 7, :2].tolist() == [3, 7]


def test_minmax_backbone_rejects_the_rescue_branch():
    x = np.zeros((1, 64, 8))
    with pytest.raises(ValueError):
        O.prefill(x, x, x, block=32, mode="cummass", mass=0.9, tau=1.0, max_blocks=2,
                  backbone="minmax")


# --------------------------------------------------------------------------
# The page's own gate (uncertainty-gated page, Metodologia steps 3-5):
# sigma = (s_(k-1) - s_(k)) / (s_(0) - s_(k)), head average per tile,
# empirical percentile q, expansion to top rho*k
# --------------------------------------------------------------------------

def test_cut_margin_closed_forms():
    # three patches 10, 9.9, 9.8 and k = 2: (9.9 - 9.8) / (10 - 9.8) = 1/2
    assert O.cut_margin(np.array([9.8, 10.0, 9.9]), 2) == pytest.approx(0.5, rel=1e-6)
    # an exact tie at the cut: ambiguous
    assert O.cut_margin(np.array([5.0, 3.0, 3.0, 1.0]), 2) == 0.0
    # all kept scores equal and the first dropped below: decisive
    assert O.cut_margin(np.array([4.0, 4.0, 4.0, 1.0]), 3) == 1.0
    # everything tied: 0 (no cut at all)
    assert O.cut_margin(np.array([2.0, 2.0, 2.0]), 1) == 0.0
    # k = 1 normalises the gap by itself
    assert O.cut_margin(np.array([9.9, 9.8]), 1) == 1.0
    with pytest.raises(ValueError):
        O.cut_margin(np.array([1.0, 2.0]), 2)


def test_cut_margin_lies_in_unit_interval_and_ignores_affine_rescaling():
    rng = np.random.default_rng(31)
    for _ in range(200):
        s = rng.standard_normal(rng.integers(3, 40)).astype(np.float32)
        k = int(rng.integers(1, len(s)))
        m = O.cut_margin(s, k)
        assert 0.0 <= m <= 1.0
        assert O.cut_margin(3.0 * s.astype(np.float64) + 7.0, k) == pytest.approx(m, abs=1e-6)


def _sigma_case(seed=32):
    rng = np.random.default_rng(seed)
    hs, nb, d = 3, 20, 8
    qbar = rng.standard_normal((hs, nb, d))
    c = rng.standard_normal((hs, nb, d))
    r = np.zeros((hs, nb))
    return qbar, c, r


def _sel(qbar, c, r, **kw):
    base = dict(block_count=qbar.shape[1], mode="topk", scale=0.5, kv_of_sel=lambda h: h,
                max_blocks=qbar.shape[1])
    base.update(kw)
    return O.select(qbar, c, r, **base)


def test_percentile_gate_extremes_reduce_to_plain_top_k():
    qbar, c, r = _sigma_case()
    k = 3
    none = _sel(qbar, c, r, top_k_=k, sigma_gate=(0.0, 2))
    plain = _sel(qbar, c, r, top_k_=k)
    assert np.array_equal(none[0], plain[0]) and not (none[2] & O.FLAG_GATE).any()
    every = _sel(qbar, c, r, top_k_=k, sigma_gate=(1.0, 2))
    double = _sel(qbar, c, r, top_k_=2 * k)
    assert np.array_equal(every[0], double[0])
    fired_rows = (every[2] & O.FLAG_GATE) != 0
    assert fired_rows[:, k + 1:].all() and not fired_rows[:, :k + 1].any()


@pytest.mark.parametrize("q", [0.25, 0.5, 0.8])
def test_percentile_gate_fires_the_floor_q_t_most_ambiguous_tiles(q):
    qbar, c, r = _sigma_case(33)
    k, rho = 2, 3
    hs, nb = qbar.shape[:2]
    idx, cnt, flags = _sel(qbar, c, r, top_k_=k, sigma_gate=(q, rho))
    eligible = list(range(k + 1, nb))
    # the head-averaged margin of every eligible tile, recomputed from its definition
    sbar = {i: np.mean([O.cut_margin(O.block_scores(qbar[h, i], c[h], i, 0.5), k)
                        for h in range(hs)]) for i in eligible}
    fired = [i for i in eligible if flags[0, i] & O.FLAG_GATE]
    assert len(fired) == int(math.floor(q * len(eligible)))
    # every head of a fired tile fires, and takes rho*k blocks plus the diagonal
    for i in eligible:
        assert len({bool(flags[h, i] & O.FLAG_GATE) for h in range(hs)}) == 1
        want = min(rho * k, i) + 1 if i in fired else k + 1
        assert all(cnt[h, i] == want for h in range(hs))
    rest = [i for i in eligible if i not in fired]
    if fired and rest:
        assert max(sbar[i] for i in fired) <= min(sbar[i] for i in rest) + 1e-12


def test_percentile_gate_breaks_equal_margins_by_lower_tile():
    assert O.percentile_fire({5: 0.2, 3: 0.2, 9: 0.1, 7: 0.9}, 0.5) == {9, 3}


# --------------------------------------------------------------------------
# Row-max tile scores (uncertainty-gated page, Metodologia step 2: the tile
# score is the largest score among the tile's query rows)
# --------------------------------------------------------------------------

def test_rowmax_equals_exact_fraction_brute_force():
    """Every tile score against exact rational arithmetic over the explicit
    rows: max_t sum_d q_td * c_jd, times the scale, rounded to float32 once."""
    from fractions import Fraction
    rng = np.random.default_rng(40)
    c = rng.standard_normal((5, 8)).astype(np.float32).astype(np.float64)
    rows = rng.standard_normal((7, 8)).astype(np.float32).astype(np.float64)
    scale = 0.125
    got = O.block_scores_rowmax(rows, c, 5, scale)
    for j in range(5):
        best = max(sum(Fraction(float(q[d])) * Fraction(float(c[j, d])) for d in range(8))
                   for q in rows)
        assert got[j] == np.float32(float(best * Fraction(scale))), j


def test_rowmax_ranks_by_the_centroids_as_given_not_rounded_to_bf16():
    """Two candidates whose order flips if the centroids were rounded to
    bfloat16 first: c0 = (1 + 2^-9, 0) would round to (1, 0), and c1 =
    (1, 2^-10) is exact in bfloat16.  Against the row q = (1, 1) the exact
    scores are 1 + 2^-9 > 1 + 2^-10, so c0 ranks first; rounded operands
    would put c1 first."""
    c = np.array([[1.0 + 2 ** -9, 0.0], [1.0, 2 ** -10]])
    rows = np.array([[1.0, 1.0], [0.0, -1.0]])
    s = O.block_scores_rowmax(rows, c, 2, 1.0).astype(np.float64)
    assert s.tolist() == [1.0 + 2 ** -9, 1.0 + 2 ** -10]
    assert O.top_k(s, 1).tolist() == [0]
    rounded = torch.tensor(c, dtype=torch.float32).bfloat16().double().numpy()
    assert (rounded @ rows[0]).tolist() == [1.0, 1.0 + 2 ** -10]   # the flip it avoids


def test_rowmax_of_identical_rows_is_the_pooled_score_and_dominates_it_otherwise():
    rng = np.random.default_rng(41)
    c = rng.standard_normal((6, 16))
    row = rng.standard_normal(16)
    same = np.tile(row, (32, 1))
    got = O.block_scores_rowmax(same, c, 6, 0.25)
    assert np.array_equal(got, O.block_scores(row, c, 6, 0.25))
    rows = rng.standard_normal((32, 16))
    mx = O.block_scores_rowmax(rows, c, 6, 0.25).astype(np.float64)
    mean = c @ rows.mean(axis=0) * 0.25
    assert (mx >= mean - 1e-6).all()
    # the order of the rows does not matter
    assert np.array_equal(O.block_scores_rowmax(rows[::-1], c, 6, 0.25), mx.astype(np.float32))


@pytest.mark.parametrize("group_shared", [False, True])
def test_rowmax_finds_the_block_one_query_row_points_at(group_shared):
    """One query row of the last tile (of one head) points at block 2; the
    mean over the tile's rows hides it, the row maximum does not."""
    rng = np.random.default_rng(42)
    hq, hk, n, b, d = 2, 1, 8 * 32, 32, 16
    q = rng.standard_normal((hq, n, d)) * 0.1
    k = rng.standard_normal((hk, n, d)) * 0.1
    v = rng.standard_normal((hk, n, d))
    k[0, 2 * b:3 * b, 4] += 1.5                  # block 2: centroid along e_4
    k[0, 5 * b:6 * b, 3] += 5.0                  # block 5: along e_3
    q[:, 7 * b:, 3] += 0.5                       # every row of the last tile leans along e_3 ...
    q[1, 7 * b + 4, 4] = 40.0                    # ... one row of head 1 points along e_4
    common = dict(block=b, mode="topk", top_k_=1, max_blocks=2, group_shared=group_shared)
    mean = O.prefill(q, k, v, tile_score="mean", **common)
    rowmax = O.prefill(q, k, v, tile_score="rowmax", **common)
    hs = 0 if group_shared else 1
    assert rowmax["idx"][hs, 7, :2].tolist() == [2, 7]
    assert mean["idx"][hs, 7, :2].tolist() != [2, 7]
