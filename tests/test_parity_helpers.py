"""The tie-band comparator used by the GPU parity tests accepts exactly the
differences the band allows and rejects planted mistakes."""
import numpy as np

import parity as PT
from block_sparse_attention_sbsa_b200 import workloads as W

TOPK = W.CONFIGS["gqa32k"].scaled(top_k=2)
GATE = W.CONFIGS["gate64k"].scaled(top_k=2)
MASS = W.CONFIGS["rbs128k"].scaled(rescue_tau=None)
RESC = W.CONFIGS["rbs128k"]


def test_exact_list_matches():
    s = np.array([3.0, 1.0, 2.0, 0.5], dtype=np.float32)
    assert PT.row_matches([0, 2, 4], s, None, 4, TOPK)


def test_swap_inside_the_band_is_accepted():
    s = np.array([3.0, 1.0, 1.0 + 2e-6, 0.5], dtype=np.float32)   # near tie at the cut
    assert PT.row_matches([0, 2, 4], s, None, 4, TOPK)
    assert PT.row_matches([0, 1, 4], s, None, 4, TOPK)


def test_planted_wrong_block_is_rejected():
    s = np.array([3.0, 1.0, 2.0, 0.5], dtype=np.float32)
    assert not PT.row_matches([0, 1, 4], s, None, 4, TOPK)       # 1.0 is not within the band of 2.0
    assert not PT.row_matches([0, 2, 3, 4], s, None, 4, TOPK)    # too many
    assert not PT.row_matches([0, 2], s, None, 4, TOPK)          # diagonal missing
    assert not PT.row_matches([0, 2, 4, 5], s, None, 4, TOPK)    # future block


def test_gate_ambiguity_accepts_both_budgets():
    # gap between 2nd and 3rd = margin * std up to the band -> k or 2k
    s = np.array([5.0, 4.0, 3.0, 0.0, -1.0], dtype=np.float32)
    std = float(np.float64(s).std())
    gap = 1.0
    w = GATE.scaled(gate_margin=gap / std)
    assert PT.row_matches([0, 1, 5], s, None, 5, w)
    assert PT.row_matches([0, 1, 2, 3, 5], s, None, 5, w)
    w_far = GATE.scaled(gate_margin=0.1 * gap / std)             # decisively not gated
    assert not PT.row_matches([0, 1, 2, 3, 5], s, None, 5, w_far)


def test_cumulative_mass_boundary():
    s = np.log(np.array([0.5, 0.4, 0.1], dtype=np.float64)).astype(np.float32)
    # masses 0.5, 0.9, 1.0: 0.9 reached exactly at two blocks (inside the band)
    assert PT.row_matches([0, 1, 3], s, None, 3, MASS)
    assert PT.row_matches([0, 1, 2, 3], s, None, 3, MASS)
    s2 = np.log(np.array([0.6, 0.2, 0.2], dtype=np.float64)).astype(np.float32)
    assert not PT.row_matches([0, 3], s2, None, 3, MASS)         # 0.6 < 0.9, decisively


def test_rescue_boundary_and_union():
    s = np.array([10.0, 0.0, 0.0], dtype=np.float32)
    ub = np.array([10.0, 60.0 + 1e-4, 30.0], dtype=np.float32)   # block 1 inside the band of tau
    assert PT.row_matches([0, 3], s, ub, 3, RESC)
    assert PT.row_matches([0, 1, 3], s, ub, 3, RESC)
    ub2 = np.array([10.0, 75.0, 30.0], dtype=np.float32)         # block 1 decisively rescued
    assert not PT.row_matches([0, 3], s, ub2, 3, RESC)
    assert PT.row_matches([0, 1, 3], s, ub2, 3, RESC)
