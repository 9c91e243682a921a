"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, its parameter struct matches the C layout, and argument
errors are rejected on the host before anything is launched."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sbsa.h")


@pytest.fixture(scope="module")
def sb():
    from block_sparse_attention_sbsa_b200 import build
    build.build()
    from block_sparse_attention_sbsa_b200 import sbsa
    return sbsa


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\*]+\s+\**(sbsa_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["sbsa_pool_blocks", "sbsa_select", "sbsa_attend", "sbsa_prefill",
                     "sbsa_prefill_workspace_bytes", "sbsa_get_status", "sbsa_status_string"]:
        assert required in names


def test_library_exports_every_declared_symbol(sb):
    out = subprocess.run(["nm", "-D", "--defined-only", sb.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (sbsa_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(sb.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n)
    assert set(sb.SYMBOLS) <= set(declared_functions())


def test_params_struct_layout_matches_c(sb):
    src = r'''
#include <stdio.h>
#include <stddef.h>
#include "sbsa.h"
#define F(m) printf("%s %zu\n", #m, offsetof(sbsa_params, m));
int main(void) {
  printf("size %zu\n", sizeof(sbsa_params));
  F(n_q_heads) F(n_kv_heads) F(seq_len) F(head_dim) F(block_size) F(dtype) F(select_mode)
  F(group_shared) F(index_dim) F(top_k) F(mass_threshold) F(rescue) F(rescue_tau) F(gate)
  F(gate_margin) F(max_blocks) F(sm_scale) F(score_scale) F(backbone) F(gate_quantile)
  F(gate_rho) F(tile_score)
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), c, "-o", exe], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    got = dict(line.split() for line in out.strip().splitlines())
    assert int(got.pop("size")) == ctypes.sizeof(sb.Params)
    for name, off in got.items():
        assert getattr(sb.Params, name).offset == int(off), name


def test_status_strings(sb):
    for code in range(7):
        assert sb.status_string(code)
    assert sb.lib.sbsa_version() >= 100


def _valid_base():
    return dict(n_q_heads=4, n_kv_heads=2, seq_len=1000, head_dim=128, block_size=128,
                dtype="bf16", select_mode="topk", top_k=4)


def _valid(sb, **kw):
    base = _valid_base()
    base.update(kw)
    return sb.make_params(**base)


FAKE = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced on the host


def r256(x):
    return (x + 255) // 256 * 256


def _centroid_scratch(p, with_table=True):
    """Bytes of the tensor-core centroid scores' scratch: tf32 hi and lo parts
    of the pooled queries and of the centroids, then the [Hs, NB, NB] table."""
    nb, hs, ds = p.n_blocks, p.n_sel_heads, p.score_dim
    parts = 2 * r256(hs * nb * ds * 4) + 2 * r256(p.n_kv_heads * nb * ds * 4)
    return parts + (r256(hs * nb * nb * 4) if with_table else 0)


def _select(sb, p):
    return sb.lib.sbsa_select(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, None)


def _attend(sb, p):
    return sb.lib.sbsa_attend(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None)


@pytest.mark.parametrize("mutate,code", [
    (dict(n_q_heads=3), 1),                      # Hq % Hkv != 0
    (dict(seq_len=0), 1),
    (dict(head_dim=96), 2),
    (dict(block_size=32), 2),
    (dict(index_dim=32), 2),
    (dict(top_k=0), 1),
    (dict(select_mode="cummass", mass_threshold=0.0), 1),
    (dict(select_mode="cummass", mass_threshold=1.5), 1),
    (dict(select_mode="cummass", mass_threshold=0.9, gate_margin=0.05), 1),
    (dict(gate_margin=-1.0), 1),
    (dict(max_blocks=4), 1),                     # needs k+1 = 5
    (dict(top_k=4, gate_margin=0.05, max_blocks=5), 1),   # gated needs 2k+1 = 9
    (dict(select_mode="cummass", mass_threshold=0.9, max_blocks=5), 1),  # needs NB
    (dict(sm_scale=-1.0), 1),
    (dict(backbone=2), 1),                       # no such backbone
    (dict(gate_quantile=1.5), 1),                # q outside [0, 1]
    (dict(gate_quantile=0.3, gate_rho=0), 1),
    (dict(gate_quantile=0.3, gate_rho=3, max_blocks=7), 1),   # needs min(rho*k, NB-1)+1 = 8
    (dict(select_mode="cummass", mass_threshold=0.9, gate_quantile=0.3), 1),
    (dict(tile_score=2), 1),                     # no such tile score
    (dict(tile_score="rowmax", backbone="minmax"), 1),
    (dict(tile_score="rowmax", dtype="fp32"), 1),
    (dict(tile_score="rowmax", select_mode="cummass", mass_threshold=0.9, rescue_tau=1.0), 1),
    (dict(select_mode="cummass", mass_threshold=0.9, rescue_tau=5.0, backbone="minmax"), 1),
])
def test_invalid_parameters_are_rejected_before_launch(sb, mutate, code):
    p = _valid(sb, **mutate)
    assert _select(sb, p) == code
    assert _attend(sb, p) == code
    assert sb.lib.sbsa_prefill_workspace_bytes(ctypes.byref(p)) == 0


def test_null_pointers_are_rejected(sb):
    p = _valid(sb)
    assert sb.lib.sbsa_select(None, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == 1
    assert sb.lib.sbsa_select(ctypes.byref(p), None, FAKE, None, FAKE, FAKE, None, None) == 1
    assert sb.lib.sbsa_attend(ctypes.byref(p), FAKE, None, FAKE, FAKE, FAKE, FAKE, None) == 1
    pr = _valid(sb, rescue_tau=1.0)
    assert sb.lib.sbsa_select(ctypes.byref(pr), FAKE, FAKE, None, FAKE, FAKE, None, None) == 1
    assert sb.lib.sbsa_pool_blocks(ctypes.byref(p), None, 2, 128, 1, FAKE, None, None) == 1


def test_misaligned_pointers_are_rejected(sb):
    p = _valid(sb)
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert sb.lib.sbsa_attend(ctypes.byref(p), odd, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert sb.lib.sbsa_pool_blocks(ctypes.byref(p), odd, 2, 128, 1, FAKE, None, None) == 1


def test_pool_argument_checks(sb):
    p = _valid(sb)
    assert sb.lib.sbsa_pool_blocks(ctypes.byref(p), FAKE, 3, 128, 2, FAKE, None, None) == 1
    assert sb.lib.sbsa_pool_blocks(ctypes.byref(p), FAKE, 4, 96, 1, FAKE, None, None) == 2
    assert sb.lib.sbsa_pool_blocks(ctypes.byref(p), FAKE, 4, 128, 2, FAKE, FAKE, None) == 1


def test_pool_minmax_argument_checks(sb):
    p = _valid(sb)
    assert sb.lib.sbsa_pool_minmax(ctypes.byref(p), None, 2, 128, FAKE, None) == 1
    assert sb.lib.sbsa_pool_minmax(ctypes.byref(p), FAKE, 0, 128, FAKE, None) == 1
    assert sb.lib.sbsa_pool_minmax(ctypes.byref(p), FAKE, 2, 96, FAKE, None) == 2
    assert sb.lib.sbsa_pool_minmax(ctypes.byref(p), FAKE, 2, 128,
                                   ctypes.c_void_p((1 << 20) + 4), None) == 1


def test_minmax_backbone_doubles_the_key_table_in_the_workspace(sb):
    mean = _valid(sb)
    mm = _valid(sb, backbone="minmax")
    nb = mean.n_blocks
    extra = r256(2 * 2 * nb * 128 * 4) - r256(2 * nb * 128 * 4)
    # the upper bound is no product: no tensor-core score scratch
    assert sb.workspace_bytes(mm) == sb.workspace_bytes(mean) - _centroid_scratch(mean) + extra


def test_centroid_scores_workspace_and_checks(sb):
    p = _valid(sb, seq_len=4096)
    need = sb.lib.sbsa_score_centroids_workspace_bytes(ctypes.byref(p))
    assert need == _centroid_scratch(p, with_table=False)
    for other in (_valid(sb, backbone="minmax"), _valid(sb, tile_score="rowmax")):
        assert sb.lib.sbsa_score_centroids_workspace_bytes(ctypes.byref(other)) == 0
        assert sb.lib.sbsa_score_centroids(ctypes.byref(other), FAKE, FAKE, FAKE, FAKE, need,
                                           None) == 2
    f = sb.lib.sbsa_score_centroids
    assert f(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, need - 1, None) == 3
    assert f(ctypes.byref(p), FAKE, FAKE, FAKE, ctypes.c_void_p((1 << 20) + 128), need, None) == 3
    assert f(ctypes.byref(p), None, FAKE, FAKE, FAKE, need, None) == 1
    assert f(ctypes.byref(p), FAKE, FAKE, ctypes.c_void_p((1 << 20) + 4), FAKE, need, None) == 1
    # sbsa_select_ws needs the table and its scratch; sbsa_select none
    assert sb.lib.sbsa_select_workspace_bytes(ctypes.byref(p)) == _centroid_scratch(p)
    ws = sb.lib.sbsa_select_ws
    assert ws(ctypes.byref(p), FAKE, FAKE, None, FAKE, FAKE, None, FAKE,
              _centroid_scratch(p) - 1, None) == 3
    assert ws(ctypes.byref(p), FAKE, FAKE, None, FAKE, FAKE, None, None, 0, None) == 3


def test_percentile_gate_needs_a_workspace(sb):
    p = _valid(sb, gate_quantile=0.3, gate_rho=2, seq_len=4096)
    nb = p.n_blocks
    need = sb.lib.sbsa_select_workspace_bytes(ctypes.byref(p))
    # per-row margins, per-tile margin sums (doubles), per-tile decisions
    gate = r256(4 * nb * 8) + r256(nb * 8) + r256(nb)
    assert need == gate + _centroid_scratch(p)
    mm = _valid(sb, gate_quantile=0.3, gate_rho=2, seq_len=4096, backbone="minmax")
    assert sb.lib.sbsa_select_workspace_bytes(ctypes.byref(mm)) == gate
    assert sb.lib.sbsa_select_workspace_bytes(ctypes.byref(_valid(sb, backbone="minmax"))) == 0
    assert _select(sb, p) == 3                   # the plain entry point has no workspace
    ws = sb.lib.sbsa_select_ws
    assert ws(ctypes.byref(p), FAKE, FAKE, None, FAKE, FAKE, None, FAKE, need - 1, None) == 3
    assert ws(ctypes.byref(p), FAKE, FAKE, None, FAKE, FAKE, None,
              ctypes.c_void_p((1 << 20) + 64), need, None) == 3
    # the prefill workspace grows by the gate's scratch
    plain = sb.workspace_bytes(_valid(sb, seq_len=4096, max_blocks=p.max_blocks))
    assert sb.workspace_bytes(p) == plain + gate


def test_percentile_gate_halves_check_their_arguments(sb):
    p = _valid(sb, gate_quantile=0.3, gate_rho=2, seq_len=4096)
    need = sb.lib.sbsa_select_workspace_bytes(ctypes.byref(p))
    part, fin = sb.lib.sbsa_select_gate_partial, sb.lib.sbsa_select_gate_finish
    args = (ctypes.byref(p), FAKE, FAKE, None, FAKE, FAKE, None, FAKE, need)
    assert part(*args, None, None) == 1                              # no tile sums
    assert part(*args, ctypes.c_void_p((1 << 20) + 4), None) == 1    # misaligned
    assert fin(*args, FAKE, p.n_sel_heads - 1, None) == 1            # fewer heads than its own
    short = (ctypes.byref(p), FAKE, FAKE, None, FAKE, FAKE, None, FAKE, need - 1)
    assert part(*short, FAKE, None) == 3 and fin(*short, FAKE, 8, None) == 3
    plain = _valid(sb)                                               # no percentile gate
    assert part(ctypes.byref(plain), FAKE, FAKE, None, FAKE, FAKE, None, FAKE, 1 << 20, FAKE,
                None) == 1
    rowmax = _valid(sb, gate_quantile=0.3, gate_rho=2, tile_score="rowmax")
    assert fin(ctypes.byref(rowmax), FAKE, FAKE, None, FAKE, FAKE, None, FAKE, 1 << 30, FAKE, 8,
               None) == 1


def test_rowmax_workspace_and_checks(sb):
    p = _valid(sb, tile_score="rowmax", seq_len=4096)
    nb = p.n_blocks
    need = sb.lib.sbsa_score_rowmax_workspace_bytes(ctypes.byref(p))
    assert need == (3 * 2 * nb * 128 * 2 + 255) // 256 * 256   # three bf16 parts
    assert sb.lib.sbsa_score_rowmax_workspace_bytes(ctypes.byref(_valid(sb))) == 0
    f = sb.lib.sbsa_score_rowmax
    assert f(ctypes.byref(_valid(sb)), FAKE, FAKE, FAKE, FAKE, need, None) == 2  # not rowmax
    assert f(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, need - 1, None) == 3
    assert f(ctypes.byref(p), None, FAKE, FAKE, FAKE, need, None) == 1
    # the prefill workspace holds the centroid parts and the score table
    # in place of the tensor-core centroid scratch
    mean = _valid(sb, seq_len=4096)
    plain = sb.workspace_bytes(mean) - _centroid_scratch(mean)
    scores = (4 * nb * nb * 4 + 255) // 256 * 256
    assert sb.workspace_bytes(p) == plain + need + scores


@pytest.mark.parametrize("kw,ok_len,bad_len", [
    # the selection kernel keeps two score rows of NB candidates in shared memory
    (dict(top_k=4), 23424 * 128, 23425 * 128),
    (dict(select_mode="cummass", mass_threshold=0.9, rescue_tau=5.0), 15616 * 128,
     15617 * 128),
    # the row-max kernel keeps the running maxima of a tile's candidates
    (dict(top_k=4, tile_score="rowmax"), 16897 * 128, 16898 * 128),
])
def test_shared_memory_limits_are_rejected_before_launch(sb, kw, ok_len, bad_len):
    base = dict(_valid_base(), **kw)
    good = sb.make_params(**dict(base, seq_len=ok_len))
    bad = sb.make_params(**dict(base, seq_len=bad_len))
    assert sb.lib.sbsa_prefill_workspace_bytes(ctypes.byref(good)) > 0
    assert sb.lib.sbsa_prefill_workspace_bytes(ctypes.byref(bad)) == 0
    assert _select(sb, bad) == 2
    assert sb.lib.sbsa_prefill(ctypes.byref(bad), FAKE, FAKE, FAKE, None, None, FAKE, FAKE,
                               1 << 40, None, None, None, None) == 2


def test_prefill_host_workspace_and_checks(sb):
    p = _valid(sb, seq_len=4096)                    # 4 query / 2 kv heads: two chunks
    need = sb.lib.sbsa_prefill_host_workspace_bytes(ctypes.byref(p))
    sub = _valid(sb, seq_len=4096, n_q_heads=2, n_kv_heads=1)
    n, d = 4096, 128
    q_chunk, kv_chunk = r256(2 * n * d * 2), r256(n * d * 2)
    staging = q_chunk + 2 * kv_chunk + q_chunk        # Q, K, V and O of one chunk
    assert need == 2 * staging + r256(sb.workspace_bytes(sub))
    f = sb.lib.sbsa_prefill_host
    assert f(ctypes.byref(p), FAKE, FAKE, FAKE, None, None, FAKE, FAKE, need - 1, None) == 3
    assert f(ctypes.byref(p), FAKE, FAKE, FAKE, None, None, FAKE,
             ctypes.c_void_p((1 << 20) + 128), need, None) == 3
    assert f(ctypes.byref(p), FAKE, None, FAKE, None, None, FAKE, FAKE, need, None) == 1
    bad = _valid(sb, head_dim=96)
    assert f(ctypes.byref(bad), FAKE, FAKE, FAKE, None, None, FAKE, FAKE, 1 << 40, None) == 2
    assert sb.lib.sbsa_prefill_host_workspace_bytes(ctypes.byref(bad)) == 0
    # the percentile gate couples heads: one chunk holding every head
    g = _valid(sb, seq_len=4096, gate_quantile=0.3, gate_rho=2)
    one = r256(4 * n * d * 2) * 2 + r256(2 * n * d * 2) * 2
    assert sb.lib.sbsa_prefill_host_workspace_bytes(ctypes.byref(g)) == \
        2 * one + r256(sb.workspace_bytes(g))


def test_fp32_attention_is_limited_to_d64_b64(sb):
    p = _valid(sb, dtype="fp32")
    assert _attend(sb, p) == 2


def test_workspace_size_and_checks(sb):
    p = _valid(sb, rescue_tau=5.0)
    nb = p.n_blocks
    ws = sb.workspace_bytes(p)
    want = (r256(4 * nb * 128 * 4) + r256(2 * nb * 128 * 4) + r256(2 * nb * 4)
            + r256(4 * nb * p.max_blocks * 4) + r256(4 * nb * 4) + r256(4 * nb)
            + _centroid_scratch(p))
    assert ws == want
    small = sb.lib.sbsa_prefill(ctypes.byref(p), FAKE, FAKE, FAKE, None, None, FAKE, FAKE,
                                ws - 1, None, None, None, None)
    assert small == 3
    unaligned = sb.lib.sbsa_prefill(ctypes.byref(p), FAKE, FAKE, FAKE, None, None, FAKE,
                                    ctypes.c_void_p((1 << 20) + 16), ws, None, None, None, None)
    assert unaligned == 3
    # index tensors are required when index_dim is set
    pi = _valid(sb, index_dim=64)
    assert sb.lib.sbsa_prefill(ctypes.byref(pi), FAKE, FAKE, FAKE, None, None, FAKE, FAKE,
                               1 << 30, None, None, None, None) == 1
