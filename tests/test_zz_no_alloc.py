"""The no-allocation prefill entry point.

sbsa_prefill_noalloc serves callers that cannot allocate device memory: a
plugin inside a framework that owns all device memory and gives operators no
allocator, a latency-critical path where cudaMalloc's implicit device
synchronisation is not acceptable, or a process whose device memory budget
is fixed at start-up.  Its temporaries live in a fixed array inside the
library instead of a caller-supplied workspace.

Each case calls it through the C ABI twice in a row and checks every result
against the workspace entry point sbsa_prefill on the same inputs, and that
a call (after the first one on the device, which looks up the array's
address) leaves the device's allocated and free memory unchanged.  This file
is collected last on purpose, and passes on its own in a fresh process too.
"""
import ctypes

import pytest
import torch

import parity as PT
from block_sparse_attention_sbsa_b200 import workloads as W

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 * 1024 * 1024          # SBSA_NOALLOC_SCRATCH_BYTES in include/sbsa.h
FAKE = ctypes.c_void_p(1 << 20)           # aligned; never dereferenced when a call is rejected


@pytest.fixture(scope="module")
def sb(cuda):
    from block_sparse_attention_sbsa_b200 import build
    build.build()
    from block_sparse_attention_sbsa_b200 import sbsa
    fn = sbsa.lib.sbsa_prefill_noalloc
    fn.argtypes = [ctypes.POINTER(sbsa.Params)] + [ctypes.c_void_p] * 10
    fn.restype = ctypes.c_int
    return sbsa


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _noalloc(sb, p, d, o, idx=None, cnt=None, flags=None):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return sb.lib.sbsa_prefill_noalloc(ctypes.byref(p), _ptr(d["q"]), _ptr(d["k"]), _ptr(d["v"]),
                                       _ptr(d["q_idx"]), _ptr(d["k_idx"]), _ptr(o), _ptr(idx),
                                       _ptr(cnt), _ptr(flags), stream)


@pytest.mark.parametrize("name", ["gqa_small", "msa_small", "tiny"])
def test_noalloc_matches_the_workspace_entry_point_twice(sb, name):
    w = W.SMALL[name]
    data = W.generate(w, "cpu")
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in data.items()}
    p = sb.params_for(w)
    o_ref, idx_ref, cnt_ref, flags_ref = sb.prefill(p, d["q"], d["k"], d["v"], d["q_idx"],
                                                    d["k_idx"])
    torch.cuda.synchronize()
    o_ref = o_ref.float().cpu().numpy()
    for _ in range(2):
        # lists returned to the caller
        o = torch.empty_like(d["q"])
        idx, cnt = torch.empty_like(idx_ref), torch.empty_like(cnt_ref)
        flags = torch.empty_like(flags_ref)
        assert _noalloc(sb, p, d, o, idx, cnt, flags) == sb.OK
        torch.cuda.synchronize()
        assert sb.get_status() == sb.OK
        assert torch.equal(idx, idx_ref) and torch.equal(cnt, cnt_ref)
        assert torch.equal(flags, flags_ref)
        mx, mean = PT.output_errors(o.float().cpu().numpy(), o_ref)
        assert mx <= PT.MAX_ABS and mean <= PT.MEAN_ABS, (mx, mean)
        # lists kept in the library's scratch as well
        o2 = torch.empty_like(d["q"])
        assert _noalloc(sb, p, d, o2) == sb.OK
        torch.cuda.synchronize()
        assert sb.get_status() == sb.OK
        mx, mean = PT.output_errors(o2.float().cpu().numpy(), o_ref)
        assert mx <= PT.MAX_ABS and mean <= PT.MEAN_ABS, (mx, mean)


def test_noalloc_allocates_no_device_memory(sb):
    w = W.SMALL["gqa_small"]
    data = W.generate(w, "cpu")
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in data.items()}
    p = sb.params_for(w)
    o = torch.empty_like(d["q"])
    assert _noalloc(sb, p, d, o) == sb.OK            # the one-time address lookup
    torch.cuda.synchronize()
    before = (torch.cuda.memory_allocated(), torch.cuda.memory_reserved(),
              torch.cuda.mem_get_info()[0])
    for _ in range(2):
        assert _noalloc(sb, p, d, o) == sb.OK
    torch.cuda.synchronize()
    after = (torch.cuda.memory_allocated(), torch.cuda.memory_reserved(),
             torch.cuda.mem_get_info()[0])
    assert after == before
    assert sb.get_status() == sb.OK


def test_noalloc_rejects_problems_larger_than_its_scratch(sb):
    # 128k tokens with the lists in the scratch: ~150 MB of temporaries
    p = sb.params_for(W.CONFIGS["rbs128k"])
    assert sb.workspace_bytes(p) > SCRATCH_BYTES
    fn = sb.lib.sbsa_prefill_noalloc
    assert fn(ctypes.byref(p), FAKE, FAKE, FAKE, None, None, FAKE, None, None, None, None) == \
        sb.ERR_WORKSPACE
    # 512k tokens x 32 heads: the pooled query table alone is 64 MB
    big = sb.make_params(n_q_heads=32, n_kv_heads=8, seq_len=524288, head_dim=128,
                         block_size=128, top_k=8)
    assert fn(ctypes.byref(big), FAKE, FAKE, FAKE, None, None, FAKE, FAKE, FAKE, None, None) == \
        sb.ERR_WORKSPACE
    # an argument error wins over the size check, as in sbsa_prefill
    assert fn(ctypes.byref(p), FAKE, FAKE, FAKE, None, None, FAKE, None, FAKE, None, None) == \
        sb.ERR_INVALID_ARG
