"""The FMA-pipe exponential of the attention softmax's option (exp2_fma.cuh).

On the CPU: the header's coefficients are the ones the documented fit
(fit_exp2_fma.py, Lawson's iteration toward the minimax relative error of
2^f on [-1/2, 1/2]) produces, and the float32 algorithm built on them meets
the stated bound against float64 exp2 over the softmax's argument range.
On the GPU: the device function itself, through sbsa_exp2_fma_eval, against
float64 exp2, and the attention kernel with the option forced against the
oracle ("RBS-Attention", method paragraph: exact softmax attention over the
kept blocks).
"""
from __future__ import annotations

import importlib.util
import os
import re
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_attention_sbsa_b200", "csrc")
BOUND = 7.6e-5  # stated bound of the relative error over [-125, 8]


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_fma", os.path.join(CSRC, "fit_exp2_fma.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_coefficients() -> np.ndarray:
    text = open(os.path.join(CSRC, "exp2_fma.cuh")).read()
    found = dict(re.findall(r"kExp2FmaC(\d) = ([-+0-9.e]+)f;", text))
    assert sorted(found) == ["0", "1", "2", "3"]
    return np.array([float(found[str(k)]) for k in range(4)], dtype=np.float32)


def test_header_coefficients_are_the_documented_fit():
    fit = _fit_module().fit()
    head = _header_coefficients()
    # the header prints 10 significant digits of each float32 coefficient
    assert np.array_equal(fit, head), (fit, head)


def test_float32_algorithm_meets_the_stated_bound():
    mod = _fit_module()
    c = _header_coefficients()
    assert mod.max_rel_error(c) <= BOUND
    # integers, halves and the interval ends of the reduction
    x = np.concatenate([np.arange(-125, 9, dtype=np.float32),
                        np.arange(-124.5, 8, 1.0, dtype=np.float32)])
    y = mod.eval32(c, x)
    assert np.max(np.abs(y / np.exp2(x.astype(np.float64)) - 1)) <= BOUND


def test_below_the_range_and_minus_infinity_give_zero():
    mod = _fit_module()
    c = _header_coefficients()
    x = np.array([-np.inf, -1e30, -126.0, -125.5, -125.0001], dtype=np.float32)
    assert np.all(mod.eval32(c, x) == 0.0)
    # the last value inside the range stays a normal float
    assert mod.eval32(c, np.array([-125.0], dtype=np.float32))[0] > 0.0


@pytest.mark.gpu
def test_device_exp2_fma_meets_the_bound():
    import torch
    from block_sparse_attention_sbsa_b200 import sbsa
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.uniform(-125.0, 8.0, 1 << 20).astype(np.float32),
                        np.arange(-125, 9, dtype=np.float32),
                        np.float32([0.5, -0.5, 7.999, -124.999])])
    y = sbsa.exp2_fma_eval(torch.from_numpy(x).cuda()).cpu().numpy()
    assert sbsa.get_status() == sbsa.OK
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= BOUND, rel.max()
    # the host restatement of the same float32 steps agrees to within an ulp
    # (the host's fused multiply-add rounds twice in rare cases)
    ref = _fit_module().eval32(_header_coefficients(), x)
    ulps = np.abs(y.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1
    z = sbsa.exp2_fma_eval(torch.tensor([-np.inf, -200.0, -125.5], dtype=torch.float32).cuda())
    assert torch.all(z == 0).item()


@pytest.mark.gpu
def test_attention_with_fma_exponentials_matches_oracle():
    """The persistent 128-token kernel with SBSA_ATTEND_EXP2=fma (forced for
    every 128-token workload with SBSA_ATTEND_KERNEL=persistent), in a child
    process, on the oracle's own lists."""
    code = (
        "import sys; sys.path.insert(0, 'tests'); sys.path.insert(0, '.');\n"
        "import test_gpu_parity as T, torch\n"
        "from block_sparse_attention_sbsa_b200 import sbsa\n"
        "import parity as PT\n"
        "for name in ['gqa_small', 'rbs_small', 'msa_small']:\n"
        "    w, data, ref = T.small_case(name)\n"
        "    d = T._dev(data)\n"
        "    o = sbsa.attend(sbsa.params_for(w), d['q'], d['k'], d['v'],\n"
        "                    torch.tensor(ref['idx'], device='cuda'), torch.tensor(ref['cnt'], device='cuda'))\n"
        "    torch.cuda.synchronize()\n"
        "    assert sbsa.get_status() == sbsa.OK\n"
        "    mx, mean = PT.output_errors(o.float().cpu().numpy(), ref['o'])\n"
        "    assert mx <= PT.MAX_ABS and mean <= PT.MEAN_ABS, (name, mx, mean)\n"
        "    print(name, mx, mean)\n"
        "print('fma ok')\n")
    env = dict(os.environ, SBSA_ATTEND_EXP2="fma", SBSA_ATTEND_KERNEL="persistent")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "fma ok" in r.stdout, r.stdout + r.stderr


def test_eval_entry_rejects_bad_arguments_on_the_host():
    """sbsa_exp2_fma_eval checks its arguments before any CUDA call."""
    import ctypes
    from block_sparse_attention_sbsa_b200 import sbsa
    fake = ctypes.c_void_p(0x10000)
    assert sbsa.lib.sbsa_exp2_fma_eval(fake, fake, -1, None) == sbsa.ERR_INVALID_ARG
    assert sbsa.lib.sbsa_exp2_fma_eval(None, fake, 4, None) == sbsa.ERR_INVALID_ARG
    assert sbsa.lib.sbsa_exp2_fma_eval(fake, None, 4, None) == sbsa.ERR_INVALID_ARG
    # nothing to do: no launch, no pointer needed
    assert sbsa.lib.sbsa_exp2_fma_eval(None, None, 0, None) == sbsa.OK


def test_binding_rejects_non_float32_or_host_tensors():
    import torch
    from block_sparse_attention_sbsa_b200 import sbsa
    with pytest.raises(ValueError):
        sbsa.exp2_fma_eval(torch.zeros(4, dtype=torch.float32))  # host memory
    with pytest.raises(ValueError):
        sbsa.exp2_fma_eval(torch.zeros(4, dtype=torch.float64))
