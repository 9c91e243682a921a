"""ctypes binding over libsbsa.so (argument marshalling only).

Every function takes torch CUDA tensors (PyTorch provides device memory and
the stream), passes raw pointers and sizes to the C ABI declared in
include/sbsa.h, and raises on a non-zero status.  All compute runs in the
library's CUDA kernels; there is no fallback of any kind: if the library is
missing or fails to load, importing this module raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsbsa.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE = range(7)
BF16, FP32 = 0, 1
TOPK, CUMMASS = 0, 1
BACKBONE_MEAN, BACKBONE_MINMAX = 0, 1
GATE_GAP, GATE_PERCENTILE = 1, 2
TILE_MEAN, TILE_ROWMAX = 0, 1
FLAG_GATE, FLAG_RESCUE = 1, 2

SYMBOLS = ["sbsa_pool_blocks", "sbsa_pool_minmax", "sbsa_select", "sbsa_select_ws",
           "sbsa_select_workspace_bytes", "sbsa_score_centroids",
           "sbsa_score_centroids_workspace_bytes", "sbsa_score_rowmax",
           "sbsa_score_rowmax_workspace_bytes",
           "sbsa_select_scores", "sbsa_select_gate_partial", "sbsa_select_gate_finish",
           "sbsa_attend", "sbsa_prefill", "sbsa_prefill_host", "sbsa_prefill_host_workspace_bytes",
           "sbsa_prefill_workspace_bytes", "sbsa_get_status", "sbsa_status_string",
           "sbsa_version", "sbsa_debug_wait_timeout", "sbsa_exp2_fma_eval"]


class SbsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (code {code})")


class Params(ctypes.Structure):
    _fields_ = [
        ("n_q_heads", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int),
        ("seq_len", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("block_size", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("select_mode", ctypes.c_int),
        ("group_shared", ctypes.c_int),
        ("index_dim", ctypes.c_int),
        ("top_k", ctypes.c_int),
        ("mass_threshold", ctypes.c_float),
        ("rescue", ctypes.c_int),
        ("rescue_tau", ctypes.c_float),
        ("gate", ctypes.c_int),
        ("gate_margin", ctypes.c_float),
        ("max_blocks", ctypes.c_int),
        ("sm_scale", ctypes.c_float),
        ("score_scale", ctypes.c_float),
        ("backbone", ctypes.c_int),
        ("gate_quantile", ctypes.c_float),
        ("gate_rho", ctypes.c_int),
        ("tile_score", ctypes.c_int),
    ]

    @property
    def n_blocks(self) -> int:
        return (self.seq_len + self.block_size - 1) // self.block_size

    @property
    def n_sel_heads(self) -> int:
        return self.n_kv_heads if self.group_shared else self.n_q_heads

    @property
    def score_dim(self) -> int:
        return self.index_dim if self.index_dim else self.head_dim


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m block_sparse_attention_sbsa_b200.build`"
            " (there is no non-CUDA fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(Params)
    vp, i32p, f32p, u8p = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
    ci = ctypes.c_int
    lib.sbsa_pool_blocks.argtypes = [P, vp, ci, ci, ci, f32p, f32p, vp]
    lib.sbsa_pool_minmax.argtypes = [P, vp, ci, ci, f32p, vp]
    lib.sbsa_select.argtypes = [P, f32p, f32p, f32p, i32p, i32p, u8p, vp]
    lib.sbsa_select_ws.argtypes = [P, f32p, f32p, f32p, i32p, i32p, u8p, vp, ctypes.c_size_t, vp]
    lib.sbsa_select_workspace_bytes.argtypes = [P]
    lib.sbsa_select_workspace_bytes.restype = ctypes.c_size_t
    lib.sbsa_score_centroids.argtypes = [P, f32p, f32p, f32p, vp, ctypes.c_size_t, vp]
    lib.sbsa_score_centroids_workspace_bytes.argtypes = [P]
    lib.sbsa_score_centroids_workspace_bytes.restype = ctypes.c_size_t
    lib.sbsa_score_rowmax.argtypes = [P, vp, f32p, f32p, vp, ctypes.c_size_t, vp]
    lib.sbsa_score_rowmax_workspace_bytes.argtypes = [P]
    lib.sbsa_score_rowmax_workspace_bytes.restype = ctypes.c_size_t
    lib.sbsa_select_scores.argtypes = [P, f32p, i32p, i32p, u8p, vp, ctypes.c_size_t, vp]
    lib.sbsa_select_gate_partial.argtypes = [P, f32p, f32p, f32p, i32p, i32p, u8p, vp,
                                             ctypes.c_size_t, vp, vp]
    lib.sbsa_select_gate_finish.argtypes = [P, f32p, f32p, f32p, i32p, i32p, u8p, vp,
                                            ctypes.c_size_t, vp, ci, vp]
    lib.sbsa_attend.argtypes = [P, vp, vp, vp, i32p, i32p, vp, vp]
    lib.sbsa_prefill.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, i32p, i32p, u8p, vp]
    lib.sbsa_prefill_workspace_bytes.argtypes = [P]
    lib.sbsa_prefill_workspace_bytes.restype = ctypes.c_size_t
    lib.sbsa_prefill_host.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.sbsa_prefill_host_workspace_bytes.argtypes = [P]
    lib.sbsa_prefill_host_workspace_bytes.restype = ctypes.c_size_t
    lib.sbsa_get_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
    lib.sbsa_status_string.argtypes = [ci]
    lib.sbsa_status_string.restype = ctypes.c_char_p
    lib.sbsa_version.argtypes = []
    lib.sbsa_debug_wait_timeout.argtypes = [ctypes.c_uint64, vp]
    lib.sbsa_exp2_fma_eval.argtypes = [f32p, f32p, ctypes.c_int64, vp]
    for name in ["sbsa_pool_blocks", "sbsa_select", "sbsa_attend", "sbsa_prefill",
                 "sbsa_get_status", "sbsa_version", "sbsa_debug_wait_timeout"]:
        getattr(lib, name).restype = ctypes.c_int
    return lib


lib = _load()


def status_string(code: int) -> str:
    return lib.sbsa_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != OK:
        raise SbsaError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def make_params(*, n_q_heads, n_kv_heads, seq_len, head_dim, block_size, dtype="bf16",
                select_mode="topk", top_k=0, mass_threshold=0.0, rescue_tau=None,
                gate_margin=None, group_shared=False, index_dim=0, max_blocks=None,
                sm_scale=0.0, score_scale=0.0, backbone="mean", gate_quantile=None,
                gate_rho=2, tile_score="mean") -> Params:
    p = Params()
    p.n_q_heads, p.n_kv_heads, p.seq_len = n_q_heads, n_kv_heads, seq_len
    p.head_dim, p.block_size = head_dim, block_size
    p.dtype = {"bf16": BF16, "fp32": FP32}[dtype] if isinstance(dtype, str) else int(dtype)
    p.select_mode = {"topk": TOPK, "cummass": CUMMASS}[select_mode] if isinstance(select_mode, str) else int(select_mode)
    p.group_shared = 1 if group_shared else 0
    p.index_dim = index_dim
    p.top_k = top_k
    p.mass_threshold = mass_threshold
    p.rescue = 0 if rescue_tau is None else 1
    p.rescue_tau = 0.0 if rescue_tau is None else float(rescue_tau)
    if gate_margin is not None and gate_quantile is not None:
        raise ValueError("choose one gate: gate_margin (gap) or gate_quantile (percentile)")
    p.gate = GATE_GAP if gate_margin is not None else (
        GATE_PERCENTILE if gate_quantile is not None else 0)
    p.gate_margin = 0.0 if gate_margin is None else float(gate_margin)
    p.gate_quantile = 0.0 if gate_quantile is None else float(gate_quantile)
    p.gate_rho = int(gate_rho)
    p.tile_score = ({"mean": TILE_MEAN, "rowmax": TILE_ROWMAX}[tile_score]
                    if isinstance(tile_score, str) else int(tile_score))
    nb = (seq_len + block_size - 1) // block_size
    if max_blocks is None:
        if p.select_mode == CUMMASS or p.rescue:
            max_blocks = nb
        else:
            budget = {0: top_k, GATE_GAP: 2 * top_k, GATE_PERCENTILE: p.gate_rho * top_k}[p.gate]
            max_blocks = min(budget, nb - 1) + 1
    p.max_blocks = max_blocks
    p.sm_scale = sm_scale
    p.score_scale = score_scale
    p.backbone = ({"mean": BACKBONE_MEAN, "minmax": BACKBONE_MINMAX}[backbone]
                  if isinstance(backbone, str) else int(backbone))
    return p


def params_for(w) -> Params:
    """Parameters of a workload description (block_sparse_attention_sbsa_b200.workloads)."""
    return make_params(n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, seq_len=w.seq_len,
                       head_dim=w.head_dim, block_size=w.block_size, dtype=w.dtype,
                       select_mode=w.select_mode, top_k=w.top_k,
                       mass_threshold=w.mass_threshold, rescue_tau=w.rescue_tau,
                       gate_margin=w.gate_margin, group_shared=w.group_shared,
                       index_dim=w.index_dim, max_blocks=w.max_blocks,
                       backbone=getattr(w, "backbone", "mean"),
                       gate_quantile=getattr(w, "gate_quantile", None),
                       gate_rho=getattr(w, "gate_rho", 2),
                       tile_score=getattr(w, "tile_score", "mean"))


_TORCH_DT = {BF16: torch.bfloat16, FP32: torch.float32}


def pool_blocks(p: Params, x: torch.Tensor, group: int = 1, radius: bool = False, stream=None):
    """Centroids [H/group, NB, dim] (and radii [H, NB]) of x [H, N, dim]."""
    _need(x, "x", _TORCH_DT[p.dtype])
    h, n, dim = x.shape
    if n != p.seq_len:
        raise ValueError("x.shape[1] must equal seq_len")
    nb = p.n_blocks
    cent = torch.empty(h // group, nb, dim, device=x.device, dtype=torch.float32)
    rad = torch.empty(h, nb, device=x.device, dtype=torch.float32) if radius else None
    _check(lib.sbsa_pool_blocks(ctypes.byref(p), _ptr(x), h, dim, group, _ptr(cent), _ptr(rad),
                                _stream(stream)), "sbsa_pool_blocks")
    return cent, rad


def pool_minmax(p: Params, x: torch.Tensor, stream=None):
    """Coordinate-wise minimum and maximum of each block of x [H, N, dim]:
    a [H, NB, 2, dim] table (minima, then maxima)."""
    _need(x, "x", _TORCH_DT[p.dtype])
    h, n, dim = x.shape
    if n != p.seq_len:
        raise ValueError("x.shape[1] must equal seq_len")
    mm = torch.empty(h, p.n_blocks, 2, dim, device=x.device, dtype=torch.float32)
    _check(lib.sbsa_pool_minmax(ctypes.byref(p), _ptr(x), h, dim, _ptr(mm), _stream(stream)),
           "sbsa_pool_minmax")
    return mm


def select(p: Params, q_cent: torch.Tensor, k_cent: torch.Tensor,
           k_radius: Optional[torch.Tensor] = None, stream=None, with_flags: bool = True,
           fma_scores: bool = False):
    """Block lists (idx [Hs, NB, Kmax], cnt [Hs, NB], flags [Hs, NB]).  k_cent
    is the centroid table [Hkv, NB, ds], or the min/max table [Hkv, NB, 2, ds]
    of pool_minmax when p.backbone is BACKBONE_MINMAX.  Calls sbsa_select_ws
    (centroid scores on the tensor cores), or with fma_scores sbsa_select
    (fp32 FMA scores inside the selection kernel; no percentile gate)."""
    nb, hs, ds = p.n_blocks, p.n_sel_heads, p.score_dim
    _need(q_cent, "q_cent", torch.float32, (hs, nb, ds))
    kshape = (p.n_kv_heads, nb, 2, ds) if p.backbone == BACKBONE_MINMAX else (p.n_kv_heads, nb, ds)
    _need(k_cent, "k_cent", torch.float32, kshape)
    if p.rescue:
        _need(k_radius, "k_radius", torch.float32, (p.n_kv_heads, nb))
    dev = q_cent.device
    idx = torch.empty(hs, nb, p.max_blocks, device=dev, dtype=torch.int32)
    cnt = torch.empty(hs, nb, device=dev, dtype=torch.int32)
    flags = torch.empty(hs, nb, device=dev, dtype=torch.uint8) if with_flags else None
    if fma_scores:
        _check(lib.sbsa_select(ctypes.byref(p), _ptr(q_cent), _ptr(k_cent),
                               _ptr(k_radius) if p.rescue else None, _ptr(idx), _ptr(cnt),
                               _ptr(flags), _stream(stream)), "sbsa_select")
        return idx, cnt, flags
    wsb = int(lib.sbsa_select_workspace_bytes(ctypes.byref(p)))
    ws = torch.empty(wsb, device=dev, dtype=torch.uint8) if wsb else None
    _check(lib.sbsa_select_ws(ctypes.byref(p), _ptr(q_cent), _ptr(k_cent),
                              _ptr(k_radius) if p.rescue else None, _ptr(idx), _ptr(cnt),
                              _ptr(flags), _ptr(ws), wsb, _stream(stream)), "sbsa_select_ws")
    return idx, cnt, flags


def score_centroids(p: Params, q_cent: torch.Tensor, k_cent: torch.Tensor, stream=None):
    """Centroid scores [Hs, NB, NB] on the tensor cores (entries j < i of row i
    are defined, the rest stay 0)."""
    nb, hs, ds = p.n_blocks, p.n_sel_heads, p.score_dim
    _need(q_cent, "q_cent", torch.float32, (hs, nb, ds))
    _need(k_cent, "k_cent", torch.float32, (p.n_kv_heads, nb, ds))
    dev = q_cent.device
    scores = torch.zeros(hs, nb, nb, device=dev, dtype=torch.float32)
    wsb = int(lib.sbsa_score_centroids_workspace_bytes(ctypes.byref(p)))
    ws = torch.empty(max(wsb, 1), device=dev, dtype=torch.uint8)
    _check(lib.sbsa_score_centroids(ctypes.byref(p), _ptr(q_cent), _ptr(k_cent), _ptr(scores),
                                    _ptr(ws), wsb, _stream(stream)), "sbsa_score_centroids")
    return scores


def score_rowmax(p: Params, q_src: torch.Tensor, k_cent: torch.Tensor, stream=None):
    """Row-max tile scores [Hs, NB, NB] (entries j < i of row i are defined)."""
    nb, hs, ds = p.n_blocks, p.n_sel_heads, p.score_dim
    _need(q_src, "q_src", torch.bfloat16, (p.n_q_heads, p.seq_len, ds))
    _need(k_cent, "k_cent", torch.float32, (p.n_kv_heads, nb, ds))
    dev = q_src.device
    scores = torch.zeros(hs, nb, nb, device=dev, dtype=torch.float32)
    wsb = int(lib.sbsa_score_rowmax_workspace_bytes(ctypes.byref(p)))
    ws = torch.empty(max(wsb, 1), device=dev, dtype=torch.uint8)
    _check(lib.sbsa_score_rowmax(ctypes.byref(p), _ptr(q_src), _ptr(k_cent), _ptr(scores),
                                 _ptr(ws), wsb, _stream(stream)), "sbsa_score_rowmax")
    return scores


def select_scores(p: Params, scores: torch.Tensor, stream=None):
    """Block lists from a precomputed tile-score table [Hs, NB, NB]."""
    nb, hs = p.n_blocks, p.n_sel_heads
    _need(scores, "scores", torch.float32, (hs, nb, nb))
    dev = scores.device
    idx = torch.empty(hs, nb, p.max_blocks, device=dev, dtype=torch.int32)
    cnt = torch.empty(hs, nb, device=dev, dtype=torch.int32)
    flags = torch.empty(hs, nb, device=dev, dtype=torch.uint8)
    wsb = int(lib.sbsa_select_workspace_bytes(ctypes.byref(p)))
    ws = torch.empty(wsb, device=dev, dtype=torch.uint8) if wsb else None
    _check(lib.sbsa_select_scores(ctypes.byref(p), _ptr(scores), _ptr(idx), _ptr(cnt),
                                  _ptr(flags), _ptr(ws), wsb, _stream(stream)),
           "sbsa_select_scores")
    return idx, cnt, flags


def attend(p: Params, q, k, v, idx, cnt, out=None, stream=None):
    """O [Hq, N, d] of attention restricted to the listed blocks."""
    dt = _TORCH_DT[p.dtype]
    _need(q, "q", dt, (p.n_q_heads, p.seq_len, p.head_dim))
    _need(k, "k", dt, (p.n_kv_heads, p.seq_len, p.head_dim))
    _need(v, "v", dt, (p.n_kv_heads, p.seq_len, p.head_dim))
    _need(idx, "idx", torch.int32, (p.n_sel_heads, p.n_blocks, p.max_blocks))
    _need(cnt, "cnt", torch.int32, (p.n_sel_heads, p.n_blocks))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", dt, q.shape)
    _check(lib.sbsa_attend(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt),
                           _ptr(out), _stream(stream)), "sbsa_attend")
    return out


def workspace_bytes(p: Params) -> int:
    n = lib.sbsa_prefill_workspace_bytes(ctypes.byref(p))
    if n == 0:
        raise SbsaError(ERR_INVALID_ARG, "sbsa_prefill_workspace_bytes")
    return int(n)


class Prefill:
    """Reusable prefill call: owns the workspace and optional list outputs so
    repeated calls allocate nothing."""

    def __init__(self, p: Params, device="cuda", keep_lists: bool = True):
        self.p = p
        self.ws = torch.empty(workspace_bytes(p), device=device, dtype=torch.uint8)
        nb, hs = p.n_blocks, p.n_sel_heads
        if keep_lists:
            self.idx = torch.empty(hs, nb, p.max_blocks, device=device, dtype=torch.int32)
            self.cnt = torch.empty(hs, nb, device=device, dtype=torch.int32)
            self.flags = torch.empty(hs, nb, device=device, dtype=torch.uint8)
        else:
            self.idx = self.cnt = self.flags = None

    def __call__(self, q, k, v, q_idx=None, k_idx=None, out=None, stream=None):
        p = self.p
        dt = _TORCH_DT[p.dtype]
        _need(q, "q", dt, (p.n_q_heads, p.seq_len, p.head_dim))
        _need(k, "k", dt, (p.n_kv_heads, p.seq_len, p.head_dim))
        _need(v, "v", dt, (p.n_kv_heads, p.seq_len, p.head_dim))
        if p.index_dim:
            _need(q_idx, "q_idx", dt, (p.n_q_heads, p.seq_len, p.index_dim))
            _need(k_idx, "k_idx", dt, (p.n_kv_heads, p.seq_len, p.index_dim))
        if out is None:
            out = torch.empty_like(q)
        _check(lib.sbsa_prefill(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
                                _ptr(q_idx) if p.index_dim else None,
                                _ptr(k_idx) if p.index_dim else None, _ptr(out), _ptr(self.ws),
                                self.ws.numel(), _ptr(self.idx), _ptr(self.cnt), _ptr(self.flags),
                                _stream(stream)), "sbsa_prefill")
        return out


class PrefillHost:
    """Reusable prefill from host tensors to a host output through
    sbsa_prefill_host (one C call per request; the library pipelines the
    copies and the computation over chunks of kv heads).  Host tensors
    should be pinned; they must stay untouched until the stream has
    completed the request."""

    def __init__(self, p: Params, device="cuda"):
        self.p = p
        n = int(lib.sbsa_prefill_host_workspace_bytes(ctypes.byref(p)))
        if n == 0:
            raise SbsaError(ERR_INVALID_ARG, "sbsa_prefill_host_workspace_bytes")
        self.ws = torch.empty(n, device=device, dtype=torch.uint8)

    def __call__(self, q, k, v, out, q_idx=None, k_idx=None, stream=None):
        p = self.p
        dt = _TORCH_DT[p.dtype]
        for t, name, shape in ((q, "q", (p.n_q_heads, p.seq_len, p.head_dim)),
                               (k, "k", (p.n_kv_heads, p.seq_len, p.head_dim)),
                               (v, "v", (p.n_kv_heads, p.seq_len, p.head_dim)),
                               (out, "out", (p.n_q_heads, p.seq_len, p.head_dim))):
            if t.device.type != "cpu" or t.dtype != dt or tuple(t.shape) != shape \
                    or not t.is_contiguous():
                raise ValueError(f"{name}: expected a contiguous host {dt} tensor of {shape}")
        _check(lib.sbsa_prefill_host(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
                                     _ptr(q_idx) if p.index_dim else None,
                                     _ptr(k_idx) if p.index_dim else None, _ptr(out),
                                     _ptr(self.ws), self.ws.numel(), _stream(stream)),
               "sbsa_prefill_host")
        return out


def prefill(p: Params, q, k, v, q_idx=None, k_idx=None, stream=None):
    """One-shot prefill; returns (O, idx, cnt, flags)."""
    call = Prefill(p, device=q.device)
    out = call(q, k, v, q_idx, k_idx, stream=stream)
    return out, call.idx, call.cnt, call.flags


def debug_wait_timeout(timeout_ns: int, stream=None):
    """Launch the bounded-wait probe (see include/sbsa.h)."""
    _check(lib.sbsa_debug_wait_timeout(int(timeout_ns), _stream(stream)),
           "sbsa_debug_wait_timeout")


def exp2_fma_eval(x: torch.Tensor, stream=None) -> torch.Tensor:
    """exp2 on the FMA pipe (the attention softmax's option) of each element
    of a float32 CUDA tensor (see include/sbsa.h)."""
    if x.dtype != torch.float32 or not x.is_cuda:
        raise ValueError("x must be a float32 CUDA tensor")
    x = x.contiguous()
    y = torch.empty_like(x)
    _check(lib.sbsa_exp2_fma_eval(_ptr(x), _ptr(y), x.numel(), _stream(stream)),
           "sbsa_exp2_fma_eval")
    return y


def get_status(stream=None) -> int:
    """Synchronise the stream and read/clear the device status word."""
    st = ctypes.c_int(0)
    _check(lib.sbsa_get_status(_stream(stream), ctypes.byref(st)), "sbsa_get_status")
    return st.value


class Staged:
    """The prefill as its separate C-ABI stages on preallocated buffers:
    pool keys (centroids + radii, or the min/max table of the upper-bound
    backbone), pool queries (or the row-max tile scores), select (with the
    mean backbone: tf32 split, tensor-core centroid scores, selection), attend.
    Each method is one or two library calls and allocates nothing; the kernels
    are the ones sbsa_prefill launches (which merges the two pooling jobs into
    one grid)."""

    def __init__(self, p: Params, device="cuda"):
        self.p = p
        nb, hs, ds, hk = p.n_blocks, p.n_sel_heads, p.score_dim, p.n_kv_heads
        f32 = dict(device=device, dtype=torch.float32)
        self.minmax = p.backbone == BACKBONE_MINMAX
        self.kc = torch.empty((hk, nb, 2, ds) if self.minmax else (hk, nb, ds), **f32)
        self.kr = torch.empty(hk, nb, **f32) if p.rescue else None
        self.qc = torch.empty(hs, nb, ds, **f32)
        self.idx = torch.empty(hs, nb, p.max_blocks, device=device, dtype=torch.int32)
        self.cnt = torch.empty(hs, nb, device=device, dtype=torch.int32)
        self.flags = torch.empty(hs, nb, device=device, dtype=torch.uint8)
        self.rowmax = p.tile_score == TILE_ROWMAX
        self.scores = torch.empty(hs, nb, nb, **f32) if self.rowmax else None
        self.rm_bytes = int(lib.sbsa_score_rowmax_workspace_bytes(ctypes.byref(p)))
        self.rm_ws = (torch.empty(self.rm_bytes, device=device, dtype=torch.uint8)
                      if self.rowmax else None)
        self.ws_bytes = int(lib.sbsa_select_workspace_bytes(ctypes.byref(p)))
        self.ws = (torch.empty(self.ws_bytes, device=device, dtype=torch.uint8)
                   if self.ws_bytes else None)
        self.tile_sums = None
        self._p = ctypes.byref(p)

    def pool(self, q_src, k_src, stream=None):
        p, s = self.p, _stream(stream)
        ds = p.score_dim
        grp = (p.n_q_heads // p.n_kv_heads) if p.group_shared else 1
        if self.minmax:
            _check(lib.sbsa_pool_minmax(self._p, _ptr(k_src), p.n_kv_heads, ds, _ptr(self.kc), s),
                   "sbsa_pool_minmax")
        else:
            _check(lib.sbsa_pool_blocks(self._p, _ptr(k_src), p.n_kv_heads, ds, 1, _ptr(self.kc),
                                        _ptr(self.kr), s), "sbsa_pool_blocks")
        if self.rowmax:
            # the tile scores read the query rows themselves
            _check(lib.sbsa_score_rowmax(self._p, _ptr(q_src), _ptr(self.kc), _ptr(self.scores),
                                         _ptr(self.rm_ws), self.rm_bytes, s), "sbsa_score_rowmax")
            return
        _check(lib.sbsa_pool_blocks(self._p, _ptr(q_src), p.n_q_heads, ds, grp, _ptr(self.qc),
                                    None, s), "sbsa_pool_blocks")

    def select(self, stream=None, exchange=None, total_heads=None):
        """The selection stage.  Under the percentile gate with several
        processes sharing one sequence by kv head, `exchange(tile_sums)` sums
        the per-tile margin sums (a device float64 tensor [NB]) over the
        processes in place (an all-reduce), and `total_heads` is the number of
        selection heads over all of them; the gate then decides every tile on
        the mean over all heads."""
        p = self.p
        if exchange is not None and p.gate == GATE_PERCENTILE and not self.rowmax:
            if self.tile_sums is None:
                self.tile_sums = torch.empty(p.n_blocks, device=self.qc.device,
                                             dtype=torch.float64)
            args = (self._p, _ptr(self.qc), _ptr(self.kc), _ptr(self.kr), _ptr(self.idx),
                    _ptr(self.cnt), _ptr(self.flags), _ptr(self.ws), self.ws_bytes)
            _check(lib.sbsa_select_gate_partial(*args, _ptr(self.tile_sums), _stream(stream)),
                   "sbsa_select_gate_partial")
            exchange(self.tile_sums)
            _check(lib.sbsa_select_gate_finish(*args, _ptr(self.tile_sums),
                                               int(total_heads or p.n_sel_heads),
                                               _stream(stream)), "sbsa_select_gate_finish")
            return
        if self.rowmax:
            _check(lib.sbsa_select_scores(self._p, _ptr(self.scores), _ptr(self.idx),
                                          _ptr(self.cnt), _ptr(self.flags), _ptr(self.ws),
                                          self.ws_bytes, _stream(stream)), "sbsa_select_scores")
            return
        _check(lib.sbsa_select_ws(self._p, _ptr(self.qc), _ptr(self.kc), _ptr(self.kr),
                                  _ptr(self.idx), _ptr(self.cnt), _ptr(self.flags),
                                  _ptr(self.ws), self.ws_bytes, _stream(stream)),
               "sbsa_select_ws")

    def attend(self, q, k, v, out, stream=None):
        _check(lib.sbsa_attend(self._p, _ptr(q), _ptr(k), _ptr(v), _ptr(self.idx),
                               _ptr(self.cnt), _ptr(out), _stream(stream)), "sbsa_attend")


def attended_pairs(p: Params, cnt: torch.Tensor) -> int:
    """Unmasked (query, key) pairs of the attention over the lists `cnt`
    describes, assuming each list holds valid ids ending with its diagonal
    block: full B x rows for every earlier block, the causal triangle for
    the diagonal block."""
    b, n, nb = p.block_size, p.seq_len, p.n_blocks
    c = cnt.to(torch.int64).cpu()
    rows = torch.full((nb,), b, dtype=torch.int64)
    rows[-1] = n - (nb - 1) * b
    diag = rows * (rows + 1) // 2
    if p.group_shared:
        c = c.repeat_interleave(p.n_q_heads // p.n_kv_heads, dim=0)
    past = ((c - 1).clamp(min=0) * rows.view(1, -1) * b).sum()
    return int(past + (diag.view(1, -1) * (c > 0)).sum())


class PrefillPipeline:
    """Prefills from and to pinned host buffers with copies overlapped.

    Each submitted request copies its inputs host -> device, runs the
    prefill (one sbsa_prefill call) and copies O device -> host.  Two device
    buffer sets and three streams let the next request's input copy and the
    previous request's output copy run while the current prefill computes;
    the order of requests is preserved.  Host tensors must be pinned and
    must stay untouched until `synchronize()` (or the request two
    submissions later) has completed.
    """

    def __init__(self, p: Params, device="cuda", with_index: bool = False):
        self.p = p
        self.device = torch.device(device)
        dt = _TORCH_DT[p.dtype]
        shapes = {"q": (p.n_q_heads, p.seq_len, p.head_dim),
                  "k": (p.n_kv_heads, p.seq_len, p.head_dim),
                  "v": (p.n_kv_heads, p.seq_len, p.head_dim)}
        if p.index_dim:
            shapes["q_idx"] = (p.n_q_heads, p.seq_len, p.index_dim)
            shapes["k_idx"] = (p.n_kv_heads, p.seq_len, p.index_dim)
        self.bufs = [{k: torch.empty(s, dtype=dt, device=self.device) for k, s in shapes.items()}
                     for _ in range(2)]
        self.outs = [torch.empty(shapes["q"], dtype=dt, device=self.device) for _ in range(2)]
        self.calls = [Prefill(p, device=self.device, keep_lists=False) for _ in range(2)]
        self.h2d = torch.cuda.Stream(self.device)
        self.comp = torch.cuda.Stream(self.device)
        self.d2h = torch.cuda.Stream(self.device)
        self.in_free = [torch.cuda.Event() for _ in range(2)]    # compute done with inputs
        self.in_ready = [torch.cuda.Event() for _ in range(2)]   # inputs copied
        self.out_ready = [torch.cuda.Event() for _ in range(2)]  # prefill done
        self.out_free = [torch.cuda.Event() for _ in range(2)]   # output copied back
        self.n = 0

    def submit(self, host_in: dict, host_out: torch.Tensor):
        s = self.n % 2
        bufs, out = self.bufs[s], self.outs[s]
        if self.n >= 2:
            self.h2d.wait_event(self.in_free[s])
        with torch.cuda.stream(self.h2d):
            for name, dev in bufs.items():
                dev.copy_(host_in[name], non_blocking=True)
            self.in_ready[s].record(self.h2d)
        self.comp.wait_event(self.in_ready[s])
        if self.n >= 2:
            self.comp.wait_event(self.out_free[s])
        self.calls[s](bufs["q"], bufs["k"], bufs["v"], bufs.get("q_idx"), bufs.get("k_idx"),
                      out=out, stream=self.comp)
        self.in_free[s].record(self.comp)
        self.out_ready[s].record(self.comp)
        self.d2h.wait_event(self.out_ready[s])
        with torch.cuda.stream(self.d2h):
            host_out.copy_(out, non_blocking=True)
            self.out_free[s].record(self.d2h)
        self.n += 1

    def synchronize(self):
        for st in (self.h2d, self.comp, self.d2h):
            st.synchronize()
