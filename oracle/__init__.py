"""fp64 CPU oracle for causal scaled dot-product attention and its gradients.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library and
its Python binding never import it, and it imports nothing from them.

The arithmetic lives in ``attention_oracle.c`` (plain C, double precision,
OpenMP over heads and rows only).  This module builds it with gcc and wraps it
with ctypes; it only marshals numpy arrays.  What each function computes, and
the passages of the pages it follows, is stated in the C file's header:
CS336 A2 Systems handout section 4.1.1 Eq. 1 and section 4.2.2 Eqs. 4-12
(forward, logsumexp), Eqs. 7-11 (standard backward through the softmax
Jacobian), and the causal rule of Problem flash_forward (c).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib: Optional[ctypes.CDLL] = None

_dp = ctypes.POINTER(ctypes.c_double)
_lp = ctypes.POINTER(ctypes.c_long)


def build(force: bool = False) -> str:
    """Compile attention_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP).

    No fast-math: the oracle keeps IEEE double semantics.
    """
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + ".tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-Wall", "-Wextra", "-Werror", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    lib.oracle_max_threads.restype = ctypes.c_int
    lib.oracle_forward.restype = ctypes.c_int
    lib.oracle_forward.argtypes = [_dp, _dp, _dp, _dp, _dp, ctypes.c_long, ctypes.c_long,
                                   ctypes.c_long, ctypes.c_long, ctypes.c_int,
                                   ctypes.c_double]
    lib.oracle_backward.restype = ctypes.c_int
    lib.oracle_backward.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                                    ctypes.c_long, ctypes.c_long, ctypes.c_long,
                                    ctypes.c_long, ctypes.c_int, ctypes.c_double]
    _up = ctypes.POINTER(ctypes.c_ubyte)
    lib.oracle_forward_bs.restype = ctypes.c_int
    lib.oracle_forward_bs.argtypes = [_dp, _dp, _dp, _dp, _dp, ctypes.c_long, ctypes.c_long,
                                      ctypes.c_long, ctypes.c_long, ctypes.c_int, ctypes.c_double,
                                      _up, ctypes.c_long, ctypes.c_long]
    lib.oracle_backward_bs.restype = ctypes.c_int
    lib.oracle_backward_bs.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _dp, ctypes.c_long,
                                       ctypes.c_long, ctypes.c_long, ctypes.c_long, ctypes.c_int,
                                       ctypes.c_double, _up, ctypes.c_long, ctypes.c_long]
    lib.oracle_head_sampled.restype = ctypes.c_int
    lib.oracle_head_sampled.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_long, ctypes.c_long,
                                        ctypes.c_long, ctypes.c_int, ctypes.c_double,
                                        _lp, ctypes.c_long, _lp, ctypes.c_long,
                                        _dp, _dp, _dp, _dp, _dp]
    return lib


def _load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def max_threads() -> int:
    """Threads the oracle's OpenMP regions use (OMP_NUM_THREADS or the core count)."""
    return int(_load().oracle_max_threads())


def _as_f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return ctypes.cast(None, _dp)
    return a.ctypes.data_as(_dp)


def _heads_view(x: np.ndarray):
    """[..., n, d] -> ([heads, n, d], leading shape)."""
    if x.ndim < 2:
        raise ValueError("expected [..., n, d]")
    lead = x.shape[:-2]
    heads = int(np.prod(lead)) if lead else 1
    return x.reshape(heads, x.shape[-2], x.shape[-1]), lead


def forward(q, k, v, causal: bool, scale: float):
    """O and L (natural-log logsumexp) for inputs of shape [..., n, d].

    Returns (o [..., nq, d], lse [..., nq]) as float64.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    qh, lead = _heads_view(q)
    kh, _ = _heads_view(k)
    vh, _ = _heads_view(v)
    heads, nq, d = qh.shape
    nk = kh.shape[1]
    if kh.shape != (heads, nk, d) or vh.shape != kh.shape:
        raise ValueError("q, k, v shapes disagree")
    o = np.empty_like(qh)
    lse = np.empty((heads, nq), dtype=np.float64)
    rc = _load().oracle_forward(_ptr(qh), _ptr(kh), _ptr(vh), _ptr(o), _ptr(lse),
                                heads, nq, nk, d, int(bool(causal)), float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle_forward failed with code {rc}")
    return o.reshape(*lead, nq, d), lse.reshape(*lead, nq)


def backward(q, k, v, dout, causal: bool, scale: float, return_stats: bool = False):
    """dQ, dK, dV (float64) through the softmax Jacobian.

    With ``return_stats`` also returns an array [..., nq, 2] holding, per query
    row, the logsumexp L_i and the Jacobian scalar c_i = sum_j P_ij dP_ij.
    """
    q, k, v, dout = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    qh, lead = _heads_view(q)
    kh, _ = _heads_view(k)
    vh, _ = _heads_view(v)
    doh, _ = _heads_view(dout)
    heads, nq, d = qh.shape
    nk = kh.shape[1]
    if kh.shape != (heads, nk, d) or vh.shape != kh.shape or doh.shape != qh.shape:
        raise ValueError("q, k, v, dout shapes disagree")
    dq = np.empty_like(qh)
    dk = np.empty_like(kh)
    dv = np.empty_like(vh)
    stats = np.empty((heads, nq, 2), dtype=np.float64) if return_stats else None
    rc = _load().oracle_backward(_ptr(qh), _ptr(kh), _ptr(vh), _ptr(doh), _ptr(dq), _ptr(dk),
                                 _ptr(dv), _ptr(stats), heads, nq, nk, d,
                                 int(bool(causal)), float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle_backward failed with code {rc}")
    out = (dq.reshape(*lead, nq, d), dk.reshape(*lead, nk, d), dv.reshape(*lead, nk, d))
    if return_stats:
        return out + (stats.reshape(*lead, nq, 2),)
    return out


def _mask_arg(block_mask, nq: int, nk: int, block_q: int, block_k: int):
    m = np.ascontiguousarray(np.asarray(block_mask) != 0, dtype=np.uint8)
    want = ((nq + block_q - 1) // block_q, (nk + block_k - 1) // block_k)
    if m.shape != want:
        raise ValueError(f"block_mask must have shape {want}, got {m.shape}")
    return m


def forward_block_sparse(q, k, v, causal: bool, scale: float, block_mask,
                         block_q: int = 128, block_k: int = 128):
    """Block-sparse O and L: key j is visible to query i iff
    block_mask[i // block_q, j // block_k] is set (and j <= i under causal).
    Rows that see no key get O = 0 and L = -inf.  Shapes as in forward()."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    qh, lead = _heads_view(q)
    kh, _ = _heads_view(k)
    vh, _ = _heads_view(v)
    heads, nq, d = qh.shape
    nk = kh.shape[1]
    if kh.shape != (heads, nk, d) or vh.shape != kh.shape:
        raise ValueError("q, k, v shapes disagree")
    m = _mask_arg(block_mask, nq, nk, block_q, block_k)
    o = np.empty_like(qh)
    lse = np.empty((heads, nq), dtype=np.float64)
    rc = _load().oracle_forward_bs(_ptr(qh), _ptr(kh), _ptr(vh), _ptr(o), _ptr(lse), heads, nq, nk,
                                   d, int(bool(causal)), float(scale),
                                   m.ctypes.data_as(ctypes.POINTER(ctypes.c_ubyte)),
                                   block_q, block_k)
    if rc != 0:
        raise RuntimeError(f"oracle_forward_bs failed with code {rc}")
    return o.reshape(*lead, nq, d), lse.reshape(*lead, nq)


def backward_block_sparse(q, k, v, dout, causal: bool, scale: float, block_mask,
                          block_q: int = 128, block_k: int = 128):
    """dQ, dK, dV of the block-sparse attention (see forward_block_sparse)."""
    q, k, v, dout = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    qh, lead = _heads_view(q)
    kh, _ = _heads_view(k)
    vh, _ = _heads_view(v)
    doh, _ = _heads_view(dout)
    heads, nq, d = qh.shape
    nk = kh.shape[1]
    if kh.shape != (heads, nk, d) or vh.shape != kh.shape or doh.shape != qh.shape:
        raise ValueError("q, k, v, dout shapes disagree")
    m = _mask_arg(block_mask, nq, nk, block_q, block_k)
    dq = np.empty_like(qh)
    dk = np.empty_like(kh)
    dv = np.empty_like(vh)
    rc = _load().oracle_backward_bs(_ptr(qh), _ptr(kh), _ptr(vh), _ptr(doh), _ptr(dq), _ptr(dk),
                                    _ptr(dv), heads, nq, nk, d, int(bool(causal)), float(scale),
                                    m.ctypes.data_as(ctypes.POINTER(ctypes.c_ubyte)),
                                    block_q, block_k)
    if rc != 0:
        raise RuntimeError(f"oracle_backward_bs failed with code {rc}")
    return dq.reshape(*lead, nq, d), dk.reshape(*lead, nk, d), dv.reshape(*lead, nk, d)


def head_sampled(q, k, v, dout, causal: bool, scale: float, qrows, krows,
                 want_forward: bool = True, want_grad: bool = True):
    """Sampled outputs of one head (q, k, v, dout: [n, d]).

    Returns a dict with 'o', 'lse', 'dq' for the query rows ``qrows`` and 'dk',
    'dv' for the key rows ``krows`` (float64).  Gradients need a full pass over
    the head for every row's normaliser; the rest is per selected row.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    if q.ndim != 2 or k.ndim != 2 or v.shape != k.shape or q.shape[1] != k.shape[1]:
        raise ValueError("head_sampled expects q [nq, d], k and v [nk, d]")
    nq, d = q.shape
    nk = k.shape[0]
    qr = np.ascontiguousarray(np.asarray(qrows, dtype=np.int64)).astype(np.int64)
    kr = np.ascontiguousarray(np.asarray(krows, dtype=np.int64)).astype(np.int64)
    res = {}
    o = np.empty((len(qr), d)) if want_forward else None
    lse = np.empty((len(qr),)) if want_forward else None
    dq = np.empty((len(qr), d)) if want_grad else None
    dk = np.empty((len(kr), d)) if want_grad else None
    dv = np.empty((len(kr), d)) if want_grad else None
    do = _as_f64(dout) if want_grad else None
    if do is not None and do.shape != q.shape:
        raise ValueError("dout must match q")
    rc = _load().oracle_head_sampled(_ptr(q), _ptr(k), _ptr(v), _ptr(do), nq, nk, d,
                                     int(bool(causal)), float(scale),
                                     qr.ctypes.data_as(_lp), len(qr), kr.ctypes.data_as(_lp),
                                     len(kr), _ptr(o), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv))
    if rc != 0:
        raise RuntimeError(f"oracle_head_sampled failed with code {rc}")
    if want_forward:
        res["o"], res["lse"] = o, lse
    if want_grad:
        res["dq"], res["dk"], res["dv"] = dq, dk, dv
    return res


def _swap_library(path: Optional[str]) -> None:
    """Point this module at another build of the oracle, or back at the default
    one when ``path`` is None.  Only the tests that plant mistakes in a copy of
    the C source use this, to show that the pins catch them."""
    global _lib
    _lib = _bind(ctypes.CDLL(path)) if path else None
