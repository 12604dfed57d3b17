"""KDA oracle -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.

A plain, slow, fp64 CPU statement of what the KDA hot path computes.  Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline leg
and its ``--impl reference`` arm) may import this package.  It shares no code
with the CUDA library in ``gated_delta_rule_123_b200`` and never calls it; the
CUDA library never calls it either.

Sources, cited by page title and section:

* "Kimi Linear: An Expressive, Efficient Attention Architecture" (research
  notes on arXiv 2510.26692) -- section Method / "From Linear Attention to KDA"
  (the DeltaNet step, its residual form, eq. KDA and its S~ reading),
  "Neural Parameterization" (the layer table), "Chunkwise Algorithm"
  (constrained DPLR, C = 64), "Mathematical Rigor" (the corrected cumulative
  decay gamma^{i->j} = prod_{k=i+1}^{j} alpha^k), "Code Verification" (the
  naive recurrence decays first, then writes the residual).
* "Kimi Linear" news rewrite (m.jxzklqfsx.com/article/828570), section
  "Hardware-efficient chunkwise algorithm" (WY representation, UT transform
  by forward substitution, inter-chunk recurrence + intra-chunk output).

Parts:

* ``kda_recurrent``           token-by-token recurrence, residual form (C, OpenMP).
* ``kda_recurrent_product``   the same through the product form of eq. KDA (C).
* ``dplr_recurrent``          untied generic DPLR recurrence, product form (C).
* ``kda_chunkwise``           naive chunkwise evaluation (numpy), any chunk size.
* ``kda_layer``               the full KDA layer (numpy + the recurrence).
* ``kda_recurrent_backward``  reverse mode of the recurrence (numpy): dq, dk, dv,
                              dg, dbeta and the initial-state gradient.
* ``kda_chunkwise_backward`` reverse mode of the chunkwise form (numpy), chunk by
                              chunk: the same six gradients through the gated grams,
                              the WY products and the UT inverse.

Every function is pinned by ``tests/test_oracle_pins.py`` against facts the
pages and plain mathematics fix (special cases, closed forms, invariants, an
autograd gradient step, a hand-derived golden example).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .backward import kda_recurrent_backward  # noqa: F401
from .chunkwise import kda_chunkwise  # noqa: F401
from .chunkwise_backward import kda_chunkwise_backward  # noqa: F401
from .layer import kda_layer, layer_reference_parts  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C part of the oracle (gcc, -O2, OpenMP) next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        llp = ctypes.POINTER(ctypes.c_longlong)
        lib.kda_oracle_recurrent.argtypes = [dp] * 5 + [dp, dp, dp, llp] + [ctypes.c_int] * 4 + [ctypes.c_double]
        lib.kda_oracle_recurrent.restype = None
        lib.kda_oracle_dplr_product.argtypes = [dp] * 7 + [dp, dp, dp, llp] + [ctypes.c_int] * 4 + [ctypes.c_double]
        lib.kda_oracle_dplr_product.restype = None
        lib.kda_oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().kda_oracle_num_threads())


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _pack(q, k, v, g, beta, cu):
    """Accept dense [B,T,H,D] (cu None) or packed [Ttot,H,D] (cu given)."""
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    if cu is None:
        if q.ndim != 4:
            raise ValueError("dense inputs must be [B,T,H,D]")
        B, T, H, DK = q.shape
        DV = v.shape[-1]
        cu = np.arange(B + 1, dtype=np.int64) * T
        shape_o = (B, T, H, DV)
        q, k, g = (a.reshape(B * T, H, DK) for a in (q, k, g))
        v = v.reshape(B * T, H, DV)
        beta = beta.reshape(B * T, H)
    else:
        cu = np.ascontiguousarray(np.asarray(cu, dtype=np.int64))
        H, DK = q.shape[1], q.shape[2]
        DV = v.shape[-1]
        shape_o = (q.shape[0], H, DV)
    return q, k, v, g, beta, cu, shape_o


def kda_recurrent(q, k, v, g, beta, s0=None, cu=None, scale=1.0):
    """KDA, token by token, residual form (decay first, then write the error).

    Returns ``(o, S_T)`` in fp64; ``S_T`` is [N,H,DK,DV].
    """
    q, k, v, g, beta, cu, shape_o = _pack(q, k, v, g, beta, cu)
    N = len(cu) - 1
    H, DK, DV = q.shape[1], q.shape[2], v.shape[2]
    o = np.zeros((q.shape[0], H, DV))
    sT = np.zeros((N, H, DK, DV))
    s0a = None if s0 is None else _f64(s0).reshape(N, H, DK, DV)
    _load().kda_oracle_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0a), _ptr(o),
                                 _ptr(sT), cu.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong)),
                                 N, H, DK, DV, float(scale))
    return o.reshape(shape_o), sT


def dplr_recurrent(q, k, v, g, beta, a, b, s0=None, cu=None, scale=1.0):
    """Generic DPLR recurrence S = (I - a b^T) Diag(exp g) S + beta k v^T, product form."""
    q, k, v, g, beta, cu, shape_o = _pack(q, k, v, g, beta, cu)
    a = _f64(a).reshape(q.shape)
    b = _f64(b).reshape(q.shape)
    N = len(cu) - 1
    H, DK, DV = q.shape[1], q.shape[2], v.shape[2]
    o = np.zeros((q.shape[0], H, DV))
    sT = np.zeros((N, H, DK, DV))
    s0a = None if s0 is None else _f64(s0).reshape(N, H, DK, DV)
    _load().kda_oracle_dplr_product(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(a), _ptr(b),
                                    _ptr(s0a), _ptr(o), _ptr(sT),
                                    cu.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong)),
                                    N, H, DK, DV, float(scale))
    return o.reshape(shape_o), sT


def kda_recurrent_product(q, k, v, g, beta, s0=None, cu=None, scale=1.0):
    """KDA through the product form (I - beta k k^T) Diag(alpha) S + beta k v^T.

    This is the DPLR product-form recurrence with the KDA binding a = beta k,
    b = k ("Chunkwise Algorithm": D = Diag(alpha), a = beta k, b = k (.) alpha,
    the alpha being applied by the Diag factor here).
    """
    kk = _f64(k)
    bb = _f64(beta)[..., None] * kk
    return dplr_recurrent(q, k, v, g, beta, bb, kk, s0=s0, cu=cu, scale=scale)
