"""ctypes front end of the float64 banded C oracle (``oracle/banded.c``).

TEST INFRASTRUCTURE ONLY: used by tests/ and by bench.py's CPU baseline.  Same equations
as ``oracle/eot_oracle.py`` (Blockwise Differentiable Sinkhorn Attention, technical
summary, §2.1-§2.3); band storage instead of a dense matrix so that long sequences fit.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "banded.c")
_LIB = os.path.join(_HERE, "libeot_banded.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile banded.c with gcc + OpenMP into oracle/libeot_banded.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", _SRC, "-o", _LIB, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        up = ctypes.c_void_p
        ip = ctypes.c_void_p
        _lib.eot_banded_forward.argtypes = [ctypes.c_int] * 7 + [ctypes.c_double, dp, dp, dp, up,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                            ip, ctypes.c_int, dp, dp, dp]
        _lib.eot_banded_forward.restype = ctypes.c_int
        _lib.eot_banded_backward.argtypes = [ctypes.c_int] * 6 + [ctypes.c_double, dp, dp, dp, up,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                             ip, ctypes.c_int, dp, dp, dp, dp, dp, dp]
        _lib.eot_banded_backward.restype = ctypes.c_int
    return _lib


def _dp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _prep(Q, K, V, mask, units):
    Q = np.ascontiguousarray(Q, np.float64)
    K = np.ascontiguousarray(K, np.float64)
    V = np.ascontiguousarray(V, np.float64)
    m = None if mask is None else np.ascontiguousarray(mask, np.uint8)
    u = None if units is None else np.ascontiguousarray(units, np.int32)
    return Q, K, V, m, u


def forward(Q, K, V, W, T, R, scale=None, mask=None, dustbin=False, dustbin_index=-1,
            dustbin_mass=0.0, dustbin_self=True, units=None):
    """Banded forward over [B,H,L,d].  ``units``: optional flattened b*H+h indices.

    Returns O [B,H,L,d] and u_tail, v_tail [B,H,R+1,L] (zeros for units not computed)."""
    Q, K, V, m, u = _prep(Q, K, V, mask, units)
    B, H, L, d = Q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.zeros_like(Q)
    ut = np.zeros((B, H, R + 1, L))
    vt = np.zeros((B, H, R + 1, L))
    rc = _load().eot_banded_forward(B, H, L, d, W, T, R, scale, _dp(Q), _dp(K), _dp(V),
                                    None if m is None else m.ctypes.data, int(dustbin), int(dustbin_index),
                                    float(dustbin_mass), int(dustbin_self),
                                    None if u is None else u.ctypes.data, 0 if u is None else len(u),
                                    _dp(O), _dp(ut), _dp(vt))
    if rc != 0:
        raise MemoryError("banded oracle: allocation failed")
    return O, ut, vt


def backward(Q, K, V, dO, u_tail, v_tail, W, scale=None, mask=None, dustbin=False, dustbin_index=-1,
             dustbin_mass=0.0, dustbin_self=True, units=None):
    """Banded tail adjoint.  Returns dQ, dK, dV [B,H,L,d]."""
    Q, K, V, m, u = _prep(Q, K, V, mask, units)
    dO = np.ascontiguousarray(dO, np.float64)
    ut = np.ascontiguousarray(u_tail, np.float64)
    vt = np.ascontiguousarray(v_tail, np.float64)
    B, H, L, d = Q.shape
    R = ut.shape[2] - 1
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(Q)
    dV = np.zeros_like(Q)
    rc = _load().eot_banded_backward(B, H, L, d, W, R, scale, _dp(Q), _dp(K), _dp(V),
                                     None if m is None else m.ctypes.data, int(dustbin), int(dustbin_index),
                                     float(dustbin_mass), int(dustbin_self),
                                     None if u is None else u.ctypes.data, 0 if u is None else len(u),
                                     _dp(ut), _dp(vt), _dp(dO), _dp(dQ), _dp(dK), _dp(dV))
    if rc != 0:
        raise MemoryError("banded oracle: allocation failed")
    return dQ, dK, dV
