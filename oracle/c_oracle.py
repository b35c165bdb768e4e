"""Binding of the plain C oracle (``oracle/c/qlora_oracle.c``): the NF4
codebook, quantiser and dequantiser, one QLoRA projection's forward and
hand-derived backward, and the gated MLP built from three projections, as
loops in binary64, for small configurations.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  ``build()`` compiles
the C file with gcc (ISO C, no fast-math, so binary32 division and products
round as written); the tests check it against the numpy oracle, which pins
each against an independent statement of the same definitions.
"""

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "c", "qlora_oracle.c")
LIB = os.path.join(HERE, "c", "libqlora_oracle.so")

_lib = None
_D = ctypes.POINTER(ctypes.c_double)


class _Proj(ctypes.Structure):
    _fields_ = [("W", _D), ("A", _D), ("B", _D), ("s", ctypes.c_double)]


_KIND = {"swiglu": 0, "geglu_tanh": 1}


def build():
    """Compile the C oracle if it is missing or older than its source."""
    if os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-o", LIB, SRC, "-lm"])
    return LIB


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.oracle_c_nf4_codebook.argtypes = [_D]
        L.oracle_c_nf4_quantize.argtypes = [ctypes.c_void_p, ctypes.c_long, ctypes.c_long, ctypes.c_void_p,
                                             ctypes.c_void_p]
        L.oracle_c_nf4_quantize.restype = ctypes.c_int
        L.oracle_c_nf4_dequantize.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_long, ctypes.c_long, _D]
        L.oracle_c_linear_fwd.argtypes = [_D, _D, _D, _D, ctypes.c_double] + [ctypes.c_long] * 4 + [_D, _D]
        L.oracle_c_linear_bwd.argtypes = ([_D, _D, _D, _D, ctypes.c_double, _D] + [ctypes.c_long] * 4 +
                                          [_D, _D, _D, _D, _D])
        L.oracle_c_mlp_fwd.argtypes = [ctypes.c_int, _D] + [ctypes.c_long] * 4 + [_Proj] * 3 + [_D] * 4
        L.oracle_c_mlp_fwd.restype = ctypes.c_int
        L.oracle_c_mlp_bwd.argtypes = [ctypes.c_int, _D] + [ctypes.c_long] * 4 + [_Proj] * 3 + [_D] * 8
        L.oracle_c_mlp_bwd.restype = ctypes.c_int
        _lib = L
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return a.ctypes.data_as(_D)


def nf4_codebook():
    out = np.empty(16, dtype=np.float64)
    lib().oracle_c_nf4_codebook(_p(out))
    return out


def nf4_quantize(w_bits, n_out, k_in):
    w = np.ascontiguousarray(w_bits, dtype=np.uint16).reshape(-1)
    codes = np.empty(n_out * k_in // 2, dtype=np.uint8)
    absmax = np.empty(n_out * k_in // 64, dtype=np.float32)
    if lib().oracle_c_nf4_quantize(w.ctypes.data, n_out, k_in, codes.ctypes.data, absmax.ctypes.data):
        raise ValueError("k_in must be a multiple of 64")
    return codes, absmax


def nf4_dequantize_f64(codes, absmax, n_out, k_in):
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    a = np.ascontiguousarray(absmax, dtype=np.float32)
    w = np.empty((n_out, k_in), dtype=np.float64)
    lib().oracle_c_nf4_dequantize(c.ctypes.data, a.ctypes.data, n_out, k_in, _p(w))
    return w


def linear_fwd(X, W, A, B, s):
    X, W, A, B = _f64(X), _f64(W), _f64(A), _f64(B)
    M, K = X.shape
    N, r = W.shape[0], A.shape[1]
    Y = np.empty((M, N))
    XA = np.empty((M, r))
    lib().oracle_c_linear_fwd(_p(X), _p(W), _p(A), _p(B), float(s), M, K, N, r, _p(Y), _p(XA))
    return Y, XA


def linear_bwd(X, W, A, B, s, dY):
    X, W, A, B, dY = _f64(X), _f64(W), _f64(A), _f64(B), _f64(dY)
    M, K = X.shape
    N, r = W.shape[0], A.shape[1]
    dX, dA, dB = np.empty((M, K)), np.empty((K, r)), np.empty((r, N))
    G, XA = np.empty((M, r)), np.empty((M, r))
    lib().oracle_c_linear_bwd(_p(X), _p(W), _p(A), _p(B), float(s), _p(dY), M, K, N, r, _p(dX), _p(dA), _p(dB),
                              _p(G), _p(XA))
    return dX, dA, dB


def _proj(p, keep):
    W, A, B = (_f64(a) for a in p[:3])
    keep.extend((W, A, B))  # the arrays must outlive the call
    return _Proj(_p(W), _p(A), _p(B), float(p[3])), W.shape, A.shape[1]


def mlp_fwd(kind, X, gate, up, down):
    """Gated MLP forward; gate/up/down are (W, A, B, s).  Returns Y, E, G, H."""
    keep = []
    X = _f64(X)
    M, d = X.shape
    pg, (h, _), r = _proj(gate, keep)
    pu, _, _ = _proj(up, keep)
    pd, _, _ = _proj(down, keep)
    E, G, H, Y = np.empty((M, h)), np.empty((M, h)), np.empty((M, h)), np.empty((M, d))
    if lib().oracle_c_mlp_fwd(_KIND[kind], _p(X), M, d, h, r, pg, pu, pd, _p(E), _p(G), _p(H), _p(Y)):
        raise MemoryError("oracle_c_mlp_fwd")
    return {"Y": Y, "E": E, "G": G, "H": H}


def mlp_bwd(kind, X, gate, up, down, dY):
    """Gated MLP backward: dX and the six adapter gradients."""
    keep = []
    X, dY = _f64(X), _f64(dY)
    M, d = X.shape
    pg, (h, _), r = _proj(gate, keep)
    pu, _, _ = _proj(up, keep)
    pd, _, _ = _proj(down, keep)
    out = {"dX": np.empty((M, d)), "dA_g": np.empty((d, r)), "dB_g": np.empty((r, h)), "dA_u": np.empty((d, r)),
           "dB_u": np.empty((r, h)), "dA_d": np.empty((h, r)), "dB_d": np.empty((r, d))}
    args = [_p(out[k]) for k in ("dX", "dA_g", "dB_g", "dA_u", "dB_u", "dA_d", "dB_d")]
    if lib().oracle_c_mlp_bwd(_KIND[kind], _p(X), M, d, h, r, pg, pu, pd, _p(dY), *args):
        raise MemoryError("oracle_c_mlp_bwd")
    return out
