"""ctypes binding of libqlora (include/qlora.h), with the same entry-point names.

Argument marshalling only: tensors are PyTorch CUDA tensors (device memory and
streams), their data pointers and the current stream are passed to the C ABI,
and every step of the computation runs in the library's CUDA kernels.  There
is no CPU fallback: if ``lib/libqlora.so`` is missing, every call raises.

With the environment variable QLORA_LIBRARY=checked the binding loads the
bounds-checked debug build ``lib/libqlora_check.so`` instead (same ABI; its
kernels report an out-of-range index through the status word rather than
touching memory out of range).
"""

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libqlora.so")
CHECK_LIB_PATH = os.path.join(_PKG, "lib", "libqlora_check.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "qlora.h")

QLORA_OK = 0
QLORA_ACT = {"swiglu": 0, "geglu_tanh": 1}
STATUS_NAMES = {0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARG", 2: "QLORA_ERR_UNSUPPORTED_SHAPE",
                3: "QLORA_ERR_MISALIGNED", 4: "QLORA_ERR_WORKSPACE_TOO_SMALL", 5: "QLORA_ERR_CUDA",
                6: "QLORA_ERR_TIMEOUT", 7: "QLORA_ERR_DEVICE"}


class QloraNF4(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("absmax", ctypes.c_void_p),
                ("n_out", ctypes.c_int64), ("k_in", ctypes.c_int64)]


class QloraLoraLinear(ctypes.Structure):
    _fields_ = [("w", QloraNF4), ("A", ctypes.c_void_p), ("B", ctypes.c_void_p),
                ("r", ctypes.c_int32), ("scale", ctypes.c_float)]


class QloraLoraLinear16(ctypes.Structure):
    _fields_ = [("w", ctypes.c_void_p), ("n_out", ctypes.c_int64), ("k_in", ctypes.c_int64), ("A", ctypes.c_void_p),
                ("B", ctypes.c_void_p), ("r", ctypes.c_int32), ("scale", ctypes.c_float)]


class QloraMlpSaved(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("E", "G", "H", "XA_g", "XA_u", "HA_d")]


class QloraTraceEntry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int64), ("total_ms", ctypes.c_double)]


class QloraError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


_lib = None

_SIGS = {
    "qlora_nf4_codebook": (ctypes.c_int, [ctypes.c_void_p]),
    "nf4_quantize": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_void_p]),
    "nf4_dequantize": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_linear_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                                       ctypes.c_int32]),
    "qlora_linear_fwd": (ctypes.c_int, [ctypes.POINTER(QloraLoraLinear), ctypes.c_void_p, ctypes.c_int64,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                        ctypes.c_void_p]),
    "qlora_linear_bwd": (ctypes.c_int, [ctypes.POINTER(QloraLoraLinear), ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_mlp_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                                    ctypes.c_int32]),
    "qlora_mlp_fwd": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(QloraLoraLinear),
                                     ctypes.POINTER(QloraLoraLinear), ctypes.POINTER(QloraLoraLinear),
                                     ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                     ctypes.POINTER(QloraMlpSaved), ctypes.c_void_p, ctypes.c_size_t,
                                     ctypes.c_void_p]),
    "qlora_mlp_bwd": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(QloraLoraLinear),
                                     ctypes.POINTER(QloraLoraLinear), ctypes.POINTER(QloraLoraLinear),
                                     ctypes.c_void_p, ctypes.POINTER(QloraMlpSaved), ctypes.c_void_p,
                                     ctypes.c_int64] + [ctypes.c_void_p] * 8 + [ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_mlp_bwd_ev": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(QloraLoraLinear),
                                        ctypes.POINTER(QloraLoraLinear), ctypes.POINTER(QloraLoraLinear),
                                        ctypes.c_void_p, ctypes.POINTER(QloraMlpSaved), ctypes.c_void_p,
                                        ctypes.c_int64] + [ctypes.c_void_p] * 8 +
                         [ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_mlp16_bwd_ev": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(QloraLoraLinear16),
                                          ctypes.POINTER(QloraLoraLinear16), ctypes.POINTER(QloraLoraLinear16),
                                          ctypes.c_void_p, ctypes.POINTER(QloraMlpSaved), ctypes.c_void_p,
                                          ctypes.c_int64] + [ctypes.c_void_p] * 8 +
                           [ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_last_device_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_test_inject_timeout": (ctypes.c_int, []),
    "qlora_test_set_grid_cap": (ctypes.c_int32, [ctypes.c_int32]),
    "qlora_test_shrink_next_slot_cap": (ctypes.c_int, []),
    "qlora_checked_build": (ctypes.c_int32, []),
    "qlora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "qlora_set_tile_config": (ctypes.c_int32, [ctypes.c_int32]),
    "qlora_mlp_tile_config": (ctypes.c_int32, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32]),
    "qlora_trace_begin": (ctypes.c_int, []),
    "qlora_trace_begin_only": (ctypes.c_int, [ctypes.c_char_p]),
    "qlora_trace_end": (ctypes.c_int32, [ctypes.POINTER(QloraTraceEntry), ctypes.c_int32]),
    "qlora_launch_count": (ctypes.c_uint64, []),
    "qlora_linear_fwd_noalloc": (ctypes.c_int, [ctypes.POINTER(QloraLoraLinear), ctypes.c_void_p, ctypes.c_int64,
                                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_rmsnorm_fwd": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_float, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_void_p]),
    "qlora_rmsnorm_bwd": (ctypes.c_int, [ctypes.c_void_p] * 4 + [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                                                 ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_qkv_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64] * 5 + [ctypes.c_int32]),
    "qlora_qkv_fwd": (ctypes.c_int, [ctypes.POINTER(QloraLoraLinear)] * 3 + [ctypes.c_void_p, ctypes.c_int64,
                                                                             ctypes.c_void_p, ctypes.c_void_p,
                                                                             ctypes.c_void_p, ctypes.c_size_t,
                                                                             ctypes.c_void_p]),
    "qlora_qkv_bwd": (ctypes.c_int, [ctypes.POINTER(QloraLoraLinear)] * 3 + [ctypes.c_void_p] * 3 +
                      [ctypes.c_int64] + [ctypes.c_void_p] * 8 + [ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_linear16_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                                         ctypes.c_int32]),
    "qlora_mlp16_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                                      ctypes.c_int32]),
    "qlora_linear16_fwd": (ctypes.c_int, [ctypes.POINTER(QloraLoraLinear16), ctypes.c_void_p, ctypes.c_int64,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                          ctypes.c_void_p]),
    "qlora_linear16_bwd": (ctypes.c_int, [ctypes.POINTER(QloraLoraLinear16), ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_mlp16_fwd": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(QloraLoraLinear16),
                                       ctypes.POINTER(QloraLoraLinear16), ctypes.POINTER(QloraLoraLinear16),
                                       ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                       ctypes.POINTER(QloraMlpSaved), ctypes.c_void_p, ctypes.c_size_t,
                                       ctypes.c_void_p]),
    "qlora_mlp16_bwd": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(QloraLoraLinear16),
                                       ctypes.POINTER(QloraLoraLinear16), ctypes.POINTER(QloraLoraLinear16),
                                       ctypes.c_void_p, ctypes.POINTER(QloraMlpSaved), ctypes.c_void_p,
                                       ctypes.c_int64] + [ctypes.c_void_p] * 8 + [ctypes.c_size_t, ctypes.c_void_p]),
}


def _load(path):
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m qlora_fine_tuning_nf4_b200.build`")
    L = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


def lib():
    """Load libqlora.so, or libqlora_check.so under QLORA_LIBRARY=checked (raises if it has not been built)."""
    global _lib
    if _lib is None:
        choice = os.environ.get("QLORA_LIBRARY", "")
        if choice not in ("", "checked"):
            raise RuntimeError(f"QLORA_LIBRARY={choice!r}: expected unset or 'checked'")
        _lib = _load(CHECK_LIB_PATH if choice == "checked" else LIB_PATH)
    return _lib


_check_lib = None


def checked_lib():
    """Load the bounds-checked debug build, libqlora_check.so (same ABI; its
    kernels report out-of-range indices as QLORA_ERR_DEVICE instead of
    touching memory out of range)."""
    global _check_lib
    if _check_lib is None:
        _check_lib = _load(CHECK_LIB_PATH)
    return _check_lib


_normal_lib = None


def normal_lib():
    """Load the normal build, libqlora.so, whatever QLORA_LIBRARY selects."""
    global _normal_lib
    if _normal_lib is None:
        _normal_lib = _load(LIB_PATH)
    return _normal_lib


class use_library:
    """Context manager that routes every wrapper of this module to another
    build of the library (e.g. checked_lib()) and restores the previous one."""

    def __init__(self, L):
        self.L = L

    def __enter__(self):
        global _lib
        self.prev = lib()
        _lib = self.L
        return self.L

    def __exit__(self, *exc):
        global _lib
        _lib = self.prev
        return False


def _check(fn, status):
    if status != QLORA_OK:
        raise QloraError(fn, status)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _dev(t, name):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    return t


def _t(t, name, shape, dtype=torch.bfloat16):
    """Marshalling check of one tensor argument: contiguous, on the current
    CUDA device, of the expected dtype and shape.  The C ABI only sees raw
    pointers, so a host tensor or a short buffer must be caught here."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor, got one on {t.device}")
    if t.get_device() != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, not on the current device cuda:{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _rows(X, name="X"):
    if not isinstance(X, torch.Tensor) or X.dim() != 2:
        raise ValueError(f"{name} must be a 2-D tensor [M, features]")
    return X.shape


# ------------------------------------------------------------------ NF4 ----

@dataclass
class NF4Weight:
    codes: torch.Tensor   # uint8 [n_out * k_in / 2]
    absmax: torch.Tensor  # float32 [n_out * k_in / 64]
    n_out: int
    k_in: int

    def c(self):
        _t(self.codes, "codes", (self.n_out * self.k_in // 2,), torch.uint8)
        _t(self.absmax, "absmax", (self.n_out * self.k_in // 64,), torch.float32)
        return QloraNF4(self.codes.data_ptr(), self.absmax.data_ptr(), self.n_out, self.k_in)


def qlora_nf4_codebook():
    out = (ctypes.c_float * 16)()
    _check("qlora_nf4_codebook", lib().qlora_nf4_codebook(out))
    return [float(v) for v in out]


def nf4_quantize(w):
    """bf16 weight [n_out, k_in] on the GPU -> NF4Weight."""
    n_out, k_in = _rows(w, "w")
    _t(w, "w", (n_out, k_in))
    codes = torch.empty(n_out * k_in // 2, dtype=torch.uint8, device=w.device)
    absmax = torch.empty(n_out * k_in // 64, dtype=torch.float32, device=w.device)
    _check("nf4_quantize", lib().nf4_quantize(_p(w), n_out, k_in, _p(codes), _p(absmax), _stream()))
    return NF4Weight(codes, absmax, n_out, k_in)


def nf4_dequantize(w: NF4Weight, out=None):
    """NF4Weight -> bf16 [n_out, k_in] (bit-exact)."""
    if out is None:
        out = torch.empty(w.n_out, w.k_in, dtype=torch.bfloat16, device=w.codes.device)
    w.c()  # checks codes and absmax
    _t(out, "out", (w.n_out, w.k_in))
    _check("nf4_dequantize", lib().nf4_dequantize(_p(w.codes), _p(w.absmax), w.n_out, w.k_in, _p(out), _stream()))
    return out


# ---------------------------------------------------------- projections ----

@dataclass
class LoraLinear:
    w: NF4Weight
    A: torch.Tensor  # bf16 [k_in, r]
    B: torch.Tensor  # bf16 [r, n_out]
    scale: float

    def c(self):
        r = self.A.shape[1] if self.A.dim() == 2 else -1
        _t(self.A, "A", (self.w.k_in, r))
        _t(self.B, "B", (r, self.w.n_out))
        return QloraLoraLinear(self.w.c(), self.A.data_ptr(), self.B.data_ptr(), r, self.scale)


@dataclass
class LoraLinear16:
    """A projection with a frozen bf16 base weight (LoRA rather than QLoRA)."""
    w: torch.Tensor  # bf16 [n_out, k_in]
    A: torch.Tensor  # bf16 [k_in, r]
    B: torch.Tensor  # bf16 [r, n_out]
    scale: float

    @property
    def n_out(self):
        return self.w.shape[0]

    @property
    def k_in(self):
        return self.w.shape[1]

    def c(self):
        if self.w.dim() != 2:
            raise ValueError("w must be a 2-D bf16 tensor [n_out, k_in]")
        _t(self.w, "w", tuple(self.w.shape))
        r = self.A.shape[1] if self.A.dim() == 2 else -1
        _t(self.A, "A", (self.k_in, r))
        _t(self.B, "B", (r, self.n_out))
        return QloraLoraLinear16(self.w.data_ptr(), self.n_out, self.k_in, self.A.data_ptr(), self.B.data_ptr(),
                                 r, self.scale)


def _dims(lin):
    """(n_out, k_in) of an NF4 or a bf16 projection."""
    return (lin.w.n_out, lin.w.k_in) if isinstance(lin, LoraLinear) else (lin.n_out, lin.k_in)


class Workspace:
    """Caller-owned device workspace (zeroed once; grows on demand)."""

    def __init__(self, device="cuda"):
        self.device = device
        self.buf = torch.zeros(256, dtype=torch.uint8, device=device)

    def get(self, nbytes):
        if self.buf.numel() < nbytes:
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        return self.buf


def qlora_linear_workspace_bytes(M, K, N, r=16):
    return int(lib().qlora_linear_workspace_bytes(M, K, N, r))


def qlora_mlp_workspace_bytes(M, d, h, r=16):
    return int(lib().qlora_mlp_workspace_bytes(M, d, h, r))


def qlora_linear16_workspace_bytes(M, K, N, r=16):
    return int(lib().qlora_linear16_workspace_bytes(M, K, N, r))


def qlora_mlp16_workspace_bytes(M, d, h, r=16):
    return int(lib().qlora_mlp16_workspace_bytes(M, d, h, r))


def _linear_fwd(fn, wsq, lin, X, ws, Y, XA):
    M = _rows(X)[0]
    n_out, k_in = _dims(lin)
    r = lin.A.shape[1]
    if Y is None:
        Y = torch.empty(M, n_out, dtype=torch.bfloat16, device=X.device)
    if XA is None:
        XA = torch.empty(M, r, dtype=torch.bfloat16, device=X.device)
    _t(X, "X", (M, k_in))
    _t(Y, "Y", (M, n_out))
    _t(XA, "XA", (M, r))
    c = lin.c()
    buf = ws.get(wsq(M, k_in, n_out, r))
    _check(fn, getattr(lib(), fn)(ctypes.byref(c), _p(X), M, _p(Y), _p(XA), _p(buf), buf.numel(), _stream()))
    return Y, XA


def qlora_linear_fwd(lin: LoraLinear, X, ws: Workspace, Y=None, XA=None):
    return _linear_fwd("qlora_linear_fwd", qlora_linear_workspace_bytes, lin, X, ws, Y, XA)


def qlora_linear16_fwd(lin: LoraLinear16, X, ws: Workspace, Y=None, XA=None):
    return _linear_fwd("qlora_linear16_fwd", qlora_linear16_workspace_bytes, lin, X, ws, Y, XA)


def qlora_linear_fwd_noalloc(lin: LoraLinear, X, Y=None, XA=None):
    """qlora_linear_fwd without a workspace, for callers that cannot allocate
    device memory; its scratch is a fixed array inside the library (shared by
    all calls, so calls must not overlap on the GPU)."""
    M = _rows(X)[0]
    r = lin.A.shape[1]
    if Y is None:
        Y = torch.empty(M, lin.w.n_out, dtype=torch.bfloat16, device=X.device)
    if XA is None:
        XA = torch.empty(M, r, dtype=torch.bfloat16, device=X.device)
    _t(X, "X", (M, lin.w.k_in))
    _t(Y, "Y", (M, lin.w.n_out))
    _t(XA, "XA", (M, r))
    c = lin.c()
    _check("qlora_linear_fwd_noalloc", lib().qlora_linear_fwd_noalloc(ctypes.byref(c), _p(X), M, _p(Y), _p(XA),
                                                                      _stream()))
    return Y, XA


def _linear_bwd(fn, wsq, lin, X, XA, dY, ws, dX, dA, dB):
    M = _rows(X)[0]
    n_out, k_in = _dims(lin)
    r = lin.A.shape[1]
    if dX is None:
        dX = torch.empty(M, k_in, dtype=torch.bfloat16, device=X.device)
    if dA is None:
        dA = torch.empty_like(lin.A)
    if dB is None:
        dB = torch.empty_like(lin.B)
    _t(X, "X", (M, k_in))
    _t(XA, "XA", (M, r))
    _t(dY, "dY", (M, n_out))
    _t(dX, "dX", (M, k_in))
    _t(dA, "dA", (k_in, r))
    _t(dB, "dB", (r, n_out))
    c = lin.c()
    buf = ws.get(wsq(M, k_in, n_out, r))
    _check(fn, getattr(lib(), fn)(ctypes.byref(c), _p(X), _p(XA), _p(dY), M, _p(dX), _p(dA), _p(dB), _p(buf),
                                  buf.numel(), _stream()))
    return dX, dA, dB


def qlora_linear_bwd(lin: LoraLinear, X, XA, dY, ws: Workspace, dX=None, dA=None, dB=None):
    return _linear_bwd("qlora_linear_bwd", qlora_linear_workspace_bytes, lin, X, XA, dY, ws, dX, dA, dB)


def qlora_linear16_bwd(lin: LoraLinear16, X, XA, dY, ws: Workspace, dX=None, dA=None, dB=None):
    return _linear_bwd("qlora_linear16_bwd", qlora_linear16_workspace_bytes, lin, X, XA, dY, ws, dX, dA, dB)


def make_mlp_saved(M, h, r, device):
    e = lambda *s: torch.empty(*s, dtype=torch.bfloat16, device=device)
    return {"E": e(M, h), "G": e(M, h), "H": e(M, h), "XA_g": e(M, r), "XA_u": e(M, r), "HA_d": e(M, r)}


def _saved_c(sv, M, h, r):
    for k in ("E", "G", "H"):
        _t(sv[k], k, (M, h))
    for k in ("XA_g", "XA_u", "HA_d"):
        _t(sv[k], k, (M, r))
    return QloraMlpSaved(*[sv[k].data_ptr() for k in ("E", "G", "H", "XA_g", "XA_u", "HA_d")])


def _mlp_dims(gate, up, down, d):
    h = _dims(gate)[0]
    if _dims(gate) != (h, d) or _dims(up) != (h, d) or _dims(down) != (d, h):
        raise ValueError(f"MLP weights must be gate, up [h, {d}] and down [{d}, h]")
    return h


def _mlp_fwd(fn, wsq, act, gate, up, down, X, ws, Y, saved):
    M, d = _rows(X)
    h = _mlp_dims(gate, up, down, d)
    r = gate.A.shape[1]
    if Y is None:
        Y = torch.empty(M, d, dtype=torch.bfloat16, device=X.device)
    if saved is None:
        saved = make_mlp_saved(M, h, r, X.device)
    _t(X, "X", (M, d))
    _t(Y, "Y", (M, d))
    g, u, dn, sv = gate.c(), up.c(), down.c(), _saved_c(saved, M, h, r)
    buf = ws.get(wsq(M, d, h, r))
    _check(fn, getattr(lib(), fn)(QLORA_ACT[act], ctypes.byref(g), ctypes.byref(u), ctypes.byref(dn), _p(X), M,
                                  _p(Y), ctypes.byref(sv), _p(buf), buf.numel(), _stream()))
    return Y, saved


def qlora_mlp_fwd(act, gate: LoraLinear, up: LoraLinear, down: LoraLinear, X, ws: Workspace, Y=None, saved=None):
    return _mlp_fwd("qlora_mlp_fwd", qlora_mlp_workspace_bytes, act, gate, up, down, X, ws, Y, saved)


def qlora_mlp16_fwd(act, gate: LoraLinear16, up: LoraLinear16, down: LoraLinear16, X, ws: Workspace, Y=None,
                    saved=None):
    return _mlp_fwd("qlora_mlp16_fwd", qlora_mlp16_workspace_bytes, act, gate, up, down, X, ws, Y, saved)


def _mlp_bwd(fn, wsq, act, gate, up, down, X, saved, dY, ws, grads, early_event=0):
    M, d = _rows(X)
    h = _mlp_dims(gate, up, down, d)
    r = gate.A.shape[1]
    if grads is None:
        grads = {"dX": torch.empty(M, d, dtype=torch.bfloat16, device=X.device),
                 "dA_g": torch.empty_like(gate.A), "dB_g": torch.empty_like(gate.B),
                 "dA_u": torch.empty_like(up.A), "dB_u": torch.empty_like(up.B),
                 "dA_d": torch.empty_like(down.A), "dB_d": torch.empty_like(down.B)}
    _t(X, "X", (M, d))
    _t(dY, "dY", (M, d))
    _t(grads["dX"], "dX", (M, d))
    for k, shp in (("dA_g", (d, r)), ("dB_g", (r, h)), ("dA_u", (d, r)), ("dB_u", (r, h)), ("dA_d", (h, r)),
                   ("dB_d", (r, d))):
        _t(grads[k], k, shp)
    g, u, dn, sv = gate.c(), up.c(), down.c(), _saved_c(saved, M, h, r)
    buf = ws.get(wsq(M, d, h, r))
    outs = [_p(grads[k]) for k in ("dX", "dA_g", "dB_g", "dA_u", "dB_u", "dA_d", "dB_d")]
    args = [QLORA_ACT[act], ctypes.byref(g), ctypes.byref(u), ctypes.byref(dn), _p(X), ctypes.byref(sv), _p(dY), M,
            *outs, _p(buf), buf.numel(), _stream()]
    if early_event:
        _check(fn + "_ev", getattr(lib(), fn + "_ev")(*args, ctypes.c_void_p(early_event)))
    else:
        _check(fn, getattr(lib(), fn)(*args))
    return grads


def qlora_mlp_bwd(act, gate: LoraLinear, up: LoraLinear, down: LoraLinear, X, saved, dY, ws: Workspace, grads=None,
                  early_event=0):
    """MLP backward; with `early_event` (a raw cudaEvent_t, e.g. torch.cuda.Event().cuda_event after its first
    record) the library records it once dA_d, dB_d, dB_g and dB_u are final (qlora_mlp_bwd_ev)."""
    return _mlp_bwd("qlora_mlp_bwd", qlora_mlp_workspace_bytes, act, gate, up, down, X, saved, dY, ws, grads,
                    early_event)


def qlora_mlp16_bwd(act, gate: LoraLinear16, up: LoraLinear16, down: LoraLinear16, X, saved, dY, ws: Workspace,
                    grads=None, early_event=0):
    return _mlp_bwd("qlora_mlp16_bwd", qlora_mlp16_workspace_bytes, act, gate, up, down, X, saved, dY, ws, grads,
                    early_event)


def qlora_rmsnorm_fwd(X, w, eps, plus_one=False, Y=None, rstd=None):
    """RMS layer norm of X [M, d] with gain w (or 1 + w): returns (Y, rstd)."""
    M, d = _rows(X)
    if Y is None:
        Y = torch.empty_like(X)
    if rstd is None:
        rstd = torch.empty(M, dtype=torch.float32, device=X.device)
    _t(X, "X", (M, d))
    _t(w, "w", (d,))
    _t(Y, "Y", (M, d))
    _t(rstd, "rstd", (M,), torch.float32)
    _check("qlora_rmsnorm_fwd", lib().qlora_rmsnorm_fwd(_p(X), _p(w), M, d, float(eps), int(bool(plus_one)), _p(Y),
                                                        _p(rstd), _stream()))
    return Y, rstd


def qlora_rmsnorm_bwd(X, w, rstd, dY, plus_one=False, dX=None):
    M, d = _rows(X)
    if dX is None:
        dX = torch.empty_like(X)
    _t(X, "X", (M, d))
    _t(w, "w", (d,))
    _t(rstd, "rstd", (M,), torch.float32)
    _t(dY, "dY", (M, d))
    _t(dX, "dX", (M, d))
    _check("qlora_rmsnorm_bwd", lib().qlora_rmsnorm_bwd(_p(X), _p(w), _p(rstd), _p(dY), M, d, int(bool(plus_one)),
                                                        _p(dX), _stream()))
    return dX


def qlora_qkv_workspace_bytes(M, K, nq, nk, nv, r=16):
    return int(lib().qlora_qkv_workspace_bytes(M, K, nq, nk, nv, r))


def qlora_qkv_fwd(q: LoraLinear, k: LoraLinear, v: LoraLinear, X, ws: Workspace, Y=None, XA=None):
    """Fused Q/K/V projection: Y = [Y_q | Y_k | Y_v] [M, nq + nk + nv], XA = [XA_q | XA_k | XA_v] [M, 3r]."""
    M, K = _rows(X)
    r = q.A.shape[1]
    nt = q.w.n_out + k.w.n_out + v.w.n_out
    if Y is None:
        Y = torch.empty(M, nt, dtype=torch.bfloat16, device=X.device)
    if XA is None:
        XA = torch.empty(M, 3 * r, dtype=torch.bfloat16, device=X.device)
    _t(X, "X", (M, K))
    _t(Y, "Y", (M, nt))
    _t(XA, "XA", (M, 3 * r))
    cq, ck, cv = q.c(), k.c(), v.c()
    buf = ws.get(qlora_qkv_workspace_bytes(M, K, q.w.n_out, k.w.n_out, v.w.n_out, r))
    _check("qlora_qkv_fwd", lib().qlora_qkv_fwd(ctypes.byref(cq), ctypes.byref(ck), ctypes.byref(cv), _p(X), M,
                                                _p(Y), _p(XA), _p(buf), buf.numel(), _stream()))
    return Y, XA


def qlora_qkv_bwd(q: LoraLinear, k: LoraLinear, v: LoraLinear, X, XA, dY, ws: Workspace, grads=None):
    M, K = _rows(X)
    r = q.A.shape[1]
    nt = q.w.n_out + k.w.n_out + v.w.n_out
    if grads is None:
        grads = {"dX": torch.empty(M, K, dtype=torch.bfloat16, device=X.device)}
        for n, l in (("q", q), ("k", k), ("v", v)):
            grads["dA_" + n] = torch.empty_like(l.A)
            grads["dB_" + n] = torch.empty_like(l.B)
    _t(X, "X", (M, K))
    _t(XA, "XA", (M, 3 * r))
    _t(dY, "dY", (M, nt))
    _t(grads["dX"], "dX", (M, K))
    for n, l in (("q", q), ("k", k), ("v", v)):
        _t(grads["dA_" + n], "dA_" + n, (K, r))
        _t(grads["dB_" + n], "dB_" + n, (r, l.w.n_out))
    cq, ck, cv = q.c(), k.c(), v.c()
    buf = ws.get(qlora_qkv_workspace_bytes(M, K, q.w.n_out, k.w.n_out, v.w.n_out, r))
    outs = [_p(grads[n]) for n in ("dX", "dA_q", "dB_q", "dA_k", "dB_k", "dA_v", "dB_v")]
    _check("qlora_qkv_bwd", lib().qlora_qkv_bwd(ctypes.byref(cq), ctypes.byref(ck), ctypes.byref(cv), _p(X), _p(XA),
                                                _p(dY), M, *outs, _p(buf), buf.numel(), _stream()))
    return grads


# ------------------------------------------------------------ utilities ----

def qlora_test_inject_timeout():
    """Arms the library's one-shot timeout injection (test hook; see include/qlora.h)."""
    _check("qlora_test_inject_timeout", lib().qlora_test_inject_timeout())


def qlora_test_shrink_next_slot_cap():
    """Arms the one-shot plan-mismatch hook (test only; see include/qlora.h)."""
    _check("qlora_test_shrink_next_slot_cap", lib().qlora_test_shrink_next_slot_cap())


def qlora_checked_build():
    return int(lib().qlora_checked_build())


def qlora_test_set_grid_cap(max_ctas):
    """Caps the CTAs of every persistent launch (test hook; 0 = no cap); returns the previous cap."""
    return int(lib().qlora_test_set_grid_cap(int(max_ctas)))


def qlora_last_device_status(ws: Workspace):
    return int(lib().qlora_last_device_status(_p(ws.buf), _stream()))


def qlora_status_string(status):
    return lib().qlora_status_string(status).decode()


TILE_CONFIGS = {0: "automatic", 1: "1 CTA, 128x256", 2: "CTA pair, 256x256", 3: "CTA pair, 512x128",
                4: "CTA pair, 256x256, staged bf16 weight"}


def qlora_set_tile_config(tiles):
    return int(lib().qlora_set_tile_config(tiles))


def qlora_mlp_tile_config(M, d, h, r=16):
    """The tile configuration the NF4 MLP calls use for these sizes under the current setting."""
    return int(lib().qlora_mlp_tile_config(M, d, h, r))


def qlora_launch_count():
    return int(lib().qlora_launch_count())


def qlora_trace_begin(only=None):
    """Start tracing every kernel launch, or only the kernel named `only`."""
    if only is None:
        _check("qlora_trace_begin", lib().qlora_trace_begin())
    else:
        _check("qlora_trace_begin_only", lib().qlora_trace_begin_only(only.encode()))


def qlora_trace_end(max_entries=64):
    arr = (QloraTraceEntry * max_entries)()
    n = int(lib().qlora_trace_end(arr, max_entries))
    if n < 0:
        raise QloraError("qlora_trace_end", 5)
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms)) for i in range(min(n, max_entries))}
