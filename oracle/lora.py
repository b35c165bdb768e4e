"""LoRA projection over a frozen base weight, and the gated MLP, in float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

All arguments are float64 arrays (bf16 inputs widened exactly); nothing here
emulates the GPU's bf16 intermediates.  Shapes follow nn.Linear:
X [M, K], frozen W [N, K] (already dequantised), A [K, r], B [r, N],
s = alpha / r, Y [M, N].  No dropout and no bias ([Mistral blog] benchmark
configuration: dropout = 0; the layers carry no bias).

Backward ([Mistral blog] "10、11. 手动 Autograd"; [Show HN] highlight 1): with
L = sum(Y * dY) and the rank-r factor bracketed first,
    G  = dY B^T                 [M, r]
    dX = dY W + s * G A^T
    dA = s * X^T G              (the page's fast bracket: X^T (dY B^T))
    dB = s * (X A)^T dY
and no gradient for the frozen W.

Gated MLP ([Reddit talk] SwiGLU kernel; [Gemma blog] "GeGLU 与 Swiglu 激活函数"):
    e = lin_g(X), g = lin_u(X), H = act(e) * g, Y = lin_d(H)
with act = SiLU (SwiGLU) or the tanh-approximate GELU (GeGLU).  The Gemma
page derives the GeGLU derivative but does not say which GELU; the
tanh approximation is the reading taken here.
"""

import numpy as np

_SQRT_2_OVER_PI = np.sqrt(2.0 / np.pi)
_GELU_C = 0.044715

ACTIVATIONS = ("swiglu", "geglu_tanh")


def _sigmoid(e):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-e))


def act_fwd(kind, e):
    """act(e): SiLU e*sigmoid(e), or GELU-tanh e/2 * (1 + tanh(sqrt(2/pi)(e + 0.044715 e^3)))."""
    if kind == "swiglu":
        return e * _sigmoid(e)
    if kind == "geglu_tanh":
        t = np.tanh(_SQRT_2_OVER_PI * (e + _GELU_C * e ** 3))
        return 0.5 * e * (1.0 + t)
    raise ValueError(kind)


def act_grad(kind, e):
    """d act / d e in closed form.

    SiLU:      sigmoid(e) * (1 + e * (1 - sigmoid(e)))
    GELU-tanh: (1 + t)/2 + e/2 * (1 - t^2) * sqrt(2/pi) * (1 + 3*0.044715*e^2),
               t = tanh(sqrt(2/pi)(e + 0.044715 e^3))
    """
    if kind == "swiglu":
        sg = _sigmoid(e)
        return sg * (1.0 + e * (1.0 - sg))
    if kind == "geglu_tanh":
        t = np.tanh(_SQRT_2_OVER_PI * (e + _GELU_C * e ** 3))
        return 0.5 * (1.0 + t) + 0.5 * e * (1.0 - t * t) * _SQRT_2_OVER_PI * (1.0 + 3.0 * _GELU_C * e * e)
    raise ValueError(kind)


def linear_fwd(X, W, A, B, s):
    """Y = X W^T + s (X A) B; also returns XA = X A (kept for the backward)."""
    XA = X @ A
    Y = X @ W.T + s * (XA @ B)
    return Y, XA


def linear_bwd(X, W, A, B, s, dY):
    """Hand-derived backward of :func:`linear_fwd`: returns (dX, dA, dB)."""
    G = dY @ B.T
    dX = dY @ W + s * (G @ A.T)
    dA = s * (X.T @ G)
    dB = s * ((X @ A).T @ dY)
    return dX, dA, dB


def mlp_fwd(kind, X, gate, up, down):
    """Gated MLP forward.  gate/up/down are (W, A, B, s) tuples.

    Returns dict with Y and the saved E (= e), G (= g), H.
    """
    E, _ = linear_fwd(X, *gate)
    G, _ = linear_fwd(X, *up)
    H = act_fwd(kind, E) * G
    Y, _ = linear_fwd(H, *down)
    return {"Y": Y, "E": E, "G": G, "H": H}


def mlp_bwd(kind, X, gate, up, down, dY, saved=None):
    """Gated MLP backward by the chain rule through the closed-form act'.

    dH = dY W_d + s_d (dY B_d^T) A_d^T, dE = dH * g * act'(e), dG = dH * act(e),
    dX = [gate bwd of dE] + [up bwd of dG].  Returns a dict of dX and the six
    adapter gradients dA_g, dB_g, dA_u, dB_u, dA_d, dB_d.
    """
    if saved is None:
        saved = mlp_fwd(kind, X, gate, up, down)
    E, G, H = saved["E"], saved["G"], saved["H"]
    dH, dA_d, dB_d = linear_bwd(H, *down, dY)
    dE = dH * G * act_grad(kind, E)
    dG = dH * act_fwd(kind, E)
    dX_g, dA_g, dB_g = linear_bwd(X, *gate, dE)
    dX_u, dA_u, dB_u = linear_bwd(X, *up, dG)
    return {"dX": dX_g + dX_u, "dA_g": dA_g, "dB_g": dB_g, "dA_u": dA_u,
            "dB_u": dB_u, "dA_d": dA_d, "dB_d": dB_d, "dE": dE, "dG": dG}
