"""RMS layer norm, forward and hand-derived backward, in fp64 (oracle; test
infrastructure only).

Sources: [Mistral blog] table "逐项性能拆解" item "8. 快速 RMS Layernorm" (a
fused RMS layernorm kernel whose derivative is worked out by the chain rule)
and [Gemma blog] "+1 to RMS LayerNorm" (Llama and Mistral scale by w, Gemma by
1 + w).  The pages print neither formula; the oracle takes the standard RMS
layer norm in its plainest reading:

    rstd = 1 / sqrt(mean_j x_j^2 + eps),   n = x * rstd,   y = n * g,
    g = w  (Llama, Mistral)  or  g = 1 + w  (Gemma).

Backward with the norm weight frozen (only the LoRA adapters train), by the
chain rule through rstd:

    dx_j = rstd * (g_j dy_j - n_j * mean_i(n_i g_i dy_i)).
"""

import numpy as np


def _gain(w, plus_one):
    w = np.asarray(w, dtype=np.float64)
    return 1.0 + w if plus_one else w


def rmsnorm_fwd(X, w, eps, plus_one=False):
    """Returns (Y, rstd) for X [M, d], w [d]."""
    X = np.asarray(X, dtype=np.float64)
    rstd = 1.0 / np.sqrt(np.mean(X * X, axis=1) + eps)
    return X * rstd[:, None] * _gain(w, plus_one)[None, :], rstd


def rmsnorm_bwd(X, w, eps, dY, plus_one=False):
    """dX for X [M, d], upstream gradient dY [M, d]."""
    X = np.asarray(X, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    rstd = 1.0 / np.sqrt(np.mean(X * X, axis=1) + eps)
    n = X * rstd[:, None]
    gdy = _gain(w, plus_one)[None, :] * dY
    c = np.mean(n * gdy, axis=1)
    return rstd[:, None] * (gdy - n * c[:, None])
