"""Full-size parity: every workload at its real shape, in the launch
configuration the benchmark uses, against expected values the oracle wrote
(``tests/golden/make_full_size_expected.py``).

Checked: NF4 codes/absmax bit-exact (SHA-256 of the oracle's arrays); sampled
rows of Y, dX (and E, G, H) and sampled entries of every adapter gradient within
2e-2 x RMS of the oracle's full tensor; the saved activations E, G, H also
elementwise within their bf16 rounding bound.
"""

import hashlib
import os

import numpy as np
import pytest
import torch

from qlora_fine_tuning_nf4_b200 import ops
from qlora_fine_tuning_nf4_b200.synth import bits_to_torch, make_linear_problem, make_mlp_problem
from qlora_fine_tuning_nf4_b200.workloads import LINEAR_WORKLOADS, MLP_WORKLOADS

from parity import TOL, gpu_f64

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    path = os.path.join(GOLDEN, f"full_{name}.npz")
    if not os.path.exists(path):
        pytest.fail(f"missing {path}: run tests/golden/make_full_size_expected.py")
    return np.load(path)


def _sha(t):
    return hashlib.sha256(t.cpu().numpy().tobytes()).hexdigest()


def _check(name, got, want, rms, tol=TOL):
    err = float(np.max(np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64))))
    assert err <= tol * float(rms), f"{name}: {err:.3e} > {tol} * {float(rms):.3e} (ratio {err / float(rms):.3e})"


def _check_saved(name, got, want, rms):
    """Elementwise: bf16 output rounding (u = 2^-8 relative, factor 2) plus fp32-accumulation slack."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    bound = 2.0 ** -7 * np.abs(want) + 2.0 ** -9 * float(rms)
    bad = np.abs(got - want) > bound
    assert not bad.any(), f"{name}: {int(bad.sum())} elements outside the bf16 rounding bound"


def _quant(w_bits, g, tag):
    w = ops.nf4_quantize(bits_to_torch(w_bits, "cuda"))
    assert _sha(w.codes) == str(g[f"sha_codes_{tag}"]), f"{tag} codes differ from the oracle"
    assert _sha(w.absmax) == str(g[f"sha_absmax_{tag}"]), f"{tag} absmax differ from the oracle"
    return w


@pytest.mark.parametrize("tiles", [4, 2])  # staged weight (default); dequantised in the mainloop
@pytest.mark.parametrize("name", [n for n in LINEAR_WORKLOADS if n != "tiny_linear"])
def test_full_size_linear(name, tiles):
    cfg = LINEAR_WORKLOADS[name]
    g = _golden(name)
    ops.qlora_set_tile_config(tiles)
    p = make_linear_problem(cfg["M"], cfg["K"], cfg["N"], cfg["r"], cfg["alpha"], cfg["seed"])
    w = _quant(p["W"], g, "W")
    lin = ops.LoraLinear(w, bits_to_torch(p["A"], "cuda"), bits_to_torch(p["B"], "cuda"), p["s"])
    X, dY = bits_to_torch(p["X"], "cuda"), bits_to_torch(p["dY"], "cuda")
    ws = ops.Workspace()
    Y, XA = ops.qlora_linear_fwd(lin, X, ws)
    dX, dA, dB = ops.qlora_linear_bwd(lin, X, XA, dY, ws)
    torch.cuda.synchronize()
    assert ops.qlora_last_device_status(ws) == 0
    rows = torch.from_numpy(g["rows"]).cuda()
    _check("Y", gpu_f64(Y[rows]), g["rows_Y"], g["rms_Y"])
    _check("dX", gpu_f64(dX[rows]), g["rows_dX"], g["rms_dX"])
    for k, t in (("dA", dA), ("dB", dB)):
        _check(k, gpu_f64(t).reshape(-1)[g[f"idx_{k}"]], g[f"val_{k}"], g[f"rms_{k}"])


@pytest.mark.parametrize("tiles", [4, 2])
@pytest.mark.parametrize("name", list(MLP_WORKLOADS))
def test_full_size_mlp(name, tiles):
    cfg = MLP_WORKLOADS[name]
    g = _golden(name)
    ops.qlora_set_tile_config(tiles)
    p = make_mlp_problem(cfg["M"], cfg["d"], cfg["h"], cfg["r"], cfg["alpha"], cfg["seed"])
    lins = {}
    for k in ("g", "u", "d"):
        w = _quant(p["W_" + k], g, "W_" + k)
        lins[k] = ops.LoraLinear(w, bits_to_torch(p["A_" + k], "cuda"), bits_to_torch(p["B_" + k], "cuda"), p["s"])
    X, dY = bits_to_torch(p["X"], "cuda"), bits_to_torch(p["dY"], "cuda")
    del p
    ws = ops.Workspace()
    act = cfg["act"]
    Y, saved = ops.qlora_mlp_fwd(act, lins["g"], lins["u"], lins["d"], X, ws)
    grads = ops.qlora_mlp_bwd(act, lins["g"], lins["u"], lins["d"], X, saved, dY, ws)
    torch.cuda.synchronize()
    assert ops.qlora_last_device_status(ws) == 0
    rows = torch.from_numpy(g["rows"]).cuda()
    wide = torch.from_numpy(g["rows_wide"]).cuda()
    _check("Y", gpu_f64(Y[rows]), g["rows_Y"], g["rms_Y"])
    _check("dX", gpu_f64(grads["dX"][rows]), g["rows_dX"], g["rms_dX"])
    for k in ("E", "G", "H"):
        _check_saved(k, gpu_f64(saved[k][wide]), g[f"rows_{k}"], g[f"rms_{k}"])
    for k in ("dA_g", "dB_g", "dA_u", "dB_u", "dA_d", "dB_d"):
        _check(k, gpu_f64(grads[k]).reshape(-1)[g[f"idx_{k}"]], g[f"val_{k}"], g[f"rms_{k}"])
