"""GPU parity of the RMS norm fused into the gated MLP behind it
(qlora_norm_mlp_fwd / qlora_norm_mlp_bwd) against the oracle composed the way
the pages define the two steps: the norm (oracle/norm.py), then the MLP oracle
on the normalised rows; the MLP oracle's backward, then the norm's backward on
its dX.  The GPU never forms Xn: the gain is folded into the staged gate/up
weights and A factors and rstd into the gate/up GEMM's epilogue, so its
roundings fall elsewhere than the unfused chain's.

Bars: rstd to 1e-5 relative (an fp32 sum of squares); E, G, H element by
element against their bf16 rounding bound, including the one rounding of the
gained weight and factor (parity.saved_bounds, input_round); every other
tensor max|err| <= tol x RMS(oracle) with tol = 2e-2 at full size.  At M =
200-1100 tokens a CPU emulation of the bf16 roundings of the chain alone (no
kernel involved; norm + MLP, fused or unfused) already gives 1.3-2.3e-2 x RMS
on Y, the rank-side products and the adapter gradients, and 2.8-4.4e-2 on dX:
the norm's backward subtracts n mean(n g dXn) from g dXn, whose bf16 copy
already carries the small-M MLP error.  Those cases use 3e-2, and 5e-2 for
dX."""

import os

import numpy as np
import pytest
import torch

import oracle
from qlora_fine_tuning_nf4_b200 import ops
from qlora_fine_tuning_nf4_b200.synth import make_norm_mlp_problem
from qlora_fine_tuning_nf4_b200.workloads import MLP_WORKLOADS

from parity import (TOL, TOL_SMALL_MLP, assert_close, assert_saved, dev, f64, gpu_f64, gpu_weight, oracle_weight,
                    saved_bounds)

pytestmark = pytest.mark.gpu

EPS = {False: 1e-5, True: 1e-6}  # Llama-style gain w, Gemma-style 1 + w
TOL_SMALL_NORM_DX = 5e-2


def _problem(M, d, h, gemma, seed, r=16):
    return make_norm_mlp_problem(M, d, h, r, 16.0, seed, plus_one=gemma)


def _run_gpu(p, act, gemma, rows=None):
    ops.qlora_set_tile_config(4)
    lins = {}
    for k in ("g", "u", "d"):
        w, _, _ = gpu_weight(p["W_" + k])
        lins[k] = ops.LoraLinear(w, dev(p["A_" + k]), dev(p["B_" + k]), p["s"])
    ws = ops.Workspace()
    X, dY, w = dev(p["X"]), dev(p["dY"]), dev(p["w"])
    Y, saved, rstd = ops.qlora_norm_mlp_fwd(act, w, EPS[gemma], lins["g"], lins["u"], lins["d"], X, ws,
                                            plus_one=gemma)
    grads = ops.qlora_norm_mlp_bwd(act, w, lins["g"], lins["u"], lins["d"], X, saved, rstd, dY, ws, plus_one=gemma)
    torch.cuda.synchronize()
    sel = (lambda t: t) if rows is None else (lambda t: t[torch.as_tensor(rows, device=t.device)])
    out = {"status": ops.qlora_last_device_status(ws), "Y": gpu_f64(sel(Y)), "rstd": sel(rstd).cpu().double().numpy()}
    for k in ("E", "G", "H", "XA_g", "XA_u", "HA_d"):
        out[k] = gpu_f64(sel(saved[k]))
    for k, v in grads.items():
        out[k] = gpu_f64(sel(v) if k == "dX" else v)
    return out


def _run_oracle(p, act, gemma):
    lin = {}
    for k in ("g", "u", "d"):
        _, _, W = oracle_weight(p["W_" + k])
        lin[k] = (W, f64(p["A_" + k]), f64(p["B_" + k]), p["s"])
    X, w, dY = f64(p["X"]), f64(p["w"]), f64(p["dY"])
    Xn, rstd = oracle.rmsnorm_fwd(X, w, EPS[gemma], plus_one=gemma)
    fwd = oracle.mlp_fwd(act, Xn, lin["g"], lin["u"], lin["d"])
    bwd = oracle.mlp_bwd(act, Xn, lin["g"], lin["u"], lin["d"], dY, saved=fwd)
    out = dict(fwd)
    out.update(bwd)
    out["dX"] = oracle.rmsnorm_bwd(X, w, EPS[gemma], bwd["dX"], plus_one=gemma)
    out["rstd"] = rstd
    out["lin"], out["X"], out["act"] = lin, Xn, act  # the MLP's input, for the rounding bounds
    out["XA_g"], out["XA_u"] = Xn @ lin["g"][1], Xn @ lin["u"][1]
    out["HA_d"] = fwd["H"] @ lin["d"][1]
    return out


@pytest.mark.parametrize("gemma", [False, True])
@pytest.mark.parametrize("act", ["swiglu", "geglu_tanh"])
@pytest.mark.parametrize("M,d,h", [(256, 256, 512), (200, 512, 768), (1100, 512, 768)])
def test_norm_mlp_parity(M, d, h, act, gemma):
    p = _problem(M, d, h, gemma, seed=M + d + h)
    g = _run_gpu(p, act, gemma)
    o = _run_oracle(p, act, gemma)
    assert g["status"] == 0
    np.testing.assert_allclose(g["rstd"], o["rstd"], rtol=1e-5)
    bounds = saved_bounds(o, p, input_round=True)
    for k in ("E", "G", "H"):
        assert_saved(k, g[k], o[k], bounds[k])
    for k in ("XA_g", "XA_u", "HA_d", "Y", "dA_g", "dB_g", "dA_u", "dB_u", "dA_d", "dB_d"):
        assert_close(k, g[k], o[k], TOL_SMALL_MLP)
    assert_close("dX", g["dX"], o["dX"], TOL_SMALL_NORM_DX)


@pytest.mark.parametrize("r", [32, 64])
def test_norm_mlp_higher_rank(r):
    """Ranks 32 and 64 (s = 16 / r) with Gemma's gain and GeGLU.  The bf16
    emulation gives 1.8-2.5e-2 x RMS on the adapter gradients here; the GPU
    also evaluates tanh on the hardware's approximate unit, whose small
    absolute error becomes a larger relative one where 1 + tanh cancels
    (negative e), and that reaches dB_u through dG = dH act(e): measured up to
    3.03e-2.  The adapter gradients use 4e-2 here."""
    p = _problem(384, 512, 768, True, seed=91, r=r)
    g = _run_gpu(p, "geglu_tanh", True)
    o = _run_oracle(p, "geglu_tanh", True)
    assert g["status"] == 0
    assert_close("Y", g["Y"], o["Y"], TOL_SMALL_MLP)
    for k in ("dA_g", "dB_g", "dA_u", "dB_u", "dA_d", "dB_d"):
        assert_close(k, g[k], o[k], 4e-2)
    assert_close("dX", g["dX"], o["dX"], TOL_SMALL_NORM_DX)


@pytest.mark.parametrize("name", ["llama7b_swiglu_mlp", "gemma7b_geglu_mlp"])
def test_norm_mlp_full_size(name):
    """Llama-7B (gain w) and Gemma-7B (gain 1 + w, GeGLU, 16384 tokens) widths
    against the oracle's stored values (tests/golden/make_full_size_expected.py):
    sampled rows of rstd, Y, dX, E, G, H and sampled entries of every adapter
    gradient; Y within 2e-2 x the RMS of the oracle's full tensor, E, G, H
    element by element against their stored rounding bounds, dX and the adapter
    gradients against the bars derived below."""
    cfg = MLP_WORKLOADS[name]
    gemma = cfg["act"] == "geglu_tanh"
    path = os.path.join(os.path.dirname(__file__), "golden", f"full_norm_{name}.npz")
    gold = np.load(path)
    p = _problem(cfg["M"], cfg["d"], cfg["h"], gemma, seed=cfg["seed"])
    rows = gold["rows"]
    g = _run_gpu(p, cfg["act"], gemma, rows=rows)
    assert g["status"] == 0
    np.testing.assert_allclose(g["rstd"], gold["rows_rstd"][:, 0], rtol=1e-5)
    _check_rows("Y", g["Y"], gold["rows_Y"], gold["rms_Y"])
    # dX: a CPU emulation of the chain's own bf16 roundings on these rows (no kernel)
    # gives 2.8e-2 (Llama) and 3.2e-2 (Gemma) x RMS, 2.35e-2 and 1.9e-2 if g dXn were
    # handed to the norm's backward in fp32: the bf16 hand-off (which the unfused chain
    # has too, as its bf16 dXn) dominates, and rows with rstd up to 1.43 (token norms
    # spread 2x) scale it against an RMS taken over all rows.  Bar 4e-2.
    _check_rows("dX", g["dX"], gold["rows_dX"], gold["rms_dX"], 4e-2)
    wide = np.searchsorted(rows, gold["rows_wide"])
    for k in ("E", "G", "H"):  # element by element, against the bound the oracle stored (see saved_bounds)
        bad = np.abs(g[k][wide] - gold[f"rows_{k}"]) > gold[f"bound_{k}"]
        assert not bad.any(), f"{k}: {int(bad.sum())} elements outside the bf16 rounding bound"
    # adapter gradients: H and the rank-side products carry the gained weight's rounding
    # (the emulation at small M gives up to 2.15e-2 on dA_d); bar 3e-2
    for k in ("dA_g", "dB_g", "dA_u", "dB_u", "dA_d", "dB_d"):
        _check_rows(k, g[k].reshape(-1)[gold[f"idx_{k}"]], gold[f"val_{k}"], gold[f"rms_{k}"], 3e-2)


def _check_rows(name, got, want, rms, tol=TOL):
    err = float(np.max(np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64))))
    assert err <= tol * float(rms), f"{name}: {err:.3e} > {tol} * {float(rms):.3e}"


def test_norm_mlp_rejects_unsupported_configurations():
    p = _problem(64, 256, 256, False, seed=3)
    w, _, _ = gpu_weight(p["W_g"])
    lin = ops.LoraLinear(w, dev(p["A_g"]), dev(p["B_g"]), p["s"])
    ops.qlora_set_tile_config(2)  # the fusion needs the staged weight feed
    try:
        with pytest.raises(ops.QloraError) as e:
            ops.qlora_norm_mlp_fwd("swiglu", dev(p["w"]), 1e-5, lin, lin, lin, dev(p["X"]), ops.Workspace())
        assert e.value.status == 2
    finally:
        ops.qlora_set_tile_config(4)
