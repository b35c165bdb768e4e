"""Where the small-M bar for the gated MLP (TOL_SMALL_MLP = 3e-2 x RMS) comes
from, derived on the CPU without any kernel.

The CUDA path accumulates every contraction in fp32 and stores in bf16 the
tensors that later contractions read: X A and H A_d, e and g (h is formed from
the fp32 e and g), s G for each projection, and dE, dG; every returned tensor
is rounded to bf16 once.  Below, that chain of roundings is applied to exact
(fp64) products of the same inputs as the GPU parity cases and compared with
the oracle.  Rounding each returned tensor alone already costs up to about
1.9e-2 x RMS at these sizes: a few hundred rows make the maximum over elements
land on single heavy-tailed products, where half a bf16 ulp is large against
the RMS.  With the stored intermediates the chain reaches 2.25e-2, so an exact
implementation of this arithmetic would fail the 2e-2 bar, while 3e-2 holds with
room.  More rows do not cure it: over whole tensors of 2088-4136 rows the chain
stays at 1.9-2.2e-2 (one multi-tile case is pinned below), so the multi-tile
parity cases use 2.5e-2.  The full-size workloads meet 2e-2 on the rows they
sample (tests/test_gpu_full.py), where the maximum runs over fewer elements.
"""

import numpy as np
import pytest

import oracle
from oracle.nf4 import nf4_dequantize_f64
from qlora_fine_tuning_nf4_b200.synth import make_mlp_problem

from parity import SMALL_MLP_CASES, TOL, TOL_SMALL_MLP, f64, rel_err

OUTS = ("Y", "dX", "dA_g", "dB_g", "dA_u", "dB_u", "dA_d", "dB_d")


def _bf(x):
    """fp32 accumulator value rounded to bf16 (round to nearest even)."""
    return oracle.bf16_bits_to_f64(oracle.f32_to_bf16_bits(np.asarray(x, dtype=np.float32).astype(np.float64)))


def _case(M, d, h, act):
    p = make_mlp_problem(M, d, h, seed=M + d + h)
    lin = {}
    for k in ("g", "u", "d"):
        n, kk = p["W_" + k].shape
        codes, absmax = oracle.nf4_quantize(p["W_" + k], n, kk)
        lin[k] = (nf4_dequantize_f64(codes, absmax, n, kk), f64(p["A_" + k]), f64(p["B_" + k]), p["s"])
    X, dY = f64(p["X"]), f64(p["dY"])
    fwd = oracle.mlp_fwd(act, X, lin["g"], lin["u"], lin["d"])
    ref = oracle.mlp_bwd(act, X, lin["g"], lin["u"], lin["d"], dY, saved=fwd)
    ref["Y"] = fwd["Y"]
    return X, dY, lin, ref


def _chain(act, X, dY, lin, rnd=_bf):
    """The CUDA path's rounding points (`rnd`) on exact products."""
    (Wg, Ag, Bg, s), (Wu, Au, Bu, su), (Wd, Ad, Bd, sd) = lin["g"], lin["u"], lin["d"]
    XAg, XAu = rnd(X @ Ag), rnd(X @ Au)
    e, g = X @ Wg.T + s * XAg @ Bg, X @ Wu.T + su * XAu @ Bu
    E, G, H = rnd(e), rnd(g), rnd(oracle.act_fwd(act, e) * g)
    HAd = rnd(H @ Ad)
    out = {"Y": rnd(H @ Wd.T + sd * HAd @ Bd)}
    sGd = rnd(sd * dY @ Bd.T)
    out["dB_d"] = rnd(sd * HAd.T @ dY)
    dH = dY @ Wd + sGd @ Ad.T
    dE, dG = rnd(dH * G * oracle.act_grad(act, E)), rnd(dH * oracle.act_fwd(act, E))
    out["dA_d"] = rnd(H.T @ sGd)
    sGg, sGu = rnd(s * dE @ Bg.T), rnd(su * dG @ Bu.T)
    out["dB_g"], out["dB_u"] = rnd(s * XAg.T @ dE), rnd(su * XAu.T @ dG)
    out["dX"] = rnd(dE @ Wg + dG @ Wu + sGg @ Ag.T + sGu @ Au.T)
    out["dA_g"], out["dA_u"] = rnd(X.T @ sGg), rnd(X.T @ sGu)
    return out


def _ratio(got, want):
    err, rms = rel_err(got, want)
    return err / rms


def test_bf16_chain_explains_the_small_mlp_bar():
    chain_max, output_only_min = 0.0, 1.0
    for M, d, h in SMALL_MLP_CASES:
        for act in ("swiglu", "geglu_tanh"):
            X, dY, lin, ref = _case(M, d, h, act)
            em = _chain(act, X, dY, lin)
            worst = max(_ratio(em[k], ref[k]) for k in OUTS)
            assert worst <= TOL_SMALL_MLP, (M, d, h, act, worst)
            chain_max = max(chain_max, worst)
            output_only_min = min(output_only_min, max(_ratio(_bf(ref[k]), ref[k]) for k in OUTS))
    # the returned tensors' own rounding takes most of the 2e-2 budget in every case ...
    assert output_only_min >= 0.7 * TOL
    # ... and the design's stored bf16 intermediates push some case past it
    assert chain_max > TOL


def test_bf16_chain_explains_the_multi_tile_mlp_bar():
    """The multi-tile parity case of tests/test_gpu_persistent.py (2344 tokens,
    d = 1024, h = 2816, SwiGLU): more rows do not bring the whole-tensor
    maximum under 2e-2.  The design's own bf16 roundings put Y above 2e-2 x RMS
    there, so that case's bar is 2.5e-2 (still below the small-M 3e-2)."""
    from test_gpu_persistent import MLP_SHAPE, TOL_MLP_FULL_TENSOR
    M, d, h = MLP_SHAPE
    X, dY, lin, ref = _case(M, d, h, "swiglu")
    em = _chain("swiglu", X, dY, lin)
    worst = max(_ratio(em[k], ref[k]) for k in OUTS)
    assert TOL < worst <= 0.9 * TOL_MLP_FULL_TENSOR, worst


@pytest.mark.parametrize("act", ["swiglu", "geglu_tanh"])
def test_chain_emulation_is_the_oracle_without_roundings(act):
    """With every rounding removed the emulated chain is the oracle itself (a
    check that it follows the same algebra, not only similar numbers)."""
    X, dY, lin, ref = _case(96, 256, 512, act)
    em = _chain(act, X, dY, lin, rnd=lambda x: np.asarray(x, dtype=np.float64))
    for k in OUTS:
        assert _ratio(em[k], ref[k]) <= 1e-12, k
