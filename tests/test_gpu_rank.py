"""GPU parity at LoRA ranks 32 and 64 (the Mistral blog's r = 64 variant) and
with the rank-stabilised scale s = alpha / sqrt(r), on the staged-feed GEMM
(NF4 base, tile configuration 4) and on the 16-bit entry points, against the
fp64 oracle.  Same bars as the rank-16 tests."""

import numpy as np
import pytest

from qlora_fine_tuning_nf4_b200.synth import make_linear_problem, make_mlp_problem

from parity import (TOL_SMALL_MLP, assert_close, assert_saved, run_linear16_gpu, run_linear_gpu,
                    run_linear_oracle, run_mlp16_gpu, run_mlp_gpu, run_mlp_oracle, saved_bounds)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("base", ["nf4", "bf16"])
@pytest.mark.parametrize("r", [32, 64])
@pytest.mark.parametrize("M,K,N", [(256, 512, 1024), (300, 768, 520), (1, 256, 256)])
def test_linear_rank_parity(base, r, M, K, N):
    p = make_linear_problem(M, K, N, r=r, alpha=2.0 * r, seed=r + M + K + N)
    g = run_linear_gpu(p, 4) if base == "nf4" else run_linear16_gpu(p)
    o = run_linear_oracle(p, base=base)
    assert g["status"] == 0
    if base == "nf4":
        assert np.array_equal(g["codes"], o["codes"]) and np.array_equal(g["absmax"], o["absmax"])
    for k in ("XA", "Y", "dX"):
        assert_close(k, g[k], o[k])
    for k in ("dA", "dB"):
        if M == 1:
            # one token row: dA and dB are outer products, each element two bf16 roundings
            # (of s G or X A, and of the result) away from the exact value, 2^-8 relative each
            assert_saved(k, g[k], o[k], 2.0 ** -7 * np.abs(o[k]) + 2.0 ** -12 * np.sqrt(np.mean(o[k] ** 2)))
        else:
            assert_close(k, g[k], o[k])


def test_linear_rslora_scale():
    """r = 64 with s = alpha / sqrt(r) (RSLoRA) instead of alpha / r."""
    p = make_linear_problem(384, 1024, 768, r=64, alpha=16.0, seed=64)
    p["s"] = 16.0 / np.sqrt(64.0)
    g = run_linear_gpu(p, 4)
    o = run_linear_oracle(p)
    for k in ("XA", "Y", "dX", "dA", "dB"):
        assert_close(k, g[k], o[k])


@pytest.mark.parametrize("base", ["nf4", "bf16"])
@pytest.mark.parametrize("act", ["swiglu", "geglu_tanh"])
@pytest.mark.parametrize("r", [32, 64])
def test_mlp_rank_parity(base, act, r):
    M, d, h = 384, 512, 768
    p = make_mlp_problem(M, d, h, r=r, alpha=2.0 * r, seed=r + 7)
    g = run_mlp_gpu(p, act, 4) if base == "nf4" else run_mlp16_gpu(p, act)
    o = run_mlp_oracle(p, act, base=base)
    assert g["status"] == 0
    bounds = saved_bounds(o, p)
    for k in ("E", "G", "H"):
        assert_saved(k, g[k], o[k], bounds[k])
    for k in ("XA_g", "XA_u", "HA_d"):
        assert_close(k, g[k], o[k])
    for k in ("Y", "dX", "dA_g", "dB_g", "dA_u", "dB_u", "dA_d", "dB_d"):
        assert_close(k, g[k], o[k], TOL_SMALL_MLP)
