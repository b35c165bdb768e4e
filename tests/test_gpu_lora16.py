"""GPU parity of the 16-bit LoRA entry points (a frozen bf16 base weight in
place of NF4: the Mistral blog's "load_in_4bit = False" variant) against the
fp64 oracle fed the same bf16 weight.  Same bar as the NF4 path: every bf16
output and gradient within max|gpu - oracle| <= 2e-2 * RMS(oracle) (3e-2 for
the small-M gated MLP, for the reason given in parity.py), saved activations
element by element."""

import numpy as np
import pytest
import torch

from qlora_fine_tuning_nf4_b200 import ops
from qlora_fine_tuning_nf4_b200.synth import bits_to_torch, make_linear_problem, make_mlp_problem
from qlora_fine_tuning_nf4_b200.workloads import MLP_WORKLOADS

from parity import (TOL, TOL_SMALL_MLP, assert_close, assert_saved, run_linear16_gpu, run_linear_oracle,
                    run_mlp16_gpu, run_mlp_oracle, saved_bounds)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,N,alpha", [(256, 512, 1024, 16.0), (200, 512, 1024, 16.0), (1, 256, 256, 16.0),
                                         (300, 768, 520, 32.0), (640, 1024, 768, 8.0)])
def test_linear16_fwd_bwd_parity(M, K, N, alpha):
    p = make_linear_problem(M, K, N, r=16, alpha=alpha, seed=M + K + N)
    g = run_linear16_gpu(p)
    o = run_linear_oracle(p, base="bf16")
    assert g["status"] == 0
    for k in ("XA", "Y", "dX", "dA", "dB"):
        assert_close(k, g[k], o[k])


@pytest.mark.parametrize("act", ["swiglu", "geglu_tanh"])
@pytest.mark.parametrize("M,d,h", [(256, 256, 512), (200, 512, 768), (1100, 512, 768)])
def test_mlp16_fwd_bwd_parity(act, M, d, h):
    p = make_mlp_problem(M, d, h, seed=M + d + h)
    g = run_mlp16_gpu(p, act)
    o = run_mlp_oracle(p, act, base="bf16")
    assert g["status"] == 0
    bounds = saved_bounds(o, p)
    for k in ("E", "G", "H"):
        assert_saved(k, g[k], o[k], bounds[k])
    for k in ("XA_g", "XA_u", "HA_d"):
        assert_close(k, g[k], o[k])
    for k in ("Y", "dX", "dA_g", "dB_g", "dA_u", "dB_u", "dA_d", "dB_d"):
        assert_close(k, g[k], o[k], TOL_SMALL_MLP)


def test_mlp16_full_size_sampled_rows():
    """Llama-7B widths at 8192 tokens: Y, dX and the saved rows of a sample of
    token rows, each a row-local function the oracle evaluates on those rows."""
    cfg = MLP_WORKLOADS["llama7b_swiglu_mlp"]
    p = make_mlp_problem(cfg["M"], cfg["d"], cfg["h"], cfg["r"], cfg["alpha"], cfg["seed"])
    rows = np.array([0, 1, 977, 4096, 5555, 8191])
    g = run_mlp16_gpu(p, cfg["act"], rows=rows)
    assert g["status"] == 0
    sub = dict(p)
    sub["X"], sub["dY"] = p["X"][rows], p["dY"][rows]
    o = run_mlp_oracle(sub, cfg["act"], base="bf16")
    bounds = saved_bounds(o, sub)
    for k in ("E", "G", "H"):
        assert_saved(k, g[k], o[k], bounds[k])
    for k in ("Y", "dX"):
        assert_close(k, g[k], o[k], TOL)


def test_lora16_matches_nf4_path_on_dequantised_weight():
    """A bf16 base equal to dequant(NF4) gives what the NF4 entry point gives (same kernels after the weight)."""
    p = make_linear_problem(512, 1024, 768, seed=11)
    w4 = ops.nf4_quantize(bits_to_torch(p["W"], "cuda"))
    deq = ops.nf4_dequantize(w4)
    A, B, X = (bits_to_torch(p[k], "cuda") for k in ("A", "B", "X"))
    ops.qlora_set_tile_config(4)
    ws = ops.Workspace()
    Y4, XA4 = ops.qlora_linear_fwd(ops.LoraLinear(w4, A, B, p["s"]), X, ws)
    Y16, XA16 = ops.qlora_linear16_fwd(ops.LoraLinear16(deq, A, B, p["s"]), X, ws)
    torch.cuda.synchronize()
    assert torch.equal(Y4, Y16) and torch.equal(XA4, XA16)
