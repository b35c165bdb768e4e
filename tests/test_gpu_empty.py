"""An empty batch (M = 0) through every entry point, against the oracle.

The adapter gradients are sums over tokens: with no tokens they are exactly
zero, which is what the oracle gives, while Y, X A and dX are empty.  The
gradients are pre-filled with NaN so that a call that leaves them untouched
fails; the comparison is bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
from qlora_fine_tuning_nf4_b200 import ops
from qlora_fine_tuning_nf4_b200.synth import bits_to_torch, make_linear_problem, make_mlp_problem, make_qkv_problem

from parity import dev, gpu_f64, gpu_weight, run_linear_oracle, run_mlp_oracle

pytestmark = pytest.mark.gpu


def _nan_like(t):
    return torch.full_like(t, float("nan"))


def _same_bits(name, gpu, ref):
    assert gpu.shape == ref.shape, name
    assert np.array_equal(gpu, ref), f"{name}: not the oracle's exact zeros"


@pytest.mark.parametrize("base,tiles", [("nf4", 4), ("nf4", 2), ("bf16", 4)])
def test_linear_empty_batch(base, tiles):
    p = make_linear_problem(0, 512, 1024, seed=11)
    ops.qlora_set_tile_config(tiles)
    A, B = dev(p["A"]), dev(p["B"])
    if base == "nf4":
        lin = ops.LoraLinear(gpu_weight(p["W"])[0], A, B, p["s"])
        fwd, bwd = ops.qlora_linear_fwd, ops.qlora_linear_bwd
    else:
        lin = ops.LoraLinear16(dev(p["W"]), A, B, p["s"])
        fwd, bwd = ops.qlora_linear16_fwd, ops.qlora_linear16_bwd
    ws = ops.Workspace()
    X, dY = dev(p["X"]), dev(p["dY"])
    Y, XA = fwd(lin, X, ws)
    dX, dA, dB = bwd(lin, X, XA, dY, ws, dA=_nan_like(A), dB=_nan_like(B))
    torch.cuda.synchronize()
    o = run_linear_oracle(p, base)
    for name, g in (("Y", Y), ("XA", XA), ("dX", dX), ("dA", dA), ("dB", dB)):
        _same_bits(name, gpu_f64(g), o[name])
    assert not o["dA"].any() and not o["dB"].any()


@pytest.mark.parametrize("base", ["nf4", "bf16"])
@pytest.mark.parametrize("act", ["swiglu", "geglu_tanh"])
def test_mlp_empty_batch(base, act):
    p = make_mlp_problem(0, 256, 512, seed=12)
    ops.qlora_set_tile_config(4)
    lins = {}
    for k in ("g", "u", "d"):
        A, B = dev(p["A_" + k]), dev(p["B_" + k])
        if base == "nf4":
            lins[k] = ops.LoraLinear(gpu_weight(p["W_" + k])[0], A, B, p["s"])
        else:
            lins[k] = ops.LoraLinear16(dev(p["W_" + k]), A, B, p["s"])
    fwd, bwd = (ops.qlora_mlp_fwd, ops.qlora_mlp_bwd) if base == "nf4" else (ops.qlora_mlp16_fwd, ops.qlora_mlp16_bwd)
    ws = ops.Workspace()
    X, dY = dev(p["X"]), dev(p["dY"])
    Y, saved = fwd(act, lins["g"], lins["u"], lins["d"], X, ws)
    grads = {"dX": torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")}
    for k in ("g", "u", "d"):
        grads["dA_" + k] = _nan_like(lins[k].A)
        grads["dB_" + k] = _nan_like(lins[k].B)
    grads = bwd(act, lins["g"], lins["u"], lins["d"], X, saved, dY, ws, grads=grads)
    torch.cuda.synchronize()
    o = run_mlp_oracle(p, act, base)
    _same_bits("Y", gpu_f64(Y), o["Y"])
    for k, v in grads.items():
        _same_bits(k, gpu_f64(v), o[k])


def test_qkv_empty_batch():
    p = make_qkv_problem(0, 512, 512, 256, 256, seed=13)
    lins = {}
    for n in "qkv":
        w = ops.nf4_quantize(bits_to_torch(p["W_" + n], "cuda"))
        lins[n] = ops.LoraLinear(w, bits_to_torch(p["A_" + n], "cuda"), bits_to_torch(p["B_" + n], "cuda"), p["s"])
    X, dY = bits_to_torch(p["X"], "cuda"), bits_to_torch(p["dY"], "cuda")
    ws = ops.Workspace()
    Y, XA = ops.qlora_qkv_fwd(lins["q"], lins["k"], lins["v"], X, ws)
    grads = {"dX": torch.empty(0, 512, dtype=torch.bfloat16, device="cuda")}
    for n in "qkv":
        grads["dA_" + n] = _nan_like(lins[n].A)
        grads["dB_" + n] = _nan_like(lins[n].B)
    grads = ops.qlora_qkv_bwd(lins["q"], lins["k"], lins["v"], X, XA, dY, ws, grads=grads)
    torch.cuda.synchronize()
    assert Y.shape == (0, 1024) and XA.shape[0] == 0
    X64, dY64 = oracle.bf16_bits_to_f64(p["X"]), oracle.bf16_bits_to_f64(p["dY"])
    col = {"q": (0, 512), "k": (512, 768), "v": (768, 1024)}
    for n in "qkv":
        A, B = oracle.bf16_bits_to_f64(p["A_" + n]), oracle.bf16_bits_to_f64(p["B_" + n])
        W = np.zeros((B.shape[1], 512))  # the base weight does not enter dA, dB
        _, dA, dB = oracle.linear_bwd(X64, W, A, B, p["s"], dY64[:, col[n][0]:col[n][1]])
        _same_bits("dA_" + n, gpu_f64(grads["dA_" + n]), dA)
        _same_bits("dB_" + n, gpu_f64(grads["dB_" + n]), dB)
