"""The plain C loop oracle (oracle/c/qlora_oracle.c) against the numpy oracle.

Two independent statements of the same definitions (different languages,
quantile routines, loop orders and summation orders) must agree: the NF4
codebook, codes and absmax bit for bit, the dequantised weight exactly, and
the projection's forward and backward to binary64 rounding on the tiny
configuration (256 x 512 -> 1024, rank 16), and the gated MLP's forward and
backward (both activations, with derivatives written separately in each) on a
small MLP.  A mistake in either (a dropped LoRA term, a transposed operand, a
wrong nibble order or tie rule, a wrong activation derivative) fails here.
"""

import numpy as np
import pytest

import oracle
from oracle import c_oracle
from oracle.nf4 import nf4_dequantize_f64
from qlora_fine_tuning_nf4_b200.synth import bf16_bits, make_linear_problem, make_mlp_problem
from qlora_fine_tuning_nf4_b200.workloads import LINEAR_WORKLOADS


def test_codebooks_agree_bit_for_bit():
    assert np.array_equal(c_oracle.nf4_codebook(), oracle.nf4_codebook())


def _adversarial_weight():
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    w[1, :64] = 0.0                                   # all-zero block
    w[2, 64:128] = -np.abs(w[2, 64:128])              # absmax element negative
    w[2, 70] = -0.5
    mids = oracle.nf4_midpoints()
    w[3, :64] = 0.0
    w[3, 0] = 1.0                                     # absmax 1: values land on (bf16 neighbours of) midpoints
    w[3, 1:16] = mids.astype(np.float32)
    w[4, 128:192] = rng.standard_normal(64) * 1e-38   # subnormal magnitudes
    return bf16_bits(w)


@pytest.mark.parametrize("case", ["tiny_linear", "adversarial"])
def test_quantise_and_dequantise_agree_bit_for_bit(case):
    if case == "tiny_linear":
        cfg = LINEAR_WORKLOADS["tiny_linear"]
        w = make_linear_problem(cfg["M"], cfg["K"], cfg["N"], seed=cfg["seed"])["W"]
    else:
        w = _adversarial_weight()
    n, k = w.shape
    cc, ca = c_oracle.nf4_quantize(w, n, k)
    nc, na = oracle.nf4_quantize(w, n, k)
    assert np.array_equal(cc, nc) and np.array_equal(ca, na)
    assert np.array_equal(c_oracle.nf4_dequantize_f64(cc, ca, n, k), nf4_dequantize_f64(nc, na, n, k))


def test_linear_forward_and_backward_agree():
    cfg = LINEAR_WORKLOADS["tiny_linear"]
    p = make_linear_problem(cfg["M"], cfg["K"], cfg["N"], cfg["r"], cfg["alpha"], cfg["seed"])
    n, k = p["W"].shape
    codes, absmax = oracle.nf4_quantize(p["W"], n, k)
    W = nf4_dequantize_f64(codes, absmax, n, k)
    X, A, B, dY = (oracle.bf16_bits_to_f64(p[t]) for t in ("X", "A", "B", "dY"))
    s = p["s"]
    cy, cxa = c_oracle.linear_fwd(X, W, A, B, s)
    ny, nxa = oracle.linear_fwd(X, W, A, B, s)
    c_b = c_oracle.linear_bwd(X, W, A, B, s, dY)
    n_b = oracle.linear_bwd(X, W, A, B, s, dY)
    for name, c, o in [("Y", cy, ny), ("XA", cxa, nxa)] + list(zip(("dX", "dA", "dB"), c_b, n_b)):
        rms = np.sqrt(np.mean(o * o))
        assert np.max(np.abs(c - o)) <= 1e-12 * rms, name


@pytest.mark.parametrize("kind", ["swiglu", "geglu_tanh"])
def test_gated_mlp_forward_and_backward_agree(kind):
    """The C loops' gated MLP (their own activations and derivatives, written
    from the definitions) against the numpy oracle, on bf16-valued inputs of a
    small MLP with the pages' structure (d -> h -> d, rank r, s = alpha / r)."""
    p = make_mlp_problem(48, 256, 512, r=16, alpha=32.0, seed=9)
    lin = {}
    for k in ("g", "u", "d"):
        n, kk = p["W_" + k].shape
        codes, absmax = oracle.nf4_quantize(p["W_" + k], n, kk)
        lin[k] = (nf4_dequantize_f64(codes, absmax, n, kk), oracle.bf16_bits_to_f64(p["A_" + k]),
                  oracle.bf16_bits_to_f64(p["B_" + k]), p["s"])
    X, dY = oracle.bf16_bits_to_f64(p["X"]), oracle.bf16_bits_to_f64(p["dY"])
    cf = c_oracle.mlp_fwd(kind, X, lin["g"], lin["u"], lin["d"])
    nf = oracle.mlp_fwd(kind, X, lin["g"], lin["u"], lin["d"])
    cb = c_oracle.mlp_bwd(kind, X, lin["g"], lin["u"], lin["d"], dY)
    nb = oracle.mlp_bwd(kind, X, lin["g"], lin["u"], lin["d"], dY)
    for name, c, o in [(k, cf[k], nf[k]) for k in ("Y", "E", "G", "H")] + [(k, cb[k], nb[k]) for k in cb]:
        rms = np.sqrt(np.mean(o * o))
        assert np.max(np.abs(c - o)) <= 1e-12 * rms, name
