"""CPU pins for the oracle's LoRA projection, gated MLP and bracket cost model.

Pins: special cases that reduce to textbook operations (B = 0, s = 0,
absmax = 0), associativity of the rank-r chain, central finite differences of
L = sum(Y * dY), closed-form activation values, torch fp64 autograd as an
independent derivation, and the speed-ups printed on the Mistral blog.
"""

import os

import numpy as np
import pytest
import torch

import oracle
from oracle.nf4 import nf4_dequantize_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _lin(rng, M, K, N, r, s=1.0):
    X = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K)) * 0.1
    A = rng.uniform(-1, 1, (K, r)) / np.sqrt(K)
    B = rng.standard_normal((r, N)) * 0.1
    dY = rng.standard_normal((M, N))
    return X, W, A, B, s, dY


def test_b_zero_reduces_to_dense_and_zero_dA():
    rng = np.random.default_rng(0)
    X, W, A, B, s, dY = _lin(rng, 8, 64, 16, 4)
    B = np.zeros_like(B)
    Y, _ = oracle.linear_fwd(X, W, A, B, s)
    assert np.array_equal(Y, X @ W.T)
    dX, dA, dB = oracle.linear_bwd(X, W, A, B, s, dY)
    assert np.all(dA == 0)
    assert np.array_equal(dX, dY @ W)


def test_s_zero_is_pure_dense_layer():
    rng = np.random.default_rng(1)
    X, W, A, B, _, dY = _lin(rng, 8, 64, 16, 4)
    Y, _ = oracle.linear_fwd(X, W, A, B, 0.0)
    assert np.array_equal(Y, X @ W.T)
    dX, dA, dB = oracle.linear_bwd(X, W, A, B, 0.0, dY)
    assert np.all(dA == 0) and np.all(dB == 0)


def test_adapter_gradients_add_over_token_shards_and_vanish_for_no_tokens():
    """dA, dB are sums over tokens: the gradients of a batch equal the sum of
    those of any split of its rows (what a data-parallel all-reduce relies
    on), and an empty batch gives exactly zero."""
    rng = np.random.default_rng(3)
    X, W, A, B, s, dY = _lin(rng, 12, 64, 16, 4, s=2.0)
    _, dA, dB = oracle.linear_bwd(X, W, A, B, s, dY)
    _, dA1, dB1 = oracle.linear_bwd(X[:5], W, A, B, s, dY[:5])
    _, dA2, dB2 = oracle.linear_bwd(X[5:], W, A, B, s, dY[5:])
    assert np.allclose(dA, dA1 + dA2, rtol=0, atol=1e-12) and np.allclose(dB, dB1 + dB2, rtol=0, atol=1e-12)
    Y0, XA0 = oracle.linear_fwd(X[:0], W, A, B, s)
    dX0, dA0, dB0 = oracle.linear_bwd(X[:0], W, A, B, s, dY[:0])
    assert Y0.shape == (0, 16) and XA0.shape == (0, 4) and dX0.shape == (0, 64)
    assert dA0.shape == A.shape and dB0.shape == B.shape and not dA0.any() and not dB0.any()
    lin = lambda n_out, k_in: (rng.standard_normal((n_out, k_in)) * 0.1, rng.uniform(-1, 1, (k_in, 4)) / np.sqrt(k_in),
                               rng.standard_normal((4, n_out)) * 0.1, 2.0)
    g, u, d = lin(32, 16), lin(32, 16), lin(16, 32)
    Xm, dYm = rng.standard_normal((9, 16)), rng.standard_normal((9, 16))
    full = oracle.mlp_bwd("swiglu", Xm, g, u, d, dYm)
    parts = [oracle.mlp_bwd("swiglu", Xm[a:b], g, u, d, dYm[a:b]) for a, b in ((0, 4), (4, 9))]
    empty = oracle.mlp_bwd("swiglu", Xm[:0], g, u, d, dYm[:0])
    for k in ("dA_g", "dB_g", "dA_u", "dB_u", "dA_d", "dB_d"):
        assert np.allclose(full[k], parts[0][k] + parts[1][k], rtol=0, atol=1e-12), k
        assert empty[k].shape == full[k].shape and not empty[k].any(), k


def test_zero_absmax_is_pure_lora():
    rng = np.random.default_rng(2)
    M, K, N, r = 6, 128, 8, 4
    q = rng.integers(0, 256, N * K // 2, dtype=np.uint8)
    W = nf4_dequantize_f64(q, np.zeros(N * K // 64, np.float32), N, K)
    assert np.all(W == 0)
    X, _, A, B, s, dY = _lin(rng, M, K, N, r, s=2.0)
    Y, XA = oracle.linear_fwd(X, W, A, B, s)
    assert np.allclose(Y, s * (X @ A) @ B, rtol=0, atol=1e-12)


def test_rank_chain_is_associative():
    rng = np.random.default_rng(3)
    X, W, A, B, s, dY = _lin(rng, 32, 256, 128, 16)
    Y, XA = oracle.linear_fwd(X, np.zeros_like(W), A, B, 1.0)
    ref = X @ (A @ B)
    assert np.max(np.abs(Y - ref)) <= 1e-12 * np.max(np.abs(ref))


def _fd(f, P, h):
    g = np.zeros_like(P)
    it = np.nditer(P, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = P[i]
        P[i] = old + h
        fp = f()
        P[i] = old - h
        fm = f()
        P[i] = old
        g[i] = (fp - fm) / (2 * h)
    return g


def test_linear_backward_matches_central_differences():
    rng = np.random.default_rng(4)
    X, W, A, B, s, dY = _lin(rng, 4, 64, 8, 2, s=1.5)
    loss = lambda: float(np.sum(oracle.linear_fwd(X, W, A, B, s)[0] * dY))
    dX, dA, dB = oracle.linear_bwd(X, W, A, B, s, dY)
    for P, g in ((X, dX), (A, dA), (B, dB)):
        num = _fd(loss, P, 1e-6)
        assert np.max(np.abs(num - g)) <= 1e-7 * max(1.0, np.max(np.abs(g)))


def test_linear_matches_torch_autograd_fp64():
    rng = np.random.default_rng(5)
    X, W, A, B, s, dY = _lin(rng, 16, 128, 48, 8, s=0.5)
    tX, tA, tB = (torch.tensor(v, requires_grad=True) for v in (X, A, B))
    tY = tX @ torch.tensor(W).T + s * (tX @ tA) @ tB
    tY.backward(torch.tensor(dY))
    Y, _ = oracle.linear_fwd(X, W, A, B, s)
    dX, dA, dB = oracle.linear_bwd(X, W, A, B, s, dY)
    np.testing.assert_allclose(Y, tY.detach().numpy(), rtol=1e-12, atol=1e-12)
    for ours, ref in ((dX, tX.grad), (dA, tA.grad), (dB, tB.grad)):
        np.testing.assert_allclose(ours, ref.numpy(), rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------- activations ----

@pytest.mark.parametrize("kind", oracle.ACTIVATIONS)
def test_activation_closed_forms(kind):
    assert oracle.act_fwd(kind, np.array([0.0]))[0] == 0.0
    assert oracle.act_grad(kind, np.array([0.0]))[0] == 0.5
    big = np.array([40.0])
    assert abs(oracle.act_fwd(kind, big)[0] - 40.0) < 1e-12
    assert abs(oracle.act_grad(kind, big)[0] - 1.0) < 1e-12
    assert abs(oracle.act_fwd(kind, -big)[0]) < 1e-12
    assert abs(oracle.act_grad(kind, -big)[0]) < 1e-12


@pytest.mark.parametrize("kind", oracle.ACTIVATIONS)
def test_activation_matches_torch_and_central_differences(kind):
    e = np.linspace(-8, 8, 4001)
    te = torch.tensor(e, requires_grad=True)
    f = torch.nn.functional.silu(te) if kind == "swiglu" else \
        torch.nn.functional.gelu(te, approximate="tanh")
    f.sum().backward()
    np.testing.assert_allclose(oracle.act_fwd(kind, e), f.detach().numpy(), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(oracle.act_grad(kind, e), te.grad.numpy(), rtol=1e-12, atol=1e-13)
    h = 1e-5
    num = (oracle.act_fwd(kind, e + h) - oracle.act_fwd(kind, e - h)) / (2 * h)
    np.testing.assert_allclose(oracle.act_grad(kind, e), num, rtol=0, atol=1e-9)


# ------------------------------------------------------------------ MLP ----

def _mlp(rng, M, d, h, r):
    X = rng.standard_normal((M, d))
    def proj(K, N, s):
        return (rng.standard_normal((N, K)) * 0.2, rng.uniform(-1, 1, (K, r)) / np.sqrt(K),
                rng.standard_normal((r, N)) * 0.3, s)
    return X, proj(d, h, 1.0), proj(d, h, 0.75), proj(h, d, 2.0), rng.standard_normal((M, d))


@pytest.mark.parametrize("kind", oracle.ACTIVATIONS)
def test_mlp_backward_matches_central_differences(kind):
    rng = np.random.default_rng(6)
    X, gate, up, down, dY = _mlp(rng, 4, 64, 128, 2)
    loss = lambda: float(np.sum(oracle.mlp_fwd(kind, X, gate, up, down)["Y"] * dY))
    g = oracle.mlp_bwd(kind, X, gate, up, down, dY)
    checks = [(X, g["dX"]), (gate[1], g["dA_g"]), (gate[2], g["dB_g"]), (up[1], g["dA_u"]),
              (up[2], g["dB_u"]), (down[1], g["dA_d"]), (down[2], g["dB_d"])]
    for P, ana in checks:
        num = _fd(loss, P, 1e-5)
        assert np.max(np.abs(num - ana)) <= 1e-6 * max(1.0, np.max(np.abs(ana)))


@pytest.mark.parametrize("kind", oracle.ACTIVATIONS)
def test_mlp_matches_torch_autograd_fp64(kind):
    rng = np.random.default_rng(7)
    X, gate, up, down, dY = _mlp(rng, 12, 64, 96, 4)
    t = lambda a: torch.tensor(a, requires_grad=True)
    tX = t(X)
    tp = [(torch.tensor(W), t(A), t(B), s) for (W, A, B, s) in (gate, up, down)]
    lin = lambda Z, p: Z @ p[0].T + p[3] * (Z @ p[1]) @ p[2]
    act = torch.nn.functional.silu if kind == "swiglu" else \
        (lambda z: torch.nn.functional.gelu(z, approximate="tanh"))
    tY = lin(act(lin(tX, tp[0])) * lin(tX, tp[1]), tp[2])
    tY.backward(torch.tensor(dY))
    out = oracle.mlp_fwd(kind, X, gate, up, down)
    g = oracle.mlp_bwd(kind, X, gate, up, down, dY)
    np.testing.assert_allclose(out["Y"], tY.detach().numpy(), rtol=1e-11, atol=1e-11)
    pairs = [(g["dX"], tX.grad), (g["dA_g"], tp[0][1].grad), (g["dB_g"], tp[0][2].grad),
             (g["dA_u"], tp[1][1].grad), (g["dB_u"], tp[1][2].grad),
             (g["dA_d"], tp[2][1].grad), (g["dB_d"], tp[2][2].grad)]
    for ours, ref in pairs:
        np.testing.assert_allclose(ours, ref.numpy(), rtol=1e-10, atol=1e-10)


# --------------------------------------------------------- bracket cost ----

def test_bracket_speedups_printed_on_the_page():
    with open(os.path.join(GOLDEN, "bracket_speedup.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) == 2
    for name, h, d, r, printed in rows:
        h, d, r, printed = int(h), int(d), int(r), float(printed)
        assert round(oracle.bracket_speedup_limit(h, d, r), 2) == printed
        slow, fast = oracle.bracket_costs(10 ** 9, h, d, r)
        assert abs(slow / fast - printed) < 0.01


def test_bracket_costs_count_the_actual_products():
    """Count the multiply-adds of each bracket order by explicit shapes."""
    m, h, d, r = 64, 40, 24, 4
    # slow: (X^T dY) is (d x m)(m x h) -> d*h*m, then (d x h)(h x r) -> d*h*r
    slow_count = d * m * h + d * h * r
    # fast: (dY B^T) is (m x h)(h x r) -> m*h*r, then (d x m)(m x r) -> d*m*r
    fast_count = m * h * r + d * m * r
    assert oracle.bracket_costs(m, h, d, r) == (slow_count, fast_count)


def test_benchmark_setup_constants():
    with open(os.path.join(GOLDEN, "lora_benchmark_setup.txt")) as f:
        kv = dict(l.split() for l in f if l.strip() and not l.startswith("#"))
    from qlora_fine_tuning_nf4_b200.workloads import LINEAR_WORKLOADS, MLP_WORKLOADS
    for w in list(LINEAR_WORKLOADS.values()) + list(MLP_WORKLOADS.values()):
        assert w["r"] == int(kv["rank"]) and w["alpha"] == float(kv["alpha"])
    assert MLP_WORKLOADS["llama7b_swiglu_mlp"]["M"] == int(kv["batch_size"]) * int(kv["max_seq_length"])
