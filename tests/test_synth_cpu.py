"""The seeded input generators follow the stated recipe: reproducible per seed,
independent per tensor, bf16 values, and the stated distributions
(X, dY ~ N(0, 1); W ~ N(0, 0.02); A ~ U(-1/sqrt(k_in), 1/sqrt(k_in)); B ~ N(0, 0.02))."""

import numpy as np

import oracle
from qlora_fine_tuning_nf4_b200.synth import make_linear_problem, make_mlp_problem, make_qkv_problem


def _f(bits):
    return oracle.bf16_bits_to_f64(bits)


def test_same_seed_same_bits_and_different_seed_different_bits():
    a = make_linear_problem(64, 256, 512, seed=3)
    b = make_linear_problem(64, 256, 512, seed=3)
    c = make_linear_problem(64, 256, 512, seed=4)
    for k in ("X", "W", "A", "B", "dY"):
        assert a[k].dtype == np.uint16 and np.array_equal(a[k], b[k]), k
        assert not np.array_equal(a[k], c[k]), k


def test_stated_distributions_and_shapes():
    M, K, N, r = 512, 1024, 768, 16
    p = make_linear_problem(M, K, N, r=r, alpha=32.0, seed=1)
    assert p["X"].shape == (M, K) and p["W"].shape == (N, K) and p["A"].shape == (K, r)
    assert p["B"].shape == (r, N) and p["dY"].shape == (M, N) and p["s"] == 2.0
    for k, std in (("X", 1.0), ("dY", 1.0), ("W", 0.02), ("B", 0.02)):
        v = _f(p[k])
        n = v.size
        assert abs(v.mean()) < 5 * std / np.sqrt(n), k          # five standard errors
        assert abs(v.std() / std - 1.0) < 5 / np.sqrt(2 * n) + 4e-3, k  # plus bf16 rounding
    a = _f(p["A"])
    bound = 1.0 / np.sqrt(K)
    assert np.max(np.abs(a)) <= bound * (1 + 2 ** -8)               # within the bound, up to one bf16 rounding
    assert abs(a.std() / (bound / np.sqrt(3)) - 1.0) < 0.03          # U(-b, b) has std b / sqrt(3)


def test_tensors_are_drawn_independently():
    """Each tensor has its own child generator: changing one shape leaves the
    others' values unchanged."""
    a = make_linear_problem(64, 256, 512, seed=5)
    b = make_linear_problem(96, 256, 512, seed=5)     # more token rows: X and dY grow
    for k in ("W", "A", "B"):
        assert np.array_equal(a[k], b[k]), k


def test_mlp_and_qkv_shapes():
    p = make_mlp_problem(32, 256, 512, r=16, seed=0)
    assert p["W_g"].shape == p["W_u"].shape == (512, 256) and p["W_d"].shape == (256, 512)
    assert p["A_d"].shape == (512, 16) and p["B_d"].shape == (16, 256) and p["dY"].shape == (32, 256)
    q = make_qkv_problem(32, 256, 512, 256, 256, r=32, seed=0)
    assert q["W_k"].shape == (256, 256) and q["B_q"].shape == (32, 512) and q["dY"].shape == (32, 1024)
