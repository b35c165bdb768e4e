"""Seeded synthetic inputs for the QLoRA projection and gated-MLP workloads.

This module only draws random numbers and casts them to bf16; it holds none
of the method's arithmetic, so both the CUDA path's tests and the CPU oracle
can take their inputs from it.

Recipe (stands in for the fine-tuning datasets and checkpoints the pages
benchmark on, which are not available): numpy ``SeedSequence(seed)`` spawns
one child generator per tensor in a fixed order; values are drawn in binary32
and rounded to bf16 (round-to-nearest-even, via torch's bf16 cast).

* activations X and upstream gradient dY ~ N(0, 1);
* frozen base weights W [N, K] ~ N(0, 0.02) (quantised to NF4 later by
  whichever side is under test);
* LoRA A [K, r] ~ U(-1/sqrt(K), 1/sqrt(K)) (kaiming-uniform, a = sqrt(5));
* LoRA B [r, N] ~ N(0, 0.02) (non-zero, so that dA is non-zero).

bf16 tensors are returned as ``uint16`` numpy arrays of bit patterns.
"""

import numpy as np
import torch


def bf16_bits(a):
    """Round a binary32 numpy array to bf16 bit patterns (uint16)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bits_to_torch(bits, device=None):
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor (optionally on device)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device) if device is not None else t


def _normal(rng, shape, std=1.0):
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return bf16_bits(x)


def _uniform(rng, shape, bound):
    u = rng.random(shape, dtype=np.float32)
    return bf16_bits((u * np.float32(2.0) - np.float32(1.0)) * np.float32(bound))


def make_linear_problem(M, K, N, r=16, alpha=16.0, seed=0):
    """One QLoRA linear: X [M,K], W [N,K], A [K,r], B [r,N], dY [M,N] (bf16 bits).

    Child order: X, W, A, B, dY.  ``s`` = alpha / r.
    """
    ch = [np.random.default_rng(c) for c in np.random.SeedSequence(seed).spawn(5)]
    return {
        "X": _normal(ch[0], (M, K)),
        "W": _normal(ch[1], (N, K), 0.02),
        "A": _uniform(ch[2], (K, r), 1.0 / np.sqrt(K)),
        "B": _normal(ch[3], (r, N), 0.02),
        "dY": _normal(ch[4], (M, N)),
        "s": float(alpha) / float(r),
        "M": M, "K": K, "N": N, "r": r,
    }


def make_mlp_problem(M, d, h, r=16, alpha=16.0, seed=0):
    """Gated MLP: X [M,d]; gate/up W [h,d], A [d,r], B [r,h]; down W [d,h],
    A [h,r], B [r,d]; dY [M,d] (bf16 bits).

    Child order: X, W_g, W_u, W_d, A_g, A_u, A_d, B_g, B_u, B_d, dY.
    """
    ch = [np.random.default_rng(c) for c in np.random.SeedSequence(seed).spawn(11)]
    return {
        "X": _normal(ch[0], (M, d)),
        "W_g": _normal(ch[1], (h, d), 0.02),
        "W_u": _normal(ch[2], (h, d), 0.02),
        "W_d": _normal(ch[3], (d, h), 0.02),
        "A_g": _uniform(ch[4], (d, r), 1.0 / np.sqrt(d)),
        "A_u": _uniform(ch[5], (d, r), 1.0 / np.sqrt(d)),
        "A_d": _uniform(ch[6], (h, r), 1.0 / np.sqrt(h)),
        "B_g": _normal(ch[7], (r, h), 0.02),
        "B_u": _normal(ch[8], (r, h), 0.02),
        "B_d": _normal(ch[9], (r, d), 0.02),
        "dY": _normal(ch[10], (M, d)),
        "s": float(alpha) / float(r),
        "M": M, "d": d, "h": h, "r": r,
    }


def make_qkv_problem(M, K, nq, nk, nv, r=16, alpha=16.0, seed=0):
    """Fused Q/K/V projections of one input: X [M,K]; W_p [n_p,K], A_p [K,r],
    B_p [r,n_p] for p in q, k, v; dY [M, nq+nk+nv] (bf16 bits).

    Child order: X, W_q, W_k, W_v, A_q, A_k, A_v, B_q, B_k, B_v, dY.
    """
    ch = [np.random.default_rng(c) for c in np.random.SeedSequence(seed).spawn(11)]
    n = {"q": nq, "k": nk, "v": nv}
    out = {"X": _normal(ch[0], (M, K))}
    for i, p in enumerate("qkv"):
        out["W_" + p] = _normal(ch[1 + i], (n[p], K), 0.02)
        out["A_" + p] = _uniform(ch[4 + i], (K, r), 1.0 / np.sqrt(K))
        out["B_" + p] = _normal(ch[7 + i], (r, n[p]), 0.02)
    out["dY"] = _normal(ch[10], (M, nq + nk + nv))
    out.update({"s": float(alpha) / float(r), "M": M, "K": K, "nq": nq, "nk": nk, "nv": nv, "r": r})
    return out
