"""CPU pins for the oracle's bf16 rounding, NF4 codebook, quantiser and dequantiser.

Each test ties the oracle to something other than itself: an independent
normal CDF (math.erfc), a brute-force nearest-level search, a hand-worked
block, torch's own bf16 cast, or an invariant of the NF4 definition.
"""

import math
import os

import numpy as np
import torch

import oracle
from oracle.nf4 import nf4_dequantize, nf4_midpoints, nf4_unpack
from qlora_fine_tuning_nf4_b200.synth import bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- bf16 -----

def test_bf16_rounding_matches_torch_cast():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(100000).astype(np.float32),
        (rng.standard_normal(1000) * 1e-38).astype(np.float32),  # subnormals
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38], dtype=np.float32),
    ])
    # exact ties: low half exactly 0x8000, both parities of the kept half
    ties = (np.arange(1000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    x = np.concatenate([x, ties])
    ours = oracle.f32_to_bf16_bits(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_widening_is_exact():
    bits = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    finite = ((bits >> 7) & 0xFF) != 0xFF
    ours = oracle.bf16_bits_to_f64(bits[finite])
    ref = torch.from_numpy(bits[finite].view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(ours, ref)


# ------------------------------------------------------------ codebook -----

def _phi(x):
    """Standard normal CDF from erfc (independent of inv_cdf)."""
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def _quantile_by_bisection(p):
    lo, hi = -10.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if _phi(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def test_codebook_structure():
    c = oracle.nf4_codebook()
    assert c.shape == (16,)
    assert np.array_equal(c.astype(np.float32).astype(np.float64), c)  # binary32
    assert np.all(np.diff(c) > 0)
    assert c[0] == -1.0 and c[7] == 0.0 and c[15] == 1.0
    assert (c < 0).sum() == 7 and (c > 0).sum() == 8


def test_codebook_from_independent_quantile():
    """Rebuild the levels with a bisection quantile on erfc: same binary32 values."""
    delta = 0.5 * ((1 - 1 / 30) + (1 - 1 / 32))
    pos = [_quantile_by_bisection(delta + (0.5 - delta) * i / 8) for i in range(8)]
    neg = [-_quantile_by_bisection(delta + (0.5 - delta) * i / 7) for i in range(7)]
    lv = sorted(neg + [0.0] + pos)
    scale = max(abs(v) for v in lv)
    ind = np.array([v / scale for v in lv]).astype(np.float32).astype(np.float64)
    c = oracle.nf4_codebook()
    ulp = np.abs(np.spacing(c.astype(np.float32))).astype(np.float64)
    assert np.all(np.abs(ind - c) <= ulp), (ind - c) / ulp


def test_codebook_defining_property_quantiles_evenly_spaced():
    """Phi(level * scale) is evenly spaced from 1/2 to delta on each side."""
    c = oracle.nf4_codebook()
    delta = 0.5 * ((1 - 1 / 30) + (1 - 1 / 32))
    scale = _quantile_by_bisection(delta)
    p_pos = np.array([_phi(v * scale) for v in c[8:]])   # ascending to delta
    p_neg = np.array([_phi(-v * scale) for v in c[:7]])  # -level, ascending order reversed
    assert np.allclose(np.diff(p_pos), (delta - 0.5) / 8, atol=1e-7)
    assert np.allclose(np.sort(p_neg)[:0:-1] - np.sort(p_neg)[-2::-1], (delta - 0.5) / 7, atol=1e-7)
    assert abs(p_pos[-1] - delta) < 1e-7 and abs(np.max(p_neg) - delta) < 1e-7


# ------------------------------------------------------------ quantise -----

def _bits(a):
    return bf16_bits(np.asarray(a, dtype=np.float32))


def test_quantize_matches_bruteforce_random_and_edges():
    rng = np.random.default_rng(7)
    N, K = 6, 256
    w = rng.standard_normal((N, K)).astype(np.float32) * 0.02
    w[0, 0:64] = 0.0                       # all-zero block
    w[1, 64:128] = 0.0
    w[1, 70] = -0.5                        # absmax element negative, lone non-zero
    w[2, 128:192] *= 1e-30                 # tiny magnitudes
    w[3, :64] = np.linspace(-1, 1, 64)     # dense sweep of the level range
    bits = _bits(w)
    q1, a1 = oracle.nf4_quantize(bits, N, K)
    q2, a2 = oracle.nf4_quantize_bruteforce(bits, N, K)
    assert np.array_equal(q1, q2) and np.array_equal(a1, a2)


def test_quantize_ties_take_lower_level():
    """Midpoints that are binary32 numbers: v exactly on them picks the lower index."""
    code = oracle.nf4_codebook()
    mids = nf4_midpoints(code)
    for i, m in enumerate(mids):
        if np.float32(m) != m:
            continue
        v = np.array([[m]])
        idx_count = int((v[0, 0] > mids).sum())
        d = np.abs(v[0, 0] - code)
        idx_brute = int(np.flatnonzero(d == d.min())[0])
        assert idx_count == idx_brute == i


def test_hand_worked_block_fixes_nibble_order():
    rows = {}
    with open(os.path.join(GOLDEN, "nf4_pack_example.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, *v = line.split()
            rows[k] = v
    w = np.zeros(64, dtype=np.float32)
    w[:8] = [float(x) for x in rows["w_first8"]]
    q, a = oracle.nf4_quantize(_bits(w), 1, 64)
    assert a[0] == float(rows["absmax"][0])
    assert bytes(q).hex() == rows["codes_hex"][0]
    assert list(nf4_unpack(q)[:8]) == [int(x) for x in rows["levels_first8"]]
    w32, wb = nf4_dequantize(q, a, 1, 64)
    assert list(w32[0, :3]) == [float(x) for x in rows["dequant_first3"]]


def test_all_zero_block():
    q, a = oracle.nf4_quantize(_bits(np.zeros((2, 128))), 2, 128)
    assert np.all(q == 0x77) and np.all(a == 0)
    w32, wb = nf4_dequantize(q, a, 2, 128)
    assert np.all(w32 == 0) and np.all(wb == 0)


def test_dequant_then_quantize_is_idempotent():
    rng = np.random.default_rng(3)
    N, K = 32, 512
    q, a = oracle.nf4_quantize(_bits(rng.standard_normal((N, K)) * 0.02), N, K)
    w32, _ = nf4_dequantize(q, a, N, K)
    # re-quantise the binary32 dequantised values with the same rule
    blocks = w32.reshape(-1, 64)
    am = np.abs(blocks).max(axis=1)
    v = (blocks / am[:, None]).astype(np.float32).astype(np.float64)
    idx = (v[..., None] > nf4_midpoints()).sum(-1)
    assert np.array_equal(am.astype(np.float32), a)
    assert np.array_equal(idx.reshape(-1), nf4_unpack(q))


def test_reconstruction_error_bounded_by_half_gap():
    rng = np.random.default_rng(4)
    N, K = 16, 1024
    wf = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    bits = _bits(wf)
    w = oracle.bf16_bits_to_f64(bits).reshape(-1, 64)
    q, a = oracle.nf4_quantize(bits, N, K)
    w32, _ = nf4_dequantize(q, a, N, K)
    half_gap = np.max(np.diff(oracle.nf4_codebook())) / 2
    err = np.abs(w - w32.reshape(-1, 64))
    bound = half_gap * a.astype(np.float64)[:, None] * (1 + 1e-6)
    assert np.all(err <= bound)
    assert abs(half_gap - 0.1519) < 1e-3   # widest gap is between -1 and -0.696


def test_dequant_is_rne_of_binary32_product():
    rng = np.random.default_rng(5)
    q = rng.integers(0, 256, 512, dtype=np.uint8)
    a = (rng.random(16) * 3).astype(np.float32)
    w32, wb = nf4_dequantize(q, a, 4, 256)
    lv = oracle.nf4_codebook()[nf4_unpack(q)].reshape(-1, 64)
    ref32 = (lv.astype(np.float32) * a[:, None]).reshape(4, 256)       # binary32 multiply
    ref16 = torch.from_numpy(ref32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(w32, ref32.astype(np.float64))
    assert np.array_equal(wb, ref16)


def test_binary32_thresholds_take_the_binary64_midpoint_decisions():
    """The quantiser may compare v = RN_binary32(w / absmax) with t_i, the
    midpoint m_i rounded toward -inf to binary32, instead of with m_i in
    binary64: for every binary32 v near each midpoint (and at it), v > m_i and
    v > t_i agree."""
    mids = oracle.nf4_midpoints()
    for m in mids:
        t = np.float32(m)
        if np.float64(t) > m:
            t = np.nextafter(t, np.float32(-np.inf))
        assert np.float64(t) <= m < np.float64(np.nextafter(t, np.float32(np.inf)))
        v = np.float32(m)
        near = [v]
        lo = hi = v
        for _ in range(6):
            lo = np.nextafter(lo, np.float32(-np.inf))
            hi = np.nextafter(hi, np.float32(np.inf))
            near += [lo, hi]
        for x in near:
            assert (np.float64(x) > m) == (x > t), (m, x)
