"""NF4 (4-bit NormalFloat) codebook, block quantiser and dequantiser.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The [Mistral blog] benchmark configuration quantises every projection
("QLoRA nf4 layers = q/k/v/o/gate/up/down"); [Show HN] links the QLoRA paper
for the format.  The pages print neither the codebook nor the block layout, so
this module takes the plainest reading of the QLoRA NormalFloat definition:

* 16 levels built from quantiles of N(0, 1), with an exact zero, normalised to
  [-1, 1], then stored as binary32;
* blocks of 64 consecutive elements along the input (K) dimension of the
  row-major [N, K] weight, one binary32 absmax per block (no double
  quantisation of the absmax);
* two codes per byte, the even-indexed element of each pair in the HIGH
  nibble, the odd-indexed one in the LOW nibble;
* a value exactly on a midpoint between two levels takes the LOWER level;
  an all-zero block (absmax = 0) stores code 7 (the level 0.0) everywhere.

Dequantisation rounds the binary32 product ``level * absmax`` to bf16 with
round-to-nearest-even: "dequantise straight to bfloat16" is item
"2. Bitsandbytes bfloat16" of the [Mistral blog] per-optimisation table.
"""

import statistics

import numpy as np

from .bf16 import bf16_bits_to_f64, f32_to_bf16_bits, f64_to_f32

NF4_BLOCK = 64


def nf4_codebook():
    """The 16 NF4 levels as float64 values that are exact binary32 numbers.

    Construction (QLoRA NormalFloat, plainest reading):
      1. offset delta = ((1 - 1/30) + (1 - 1/32)) / 2;
      2. positive half: 9 evenly spaced probabilities from delta down to 1/2,
         drop the 1/2 end, map each through the N(0,1) quantile -> 8 values;
      3. negative half: 8 evenly spaced probabilities from delta to 1/2, drop
         the 1/2 end, negate the quantiles -> 7 values;
      4. add 0, sort ascending, divide by the largest magnitude, round to
         binary32.
    "Evenly spaced" is a + (b - a) * i / (n - 1); the quantile is
    ``statistics.NormalDist().inv_cdf`` in binary64.
    """
    delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0))
    nd = statistics.NormalDist()

    def spaced(a, b, n):
        return [a + (b - a) * i / (n - 1) for i in range(n)]

    pos = [nd.inv_cdf(p) for p in spaced(delta, 0.5, 9)[:-1]]
    neg = [-nd.inv_cdf(p) for p in spaced(delta, 0.5, 8)[:-1]]
    levels = sorted(neg + [0.0] + pos)
    scale = max(abs(v) for v in levels)
    return f64_to_f32(np.array([v / scale for v in levels], dtype=np.float64))


def nf4_midpoints(code=None):
    """Decision thresholds between adjacent levels, exact in binary64."""
    c = nf4_codebook() if code is None else code
    return (c[:-1] + c[1:]) / 2.0


def _blocks_of(w_bits, n_out, k_in):
    if k_in % NF4_BLOCK:
        raise ValueError("k_in must be a multiple of 64")
    w = bf16_bits_to_f64(np.asarray(w_bits).reshape(n_out, k_in))
    return w.reshape(-1, NF4_BLOCK)


def _normalised(blocks):
    """absmax per block and v = RN_binary32(w / absmax).

    binary64 division then rounding to binary32 equals the correctly rounded
    binary32 quotient of two binary32 operands (53 >= 2*24 + 2).
    """
    absmax = np.abs(blocks).max(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = f64_to_f32(blocks / absmax[:, None])
    return absmax, v


def _pack(idx):
    idx = idx.reshape(-1).astype(np.uint8)
    return ((idx[0::2] << 4) | idx[1::2]).astype(np.uint8)


def nf4_quantize(w_bits, n_out, k_in, rows_per_chunk=2048):
    """Quantise a bf16 weight [n_out, k_in] (uint16 bit patterns).

    Returns ``(codes, absmax)``: codes uint8 [n_out * k_in / 2] (two per byte,
    even element in the high nibble) and absmax float32 [n_out * k_in / 64].
    The level index of v is the number of midpoints strictly below v.
    Rows are processed in chunks only to bound memory; blocks are independent.
    """
    code = nf4_codebook()
    mids = nf4_midpoints(code)
    w_bits = np.asarray(w_bits).reshape(n_out, k_in)
    codes = np.empty(n_out * k_in // 2, dtype=np.uint8)
    absmax_out = np.empty(n_out * k_in // NF4_BLOCK, dtype=np.float32)
    for r0 in range(0, n_out, rows_per_chunk):
        r1 = min(n_out, r0 + rows_per_chunk)
        blocks = _blocks_of(w_bits[r0:r1], r1 - r0, k_in)
        absmax, v = _normalised(blocks)
        idx = np.zeros(v.shape, dtype=np.int64)
        for m in mids:
            idx += v > m
        idx[absmax == 0.0] = 7
        codes[r0 * k_in // 2:r1 * k_in // 2] = _pack(idx)
        absmax_out[r0 * k_in // NF4_BLOCK:r1 * k_in // NF4_BLOCK] = absmax.astype(np.float32)
    return codes, absmax_out


def nf4_quantize_bruteforce(w_bits, n_out, k_in):
    """Same mapping written as a nearest-level search (for small inputs).

    For each element take the level with the smallest |v - level| (distances
    are exact in binary64); on a tie take the lower index.  Used to pin
    :func:`nf4_quantize`'s midpoint counting against an independent statement.
    """
    code = nf4_codebook()
    blocks = _blocks_of(w_bits, n_out, k_in)
    absmax, v = _normalised(blocks)
    idx = np.empty(v.shape, dtype=np.int64)
    for b in range(v.shape[0]):
        for j in range(NF4_BLOCK):
            if absmax[b] == 0.0:
                idx[b, j] = 7
                continue
            best, best_d = 0, abs(v[b, j] - code[0])
            for q in range(1, 16):
                d = abs(v[b, j] - code[q])
                if d < best_d:
                    best, best_d = q, d
            idx[b, j] = best
    return _pack(idx), absmax.astype(np.float32)


def nf4_unpack(codes):
    """uint8 codes -> level indices in element order (high nibble first)."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1)
    idx = np.empty(c.size * 2, dtype=np.int64)
    idx[0::2] = c >> 4
    idx[1::2] = c & 0x0F
    return idx


def nf4_dequantize(codes, absmax, n_out, k_in):
    """Dequantise to ``(w_f32, w_bf16_bits)`` of shape [n_out, k_in].

    w_f32 = RN_binary32(level[q] * absmax): the binary64 product of two binary32
    numbers is exact (48 significant bits), so rounding it once to binary32 is
    the binary32 product.  w_bf16 = RNE_bf16(w_f32).
    """
    code = nf4_codebook()
    idx = nf4_unpack(codes).reshape(-1, NF4_BLOCK)
    a = np.asarray(absmax, dtype=np.float32).astype(np.float64).reshape(-1, 1)
    w32 = f64_to_f32(code[idx] * a).reshape(n_out, k_in)
    return w32, f32_to_bf16_bits(w32)


def nf4_dequantize_f64(codes, absmax, n_out, k_in):
    """The bf16 dequantised weight widened to float64 (the frozen base W)."""
    _, bits = nf4_dequantize(codes, absmax, n_out, k_in)
    return bf16_bits_to_f64(bits)
