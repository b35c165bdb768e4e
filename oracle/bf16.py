"""bf16 <-> binary64 conversions, written out with integer arithmetic.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

bf16 values travel as ``uint16`` bit patterns (the top half of an IEEE
binary32).  Rounding to bf16 is round-to-nearest-even on the 16 dropped bits,
which is the rounding the [Mistral blog] item "2. Bitsandbytes bfloat16" needs
when it dequantises straight to bfloat16.  Inputs here are always finite.
"""

import numpy as np


def bf16_bits_to_f64(bits):
    """Widen bf16 bit patterns (uint16) to float64 exactly."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f64_to_f32(x):
    """Round float64 to the nearest binary32 (ties to even), back as float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def f32_to_bf16_bits(x):
    """Round binary32 values (given as float32 or exactly-representable float64)
    to bf16, round-to-nearest-even, returning uint16 bit patterns.

    The kept half is the high 16 bits; the dropped half decides: above 0x8000
    rounds up, below rounds down, exactly 0x8000 rounds to the even kept half.
    """
    f = np.asarray(x, dtype=np.float64)
    f32 = f.astype(np.float32)
    if not np.array_equal(f32.astype(np.float64), f):
        raise ValueError("f32_to_bf16_bits expects values exactly representable in binary32")
    u = f32.view(np.uint32).astype(np.uint64)
    hi = u >> np.uint64(16)
    lo = u & np.uint64(0xFFFF)
    round_up = (lo > 0x8000) | ((lo == 0x8000) & ((hi & np.uint64(1)) == 1))
    out = hi + round_up.astype(np.uint64)
    return out.astype(np.uint16)
