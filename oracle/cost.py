"""Multiply-add cost of the two bracket orders of the LoRA backward product.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

[Mistral blog] "10、11. 手动 Autograd": for X (m x d), the upstream gradient
(m x h) and the LoRA factor B^T (h x r),
  slow  (X^T dY) B^T  costs (h*d)(m + r),
  fast  X^T (dY B^T)  costs (m*r)(h + d).
Dropping r against m gives the speed-up h*d / (r*(h + d)); the page quotes
186.58 for Llama-7B (h=11008, d=4096, r=16) and 398.22 for Llama-70B
(h=28672, d=8192, r=16).  The page counts multiply-adds; the ratio is the
same in FLOPs.
"""


def bracket_costs(m, h, d, r):
    """(slow, fast) multiply-add counts for the two bracket orders."""
    slow = (h * d) * (m + r)
    fast = (m * r) * (h + d)
    return slow, fast


def bracket_speedup_limit(h, d, r):
    """The page's simplified ratio h*d / (r*(h + d)) (m >> r)."""
    return (h * d) / (r * (h + d))
