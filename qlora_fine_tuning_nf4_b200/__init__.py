"""libqlora: QLoRA NF4 projection and gated MLP, forward and hand-derived
backward, as hand-written CUDA for sm_100a behind a C ABI.

The Python surface is a thin ctypes binding (``qlora_fine_tuning_nf4_b200.ops``)
with the same names as the C entry points; it only marshals pointers, sizes
and the caller's CUDA stream.  The shared library is loaded on first use and
the binding raises if it is missing: there is no CPU fallback.
"""

__all__ = ["ops", "synth", "workloads"]
