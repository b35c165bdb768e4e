"""The bounds-checked debug build, libqlora_check.so (the same sources
compiled with QLORA_CHECK).  On valid calls it computes what the normal build
computes (checked here against the oracle).  Given a plan that does not match
what its kernels are told -- a CPU-side test hook makes the next rank-side pass
announce one partial slot fewer than it uses, while every access still stays
inside the workspace -- it records QL_DEV_BAD_CONFIG instead of writing where
the plan does not allow, reports QLORA_ERR_DEVICE through
qlora_last_device_status, does not trap, and the next call on the same context
is clean.  The normal build does not look (its checks compile away)."""

import numpy as np
import pytest
import torch

from qlora_fine_tuning_nf4_b200 import ops
from qlora_fine_tuning_nf4_b200.synth import bits_to_torch, make_linear_problem

from parity import assert_close, gpu_f64, run_linear_gpu, run_linear_oracle

pytestmark = pytest.mark.gpu

QLORA_ERR_DEVICE = 7


def _lin(p):
    w = ops.nf4_quantize(bits_to_torch(p["W"], "cuda"))
    return ops.LoraLinear(w, bits_to_torch(p["A"], "cuda"), bits_to_torch(p["B"], "cuda"), p["s"])


def test_checked_build_computes_what_the_oracle_computes():
    L = ops.checked_lib()
    assert L.qlora_checked_build() == 1 and ops.normal_lib().qlora_checked_build() == 0
    p = make_linear_problem(300, 768, 520, r=16, alpha=32.0, seed=21)
    with ops.use_library(L):
        g = run_linear_gpu(p, 4)
    o = run_linear_oracle(p)
    assert g["status"] == 0
    for k in ("XA", "Y", "dX", "dA", "dB"):
        assert_close(k, g[k], o[k])


def _forward_with_shrunk_plan(p):
    """X A over X [256, 4096]: 4 row groups of 64 units each spread over 256
    CTAs, so every group has 64 partial slots; the hook announces 63."""
    lin = _lin(p)
    X = bits_to_torch(p["X"], "cuda")
    ws = ops.Workspace()
    ops.qlora_test_shrink_next_slot_cap()
    ops.qlora_linear_fwd(lin, X, ws)
    torch.cuda.synchronize()
    st = ops.qlora_last_device_status(ws)
    Y, XA = ops.qlora_linear_fwd(lin, X, ws)  # the next call, on the same context and workspace
    torch.cuda.synchronize()
    return st, ops.qlora_last_device_status(ws), gpu_f64(Y), gpu_f64(XA)


def test_checked_build_reports_a_plan_mismatch_without_trapping():
    p = make_linear_problem(256, 4096, 256, r=16, alpha=16.0, seed=22)
    o = run_linear_oracle(p)
    with ops.use_library(ops.checked_lib()):
        ops.qlora_set_tile_config(4)
        st, st_next, y, xa = _forward_with_shrunk_plan(p)
    assert st == QLORA_ERR_DEVICE
    assert st_next == 0
    assert np.isfinite(y).all()
    assert_close("Y", y, o["Y"])
    assert_close("XA", xa, o["XA"])


def test_normal_build_does_not_check():
    p = make_linear_problem(256, 4096, 256, r=16, alpha=16.0, seed=22)
    with ops.use_library(ops.normal_lib()):  # also when QLORA_LIBRARY=checked runs the suite on the checked build
        prev = ops.qlora_set_tile_config(4)
        try:
            st, st_next, _, _ = _forward_with_shrunk_plan(p)
        finally:
            ops.qlora_set_tile_config(prev)
    assert st == 0 and st_next == 0
