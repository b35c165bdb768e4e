"""qlora_linear_fwd_noalloc: the forward projection for callers that cannot
allocate device memory, for example a plugin that only receives its tensors'
device pointers from a host framework which owns all device memory.  Its
scratch is a fixed array inside the library, shared by every call, so two
calls in a row (outputs poisoned with NaN each time) must each give exactly
what the workspace entry point gives on the same GEMM configuration, and agree
with the fp64 oracle.  Kept in its own file, collected last; the library's
tile configuration is restored after every test (tests/conftest.py)."""

import ctypes

import numpy as np
import pytest
import torch

from qlora_fine_tuning_nf4_b200 import ops
from qlora_fine_tuning_nf4_b200.synth import bits_to_torch, make_linear_problem

from parity import TOL, assert_close, gpu_f64, run_linear_oracle

pytestmark = pytest.mark.gpu


def _lin(p):
    w = ops.nf4_quantize(bits_to_torch(p["W"], "cuda"))
    return ops.LoraLinear(w, bits_to_torch(p["A"], "cuda"), bits_to_torch(p["B"], "cuda"), p["s"])


def _twice(lin, X, Y_ref, XA_ref):
    """Two noalloc calls in a row, outputs NaN-poisoned before each."""
    outs = []
    for _ in range(2):
        Y = torch.full_like(Y_ref, float("nan"))
        XA = torch.full_like(XA_ref, float("nan"))
        ops.qlora_linear_fwd_noalloc(lin, X, Y=Y, XA=XA)
        torch.cuda.synchronize()
        outs.append((Y, XA))
    return outs


@pytest.mark.parametrize("alpha", [16.0, 32.0])  # s = 1 and s = 2 (the scaled copy of X A lives in the scratch)
def test_noalloc_forward_is_bitwise_the_workspace_forward_twice(alpha):
    """Under configuration 2 both entry points run the same kernels on the same
    partition of the work, so every bit of Y and X A must agree."""
    ops.qlora_set_tile_config(2)
    p = make_linear_problem(1000, 1024, 768, r=16, alpha=alpha, seed=7)
    lin = _lin(p)
    X = bits_to_torch(p["X"], "cuda")
    Y_ref, XA_ref = ops.qlora_linear_fwd(lin, X, ops.Workspace())
    torch.cuda.synchronize()
    o = run_linear_oracle(p)
    for Y, XA in _twice(lin, X, Y_ref, XA_ref):
        assert torch.equal(Y, Y_ref) and torch.equal(XA, XA_ref)
        assert_close("Y", gpu_f64(Y), o["Y"], TOL)
        assert_close("XA", gpu_f64(XA), o["XA"], TOL)


@pytest.mark.parametrize("tiles", [0, 4])
def test_noalloc_under_the_default_and_the_staged_configuration(tiles):
    """Under the automatic setting (the library's default) and under the staged
    configuration 4 the workspace forward stages the weight, which the fixed
    scratch has no room for, so this call runs configuration 2; its outputs
    agree with qlora_linear_fwd under the same setting and with the oracle."""
    ops.qlora_set_tile_config(tiles)
    p = make_linear_problem(777, 512, 1032, r=16, alpha=16.0, seed=8)
    lin = _lin(p)
    X = bits_to_torch(p["X"], "cuda")
    Y_ref, XA_ref = ops.qlora_linear_fwd(lin, X, ops.Workspace())
    torch.cuda.synchronize()
    o = run_linear_oracle(p)
    for Y, XA in _twice(lin, X, Y_ref, XA_ref):
        assert torch.equal(XA, XA_ref)  # the same X A pass and partition
        assert_close("Y", gpu_f64(Y), gpu_f64(Y_ref), TOL)
        assert_close("Y", gpu_f64(Y), o["Y"], TOL)
        assert_close("XA", gpu_f64(XA), o["XA"], TOL)


def test_noalloc_beyond_the_usual_partition():
    """20,000 rows of k_in = 4096: the usual split of the X A pass would need
    more partial sums than the fixed scratch holds, so the call gives every
    64-row group to one CTA instead; results still match the oracle."""
    p = make_linear_problem(20000, 4096, 256, r=16, alpha=16.0, seed=9)
    lin = _lin(p)
    X = bits_to_torch(p["X"], "cuda")
    Y_ref, XA_ref = ops.qlora_linear_fwd(lin, X, ops.Workspace())
    torch.cuda.synchronize()
    o = run_linear_oracle(p)
    for Y, XA in _twice(lin, X, Y_ref, XA_ref):
        assert_close("Y", gpu_f64(Y), o["Y"], TOL)
        assert_close("XA", gpu_f64(XA), o["XA"], TOL)
        assert_close("Y", gpu_f64(Y), gpu_f64(Y_ref), TOL)


def _raw_call(lin, X, M, Y, XA):
    c = lin.c()
    return ops.STATUS_NAMES[ops.lib().qlora_linear_fwd_noalloc(ctypes.byref(c), X.data_ptr(), M, Y.data_ptr(),
                                                               XA.data_ptr(), None)]


def test_noalloc_rejects_what_it_cannot_run_before_enqueueing_anything():
    p = make_linear_problem(16, 256, 256, r=32, alpha=32.0, seed=1)
    lin32 = _lin(p)
    X = bits_to_torch(p["X"], "cuda")
    Y = torch.full((16, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    XA = torch.full((16, 32), 7.0, dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    # rank 32: the in-mainloop feeds take rank 16 only, under the default configuration too
    assert _raw_call(lin32, X, 16, Y, XA) == "QLORA_ERR_UNSUPPORTED_SHAPE"
    torch.cuda.synchronize()
    assert bool((Y == 7.0).all()) and bool((XA == 7.0).all())  # nothing was written
    # M beyond 43,648 rows needs more than the fixed scratch (256 + 32 M + 4096 ceil(M / 64) bytes);
    # the buffers are sized for M rows all the same
    lin16 = _lin(make_linear_problem(16, 256, 256, seed=2))
    for M in (43649, 100000):
        Xm = torch.zeros(M, 256, dtype=torch.bfloat16, device="cuda")
        Ym = torch.full((M, 256), 7.0, dtype=torch.bfloat16, device="cuda")
        XAm = torch.full((M, 16), 7.0, dtype=torch.bfloat16, device="cuda")
        assert _raw_call(lin16, Xm, M, Ym, XAm) == "QLORA_ERR_WORKSPACE_TOO_SMALL"
        torch.cuda.synchronize()
        assert bool((Ym == 7.0).all()) and bool((XAm == 7.0).all())


def test_noalloc_accepts_the_largest_documented_size():
    p = make_linear_problem(43648, 256, 256, seed=3)
    lin = _lin(p)
    X = bits_to_torch(p["X"], "cuda")
    Y, XA = ops.qlora_linear_fwd_noalloc(lin, X)
    torch.cuda.synchronize()
    Y_ref, XA_ref = ops.qlora_linear_fwd(lin, X, ops.Workspace())
    torch.cuda.synchronize()
    assert np.isfinite(gpu_f64(Y)).all()
    assert_close("Y", gpu_f64(Y), gpu_f64(Y_ref), TOL)
    assert_close("XA", gpu_f64(XA), gpu_f64(XA_ref), TOL)
