"""qlora_linear_fwd_noalloc: the forward projection for callers that cannot
allocate device memory (for example a plugin that only gets its tensors' device
pointers from a host framework owning all device memory).  Its scratch is a
fixed array inside the library, shared by every call, so this checks that two
calls in a row, each with poisoned outputs, give what the workspace entry point
gives.  Kept in its own file, collected last."""

import numpy as np
import pytest
import torch

from qlora_fine_tuning_nf4_b200 import ops
from qlora_fine_tuning_nf4_b200.synth import bits_to_torch, make_linear_problem

from parity import TOL, assert_close, gpu_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("alpha", [16.0, 32.0])  # s = 1 and s = 2 (the scaled copy of X A lives in the scratch)
def test_noalloc_forward_matches_workspace_forward_twice(alpha):
    ops.qlora_set_tile_config(2)
    p = make_linear_problem(1000, 1024, 768, r=16, alpha=alpha, seed=7)
    w = ops.nf4_quantize(bits_to_torch(p["W"], "cuda"))
    lin = ops.LoraLinear(w, bits_to_torch(p["A"], "cuda"), bits_to_torch(p["B"], "cuda"), p["s"])
    X = bits_to_torch(p["X"], "cuda")
    ws = ops.Workspace()
    Y_ref, XA_ref = ops.qlora_linear_fwd(lin, X, ws)
    torch.cuda.synchronize()
    y_ref, xa_ref = gpu_f64(Y_ref), gpu_f64(XA_ref)
    for _ in range(2):
        Y = torch.full_like(Y_ref, float("nan"))
        XA = torch.full_like(XA_ref, float("nan"))
        ops.qlora_linear_fwd_noalloc(lin, X, Y=Y, XA=XA)
        torch.cuda.synchronize()
        y, xa = gpu_f64(Y), gpu_f64(XA)
        assert np.isfinite(y).all() and np.isfinite(xa).all()
        assert_close("Y", y, y_ref, TOL)
        assert_close("XA", xa, xa_ref, TOL)


def test_noalloc_rejects_problems_beyond_its_scratch():
    p = make_linear_problem(16, 256, 256, seed=1)
    w = ops.nf4_quantize(bits_to_torch(p["W"], "cuda"))
    lin = ops.LoraLinear(w, bits_to_torch(p["A"], "cuda"), bits_to_torch(p["B"], "cuda"), p["s"])
    X = bits_to_torch(p["X"], "cuda")
    Y = torch.empty(16, 256, dtype=torch.bfloat16, device="cuda")
    XA = torch.empty(16, 16, dtype=torch.bfloat16, device="cuda")
    c = lin.c()
    import ctypes
    # 100,000 rows need more than the fixed scratch: rejected on the host, nothing enqueued
    st = ops.lib().qlora_linear_fwd_noalloc(ctypes.byref(c), X.data_ptr(), 100000, Y.data_ptr(), XA.data_ptr(),
                                            None)
    assert ops.STATUS_NAMES[st] == "QLORA_ERR_WORKSPACE_TOO_SMALL"
