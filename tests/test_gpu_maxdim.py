"""The largest M the library accepts, 2^23 = 8,388,608 token rows (one more is
rejected on the host: tests/test_abi_cpu.py), on a projection narrow enough
to fit a few GB: k_in = 64, n_out = 64, rank 16.  At this size the rank-side
passes split 131,072 row groups over all CTAs, the GEMMs walk 32,768 row tiles
and the reductions index about 2^25 partial columns, all in 32-bit integers.

Y and dX are row-local, so the oracle evaluates them on sampled rows.  dA and
dB are sums over all rows; the oracle's projection backward is linear in the
rows, so it is applied to consecutive row chunks and the chunks' results are
added in fp64 (the full-batch value in exact arithmetic)."""

import numpy as np
import pytest
import torch

import oracle
from qlora_fine_tuning_nf4_b200 import ops
from qlora_fine_tuning_nf4_b200.synth import bits_to_torch, make_linear_problem

from parity import TOL, assert_close, f64, gpu_f64, oracle_weight

pytestmark = pytest.mark.gpu

M_MAX = 1 << 23


def test_linear_at_the_largest_accepted_M():
    K, N = 64, 64
    p = make_linear_problem(M_MAX, K, N, r=16, alpha=16.0, seed=23)
    w = ops.nf4_quantize(bits_to_torch(p["W"], "cuda"))
    lin = ops.LoraLinear(w, bits_to_torch(p["A"], "cuda"), bits_to_torch(p["B"], "cuda"), p["s"])
    X, dY = bits_to_torch(p["X"], "cuda"), bits_to_torch(p["dY"], "cuda")
    ws = ops.Workspace()
    Y, XA = ops.qlora_linear_fwd(lin, X, ws)
    dX, dA, dB = ops.qlora_linear_bwd(lin, X, XA, dY, ws)
    torch.cuda.synchronize()
    assert ops.qlora_last_device_status(ws) == 0

    codes, absmax, Wq = oracle_weight(p["W"])
    A, B, s = f64(p["A"]), f64(p["B"]), p["s"]
    rows = np.array([0, 1, 63, 64, 4095, 1 << 20, (1 << 22) + 17, M_MAX - 65, M_MAX - 2, M_MAX - 1])
    Yo, XAo = oracle.linear_fwd(f64(p["X"][rows]), Wq, A, B, s)
    dXo, _, _ = oracle.linear_bwd(f64(p["X"][rows]), Wq, A, B, s, f64(p["dY"][rows]))
    sel = torch.as_tensor(rows, device="cuda")
    assert_close("Y", gpu_f64(Y[sel]), Yo, TOL)
    assert_close("XA", gpu_f64(XA[sel]), XAo, TOL)
    assert_close("dX", gpu_f64(dX[sel]), dXo, TOL)

    dA_o = np.zeros((K, 16))
    dB_o = np.zeros((16, N))
    chunk = 1 << 20
    for lo in range(0, M_MAX, chunk):
        _, a, b = oracle.linear_bwd(f64(p["X"][lo:lo + chunk]), Wq, A, B, s, f64(p["dY"][lo:lo + chunk]))
        dA_o += a
        dB_o += b
    assert_close("dA", gpu_f64(dA), dA_o, TOL)
    assert_close("dB", gpu_f64(dB), dB_o, TOL)
