"""GPU parity of the fused Q/K/V projection (qlora_qkv_fwd / qlora_qkv_bwd)
against the fp64 oracle's three separate projections: Y = [Y_q | Y_k | Y_v],
dX = dX_q + dX_k + dX_v, and each projection's dA, dB.  Grouped-query shapes
(k and v narrower than q), ranks 16, 32 and 64, and the Mistral-7B widths at
8192 tokens on sampled rows."""

import numpy as np
import pytest

import oracle
from qlora_fine_tuning_nf4_b200 import ops
from qlora_fine_tuning_nf4_b200.synth import bits_to_torch, make_qkv_problem

from parity import TOL, assert_close, assert_saved, f64, gpu_f64, oracle_weight

pytestmark = pytest.mark.gpu


def run_qkv_gpu(p, rows=None):
    lins = {}
    for n in "qkv":
        w = ops.nf4_quantize(bits_to_torch(p["W_" + n], "cuda"))
        lins[n] = ops.LoraLinear(w, bits_to_torch(p["A_" + n], "cuda"), bits_to_torch(p["B_" + n], "cuda"), p["s"])
    X, dY = bits_to_torch(p["X"], "cuda"), bits_to_torch(p["dY"], "cuda")
    ws = ops.Workspace()
    Y, XA = ops.qlora_qkv_fwd(lins["q"], lins["k"], lins["v"], X, ws)
    g = ops.qlora_qkv_bwd(lins["q"], lins["k"], lins["v"], X, XA, dY, ws)
    import torch
    torch.cuda.synchronize()
    sel = (lambda t: t) if rows is None else (lambda t: t[torch.as_tensor(rows, device=t.device)])
    out = {"Y": gpu_f64(sel(Y)), "XA": gpu_f64(sel(XA)), "dX": gpu_f64(sel(g["dX"])),
           "status": ops.qlora_last_device_status(ws)}
    for k, v in g.items():
        if k != "dX":
            out[k] = gpu_f64(v)
    return out


def run_qkv_oracle(p, rows=None):
    X, dY = f64(p["X"]), f64(p["dY"])
    if rows is not None:
        X, dY = X[rows], dY[rows]
    cols = np.cumsum([0, p["nq"], p["nk"], p["nv"]])
    out = {"Y": [], "XA": [], "dX": 0.0}
    for i, n in enumerate("qkv"):
        _, _, W = oracle_weight(p["W_" + n])
        A, B = f64(p["A_" + n]), f64(p["B_" + n])
        Yp, XAp = oracle.linear_fwd(X, W, A, B, p["s"])
        dXp, dAp, dBp = oracle.linear_bwd(X, W, A, B, p["s"], dY[:, cols[i]:cols[i + 1]])
        out["Y"].append(Yp)
        out["XA"].append(XAp)
        out["dX"] = out["dX"] + dXp
        out["dA_" + n], out["dB_" + n] = dAp, dBp
    out["Y"] = np.concatenate(out["Y"], axis=1)
    out["XA"] = np.concatenate(out["XA"], axis=1)
    return out


@pytest.mark.parametrize("r", [16, 32, 64])
@pytest.mark.parametrize("M,K,nq,nk,nv", [(300, 512, 512, 256, 256), (256, 1024, 1024, 256, 256),
                                           (200, 512, 768, 256, 136), (130, 320, 512, 256, 256),
                                           (1, 256, 256, 256, 8)])  # one token, an 8-wide v
def test_qkv_parity(r, M, K, nq, nk, nv):
    p = make_qkv_problem(M, K, nq, nk, nv, r=r, alpha=2.0 * r, seed=M + K + nq + nv + r)
    g = run_qkv_gpu(p)
    o = run_qkv_oracle(p)
    assert g["status"] == 0
    for k in ("Y", "XA", "dX"):
        assert_close(k, g[k], o[k])
    for n in "qkv":
        for k in ("dA_" + n, "dB_" + n):
            if M == 1:
                # one token row: dA and dB are outer products, each element two bf16 roundings
                # (of s G or X A, and of the result) away from the exact value, 2^-8 relative each
                assert_saved(k, g[k], o[k], 2.0 ** -7 * np.abs(o[k]) + 2.0 ** -12 * np.sqrt(np.mean(o[k] ** 2)))
            else:
                assert_close(k, g[k], o[k])


def test_qkv_mistral_widths_sampled_rows():
    """Mistral-7B attention widths (q 4096, k/v 1024 with grouped-query heads) at 8192 tokens:
    Y and dX rows are row-local, so the oracle evaluates them on a sample of rows."""
    p = make_qkv_problem(8192, 4096, 4096, 1024, 1024, r=16, alpha=16.0, seed=3)
    rows = np.array([0, 2047, 4096, 8191])
    g = run_qkv_gpu(p, rows=rows)
    o = run_qkv_oracle(p, rows=rows)
    assert g["status"] == 0
    for k in ("Y", "XA", "dX"):
        assert_close(k, g[k], o[k], TOL)
