"""Shared helpers for the GPU parity tests: run a problem through the CUDA path
(via the C ABI binding) and through the fp64 oracle, and compare.

Inputs come from the seeded generators in ``qlora_fine_tuning_nf4_b200.synth``;
each side quantises the base weights with its own NF4 implementation, and the
tests assert that the two quantisations are bit-identical.
"""

import numpy as np
import torch

import oracle
from oracle.nf4 import nf4_dequantize_f64
from qlora_fine_tuning_nf4_b200 import ops
from qlora_fine_tuning_nf4_b200.synth import bits_to_torch

TOL = 2e-2  # max |gpu - oracle| <= TOL * RMS(oracle), per tensor (every workload at full size)
# Small-M gated-MLP cases: the saved activations (E, G, H), dE/dG, X A and s G
# are bf16 by design; a CPU emulation of exactly those bf16 roundings (no
# kernel involved) already gives max|err| = 1.5-2.2e-2 x RMS on the MLP outputs
# at M = 200-1024 tokens, because the max over elements of few-row sums is
# dominated by single heavy-tailed products.  These cases use 3e-2.
TOL_SMALL_MLP = 3e-2
# (M, d, h) of the small gated-MLP parity cases (seed M + d + h): several tiles of
# every kernel, ragged M and a width that is not a multiple of the 256-wide tile.
# tests/test_tolerance_emulation.py derives TOL_SMALL_MLP on exactly these.
SMALL_MLP_CASES = [
    (256, 256, 512),
    (200, 512, 768),
    (384, 768, 1280),
    (1100, 512, 768),
]


def f64(bits):
    return oracle.bf16_bits_to_f64(bits)


def gpu_f64(t):
    return t.float().cpu().double().numpy()


def rel_err(gpu, ref):
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    err = float(np.max(np.abs(np.asarray(gpu, dtype=np.float64) - ref))) if ref.size else 0.0
    return err, rms


def assert_close(name, gpu, ref, tol=TOL):
    err, rms = rel_err(gpu, ref)
    assert err <= tol * rms, f"{name}: max|err| {err:.3e} > {tol} * RMS {rms:.3e} (ratio {err / max(rms, 1e-300):.3e})"
    return err / max(rms, 1e-300)


def saved_bounds(o, p):
    """Elementwise error bounds of the saved bf16 activations E, G, H.

    bf16 keeps 8 significant bits, so one round-to-nearest-even costs at most
    u = 2^-8 relative.  e and g are fp32 accumulations whose LoRA operand s*XA
    is rounded to bf16: |de| <= u s |XA||B| plus an fp32 accumulation slack
    2^-16 |X||W|^T; both carry a safety factor 4, and the stored value's own
    rounding (u |e|) a factor 2.  h = act(e) g is formed from the fp32 e, g:
    |dh| <= 2u |h| + |act'(e) g| |de| + |act(e)| |dg|.
    """
    u = 2.0 ** -8
    act = o["act"]
    out = {}
    de = {}
    for k, key in (("g", "E"), ("u", "G")):
        W, A, B, s = o["lin"][k]
        de[key] = 4 * u * s * (np.abs(o["X"] @ A) @ np.abs(B)) + 2.0 ** -14 * (np.abs(o["X"]) @ np.abs(W).T)
        out[key] = 2 * u * np.abs(o[key]) + de[key]
    out["H"] = (2 * u * np.abs(o["H"]) + np.abs(oracle.act_grad(act, o["E"]) * o["G"]) * de["E"]
                + np.abs(oracle.act_fwd(act, o["E"])) * de["G"])
    return out


def assert_saved(name, gpu, ref, bound):
    """Saved bf16 activations, elementwise against `saved_bounds`."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    bad = np.abs(gpu - ref) > bound
    assert not bad.any(), f"{name}: {int(bad.sum())} of {bad.size} elements outside the bf16 rounding bound"


def dev(bits):
    return bits_to_torch(bits, "cuda")


def gpu_weight(w_bits):
    """Quantise on the GPU; returns (NF4Weight, codes np, absmax np)."""
    n, k = w_bits.shape
    w = ops.nf4_quantize(dev(w_bits))
    return w, w.codes.cpu().numpy(), w.absmax.cpu().numpy()


def oracle_weight(w_bits):
    n, k = w_bits.shape
    codes, absmax = oracle.nf4_quantize(w_bits, n, k)
    return codes, absmax, nf4_dequantize_f64(codes, absmax, n, k)


def run_linear_gpu(p, tiles=4, ws=None):
    ops.qlora_set_tile_config(tiles)
    w, codes, absmax = gpu_weight(p["W"])
    lin = ops.LoraLinear(w, dev(p["A"]), dev(p["B"]), p["s"])
    ws = ws or ops.Workspace()
    X, dY = dev(p["X"]), dev(p["dY"])
    Y, XA = ops.qlora_linear_fwd(lin, X, ws)
    dX, dA, dB = ops.qlora_linear_bwd(lin, X, XA, dY, ws)
    torch.cuda.synchronize()
    st = ops.qlora_last_device_status(ws)
    return {"Y": gpu_f64(Y), "XA": gpu_f64(XA), "dX": gpu_f64(dX), "dA": gpu_f64(dA), "dB": gpu_f64(dB),
            "codes": codes, "absmax": absmax, "status": st}


def run_linear16_gpu(p, ws=None):
    """The 16-bit entry points: the bf16 weight itself is the frozen base."""
    lin = ops.LoraLinear16(dev(p["W"]), dev(p["A"]), dev(p["B"]), p["s"])
    ws = ws or ops.Workspace()
    X, dY = dev(p["X"]), dev(p["dY"])
    Y, XA = ops.qlora_linear16_fwd(lin, X, ws)
    dX, dA, dB = ops.qlora_linear16_bwd(lin, X, XA, dY, ws)
    torch.cuda.synchronize()
    st = ops.qlora_last_device_status(ws)
    return {"Y": gpu_f64(Y), "XA": gpu_f64(XA), "dX": gpu_f64(dX), "dA": gpu_f64(dA), "dB": gpu_f64(dB), "status": st}


def run_linear_oracle(p, base="nf4"):
    """base = "nf4": the oracle's own NF4 quantisation of W; "bf16": W itself."""
    if base == "nf4":
        codes, absmax, W = oracle_weight(p["W"])
    else:
        codes, absmax, W = None, None, f64(p["W"])
    X, A, B, dY = f64(p["X"]), f64(p["A"]), f64(p["B"]), f64(p["dY"])
    Y, XA = oracle.linear_fwd(X, W, A, B, p["s"])
    dX, dA, dB = oracle.linear_bwd(X, W, A, B, p["s"], dY)
    return {"Y": Y, "XA": XA, "dX": dX, "dA": dA, "dB": dB, "codes": codes, "absmax": absmax}


def run_mlp_gpu(p, act, tiles=4, ws=None):
    ops.qlora_set_tile_config(tiles)
    lins = {}
    qs = {}
    for k in ("g", "u", "d"):
        w, c, a = gpu_weight(p["W_" + k])
        lins[k] = ops.LoraLinear(w, dev(p["A_" + k]), dev(p["B_" + k]), p["s"])
        qs[k] = (c, a)
    ws = ws or ops.Workspace()
    X, dY = dev(p["X"]), dev(p["dY"])
    Y, saved = ops.qlora_mlp_fwd(act, lins["g"], lins["u"], lins["d"], X, ws)
    grads = ops.qlora_mlp_bwd(act, lins["g"], lins["u"], lins["d"], X, saved, dY, ws)
    torch.cuda.synchronize()
    out = {"Y": gpu_f64(Y), "status": ops.qlora_last_device_status(ws), "q": qs}
    for k in ("E", "G", "H", "XA_g", "XA_u", "HA_d"):
        out[k] = gpu_f64(saved[k])
    for k, v in grads.items():
        out[k] = gpu_f64(v)
    return out


def run_mlp16_gpu(p, act, ws=None, rows=None):
    """The 16-bit MLP entry points; `rows` selects returned rows of Y, dX and the saved tensors."""
    lins = {k: ops.LoraLinear16(dev(p["W_" + k]), dev(p["A_" + k]), dev(p["B_" + k]), p["s"]) for k in ("g", "u", "d")}
    ws = ws or ops.Workspace()
    X, dY = dev(p["X"]), dev(p["dY"])
    Y, saved = ops.qlora_mlp16_fwd(act, lins["g"], lins["u"], lins["d"], X, ws)
    grads = ops.qlora_mlp16_bwd(act, lins["g"], lins["u"], lins["d"], X, saved, dY, ws)
    torch.cuda.synchronize()
    sel = (lambda t: t) if rows is None else (lambda t: t[torch.as_tensor(rows, device=t.device)])
    out = {"Y": gpu_f64(sel(Y)), "status": ops.qlora_last_device_status(ws)}
    for k in ("E", "G", "H", "XA_g", "XA_u", "HA_d"):
        out[k] = gpu_f64(sel(saved[k]))
    for k, v in grads.items():
        out[k] = gpu_f64(sel(v) if k == "dX" else v)
    return out


def run_mlp_oracle(p, act, base="nf4"):
    lin, qs = {}, {}
    for k in ("g", "u", "d"):
        if base == "nf4":
            c, a, W = oracle_weight(p["W_" + k])
        else:
            c, a, W = None, None, f64(p["W_" + k])
        lin[k] = (W, f64(p["A_" + k]), f64(p["B_" + k]), p["s"])
        qs[k] = (c, a)
    X, dY = f64(p["X"]), f64(p["dY"])
    fwd = oracle.mlp_fwd(act, X, lin["g"], lin["u"], lin["d"])
    bwd = oracle.mlp_bwd(act, X, lin["g"], lin["u"], lin["d"], dY, saved=fwd)
    out = dict(fwd)
    out.update(bwd)
    out["XA_g"] = X @ lin["g"][1]
    out["XA_u"] = X @ lin["u"][1]
    out["HA_d"] = fwd["H"] @ lin["d"][1]
    out["q"] = qs
    out["lin"], out["X"], out["act"] = lin, X, act
    return out
