"""Write the oracle's expected values for the full-size workloads.

    python tests/golden/make_full_size_expected.py [workload ...]

Calls only ``oracle/`` and the seeded input generators.  For every workload it
stores, in ``tests/golden/full_<workload>.npz``:
  * SHA-256 of the oracle's NF4 codes and absmax of every base weight (the GPU
    quantiser must match them bit for bit);
  * the RMS of every returned tensor over the whole workload (the tolerance is
    2e-2 x RMS);
  * a few sampled rows of Y, dX (and E, G, H for the MLP), including the first
    and last row;
  * 4096 sampled entries of every adapter gradient dA / dB.
The forward/backward runs in chunks of rows; the adapter gradients (sums over
rows) are accumulated over the chunks.
"""

import hashlib
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from oracle.nf4 import nf4_dequantize_f64  # noqa: E402
from qlora_fine_tuning_nf4_b200.synth import make_linear_problem, make_mlp_problem  # noqa: E402
from qlora_fine_tuning_nf4_b200.workloads import LINEAR_WORKLOADS, MLP_WORKLOADS  # noqa: E402

CHUNK = 2048
N_ROWS = 8
N_ROWS_WIDE = 4
N_ENTRIES = 4096


def sha(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def sample_rows(M, n, seed):
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, M - 1), size=max(0, n - 2), replace=False)
    return np.unique(np.concatenate([[0, M - 1], mid])).astype(np.int64)


def sample_entries(shape, seed):
    rng = np.random.default_rng(seed)
    size = int(np.prod(shape))
    return np.sort(rng.choice(size, size=min(N_ENTRIES, size), replace=False)).astype(np.int64)


def quantised(w_bits, out, tag):
    n, k = w_bits.shape
    codes, absmax = oracle.nf4_quantize(w_bits, n, k)
    out[f"sha_codes_{tag}"] = np.array(sha(codes))
    out[f"sha_absmax_{tag}"] = np.array(sha(absmax))
    return nf4_dequantize_f64(codes, absmax, n, k)


def linear(name, cfg):
    M, K, N, r = cfg["M"], cfg["K"], cfg["N"], cfg["r"]
    p = make_linear_problem(M, K, N, r, cfg["alpha"], cfg["seed"])
    out = {}
    W = quantised(p["W"], out, "W")
    A, B, s = oracle.bf16_bits_to_f64(p["A"]), oracle.bf16_bits_to_f64(p["B"]), p["s"]
    rows = sample_rows(M, N_ROWS, 1)
    ss = {"Y": 0.0, "dX": 0.0}
    dA = np.zeros((K, r))
    dB = np.zeros((r, N))
    row_vals = {"Y": np.zeros((len(rows), N), np.float32), "dX": np.zeros((len(rows), K), np.float32)}
    for m0 in range(0, M, CHUNK):
        m1 = min(M, m0 + CHUNK)
        X = oracle.bf16_bits_to_f64(p["X"][m0:m1])
        dY = oracle.bf16_bits_to_f64(p["dY"][m0:m1])
        Y, _ = oracle.linear_fwd(X, W, A, B, s)
        dX, a, b = oracle.linear_bwd(X, W, A, B, s, dY)
        dA += a
        dB += b
        for k, v in (("Y", Y), ("dX", dX)):
            ss[k] += float(np.sum(v * v))
            sel = (rows >= m0) & (rows < m1)
            row_vals[k][sel] = v[rows[sel] - m0]
    out["rows"] = rows
    for k in ("Y", "dX"):
        out[f"rms_{k}"] = np.array(np.sqrt(ss[k] / (M * (N if k == "Y" else K))))
        out[f"rows_{k}"] = row_vals[k]
    for k, v in (("dA", dA), ("dB", dB)):
        idx = sample_entries(v.shape, 2)
        out[f"rms_{k}"] = np.array(np.sqrt(np.mean(v * v)))
        out[f"idx_{k}"] = idx
        out[f"val_{k}"] = v.reshape(-1)[idx]
    return out


def mlp(name, cfg):
    M, d, h, r, act = cfg["M"], cfg["d"], cfg["h"], cfg["r"], cfg["act"]
    p = make_mlp_problem(M, d, h, r, cfg["alpha"], cfg["seed"])
    out = {}
    lin = {}
    for k in ("g", "u", "d"):
        W = quantised(p["W_" + k], out, "W_" + k)
        lin[k] = (W, oracle.bf16_bits_to_f64(p["A_" + k]), oracle.bf16_bits_to_f64(p["B_" + k]), p["s"])
    rows = sample_rows(M, N_ROWS, 1)
    rows_wide = rows[np.linspace(0, len(rows) - 1, N_ROWS_WIDE).astype(int)]
    widths = {"Y": d, "dX": d, "E": h, "G": h, "H": h}
    ss = {k: 0.0 for k in widths}
    row_vals = {k: np.zeros((len(rows if k in ("Y", "dX") else rows_wide), w), np.float32)
                for k, w in widths.items()}
    grads = {"dA_g": np.zeros((d, r)), "dB_g": np.zeros((r, h)), "dA_u": np.zeros((d, r)),
             "dB_u": np.zeros((r, h)), "dA_d": np.zeros((h, r)), "dB_d": np.zeros((r, d))}
    for m0 in range(0, M, CHUNK):
        m1 = min(M, m0 + CHUNK)
        X = oracle.bf16_bits_to_f64(p["X"][m0:m1])
        dY = oracle.bf16_bits_to_f64(p["dY"][m0:m1])
        fwd = oracle.mlp_fwd(act, X, lin["g"], lin["u"], lin["d"])
        bwd = oracle.mlp_bwd(act, X, lin["g"], lin["u"], lin["d"], dY, saved=fwd)
        for k in grads:
            grads[k] += bwd[k]
        vals = {"Y": fwd["Y"], "dX": bwd["dX"], "E": fwd["E"], "G": fwd["G"], "H": fwd["H"]}
        for k, v in vals.items():
            ss[k] += float(np.sum(v * v))
            rr = rows if k in ("Y", "dX") else rows_wide
            sel = (rr >= m0) & (rr < m1)
            row_vals[k][sel] = v[rr[sel] - m0]
        del fwd, bwd, vals
    out["rows"] = rows
    out["rows_wide"] = rows_wide
    for k, w in widths.items():
        out[f"rms_{k}"] = np.array(np.sqrt(ss[k] / (M * w)))
        out[f"rows_{k}"] = row_vals[k]
    for k, v in grads.items():
        idx = sample_entries(v.shape, 2)
        out[f"rms_{k}"] = np.array(np.sqrt(np.mean(v * v)))
        out[f"idx_{k}"] = idx
        out[f"val_{k}"] = v.reshape(-1)[idx]
    return out


def main(names):
    todo = names or [n for n in LINEAR_WORKLOADS if n != "tiny_linear"] + list(MLP_WORKLOADS)
    for name in todo:
        t0 = time.time()
        out = linear(name, LINEAR_WORKLOADS[name]) if name in LINEAR_WORKLOADS else mlp(name, MLP_WORKLOADS[name])
        np.savez(os.path.join(HERE, f"full_{name}.npz"), **out)
        print(f"{name}: {time.time() - t0:.1f} s", flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
