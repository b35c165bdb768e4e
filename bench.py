"""Benchmark: QLoRA gated-MLP forward + backward (Llama-7B shapes) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

One step = ``qlora_mlp_fwd`` + ``qlora_mlp_bwd`` of the SwiGLU MLP
(M = 8192 tokens = batch 4 x seq 2048, d = 4096, h = 11008, NF4 block 64,
LoRA rank 16, alpha 16) through the library's C ABI, on synthetic seeded
inputs resident in HBM.  With N > 1 (one rank per GPU, started by torchrun;
a plain `python bench.py --gpus N` starts them itself) every rank runs its
own 8192-token batch (weak scaling) and the six LoRA gradients are summed
across ranks with NCCL, as data-parallel training does: the four that are
final before the gate/up dX GEMM on a side stream while that GEMM runs, the
other two after the backward (qlora_fine_tuning_nf4_b200.dp).

Rank 0 prints one JSON line.  The dominant tensor-core kernel (the one that
takes the most time in the traced warm-up steps) has its launches bracketed
by CUDA events inside the timed region (its roofline); the other kernels'
shares come from a traced run just after it.  ``--impl reference``
times the fp64 CPU oracle instead (rank 0 only) on a bounded row sample of
the same workload.
"""

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from qlora_fine_tuning_nf4_b200.workloads import LINEAR_WORKLOADS, MLP_WORKLOADS, mlp_flops  # noqa: E402

METRIC = "QLoRA MLP fwd+bwd TFLOP/s & tokens/s (Llama-7B shape), % of bf16 peak"
UNIT = "TFLOP/s"


def l2_note(op, M, d, h, extra):
    """How the timed steps avoid running out of a warm L2 (126 MB): every step streams more than that."""
    mib = lambda n: f"{n * 2 / 2 ** 20:.0f} MiB"
    if op == "linear":
        return f"inputs larger than L2 (X and dX {mib(M * d)} each, dY and Y {mib(M * extra['N'])} each per step)"
    if op == "qkv":
        nt = extra["nq"] + extra["nk"] + extra["nv"]
        return f"inputs larger than L2 (X and dX {mib(M * d)} each, dY and Y {mib(M * nt)} each per step)"
    return f"inputs larger than L2 (saved E/G/H and dE/dG are 5 x {mib(M * h)} per step)"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama7b_swiglu_mlp", choices=sorted(MLP_WORKLOADS) + sorted(LINEAR_WORKLOADS),
                    help="an MLP workload (ops mlp, norm_mlp, qkv) or a single-projection one (op linear)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tiles", type=int, default=0, choices=[0, 1, 2, 3, 4],
                    help="GEMM tile configuration: 0 = the library's automatic choice (the default), 1-3 dequantise "
                         "in the mainloop, 4 = staged bf16 weight")
    ap.add_argument("--op", default="mlp", choices=["mlp", "norm_mlp", "qkv", "linear"],
                    help="the timed step: the gated MLP (the metric), the MLP behind its RMS layer norm (norm "
                         "forward and backward added), the fused Q/K/V projection (GQA widths), or one QLoRA "
                         "projection (qlora_linear_fwd + qlora_linear_bwd)")
    ap.add_argument("--rank", type=int, default=0, choices=[0, 16, 32, 64],
                    help="LoRA rank (0 = the workload's, 16); s = alpha / r with alpha = the rank")
    ap.add_argument("--weights", default="nf4", choices=["nf4", "bf16"],
                    help="frozen base format: NF4 (QLoRA, the metric) or bf16 (plain LoRA, for comparison)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override M (tokens per GPU) for small profiling cases; 0 = the workload's M")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"bf16": p["bf16_tflops"], "bf16_sustained": p["bf16_tflops_sustained"], "hbm": p["hbm_gbs"],
                "sustained_mhz": p.get("clocks_under_load", {}).get("sm_mhz_median") or 1300.0,
                "max_mhz": p.get("sm_max_mhz") or 1965.0, "src": "measured"}
    except Exception:
        return {"bf16": 1590.0, "bf16_sustained": 1400.0, "hbm": 6650.0, "sustained_mhz": 1300.0, "max_mhz": 1965.0,
                "src": "fallback"}


def tensor_peak(pk, clocks):
    """The bf16 peak that matches the clock the timed region ran at: the
    sustained figure (a seconds-long GEMM loop held at the power cap) when the
    median SM clock is nearer that loop's clock, the burst figure (a GEMM at
    full clock) otherwise.  Returns (TFLOP/s, description)."""
    mhz = (clocks or {}).get("sm_mhz")
    if mhz is None:
        return pk["bf16_sustained"], f"bf16 dense, sustained, {pk['src']} (no clock record)"
    mid = 0.5 * (pk["sustained_mhz"] + pk["max_mhz"])
    if mhz <= mid:
        return pk["bf16_sustained"], (f"bf16 dense, sustained, {pk['src']} (timed region at {mhz:.0f} MHz, "
                                      f"nearer the power-capped {pk['sustained_mhz']:.0f} MHz)")
    return pk["bf16"], f"bf16 dense, burst, {pk['src']} (timed region at {mhz:.0f} MHz, nearer full clock)"


def kernel_flops(name, M, d, h, r):
    """Algorithmic FLOP of one launch of each tensor-core kernel of the MLP step."""
    return {
        "gemm_nf4_gateup_glu_fwd": 2 * M * d * (2 * h) + 2 * M * r * (2 * h),
        "gemm_nf4_fwd": 2 * M * h * d + 2 * M * r * d,
        "gemm_nf4_down_bwd_glu": 2 * M * d * h + 2 * M * r * h,
        "gemm_nf4_bwd_dx": 2 * M * (2 * h) * d + 2 * M * (2 * r) * d,
    }.get(name)


def source_hash():
    h = hashlib.sha1()
    for f in ("gemm_nf4.cu", "ptx.cuh", "kernels.cuh"):
        with open(os.path.join(ROOT, "qlora_fine_tuning_nf4_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


def traffic_for(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it matches this source."""
    try:
        with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
            t = json.load(f)
        e = t.get(kernel, {})
        if e.get("source_sha1") == source_hash() and e.get("workload") == workload:
            return e.get("dram_bytes_per_launch")
    except Exception:
        pass
    return None


def smi_device_id(local):
    """nvidia-smi -i argument for this process's GPU (its UUID when torch knows it)."""
    import torch
    try:
        u = str(torch.cuda.get_device_properties(local).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(local)


class ClockSampler:
    """nvidia-smi clocks/throttle sampling; only samples stamped inside the timed window count."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index):
        self.dev = dev_index
        self.proc = None

    def start(self):
        # samples go to a file, not a pipe: nothing reads them until stop(), and a full
        # pipe would stall nvidia-smi (and drop the later samples) in a long run.  Every 20 ms,
        # so that a 20-step window (about 75 ms) holds a few samples (the driver refreshes the
        # clock and power readings about every 100 ms, so neighbouring samples may repeat).
        try:
            self.out = tempfile.TemporaryFile(mode="w+")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "20", "-i", str(self.dev)], stdout=self.out,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self, t0, t1, slack=0.3):
        """Summary of the samples stamped in [t0, t1] (host wall-clock seconds).  A window shorter than the
        sampling interval may hold no sample; then the samples within `slack` seconds of it are used (the GPU is
        busy with the same steps just before and after) and the summary says so."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.proc.wait(timeout=10)
        self.out.seek(0)
        out = self.out.read()
        self.out.close()
        return self.summarize(out, t0, t1, slack)

    @staticmethod
    def summarize(out, t0, t1, slack=0.3):
        """Median SM clock, power and the throttle reasons seen in nvidia-smi's CSV lines `out`."""
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = []
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                clk, top, power = float(f[2]), float(f[3]), float(f[4])
            except ValueError:
                continue
            rows.append((ts, clk, top, power, [n for n, v in zip(names, f[6:10]) if v.lower().startswith("active")]))
        window = "timed region"
        sel = [r for r in rows if t0 <= r[0] <= t1]
        if not sel:
            sel = [r for r in rows if t0 - slack <= r[0] <= t1 + slack]
            window = f"no sample inside the {1e3 * (t1 - t0):.0f} ms timed region; samples within {slack} s of it"
        sm = [r[1] for r in sel]
        pw = [r[3] for r in sel]
        reasons = sorted({n for r in sel for n in r[4]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": sel[-1][2] if sel else None,
                "reasons": reasons, "power_w": statistics.median(pw) if pw else None, "samples": len(sm),
                "window": window}


# ------------------------------------------------------------ oracle arm ---

def _oracle_step(wl, op):
    """(run, flops): run(n, off) times the fp64 oracle's fwd+bwd on token rows [off, off + n) of the workload
    (a gated MLP, or one projection for op "linear"); flops(n) is its algorithmic FLOP count.  Weights are
    quantised and dequantised by the oracle itself first (one-time, like the GPU side's quantisation)."""
    import oracle
    from oracle.nf4 import nf4_dequantize_f64
    from qlora_fine_tuning_nf4_b200.synth import make_linear_problem, make_mlp_problem
    from qlora_fine_tuning_nf4_b200.workloads import linear_flops

    f64 = oracle.bf16_bits_to_f64
    if op == "linear":
        p = make_linear_problem(wl["M"], wl["K"], wl["N"], wl["r"], wl["alpha"], wl["seed"])
        n_out, k_in = p["W"].shape
        c, a = oracle.nf4_quantize(p["W"], n_out, k_in)
        W, A, B = nf4_dequantize_f64(c, a, n_out, k_in), f64(p["A"]), f64(p["B"])

        def run(n, off):
            X, dY = f64(p["X"][off:off + n]), f64(p["dY"][off:off + n])
            t0 = time.perf_counter()
            oracle.linear_fwd(X, W, A, B, p["s"])
            oracle.linear_bwd(X, W, A, B, p["s"], dY)
            return time.perf_counter() - t0

        return run, lambda n: linear_flops(n, wl["K"], wl["N"], wl["r"])
    p = make_mlp_problem(wl["M"], wl["d"], wl["h"], wl["r"], wl["alpha"], wl["seed"])
    lin = {}
    for k in ("g", "u", "d"):
        n_out, k_in = p["W_" + k].shape
        c, a = oracle.nf4_quantize(p["W_" + k], n_out, k_in)
        lin[k] = (nf4_dequantize_f64(c, a, n_out, k_in), f64(p["A_" + k]), f64(p["B_" + k]), p["s"])

    def run(n, off):
        X, dY = f64(p["X"][off:off + n]), f64(p["dY"][off:off + n])
        t0 = time.perf_counter()
        fwd = oracle.mlp_fwd(wl["act"], X, lin["g"], lin["u"], lin["d"])
        oracle.mlp_bwd(wl["act"], X, lin["g"], lin["u"], lin["d"], dY, saved=fwd)
        return time.perf_counter() - t0

    return run, lambda n: mlp_flops(n, wl["d"], wl["h"], wl["r"])


def oracle_sample(wl, rows=None, seed_rows=0, target_s=12.0, op="mlp"):
    """Time the fp64 oracle's fwd+bwd (gated MLP, or one projection for op "linear") on `rows` tokens.

    With rows None, a 64-row probe sizes the sample to about `target_s` seconds
    of CPU work; when the whole batch takes less, whole-batch steps repeat
    until `target_s` has passed.  Returns (seconds, flop, threads, rows,
    steps).
    """
    run, flops = _oracle_step(wl, op)
    steps = 1
    if rows is None:
        probe = min(64, wl["M"] - seed_rows)
        per_row = run(probe, seed_rows) / probe
        rows = int(min(wl["M"] - seed_rows, max(64, target_s / max(per_row, 1e-9))))
        rows -= rows % 64
        if 2 * rows >= wl["M"] - seed_rows:  # the probe overestimates: take whole batches
            rows = wl["M"] - seed_rows
            dt = run(rows, seed_rows)
            while dt < target_s:
                dt += run(rows, seed_rows)
                steps += 1
            return dt, steps * flops(rows), len(os.sched_getaffinity(0)), rows, steps
    dt = run(rows, seed_rows)
    return dt, flops(rows), len(os.sched_getaffinity(0)), rows, steps


def c_loop_oracle_sample():
    """Time the plain C loop oracle's projection fwd+bwd on the tiny configuration
    (256 tokens, 512 -> 1024, rank 16; one thread).  Returns a summary dict."""
    from oracle import c_oracle
    from qlora_fine_tuning_nf4_b200.synth import make_linear_problem
    from qlora_fine_tuning_nf4_b200.workloads import linear_flops

    cfg = LINEAR_WORKLOADS["tiny_linear"]
    p = make_linear_problem(cfg["M"], cfg["K"], cfg["N"], cfg["r"], cfg["alpha"], cfg["seed"])
    n, k = p["W"].shape
    codes, absmax = c_oracle.nf4_quantize(p["W"], n, k)
    W = c_oracle.nf4_dequantize_f64(codes, absmax, n, k)
    wide = lambda b: (np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64)
    X, A, B, dY = (wide(p[t]) for t in ("X", "A", "B", "dY"))
    t0 = time.perf_counter()
    c_oracle.linear_fwd(X, W, A, B, p["s"])
    c_oracle.linear_bwd(X, W, A, B, p["s"], dY)
    dt = time.perf_counter() - t0
    fl = linear_flops(cfg["M"], cfg["K"], cfg["N"], cfg["r"])
    return {"workload": "tiny_linear (256 tokens, 512 -> 1024, r 16)", "value": fl / dt / 1e12, "unit": UNIT,
            "ms": dt * 1e3, "threads": 1, "kind": "C loop oracle, binary64"}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    run, flops = _oracle_step(wl, args.op)

    def step(rows, off):
        run(rows, off)

    # size the per-step row sample so the whole run takes about two minutes
    t0 = time.perf_counter()
    step(32, 0)
    per_row = (time.perf_counter() - t0) / 32
    budget = 120.0 / max(1, args.steps + args.warmup)
    rows = int(max(16, min(wl["M"], budget / max(per_row, 1e-9))))
    rows -= rows % 16
    rows = max(rows, 16)
    for i in range(args.warmup):
        step(rows, (i * rows) % (wl["M"] - rows + 1))
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(rows, (i * rows) % (wl["M"] - rows + 1))
    dt = time.perf_counter() - t0
    flop = flops(rows) * args.steps
    value = flop / dt / 1e12
    cores = len(os.sched_getaffinity(0))
    sample = f"{rows} of {wl['M']} token rows per step (fp64 numpy, BLAS threads = cores)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "op": args.op, "M": wl["M"],
                   **({"K": wl["K"], "N": wl["N"]} if args.op == "linear" else {"d": wl["d"], "h": wl["h"],
                                                                               "act": wl["act"]}),
                   "r": wl["r"], "sample_rows": rows},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# -------------------------------------------------------------- GPU arm ----

def setup_mlp(args, wl, M, d, h, r, act, rank, world, dev):
    """Tensors and step of the gated MLP fwd + bwd (the metric's workload)."""
    import torch

    from qlora_fine_tuning_nf4_b200 import dp, ops
    from qlora_fine_tuning_nf4_b200.synth import bits_to_torch, make_mlp_problem

    # Inputs: same seeded recipe as the tests; each rank draws its own batch.
    p = make_mlp_problem(M, d, h, r, wl["alpha"], wl["seed"] + 1000 * rank)
    lins = {}
    for k in ("g", "u", "d"):
        A, B = bits_to_torch(p["A_" + k], dev), bits_to_torch(p["B_" + k], dev)
        if args.weights == "nf4":
            lins[k] = ops.LoraLinear(ops.nf4_quantize(bits_to_torch(p["W_" + k], dev)), A, B, p["s"])
        else:
            lins[k] = ops.LoraLinear16(bits_to_torch(p["W_" + k], dev), A, B, p["s"])
    mlp_fwd = ops.qlora_mlp_fwd if args.weights == "nf4" else ops.qlora_mlp16_fwd
    mlp_bwd = ops.qlora_mlp_bwd if args.weights == "nf4" else ops.qlora_mlp16_bwd
    X = bits_to_torch(p["X"], dev)
    dY = bits_to_torch(p["dY"], dev)
    del p
    ws = ops.Workspace(dev)
    saved = ops.make_mlp_saved(M, h, r, dev)
    Y = torch.empty(M, d, dtype=torch.bfloat16, device=dev)
    # LoRA gradients as views of one flat buffer; with N > 1 ranks the four that are final before the gate/up
    # dX GEMM are summed on a side stream while it runs, the other two after the backward
    flat, views, early = dp.flat_lora_grads(d, h, r, dev)
    grads = dict(views)
    grads["dX"] = torch.empty(M, d, dtype=torch.bfloat16, device=dev)
    sync = dp.GradAllReduce(flat, early)
    step = dp.make_step(lambda: mlp_fwd(act, lins["g"], lins["u"], lins["d"], X, ws, Y=Y, saved=saved),
                        lambda ev: mlp_bwd(act, lins["g"], lins["u"], lins["d"], X, saved, dY, ws, grads=grads,
                                           early_event=ev),
                        sync)

    kflops = {k: kernel_flops(k, M, d, h, r) for k in ("gemm_nf4_gateup_glu_fwd", "gemm_nf4_fwd",
                                                         "gemm_nf4_down_bwd_glu", "gemm_nf4_bwd_dx")}
    dq = 2 * (2 * h * d + h * d) * (0.5 + 4 / 64 + 2)  # gate, up, down in the forward and in the backward
    return X, dY, Y, grads, flat, step, mlp_flops(M, d, h, r), kflops, dq, ws, {"h": h, "act": act}


def setup_norm_mlp(args, wl, M, d, h, r, act, rank, world, dev):
    """The MLP behind its RMS layer norm: X -> norm -> MLP fwd + bwd -> norm backward (frozen gain)."""
    import torch

    from qlora_fine_tuning_nf4_b200 import ops

    Xn, dY, Y, grads, flat, mlp_step, flop, kflops, dq, ws, extra = setup_mlp(args, wl, M, d, h, r, act, rank,
                                                                              world, dev)
    gemma = act == "geglu_tanh"
    g = torch.Generator(device="cpu").manual_seed(wl["seed"] + 77)
    w = (torch.randn(d, generator=g) * 0.1 + (0.0 if gemma else 1.0)).to(torch.bfloat16).to(dev)
    X = Xn.clone()  # the norm's input (the MLP's own input buffer receives the normalised rows)
    rstd = torch.empty(M, dtype=torch.float32, device=dev)
    dXn = grads["dX"]
    dX = torch.empty_like(X)
    eps = 1e-6 if gemma else 1e-5
    out = dict(grads)
    out["dX"] = dX

    def step():
        ops.qlora_rmsnorm_fwd(X, w, eps, plus_one=gemma, Y=Xn, rstd=rstd)
        mlp_step()
        ops.qlora_rmsnorm_bwd(X, w, rstd, dXn, plus_one=gemma, dX=dX)

    extra = dict(extra, norm="rms, gain 1 + w" if gemma else "rms, gain w")
    return X, dY, Y, out, flat, step, flop, kflops, dq, ws, extra


def setup_qkv(args, wl, M, d, r, rank, world, dev):
    """Tensors and step of the fused Q/K/V projection fwd + bwd at the workload's attention widths."""
    import torch

    from qlora_fine_tuning_nf4_b200 import dp, ops
    from qlora_fine_tuning_nf4_b200.synth import bits_to_torch, make_qkv_problem
    from qlora_fine_tuning_nf4_b200.workloads import linear_flops

    nq, nkv = wl["nq"], wl["nkv"]
    p = make_qkv_problem(M, d, nq, nkv, nkv, r, wl["alpha"], wl["seed"] + 1000 * rank)
    lins = {}
    for n in "qkv":
        lins[n] = ops.LoraLinear(ops.nf4_quantize(bits_to_torch(p["W_" + n], dev)), bits_to_torch(p["A_" + n], dev),
                                 bits_to_torch(p["B_" + n], dev), p["s"])
    X = bits_to_torch(p["X"], dev)
    dY = bits_to_torch(p["dY"], dev)
    del p
    ws = ops.Workspace(dev)
    nt = nq + 2 * nkv
    Y = torch.empty(M, nt, dtype=torch.bfloat16, device=dev)
    XA = torch.empty(M, 3 * r, dtype=torch.bfloat16, device=dev)
    sizes = [(f"d{m}_{n}", (d, r) if m == "A" else (r, wn)) for n, wn in (("q", nq), ("k", nkv), ("v", nkv))
             for m in "AB"]
    flat, views, _ = dp.flat_buffer(sizes, dev)
    grads = dict(views)
    grads["dX"] = torch.empty(M, d, dtype=torch.bfloat16, device=dev)
    step = dp.make_step(lambda: ops.qlora_qkv_fwd(lins["q"], lins["k"], lins["v"], X, ws, Y=Y, XA=XA),
                        lambda ev: ops.qlora_qkv_bwd(lins["q"], lins["k"], lins["v"], X, XA, dY, ws, grads=grads),
                        dp.GradAllReduce(flat))

    flop = sum(linear_flops(M, d, n, r) for n in (nq, nkv, nkv))
    kflops = {"gemm_nf4_fwd": 2 * M * d * nt + 2 * M * r * nt, "gemm_nf4_bwd_dx": 2 * M * nt * d + 2 * M * 3 * r * d}
    dq = 2 * nt * d * (0.5 + 4 / 64 + 2)
    return X, dY, Y, grads, flat, step, flop, kflops, dq, ws, {"nq": nq, "nk": nkv, "nv": nkv}


def setup_linear(args, wl, rank, world, dev):
    """Tensors and step of one QLoRA projection fwd + bwd (qlora_linear_fwd / qlora_linear_bwd)."""
    import torch

    from qlora_fine_tuning_nf4_b200 import dp, ops
    from qlora_fine_tuning_nf4_b200.synth import bits_to_torch, make_linear_problem
    from qlora_fine_tuning_nf4_b200.workloads import linear_flops

    M, K, N, r = wl["M"], wl["K"], wl["N"], wl["r"]
    p = make_linear_problem(M, K, N, r, wl["alpha"], wl["seed"] + 1000 * rank)
    A, B = bits_to_torch(p["A"], dev), bits_to_torch(p["B"], dev)
    if args.weights == "nf4":
        lin = ops.LoraLinear(ops.nf4_quantize(bits_to_torch(p["W"], dev)), A, B, p["s"])
        fwd, bwd = ops.qlora_linear_fwd, ops.qlora_linear_bwd
    else:
        lin = ops.LoraLinear16(bits_to_torch(p["W"], dev), A, B, p["s"])
        fwd, bwd = ops.qlora_linear16_fwd, ops.qlora_linear16_bwd
    X = bits_to_torch(p["X"], dev)
    dY = bits_to_torch(p["dY"], dev)
    del p
    ws = ops.Workspace(dev)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    XA = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    flat, views, _ = dp.flat_buffer([("dA", (K, r)), ("dB", (r, N))], dev)
    grads = dict(views, dX=torch.empty(M, K, dtype=torch.bfloat16, device=dev))
    step = dp.make_step(lambda: fwd(lin, X, ws, Y=Y, XA=XA),
                        lambda ev: bwd(lin, X, XA, dY, ws, dX=grads["dX"], dA=grads["dA"], dB=grads["dB"]),
                        dp.GradAllReduce(flat))

    kflops = {"gemm_nf4_fwd": 2 * M * K * N + 2 * M * r * N, "gemm_nf4_bwd_dx": 2 * M * N * K + 2 * M * r * K}
    dq = 2 * N * K * (0.5 + 4 / 64 + 2) if args.weights == "nf4" else 0  # the forward's and the backward's
    return X, dY, Y, grads, flat, step, linear_flops(M, K, N, r), kflops, dq, ws, {"N": N}


def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    from qlora_fine_tuning_nf4_b200 import ops
    from qlora_fine_tuning_nf4_b200.synth import bits_to_torch, make_mlp_problem

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but {world} rank(s) were started (WORLD_SIZE)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    ops.lib()
    ops.qlora_set_tile_config(args.tiles)
    M, r = wl["M"], wl["r"]
    d, h, act = wl.get("d", wl.get("K")), wl.get("h"), wl.get("act")
    norm_step_bytes = 0
    if args.op == "linear":
        (X, dY, Y, grads, flat, step, flop_step, kflops, dq_step_bytes, ws, cfg_extra) = \
            setup_linear(args, wl, rank, world, dev)
    elif args.op == "qkv":
        (X, dY, Y, grads, flat, step, flop_step, kflops, dq_step_bytes, ws, cfg_extra) = \
            setup_qkv(args, wl, M, d, r, rank, world, dev)
    elif args.op == "norm_mlp":
        (X, dY, Y, grads, flat, step, flop_step, kflops, dq_step_bytes, ws, cfg_extra) = \
            setup_norm_mlp(args, wl, M, d, h, r, act, rank, world, dev)
        norm_step_bytes = 10 * M * d  # forward reads X, writes Xn; backward reads X and dXn, writes dX
    else:
        (X, dY, Y, grads, flat, step, flop_step, kflops, dq_step_bytes, ws, cfg_extra) = \
            setup_mlp(args, wl, M, d, h, r, act, rank, world, dev)

    stream = torch.cuda.current_stream()
    clk = ClockSampler(smi_device_id(local))
    clk.start()
    time.sleep(0.5)  # the sampler's first sample lands before the timed window
    # The warm-up steps are traced (every launch bracketed by events) to name the dominant tensor-core kernel
    # of the step; the timed region then brackets that kernel's launches only.
    ops.qlora_trace_begin()
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    warm = ops.qlora_trace_end()
    if ops.qlora_last_device_status(ws) != 0:
        raise RuntimeError("device status error during warm-up")
    tw = {k: v for k, v in warm.items() if kflops.get(k)}
    top = max(tw, key=lambda k: tw[k][1]) if tw else None

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # The timed region.  Only the dominant kernel's launches are bracketed by events (the roofline's duration is
    # measured here, over the timed steps themselves); every other launch keeps its programmatic overlap.
    launches0 = ops.qlora_launch_count()
    barrier()
    if top:
        ops.qlora_trace_begin(only=top)
    t_begin = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    barrier()
    t_end = time.time()
    ms = e0.elapsed_time(e1)
    top_live = ops.qlora_trace_end().get(top) if top else None  # (launches, total ms) inside the timed region
    clocks = clk.stop(t_begin, t_end)
    launches = ops.qlora_launch_count() - launches0
    if ops.qlora_last_device_status(ws) != 0:
        raise RuntimeError("device status error during the timed region")
    # Per-kernel shares come from a traced run after the timed region: events that bracket every launch would
    # serialise the kernels' programmatic overlap.
    trace_steps = min(args.steps, 30)
    barrier()
    ops.qlora_trace_begin()
    e0.record(stream)
    for _ in range(trace_steps):
        step()
    e1.record(stream)
    barrier()
    trace_ms = e0.elapsed_time(e1)
    trace = {k: (n * args.steps / trace_steps, t * args.steps / trace_steps) for k, (n, t) in
             ops.qlora_trace_end().items()}  # scaled to the timed step count
    traced_total = trace_ms * args.steps / trace_steps  # the traced run's time, scaled to the timed step count
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item())
    value = flop_step * args.steps * world / (ms / 1e3) / 1e12
    tokens = M * args.steps * world / (ms / 1e3)
    pk = peaks()

    # ---- end-to-end through the public API with host buffers ----
    # Every step copies its inputs (X, dY) from pinned host memory and reads its result back to pinned host
    # memory, inside the timed region.  `e2e`: the result is the adapter gradients (what the optimiser
    # consumes; Y and dX feed neighbouring layers on the device).  `e2e_outputs`: Y and dX are read back every
    # step as well.  As a training loop prefetches its next batch, the next step's inputs are copied on one
    # copy stream into the other of two device buffers while the current step computes; the read-backs go on
    # a second copy stream (the two PCIe directions overlap), the gradients first, then Y and dX from the
    # step's own slot of two output buffers.  The adapter gradients alternate between two flat buffers as
    # well, so a step's backward never waits for the previous step's gradients to leave the device.
    Yt, dXt = Y, grads["dX"]
    home = (flat.untyped_storage(), flat.storage_offset())
    gviews = [t for t in grads.values() if t.untyped_storage().data_ptr() == home[0].data_ptr()]
    goffs = [t.storage_offset() - home[1] for t in gviews]
    gbufs = [torch.empty_like(flat), torch.empty_like(flat)]

    def point_grads(storage, offset):
        """Re-point the flat gradient buffer and its views (the step writes through them) at a buffer."""
        flat.set_(storage, offset, flat.size(), flat.stride())
        for t, o in zip(gviews, goffs):
            t.set_(storage, offset + o, t.size(), t.stride())

    hX = torch.empty(X.shape, dtype=torch.bfloat16, pin_memory=True)
    hdY = torch.empty(dY.shape, dtype=torch.bfloat16, pin_memory=True)
    hX.copy_(X.cpu())
    hdY.copy_(dY.cpu())
    hflat = torch.empty(flat.numel(), dtype=flat.dtype, pin_memory=True)
    hY = torch.empty(Yt.shape, dtype=torch.bfloat16, pin_memory=True)
    hdX = torch.empty(dXt.shape, dtype=torch.bfloat16, pin_memory=True)
    bufX = [torch.empty_like(X), torch.empty_like(X)]
    bufdY = [torch.empty_like(dY), torch.empty_like(dY)]
    bufY = [torch.empty_like(Yt), torch.empty_like(Yt)]
    bufdX = [torch.empty_like(dXt), torch.empty_like(dXt)]
    h2d_stream = torch.cuda.Stream(device=dev)
    d2h_stream = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event(), torch.cuda.Event()]
    ev_used = [torch.cuda.Event(), torch.cuda.Event()]
    ev_outs = [torch.cuda.Event(), torch.cuda.Event()]
    ev_grads = [torch.cuda.Event(), torch.cuda.Event()]
    e2e_steps = max(3, args.steps)  # as many as the timed region, so that both see the same clocks

    def h2d(slot):
        with torch.cuda.stream(h2d_stream):
            h2d_stream.wait_event(ev_used[slot])  # the step that last read this buffer is done
            bufX[slot].copy_(hX, non_blocking=True)
            bufdY[slot].copy_(hdY, non_blocking=True)
            ev_in[slot].record(h2d_stream)

    def run_e2e(n, outputs):
        h2d_stream.wait_stream(stream)
        d2h_stream.wait_stream(stream)
        h2d(0)
        for i in range(n):
            sl = i % 2
            stream.wait_event(ev_in[sl])
            X.set_(bufX[sl])
            dY.set_(bufdY[sl])
            stream.wait_event(ev_grads[sl])  # step i - 2's gradients have left this buffer
            point_grads(gbufs[sl].untyped_storage(), gbufs[sl].storage_offset())
            if outputs:
                stream.wait_event(ev_outs[sl])  # step i - 2's Y and dX have left this slot
                Yt.set_(bufY[sl])
                dXt.set_(bufdX[sl])
            step()
            ev_used[sl].record(stream)
            if i + 1 < n:
                h2d((i + 1) % 2)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(ev_used[sl])
                hflat.copy_(gbufs[sl], non_blocking=True)
                ev_grads[sl].record(d2h_stream)
                if outputs:
                    hY.copy_(bufY[sl], non_blocking=True)
                    hdX.copy_(bufdX[sl], non_blocking=True)
                    ev_outs[sl].record(d2h_stream)
        stream.wait_stream(h2d_stream)
        stream.wait_stream(d2h_stream)
        point_grads(*home)

    def time_e2e(outputs):
        run_e2e(2, outputs)
        barrier()
        e0.record(stream)
        run_e2e(e2e_steps, outputs)
        e1.record(stream)
        barrier()
        t = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return flop_step * e2e_steps * world / (float(t.item()) / 1e3) / 1e12

    e2e_value = time_e2e(False)
    e2e_out_value = time_e2e(True)
    h2d_bytes = (X.numel() + dY.numel()) * 2
    d2h_bytes = flat.numel() * flat.element_size()
    d2h_out_bytes = d2h_bytes + (Yt.numel() + dXt.numel()) * 2

    # ---- roofline of the dominant kernel (CUDA events around its launches in the timed region) ----
    roof = None
    if top and top_live:
        n_l, tot = top_live
        avg_s = tot / n_l / 1e3
        ach = kflops[top] / avg_s / 1e12
        peak, kind = tensor_peak(pk, clocks)
        roof = {"bound": "tensor", "kernel": top, "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": ach / peak, "peak_kind": kind,
                "traffic": traffic_for(top, args.workload), "avg_launch_ms": avg_s * 1e3,
                "launches": n_l, "share_of_step": tot / ms,
                "measured": "CUDA events around each of its launches inside the timed region"}
    kernels = {k: {"launches": int(round(v[0])), "ms_total": round(v[1], 4), "share": round(v[1] / traced_total, 4)}
               for k, v in sorted(trace.items(), key=lambda kv: -kv[1][1])}
    # HBM-bound staging dequantisation: algorithmic bytes (codes + absmax read, bf16 written) per step
    dq = None
    if "nf4_dequantize" in trace:
        n_l, tot = trace["nf4_dequantize"]
        gbs = args.steps * dq_step_bytes / (tot / 1e3) / 1e9
        dq = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s", "frac": gbs / pk["hbm"],
              "launches": n_l, "ms_per_step": tot / args.steps}

    nrm = None
    if norm_step_bytes and "rmsnorm_fwd" in trace:
        tot = trace["rmsnorm_fwd"][1] + trace["rmsnorm_bwd"][1]
        gbs = args.steps * norm_step_bytes / (tot / 1e3) / 1e9
        nrm = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s", "frac": gbs / pk["hbm"],
               "ms_per_step": tot / args.steps}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.op in ("mlp", "linear"):
        dt, fl, cores, rows, n = oracle_sample(wl, op=args.op)
        what = f"{n} fwd+bwd steps of all {M} token rows" if rows == M else f"{rows} of {M} token rows, one fwd+bwd"
        cpu = {"value": fl / dt / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{what} (fp64 numpy, {dt:.1f} s)",
               "c_loop_oracle": c_loop_oracle_sample()}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "tokens_per_s": tokens, "frac_of_bf16_peak": value / world / pk["bf16"],
        "frac_of_bf16_peak_sustained": value / world / pk["bf16_sustained"],
        "config": {"workload": args.workload, "op": args.op, "M_per_gpu": M, "d": d, **cfg_extra, "r": r,
                   "nf4_block": 64, "global_batch_tokens": M * world, "parallelism": f"dp{world}",
                   "gemm_tiles": ops.TILE_CONFIGS[effective_tiles(args, ops, M, d, h, r)],
                   "base_weights": args.weights, "l2": l2_note(args.op, M, d, h, cfg_extra)},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
                "steps": e2e_steps,
                "io": "inputs X, dY from pinned host memory every step (the next step's copied on a copy stream "
                      "during the current one); result read back every step on a second copy stream: the adapter "
                      "gradients, from two alternating device gradient buffers"},
        "e2e_outputs": {"value": e2e_out_value, "unit": UNIT, "h2d_bytes_per_step": h2d_bytes,
                        "d2h_bytes_per_step": d2h_out_bytes, "steps": e2e_steps,
                        "io": "as e2e, and Y and dX (the step's own outputs) read back every step too, from two "
                              "alternating device output buffers"},
        "gpu_launches": launches,
        "roofline": roof,
        "dequant": dq,
        "norm": nrm,
        "kernels": kernels,
        "cpu_baseline": cpu,
        "clocks": clocks,
    }), flush=True)


def effective_tiles(args, ops, M, d, h, r):
    """The GEMM configuration the timed step's calls use (the automatic setting resolved)."""
    if args.weights == "bf16" or args.op == "qkv":
        return 4  # the 16-bit and fused Q/K/V calls always stream a bf16 weight by TMA
    if args.op in ("mlp", "norm_mlp"):
        return ops.qlora_mlp_tile_config(M, d, h, r)
    return args.tiles or 4


def torchrun_command(argv, gpus, port, limit_s=1800):
    """The command that runs this script as `gpus` ranks on one node (one process per GPU), bounded by
    `timeout` well above the process group's own 120 s collective timeout."""
    import shutil
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]
    if shutil.which("timeout"):
        cmd = ["timeout", "-k", "60", str(limit_s)] + cmd
    return cmd


def free_port():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def main():
    args = parse()
    if args.impl == "ours" and args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # started as a plain process: start the ranks (the driver's torchrun launch sets WORLD_SIZE itself)
        sys.exit(subprocess.call(torchrun_command(sys.argv[1:], args.gpus, free_port())))
    if (args.op == "linear") != (args.workload in LINEAR_WORKLOADS):
        sys.exit(f"--op {args.op} needs {'a single-projection' if args.op == 'linear' else 'an MLP'} workload")
    if args.impl == "reference" and args.op not in ("mlp", "linear"):
        sys.exit("--impl reference times the MLP (--op mlp) and single-projection (--op linear) workloads")
    wl = dict(LINEAR_WORKLOADS[args.workload] if args.op == "linear" else MLP_WORKLOADS[args.workload])
    if args.tokens:
        wl["M"] = args.tokens
    if args.rank:
        wl["r"], wl["alpha"] = args.rank, float(args.rank)
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
