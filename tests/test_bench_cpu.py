"""Host logic of the benchmark: the FLOP counts it divides by and the choice
of the roofline denominator (no GPU needed)."""

import bench


def test_mlp_flops_is_the_sum_of_its_gemms_and_lora_terms():
    M, d, h, r = 8192, 4096, 11008, 16
    dense = 4 * M * d * 2 * h + 4 * M * h * d          # fwd + dX of gate/up (N = 2h) and of down
    lora = 6 * M * r * (d + h) * 2 + 6 * M * r * (h + d)  # 6 M r (K + N) per projection
    assert bench.mlp_flops(M, d, h, r) == dense + lora
    per_gemm = sum(bench.kernel_flops(k, M, d, h, r) for k in
                   ("gemm_nf4_gateup_glu_fwd", "gemm_nf4_fwd", "gemm_nf4_down_bwd_glu", "gemm_nf4_bwd_dx"))
    assert per_gemm <= bench.mlp_flops(M, d, h, r)     # the skinny passes carry the rest of the LoRA work
    assert per_gemm >= dense


def test_roofline_peak_follows_the_measured_clock():
    pk = {"bf16": 1637.6, "bf16_sustained": 1390.6, "sustained_mhz": 1342.0, "max_mhz": 1965.0, "src": "measured"}
    peak, kind = bench.tensor_peak(pk, {"sm_mhz": 1320.0})   # held at the power cap: the sustained loop's figure
    assert peak == 1390.6 and "sustained" in kind
    peak, kind = bench.tensor_peak(pk, {"sm_mhz": 1965.0})   # full clock: the burst figure
    assert peak == 1637.6 and "burst" in kind
    peak, kind = bench.tensor_peak(pk, {"sm_mhz": None})
    assert peak == 1390.6 and "no clock record" in kind


def test_cpu_baseline_repeats_whole_batches_until_the_target_time():
    """A batch the probe finds cheap is timed as whole-batch steps repeated
    until the target has passed, and the FLOP count covers every step."""
    wl = {"M": 128, "d": 256, "h": 512, "r": 16, "alpha": 16.0, "seed": 0, "act": "swiglu"}
    dt, flop, cores, rows, steps = bench.oracle_sample(wl, target_s=0.5)
    assert rows == 128 and steps >= 1 and dt >= 0.5
    assert flop == steps * bench.mlp_flops(128, 256, 512, 16)
    assert cores >= 1
    dt, flop, _, rows, steps = bench.oracle_sample(wl, rows=64)
    assert rows == 64 and steps == 1 and flop == bench.mlp_flops(64, 256, 512, 16)


def test_c_loop_baseline_record():
    rec = bench.c_loop_oracle_sample()
    assert rec["value"] > 0 and rec["ms"] > 0 and rec["threads"] == 1 and rec["unit"] == bench.UNIT


def test_gpus_n_starts_n_ranks_on_one_node():
    """`bench.py --gpus N` started as one process re-runs itself under torchrun
    with N ranks on this node (rendezvous on 127.0.0.1), bounded by `timeout`."""
    cmd = bench.torchrun_command(["--gpus", "4", "--steps", "20"], 4, 29511)
    assert "--nproc-per-node=4" in cmd and "--nnodes=1" in cmd
    i = cmd.index("--master-addr")
    assert cmd[i + 1] == "127.0.0.1" and cmd[cmd.index("--master-port") + 1] == "29511"
    assert cmd[-3:] == ["4", "--steps", "20"] and cmd[-5].endswith("bench.py")
    if cmd[0] == "timeout":
        assert cmd[1:3] == ["-k", "60"] and int(cmd[3]) > 120  # well above the process group's own timeout


def test_clock_summary_uses_the_timed_window_or_its_nearest_samples():
    import datetime
    base = datetime.datetime(2026, 1, 1, 12, 0, 0)
    line = lambda dt, mhz, cap: (f"{(base + datetime.timedelta(seconds=dt)).strftime('%Y/%m/%d %H:%M:%S.%f')[:-3]}, "
                                 f"0, {mhz}, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, "
                                 f"{'Active' if cap else 'Not Active'}")
    out = "\n".join([line(0.00, 1965, False), line(0.05, 1800, True), line(0.10, 1700, True), line(0.40, 1965, False)])
    t = base.timestamp()
    inside = bench.ClockSampler.summarize(out, t + 0.04, t + 0.11)
    assert inside["samples"] == 2 and inside["sm_mhz"] == 1750 and inside["reasons"] == ["sw_power_cap"]
    assert inside["window"] == "timed region"
    short = bench.ClockSampler.summarize(out, t + 0.65, t + 0.655)  # a 5 ms window holds no sample
    assert short["samples"] == 1 and short["sm_mhz"] == 1965 and short["reasons"] == []
    assert "no sample inside" in short["window"]


def test_cpu_baseline_for_a_single_projection():
    """The projection workloads are timed against the oracle's projection fwd+bwd too."""
    from qlora_fine_tuning_nf4_b200.workloads import LINEAR_WORKLOADS, linear_flops
    wl = dict(LINEAR_WORKLOADS["tiny_linear"])
    dt, flop, cores, rows, steps = bench.oracle_sample(wl, op="linear", target_s=0.3)
    assert rows == wl["M"] and steps >= 1 and dt >= 0.3
    assert flop == steps * linear_flops(wl["M"], wl["K"], wl["N"], wl["r"])
