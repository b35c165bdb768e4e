"""Multi-process (gloo, CPU) check of the data-parallel step logic: each rank
computes the adapter gradients of its token shard (oracle, fp64), the flat
buffer is all-reduced, and the sum equals the full-batch gradients.  One case
leaves a rank with no tokens: its gradients are zero and the sum is unchanged.

The second test runs the step plumbing the benchmark times (dp.make_step with
dp.GradAllReduce's two-part sum over dp.flat_lora_grads), with the oracle
standing in for the library's forward and backward."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from qlora_fine_tuning_nf4_b200 import dp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _problem(M=24):
    rng = np.random.default_rng(0)
    d, h, r = 64, 96, 4
    X = rng.standard_normal((M, d))
    proj = lambda K, N, s: (rng.standard_normal((N, K)) * 0.2, rng.uniform(-1, 1, (K, r)) / np.sqrt(K),
                            rng.standard_normal((r, N)) * 0.3, s)
    gate, up, down = proj(d, h, 1.0), proj(d, h, 1.0), proj(h, d, 2.0)
    dY = rng.standard_normal((M, d))
    return M, d, h, r, X, gate, up, down, dY


def _worker(rank, world, port, q, M):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        M, d, h, r, X, gate, up, down, dY = _problem(M)
        lo, hi = dp.shard_rows(M, rank, world)
        g = oracle.mlp_bwd("swiglu", X[lo:hi], gate, up, down, dY[lo:hi])
        flat, views, _ = dp.flat_lora_grads(d, h, r, "cpu", dtype=torch.float64)
        for k in dp.GRAD_ORDER:
            views[k].copy_(torch.from_numpy(g[k]))
        dp.allreduce_lora_grads(flat)
        if rank == 0:
            q.put({k: views[k].numpy().copy() for k in dp.GRAD_ORDER})
    finally:
        dist.destroy_process_group()


def _step_worker(rank, world, port, q, M):
    """The benchmark's step (dp.make_step) on this rank's shard, oracle kernels."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        M, d, h, r, X, gate, up, down, dY = _problem(M)
        lo, hi = dp.shard_rows(M, rank, world)
        flat, views, early = dp.flat_lora_grads(d, h, r, "cpu", dtype=torch.float64)
        sync = dp.GradAllReduce(flat, early)
        state = {"bwd": 0}

        def forward():
            state["fwd"] = oracle.mlp_fwd("swiglu", X[lo:hi], gate, up, down)

        def backward(ready):
            assert ready == 0  # no CUDA event on the CPU: both parts are summed after the backward
            g = oracle.mlp_bwd("swiglu", X[lo:hi], gate, up, down, dY[lo:hi], saved=state["fwd"])
            for k in dp.GRAD_ORDER:
                views[k].copy_(torch.from_numpy(g[k]))
            state["bwd"] += 1

        step = dp.make_step(forward, backward, sync)
        step()
        step()  # a second step rewrites the gradients: the sums must not accumulate across steps
        if rank == 0:
            q.put(({k: views[k].numpy().copy() for k in dp.GRAD_ORDER}, state["bwd"]))
    finally:
        dist.destroy_process_group()


def _spawn(target, M, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(rk, world, port, q, M)) for rk in range(world)]
    for p in procs:
        p.start()
    got = q.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    return got


@pytest.mark.parametrize("M,world", [(24, 2), (2, 3)])
def test_benchmark_step_plumbing_sums_shards_to_full_batch(M, world):
    got, nbwd = _spawn(_step_worker, M, world)
    assert nbwd == 2
    M, d, h, r, X, gate, up, down, dY = _problem(M)
    full = oracle.mlp_bwd("swiglu", X, gate, up, down, dY)
    for k in dp.GRAD_ORDER:
        np.testing.assert_allclose(got[k], full[k], rtol=1e-12, atol=1e-12)


def _bf16_contrib(rank, n=4096):
    """Rank `rank`'s bf16 contribution: magnitudes within a factor 2^6 of each other, so the sum of
    four of them is exact in binary32 and its bf16 rounding is the correctly rounded sum."""
    g = torch.Generator().manual_seed(100 + rank)
    mag = torch.exp2(torch.randint(-3, 3, (n,), generator=g).float())
    return (torch.randn(n, generator=g) * mag).to(torch.bfloat16)


def _bf16_sum_worker(rank, world, port, q, early):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        flat = _bf16_contrib(rank).clone()
        sync = dp.GradAllReduce(flat, early)
        sync.launch()
        sync.wait()
        if rank == 0:
            q.put(flat.clone())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("early", [0, 1000])
def test_bf16_gradients_are_summed_in_binary32_and_rounded_once(early):
    world = 4
    got = _spawn(_bf16_sum_worker, early, world)
    parts = [_bf16_contrib(rk) for rk in range(world)]
    exact = sum(p.float() for p in parts)  # exact in binary32 (see _bf16_contrib)
    assert torch.equal(got, exact.to(torch.bfloat16))
    # the check has teeth: adding in bf16, rank after rank, rounds differently for many elements
    seq = parts[0]
    for p in parts[1:]:
        seq = (seq.float() + p.float()).to(torch.bfloat16)
    assert (seq != exact.to(torch.bfloat16)).sum() > 100


def test_early_part_of_the_flat_buffer_is_the_four_gradients_final_before_the_gate_up_dx_gemm():
    d, h, r = 4096, 11008, 16
    flat, views, early = dp.flat_lora_grads(d, h, r, "cpu")
    first = dp.GRAD_ORDER[:dp.MLP_EARLY]
    assert set(first) == {"dA_d", "dB_d", "dB_g", "dB_u"}
    assert early == sum(views[k].numel() for k in first)
    for k in first:
        assert views[k].data_ptr() < flat.data_ptr() + early * flat.element_size()
    for k in dp.GRAD_ORDER[dp.MLP_EARLY:]:
        assert views[k].data_ptr() >= flat.data_ptr() + early * flat.element_size()


@pytest.mark.parametrize("M,world", [(24, 2), (2, 3)])  # (2, 3): the third rank's shard is empty
def test_sharded_gradients_sum_to_full_batch(M, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(rk, world, port, q, M)) for rk in range(world)]
    for p in procs:
        p.start()
    got = q.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    M, d, h, r, X, gate, up, down, dY = _problem(M)
    full = oracle.mlp_bwd("swiglu", X, gate, up, down, dY)
    for k in dp.GRAD_ORDER:
        np.testing.assert_allclose(got[k], full[k], rtol=1e-12, atol=1e-12)


def test_flat_buffer_views_are_aligned_and_disjoint():
    flat, views, _ = dp.flat_lora_grads(4096, 11008, 16, "cpu")
    offs = []
    for k in dp.GRAD_ORDER:
        v = views[k]
        assert v.is_contiguous()
        off = (v.data_ptr() - flat.data_ptr())
        assert off % 16 == 0
        offs.append((off, off + v.numel() * v.element_size()))
    offs.sort()
    assert all(a[1] <= b[0] for a, b in zip(offs, offs[1:]))
    assert offs[-1][1] == flat.numel() * flat.element_size()


@pytest.mark.parametrize("M,world", [(8192, 1), (8192, 8), (100, 3), (2, 4)])
def test_shard_rows_partition(M, world):
    seen = []
    for rk in range(world):
        lo, hi = dp.shard_rows(M, rk, world)
        seen.extend(range(lo, hi))
    assert seen == list(range(M))
