"""The data-parallel step on the GPU: two ranks on cuda:0 with the gloo
backend.  The collective runs on the host, so no kernel of one rank waits for
the other's.  Each rank runs the library's MLP forward and backward on its
token shard inside dp.make_step.  The backward records the early-gradient
event (qlora_mlp_bwd_ev); dp.GradAllReduce sums dA_d, dB_d, dB_g, dB_u on a
side stream that waits for that event, and the rest after the backward.
Checked: the summed buffer equals the two shards' gradients computed one after
the other without the plumbing and added, within one bf16 rounding per
element (the all-reduce adds bf16 values).  A sum that started before its
gradients were final would be far off."""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    from qlora_fine_tuning_nf4_b200 import dp, ops
    from qlora_fine_tuning_nf4_b200.synth import bits_to_torch, make_mlp_problem

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        ops.qlora_set_tile_config(4)
        M, d, h, r = 1024, 512, 768, 16
        p = make_mlp_problem(M, d, h, r, 16.0, seed=5)
        lins = {k: ops.LoraLinear(ops.nf4_quantize(bits_to_torch(p["W_" + k], "cuda")),
                                  bits_to_torch(p["A_" + k], "cuda"), bits_to_torch(p["B_" + k], "cuda"), p["s"])
                for k in ("g", "u", "d")}
        X, dY = bits_to_torch(p["X"], "cuda"), bits_to_torch(p["dY"], "cuda")
        lo, hi = dp.shard_rows(M, rank, world)
        Xs, dYs = X[lo:hi].contiguous(), dY[lo:hi].contiguous()
        ws = ops.Workspace()
        flat, views, early = dp.flat_lora_grads(d, h, r, "cuda")
        grads = dict(views, dX=torch.empty(hi - lo, d, dtype=torch.bfloat16, device="cuda"))
        sync = dp.GradAllReduce(flat, early)
        assert sync.ready_handle() != 0
        saved = {}

        def fwd():
            saved["Y"], saved["s"] = ops.qlora_mlp_fwd("swiglu", lins["g"], lins["u"], lins["d"], Xs, ws)

        def bwd(ev):
            ops.qlora_mlp_bwd("swiglu", lins["g"], lins["u"], lins["d"], Xs, saved["s"], dYs, ws, grads=grads,
                              early_event=ev)

        step = dp.make_step(fwd, bwd, sync)
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        status = ops.qlora_last_device_status(ws)
        result = None
        if rank == 0:
            ref = {}
            for r_ in range(world):
                a, b = dp.shard_rows(M, r_, world)
                Y, sv = ops.qlora_mlp_fwd("swiglu", lins["g"], lins["u"], lins["d"], X[a:b].contiguous(), ws)
                g = ops.qlora_mlp_bwd("swiglu", lins["g"], lins["u"], lins["d"], X[a:b].contiguous(), sv,
                                      dY[a:b].contiguous(), ws)
                for k in dp.GRAD_ORDER:
                    ref[k] = ref.get(k, 0) + g[k].float()
            torch.cuda.synchronize()
            result = {}
            for k in dp.GRAD_ORDER:
                got, want = views[k].float(), ref[k]
                result[k] = int(((got - want).abs() > 2.0 ** -8 * want.abs()).sum())
        q.put((rank, status, result))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_gradient_sum_on_one_gpu_matches_the_shard_sum():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(rk, 2, port, q)) for rk in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=300) for _ in range(2)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, status, result in out:
        assert status == 0
        if rank == 0:
            assert result is not None and all(v == 0 for v in result.values()), result
