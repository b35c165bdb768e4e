"""Reproducibility and graph capture of the CUDA path.

Every reduction in the library runs in a fixed order (the skinny passes write
one partial per CTA and group, the reduction adds them in slot order; the GEMMs
accumulate in a fixed k order), so a step repeated on the same inputs gives the
same bits.  The entry points neither allocate nor synchronise, so a whole
forward + backward step can be captured into a CUDA graph (the programmatic
launches become graph edges) and replayed with the same bits.
"""

import pytest
import torch

from qlora_fine_tuning_nf4_b200 import ops
from qlora_fine_tuning_nf4_b200.synth import make_mlp_problem

from parity import dev, gpu_weight

pytestmark = pytest.mark.gpu


def _mlp_setup(M=1100, d=512, h=768, act="swiglu", seed=3):
    ops.qlora_set_tile_config(4)
    p = make_mlp_problem(M, d, h, seed=seed)
    lins = {}
    for k in ("g", "u", "d"):
        w, _, _ = gpu_weight(p["W_" + k])
        lins[k] = ops.LoraLinear(w, dev(p["A_" + k]), dev(p["B_" + k]), p["s"])
    X, dY = dev(p["X"]), dev(p["dY"])
    ws = ops.Workspace()
    saved = ops.make_mlp_saved(M, h, 16, "cuda")
    Y = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    grads = {"dX": torch.empty(M, d, dtype=torch.bfloat16, device="cuda")}
    for k in ("g", "u", "d"):
        grads["dA_" + k] = torch.empty_like(lins[k].A)
        grads["dB_" + k] = torch.empty_like(lins[k].B)

    def step():
        ops.qlora_mlp_fwd(act, lins["g"], lins["u"], lins["d"], X, ws, Y=Y, saved=saved)
        ops.qlora_mlp_bwd(act, lins["g"], lins["u"], lins["d"], X, saved, dY, ws, grads=grads)

    def snapshot():
        out = {"Y": Y.clone()}
        out.update({k: v.clone() for k, v in saved.items()})
        out.update({k: v.clone() for k, v in grads.items()})
        return out

    ws.get(ops.qlora_mlp_workspace_bytes(M, d, h, 16))  # size the workspace before any capture
    return step, snapshot, ws


def _same(a, b):
    for k in a:
        assert torch.equal(a[k], b[k]), f"{k} differs"


def test_mlp_step_is_bitwise_reproducible():
    step, snapshot, ws = _mlp_setup()
    step()
    torch.cuda.synchronize()
    first = snapshot()
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    assert ops.qlora_last_device_status(ws) == 0
    _same(first, snapshot())


def test_mlp_step_captured_in_a_cuda_graph_replays_the_same_bits():
    step, snapshot, ws = _mlp_setup(act="geglu_tanh", seed=4)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # eager reference (and warm-up) on the capture stream
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    eager = snapshot()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    assert ops.qlora_last_device_status(ws) == 0
    _same(eager, snapshot())
    del graph
