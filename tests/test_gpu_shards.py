"""Data-parallel semantics of the CUDA path without a collective: the MLP step
run on token shards (one of them empty) gives adapter gradients whose sum is
the full batch's, compared with the fp64 oracle.

Each shard's gradients are rounded to bf16 once, so the sum of two shards
carries at most two such errors; each is within the small-M bar (3e-2 x the
shard's RMS), and a shard of about half the tokens has an RMS of about
1/sqrt(2) of the full batch's, so the sum stays within 3e-2 x sqrt(2) < 5e-2
of the full batch's RMS.
"""

import numpy as np
import pytest
import torch

from qlora_fine_tuning_nf4_b200 import ops
from qlora_fine_tuning_nf4_b200.synth import make_mlp_problem

from parity import assert_close, dev, gpu_f64, gpu_weight, run_mlp_oracle

pytestmark = pytest.mark.gpu

GRADS = ("dA_g", "dB_g", "dA_u", "dB_u", "dA_d", "dB_d")


@pytest.mark.parametrize("act", ["swiglu", "geglu_tanh"])
def test_shard_gradients_sum_to_the_full_batch(act):
    M, d, h = 1100, 512, 768
    p = make_mlp_problem(M, d, h, seed=21)
    ops.qlora_set_tile_config(4)
    lins = {}
    for k in ("g", "u", "d"):
        lins[k] = ops.LoraLinear(gpu_weight(p["W_" + k])[0], dev(p["A_" + k]), dev(p["B_" + k]), p["s"])
    X, dY = dev(p["X"]), dev(p["dY"])
    ws = ops.Workspace()
    total = {k: np.zeros(tuple(getattr(lins[k[-1]], "A" if k.startswith("dA") else "B").shape)) for k in GRADS}
    for lo, hi in ((0, 600), (600, 1100), (1100, 1100)):
        Xs, dYs = X[lo:hi].contiguous(), dY[lo:hi].contiguous()
        _, saved = ops.qlora_mlp_fwd(act, lins["g"], lins["u"], lins["d"], Xs, ws)
        g = ops.qlora_mlp_bwd(act, lins["g"], lins["u"], lins["d"], Xs, saved, dYs, ws)
        torch.cuda.synchronize()
        assert ops.qlora_last_device_status(ws) == 0
        for k in GRADS:
            total[k] += gpu_f64(g[k])
    o = run_mlp_oracle(p, act)
    for k in GRADS:
        assert_close(k, total[k], o[k], tol=5e-2)
