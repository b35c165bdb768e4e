"""The timeout path on the GPU, exercised without a fault.

A one-shot test hook (qlora_test_inject_timeout) makes the first CTA of the
next skinny pass leave one tile unloaded.  Its consumers' bounded wait
(about 4 s) expires and records a timeout in the status word; the kernels
after it in the same call see the status and return early (bounded waits,
copies already issued landing before their CTA exits, TMEM released).  The
test checks that qlora_last_device_status reports QLORA_ERR_TIMEOUT and
clears it, and that the same context then computes exactly the bits of a
run made before the injection.
"""

import pytest
import torch

from qlora_fine_tuning_nf4_b200 import ops
from qlora_fine_tuning_nf4_b200.synth import make_linear_problem

from parity import dev, gpu_weight

pytestmark = pytest.mark.gpu

QLORA_ERR_TIMEOUT = 6


def test_bounded_wait_reports_timeout_and_the_context_recovers():
    ops.qlora_set_tile_config(4)
    # 4096 tokens x 4096 inputs: every CTA of the X A pass streams several tiles,
    # so the injected one has a tile 1 to miss
    p = make_linear_problem(4096, 4096, 1024, seed=21)
    w, _, _ = gpu_weight(p["W"])
    lin = ops.LoraLinear(w, dev(p["A"]), dev(p["B"]), p["s"])
    ws = ops.Workspace()
    X, dY = dev(p["X"]), dev(p["dY"])

    def run():
        Y, XA = ops.qlora_linear_fwd(lin, X, ws)
        dX, dA, dB = ops.qlora_linear_bwd(lin, X, XA, dY, ws)
        torch.cuda.synchronize()
        return [t.clone() for t in (Y, XA, dX, dA, dB)]

    before = run()
    assert ops.qlora_last_device_status(ws) == 0

    ops.qlora_test_inject_timeout()
    ops.qlora_linear_fwd(lin, X, ws)
    torch.cuda.synchronize()
    assert ops.STATUS_NAMES[ops.qlora_last_device_status(ws)] == ops.STATUS_NAMES[QLORA_ERR_TIMEOUT]
    assert ops.qlora_last_device_status(ws) == 0  # reading it cleared it

    after = run()
    assert ops.qlora_last_device_status(ws) == 0
    for name, a, b in zip(("Y", "XA", "dX", "dA", "dB"), before, after):
        assert torch.equal(a, b), f"{name} differs after the recovered timeout"
