"""GPU parity of qlora_rmsnorm_fwd / qlora_rmsnorm_bwd against the fp64 oracle
(oracle/norm.py): Llama-style gain w and Gemma-style 1 + w, ragged widths (d
not a multiple of 256), a single row, and the Llama and Gemma model widths at
full token counts.

Bounds from the arithmetic, element by element: y = bf16(x * rstd * g) is one
bf16 rounding (2^-8 relative) of an fp32 expression whose own error is far
below it; dx = rstd * (g dy - n c) is one rounding of a difference whose fp32
error scales with the magnitudes of its two terms, not with dx.  Where half an
ulp of a tensor's largest element is within 2e-2 * RMS, the tensor also meets
max|err| <= 2e-2 * RMS."""

import numpy as np
import pytest
import torch

import oracle
from qlora_fine_tuning_nf4_b200 import ops
from qlora_fine_tuning_nf4_b200.synth import bf16_bits, bits_to_torch

from parity import assert_close, f64, gpu_f64

pytestmark = pytest.mark.gpu


def _problem(M, d, gemma, seed):
    rng = np.random.default_rng(seed)
    # token rows whose norms spread by 2x (hidden states entering a norm); a wider spread makes the
    # largest dx elements, and so their single bf16 rounding, large against the tensor's RMS
    X = bf16_bits((rng.standard_normal((M, d), dtype=np.float32) *
                   rng.uniform(0.7, 1.4, size=(M, 1)).astype(np.float32)))
    w = bf16_bits((rng.standard_normal(d, dtype=np.float32) * np.float32(0.1) +
                   np.float32(0.0 if gemma else 1.0)))
    dY = bf16_bits(rng.standard_normal((M, d), dtype=np.float32))
    return X, w, dY


@pytest.mark.parametrize("gemma", [False, True])
@pytest.mark.parametrize("M,d", [(1, 8), (300, 4096), (257, 3072), (64, 520), (8192, 4096), (16384, 3072)])
def test_rmsnorm_parity(M, d, gemma):
    eps = 1e-6 if gemma else 1e-5
    X, w, dY = _problem(M, d, gemma, M + d + gemma)
    Xt, wt, dYt = bits_to_torch(X, "cuda"), bits_to_torch(w, "cuda"), bits_to_torch(dY, "cuda")
    Y, rstd = ops.qlora_rmsnorm_fwd(Xt, wt, eps, plus_one=gemma)
    dX = ops.qlora_rmsnorm_bwd(Xt, wt, rstd, dYt, plus_one=gemma)
    torch.cuda.synchronize()
    x, wf, dy = f64(X), f64(w), f64(dY)
    y_ref, rstd_ref = oracle.rmsnorm_fwd(x, wf, eps, plus_one=gemma)
    dx_ref = oracle.rmsnorm_bwd(x, wf, eps, dy, plus_one=gemma)
    y, dx, rs = gpu_f64(Y), gpu_f64(dX), rstd.cpu().double().numpy()
    assert np.all(np.abs(rs - rstd_ref) <= 1e-5 * rstd_ref)
    rms_y = np.sqrt(np.mean(y_ref ** 2))
    assert np.all(np.abs(y - y_ref) <= (2.0 ** -8 + 2.0 ** -12) * np.abs(y_ref) + 2.0 ** -16 * rms_y)
    g = 1.0 + wf if gemma else wf
    n = x * rstd_ref[:, None]
    c = np.mean(n * g[None, :] * dy, axis=1)
    terms = rstd_ref[:, None] * (np.abs(g[None, :] * dy) + np.abs(n * c[:, None]))
    assert np.all(np.abs(dx - dx_ref) <= 2.0 ** -8 * np.abs(dx_ref) + 2.0 ** -12 * terms)
    for name, got, want in (("Y", y, y_ref), ("dX", dx, dx_ref)):
        # the per-tensor bar max|err| <= 2e-2 * RMS is reachable by a bf16 result only while half an ulp
        # of its largest element fits under it (33 M Gaussian-tailed elements can reach 8 x RMS)
        top = float(np.max(np.abs(want)))
        half_ulp = 2.0 ** (np.floor(np.log2(top)) - 8)
        if half_ulp <= 2e-2 * np.sqrt(np.mean(want ** 2)):
            assert_close(name, got, want)


def test_rmsnorm_rejects_bad_widths():
    X = torch.zeros(4, 12, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(12, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ops.QloraError):
        ops.qlora_rmsnorm_fwd(X, w, 1e-5)
