"""CPU checks of the C ABI: the library builds and loads, exports every entry
point declared in include/qlora.h, returns the oracle's NF4 levels, and rejects
bad arguments on the host (no GPU is touched by any call here)."""

import ctypes
import re

import numpy as np
import pytest

import oracle
from qlora_fine_tuning_nf4_b200 import build, ops


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.lib()


def _declared():
    src = open(ops.HEADER_PATH).read()
    return sorted(set(re.findall(r"QLORA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(ops._SIGS), "binding and header disagree"


def test_codebook_matches_oracle_construction_bit_for_bit(lib):
    ours = np.array(ops.qlora_nf4_codebook(), dtype=np.float32)
    ref = oracle.nf4_codebook().astype(np.float32)
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_status_strings(lib):
    for code, name in ops.STATUS_NAMES.items():
        assert ops.qlora_status_string(code) == name


def test_workspace_queries(lib):
    small = ops.qlora_linear_workspace_bytes(256, 512, 1024)
    big = ops.qlora_linear_workspace_bytes(8192, 4096, 4096)
    assert 256 < small < big
    m = ops.qlora_mlp_workspace_bytes(8192, 4096, 11008)
    assert m >= 2 * 8192 * 11008 * 2  # dE and dG live in the workspace
    assert ops.qlora_linear_workspace_bytes(0, 512, 1024) == 256
    assert ops.qlora_linear_workspace_bytes(16, 512, 1024, 8) == 256  # r != 16 unsupported


def _lin(codes=16, absmax=16, A=16, B=16, n=512, k=512, r=16, scale=1.0):
    # fake device addresses: every call below is rejected before any CUDA call
    return ops.QloraLoraLinear(ops.QloraNF4(codes, absmax, n, k), A, B, r, scale)


def test_host_side_rejections(lib):
    c = _lin()
    f = lib.qlora_linear_fwd
    assert f(ctypes.byref(c), 16, 0, 16, 16, 16, 1 << 30, None) == 0          # M = 0: nothing to do
    assert f(ctypes.byref(c), 16, -1, 16, 16, 16, 1 << 30, None) == 1         # negative M
    assert f(None, 16, 8, 16, 16, 16, 1 << 30, None) == 1                     # null struct
    assert f(ctypes.byref(c), None, 8, 16, 16, 16, 1 << 30, None) == 1        # null X
    assert f(ctypes.byref(c), 24, 8, 16, 16, 16, 1 << 30, None) == 3          # misaligned X
    assert f(ctypes.byref(c), 16, 8, 16, 16, 16, 64, None) == 4               # workspace too small
    assert f(ctypes.byref(_lin(r=8)), 16, 8, 16, 16, 16, 1 << 30, None) == 2  # r != 16
    assert f(ctypes.byref(_lin(k=100)), 16, 8, 16, 16, 16, 1 << 30, None) == 2  # k_in % 64
    # k_in = 320 (a multiple of 64, not of 256) passes the shape check under the default staged feed
    # (rejected next for the 64-byte workspace, still before any CUDA call) ...
    assert f(ctypes.byref(_lin(k=320)), 16, 8, 16, 16, 16, 64, None) == 4
    prev = ops.qlora_set_tile_config(2)
    try:  # ... and is unsupported by the feeds that dequantise in the mainloop
        assert f(ctypes.byref(_lin(k=320)), 16, 8, 16, 16, 16, 1 << 30, None) == 2
    finally:
        ops.qlora_set_tile_config(prev)
    assert f(ctypes.byref(_lin(n=500)), 16, 8, 16, 16, 16, 1 << 30, None) == 2  # n_out % 8
    assert f(ctypes.byref(c), 16, (1 << 23) + 1, 16, 16, 16, 1 << 62, None) == 2  # M above 2^23
    assert f(ctypes.byref(_lin(k=(1 << 23) + 256)), 16, 8, 16, 16, 16, 1 << 30, None) == 2  # k_in above 2^23
    assert f(ctypes.byref(_lin(n=(1 << 23) + 8)), 16, 8, 16, 16, 16, 1 << 30, None) == 2    # n_out above 2^23
    assert f(ctypes.byref(_lin(codes=8)), 16, 8, 16, 16, 16, 1 << 30, None) == 3
    assert lib.nf4_dequantize(16, 16, 4, 100, 16, None) == 2                    # k_in % 64
    assert lib.nf4_dequantize(16, 16, 4, 64, 8, None) == 3
    assert lib.nf4_quantize(16, 0, 64, 16, 16, None) == 0                       # empty
    b = lib.qlora_linear_bwd  # M = 0 clears dA, dB: their pointers are still checked before any CUDA call
    assert b(ctypes.byref(c), None, None, None, 0, None, None, 16, None, 0, None) == 1  # null dA
    assert b(ctypes.byref(c), None, None, None, 0, None, 16, 24, None, 0, None) == 3    # misaligned dB
    g, u, d = _lin(n=512, k=256), _lin(n=512, k=256), _lin(n=256, k=512)
    sv = ops.QloraMlpSaved(16, 16, 16, 16, 16, 16)
    mf = lib.qlora_mlp_fwd
    assert mf(5, ctypes.byref(g), ctypes.byref(u), ctypes.byref(d), 16, 8, 16, ctypes.byref(sv), 16, 1 << 40, None) == 1
    bad_d = _lin(n=256, k=768)
    assert mf(0, ctypes.byref(g), ctypes.byref(u), ctypes.byref(bad_d), 16, 8, 16, ctypes.byref(sv), 16, 1 << 40,
              None) == 1                                                        # shapes do not chain
    assert mf(0, ctypes.byref(g), ctypes.byref(u), ctypes.byref(d), 16, 8, 16, ctypes.byref(sv), 16, 10, None) == 4


def test_noalloc_host_side_rejections(lib):
    """qlora_linear_fwd_noalloc rejects, before any CUDA call, what its fixed
    scratch or its in-mainloop GEMM cannot run (fake device addresses: none of
    these calls reaches the GPU)."""
    f = lib.qlora_linear_fwd_noalloc
    c = _lin(k=256)
    assert f(ctypes.byref(c), 16, (43648 // 64 + 1) * 64, 16, 16, None) == 4  # beyond the documented 43,648 rows
    assert f(ctypes.byref(c), 16, 43649, 16, 16, None) == 4
    assert f(ctypes.byref(_lin(r=32)), 16, 8, 16, 16, None) == 2            # rank 16 only
    assert f(ctypes.byref(_lin(k=320)), 16, 8, 16, 16, None) == 2           # in-mainloop feed: k_in % 256
    assert f(ctypes.byref(c), 16, 0, 16, 16, None) == 0                     # M = 0: nothing to do
    assert f(None, 16, 8, 16, 16, None) == 1


def _noalloc_need(M):
    a256 = lambda x: (x + 255) & ~255
    return 256 + a256(32 * M) + a256(4096 * -(-M // 64))


def test_noalloc_documented_limit_is_the_scratch_formula():
    """43,648 is the largest M whose scratch, 256 + 32 M + 4096 ceil(M / 64)
    bytes rounded per term to 256, fits the 4 MiB array."""
    assert _noalloc_need(43648) <= 4 << 20 < _noalloc_need(43649)


def test_rank_support_follows_the_tile_configuration(lib):
    prev = ops.qlora_set_tile_config(4)
    try:
        for r in (16, 32, 64):  # staged feed: ranks 16, 32, 64
            assert ops.qlora_linear_workspace_bytes(256, 512, 1024, r) > 256
            assert ops.qlora_mlp16_workspace_bytes(256, 512, 1024, r) > 256
        assert ops.qlora_linear_workspace_bytes(256, 512, 1024, 48) == 256
        f = lib.qlora_linear_fwd
        assert f(ctypes.byref(_lin(r=48)), 16, 8, 16, 16, 16, 1 << 30, None) == 2
        ops.qlora_set_tile_config(2)  # dequantised in the mainloop: rank 16 only
        assert ops.qlora_linear_workspace_bytes(256, 512, 1024, 32) == 256
        assert f(ctypes.byref(_lin(r=32)), 16, 8, 16, 16, 16, 1 << 30, None) == 2
    finally:
        ops.qlora_set_tile_config(prev)


def test_tile_config_setting(lib):
    prev = ops.qlora_set_tile_config(1)
    assert ops.qlora_set_tile_config(prev) == 1
    assert ops.qlora_set_tile_config(7) == prev  # invalid values are ignored
    assert ops.qlora_set_tile_config(prev) == prev


def test_binding_rejects_host_tensors_before_any_library_call():
    """The C ABI only sees raw pointers: the binding must refuse a host tensor
    (whose address would be an illegal device access) before calling it."""
    import torch
    n, k, r = 512, 256, 16
    w = ops.NF4Weight(torch.zeros(n * k // 2, dtype=torch.uint8), torch.zeros(n * k // 64, dtype=torch.float32), n, k)
    lin = ops.LoraLinear(w, torch.zeros(k, r, dtype=torch.bfloat16), torch.zeros(r, n, dtype=torch.bfloat16), 1.0)
    X = torch.zeros(8, k, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ops.qlora_linear_fwd(lin, X, ws=None)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ops.qlora_linear_bwd(lin, X, torch.zeros(8, r, dtype=torch.bfloat16), torch.zeros(8, n, dtype=torch.bfloat16),
                             ws=None)
    with pytest.raises(ValueError, match="2-D"):
        ops.qlora_linear_fwd(lin, X.view(-1), ws=None)
    down = ops.LoraLinear(ops.NF4Weight(w.codes, w.absmax, k, n), torch.zeros(n, r, dtype=torch.bfloat16),
                          torch.zeros(r, k, dtype=torch.bfloat16), 1.0)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ops.qlora_mlp_fwd("swiglu", lin, lin, down, X, ws=None)
    with pytest.raises(ValueError, match="MLP weights"):
        ops.qlora_mlp_fwd("swiglu", lin, lin, lin, X, ws=None)


def test_workspace_holds_the_staged_weight_only_under_the_staged_feed(lib):
    """Configuration 4 dequantises each weight once per call into the workspace
    (n_out * k_in bf16 for a projection, the gate and up weights side by side
    for the MLP); the in-mainloop configurations and the 16-bit base need no
    such room."""
    M, d, h = 8192, 4096, 11008
    prev = ops.qlora_set_tile_config(4)
    try:
        lin4 = ops.qlora_linear_workspace_bytes(M, d, d)
        mlp4 = ops.qlora_mlp_workspace_bytes(M, d, h)
        ops.qlora_set_tile_config(2)
        lin2 = ops.qlora_linear_workspace_bytes(M, d, d)
        mlp2 = ops.qlora_mlp_workspace_bytes(M, d, h)
    finally:
        ops.qlora_set_tile_config(prev)
    assert lin4 - lin2 >= d * d * 2
    assert mlp4 - mlp2 >= 2 * h * d * 2
    assert ops.qlora_linear16_workspace_bytes(M, d, d) < lin4
    assert ops.qlora_mlp16_workspace_bytes(M, d, h) < mlp4
    sizes = [ops.qlora_mlp_workspace_bytes(m, d, h) for m in (1, 256, 1024, 8192, 16384)]
    assert sizes == sorted(sizes)


def test_checked_build_exports_the_same_abi():
    """libqlora_check.so (QLORA_CHECK) exports every symbol the normal build
    does and says it is the checked build (a host-only call)."""
    import subprocess
    syms = lambda path: {l.split()[-1] for l in subprocess.run(["nm", "-D", "--defined-only", path], check=True,
                                                                  capture_output=True, text=True).stdout.splitlines()
                         if " T " in l}
    assert syms(ops.CHECK_LIB_PATH) == syms(ops.LIB_PATH)
    assert ops.checked_lib().qlora_checked_build() == 1
    assert ops.lib().qlora_checked_build() == 0


def test_automatic_tile_configuration(lib):
    """Configuration 0 (the default): the NF4 MLP calls dequantise in the mainloop
    (configuration 2) up to 512 tokens when rank and width allow it, and stage
    the weights (configuration 4) otherwise; an explicit choice is kept."""
    prev = ops.qlora_set_tile_config(0)
    try:
        assert ops.qlora_mlp_tile_config(256, 4096, 11008, 16) == 2
        assert ops.qlora_mlp_tile_config(512, 4096, 11008, 16) == 2
        assert ops.qlora_mlp_tile_config(513, 4096, 11008, 16) == 4
        assert ops.qlora_mlp_tile_config(8192, 4096, 11008, 16) == 4
        assert ops.qlora_mlp_tile_config(256, 4096, 11008, 32) == 4   # configuration 2 takes rank 16 only
        assert ops.qlora_mlp_tile_config(256, 320, 512, 16) == 4      # ... and d % 256 == 0
        # the workspace follows: no staging room below the threshold
        assert ops.qlora_mlp_workspace_bytes(256, 4096, 11008) < ops.qlora_mlp_workspace_bytes(256, 4096, 11008, 32)
        ops.qlora_set_tile_config(3)
        assert ops.qlora_mlp_tile_config(8192, 4096, 11008, 16) == 3
    finally:
        ops.qlora_set_tile_config(prev)
