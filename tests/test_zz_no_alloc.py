"""conv_wgrad_noalloc, the weight gradient that allocates nothing (needs a B200).

Some callers cannot allocate device memory at all: a plugin inside a framework
whose caching allocator owns the device's memory, a real-time loop where
cudaMalloc/cudaFree may block or synchronise the device, a runtime that
reserved its whole budget at start-up.  They cannot hand conv_wgrad its fp32
workspace, so conv_wgrad_noalloc takes its scratch from a fixed array inside
the library.  These tests call it through the C ABI and check it against
conv_wgrad, the entry point with a caller workspace, on two calls in a row: the
array keeps the previous call's contents, so the second call (a smaller
problem after a larger one, split into fewer ranges) shows whether a call
reads anything it did not write itself.
This file is collected last on purpose.
"""
from __future__ import annotations

import zlib

import numpy as np
import pytest
import torch

import oracle
from tests.parity import TOL, assert_parity

pytestmark = pytest.mark.gpu

C = pytest.importorskip("implicit_gemm_convolution_conv2d_b200")

CODE = {"f32": 0, "f16": 1, "bf16": 2}
DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
STATIC_SCRATCH_BYTES = 16 << 20
ESCRATCH = -9

# (name, N, D, H, W, C, O, k, stride, pad_lo, pad_hi, dil, groups), in call
# order, each needing less scratch than the one before, so stale partial sums
# would show.  The first runs on the tensor-core path with more ranges than the
# static array holds slices for (conv_wgrad: 4 ranges of 4.5 MiB; here 3);
# the other two run the FP32 kernel.
CALLS = [
    ("na_tc_capped_ranges", 2, 1, 32, 32, 256, 512, (1, 3, 3), (1, 1, 1), (0, 1, 1), (0, 1, 1), (1, 1, 1), 1),
    ("na_large_3d", 4, 8, 16, 16, 48, 64, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), (1, 1, 1), 1),
    ("na_small_2d_groups", 3, 1, 13, 11, 32, 24, (1, 3, 3), (1, 2, 1), (0, 1, 1), (0, 2, 1), (1, 1, 2), 2),
]


def _inputs(case, dtype):
    name, N, D, H, W, Cc, O, k, s, p, ph, d, G = case
    gen = torch.Generator().manual_seed(zlib.crc32(name.encode()) % 1000)
    Do, Ho, Wo = C.out_dims(D, H, W, *k, s, p, d, ph)
    x = (torch.rand((N, D, H, W, Cc), generator=gen) * 2 - 1).to(DT[dtype])
    dy = (torch.rand((N, Do, Ho, Wo, O), generator=gen) * 2 - 1).to(DT[dtype])
    return x, dy, (N, D, H, W, Cc, O, *k, s, p, ph, d, G)


def _noalloc(xd, dyd, shape, geom, dtype):
    dw = torch.full(shape, float("nan"), dtype=DT[dtype], device="cuda")
    rc = C.conv_wgrad_noalloc_raw(xd.data_ptr(), dyd.data_ptr(), dw.data_ptr(), geom, CODE[dtype],
                                  torch.cuda.current_stream().cuda_stream)
    return rc, dw


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
def test_noalloc_matches_conv_wgrad_on_two_calls(dtype):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    for case in CALLS:
        name, N, D, H, W, Cc, O, k, s, p, ph, d, G = case
        x, dy, geom = _inputs(case, dtype)
        xd, dyd = x.cuda(), dy.cuda()
        shape = (O, *k, Cc // G)
        slice_bytes = O * k[0] * k[1] * k[2] * (Cc // G) * 4
        assert slice_bytes <= STATIC_SCRATCH_BYTES
        g_ws = C.conv_wgrad(xd, dyd, k, stride=s, padding=p, dilation=d, groups=G, padding_hi=ph)
        rc, g_na = _noalloc(xd, dyd, shape, geom, dtype)
        assert rc == 0, C.strerror(rc)
        torch.cuda.synchronize()
        assert C.last_status() == 0
        g_ref, s_ref = oracle.conv_wgrad(x, dy, k, s, p, d, G, pad_hi=ph)
        # the two entry points agree within the parity tolerance ...
        rel, ab = TOL[dtype]
        a = g_na.cpu().double().numpy().ravel()
        b = g_ws.cpu().double().numpy().ravel()
        tol = rel * np.asarray(s_ref, np.float64).ravel() + ab
        assert np.all(np.abs(a - b) <= tol), f"{name}/{dtype}: no-alloc and workspace results differ"
        # ... and each meets the oracle
        assert_parity(g_na.cpu(), g_ref, s_ref, dtype, f"{name}/{dtype}/noalloc")
        assert_parity(g_ws.cpu(), g_ref, s_ref, dtype, f"{name}/{dtype}/workspace")


def test_noalloc_rejects_problems_beyond_the_static_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # 16-bit output, O * taps * C = 1024 * 9 * 1024 fp32 values = 36 MiB of scratch
    N, H, W, Cc, O = 1, 4, 4, 1024, 1024
    geom = (N, 1, H, W, Cc, O, 1, 3, 3, (1, 1, 1), (0, 1, 1), (0, 1, 1), (1, 1, 1), 1)
    need = C.wgrad_workspace_size(N, 1, H, W, Cc, O, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 1, "bf16")
    assert need > STATIC_SCRATCH_BYTES
    xd = torch.zeros((N, 1, H, W, Cc), dtype=torch.bfloat16, device="cuda")
    dyd = torch.zeros((N, 1, H, W, O), dtype=torch.bfloat16, device="cuda")
    sentinel = torch.full((O, 1, 3, 3, Cc), 7.0, dtype=torch.bfloat16, device="cuda")
    rc = C.conv_wgrad_noalloc_raw(xd.data_ptr(), dyd.data_ptr(), sentinel.data_ptr(), geom, CODE["bf16"],
                                  torch.cuda.current_stream().cuda_stream)
    assert rc == ESCRATCH
    assert "scratch" in C.strerror(rc)
    torch.cuda.synchronize()
    assert torch.all(sentinel == 7.0), "a rejected call wrote its output"
    assert C.last_status() == 0
