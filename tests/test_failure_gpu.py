"""Failure detection on the GPU without a fault: an injected pipeline stall.

`conv_debug_inject_stall` makes the next tensor-core launch's MMA thread wait
on a barrier that nothing arrives at, with a short limit.  The kernel must
give up, drain, free its tensor memory and return; the host must read
CONV_ETIMEOUT from the status word; and the context must stay usable: the
very next launch is checked against the oracle.
"""
from __future__ import annotations

import time

import pytest
import torch

import oracle
import workloads as WL
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu

C = pytest.importorskip("implicit_gemm_convolution_conv2d_b200")
ETIMEOUT = -6


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield


def _geom(wl):
    return (wl.N, wl.D, wl.H, wl.W, wl.C, wl.O, *wl.k, wl.stride, wl.pad, wl.dil, wl.groups)


@pytest.mark.parametrize("variant", ["TC_GATHER", "TC_TMA", "TC_TMA_PAIR", "TC_HALO", "TC_HALO_PAIR", "TC_TMA_T",
                                     "TC_HALO_T", "TC_HALO_T_PAIR", "TC_PHASE", "DEPTHWISE", "TC_STAGED"])
def test_injected_stall_times_out_and_recovers(variant):
    v = getattr(C, "VARIANT_" + variant)
    O = {"TC_TMA_T": 128, "TC_HALO_T": 128, "TC_HALO_T_PAIR": 256}.get(variant, 64)
    if variant == "TC_PHASE":   # a stem-like layer: 3 input channels, 7x7 at stride 2
        wl = WL.case(2, 1, 20, 24, 3, O, (1, 7, 7), (1, 2, 2), (0, 3, 3), dtype="f16", seed=21)
    elif variant == "DEPTHWISE":   # one filter per channel; the TMA-staged slabs
        wl = WL.case(2, 1, 30, 28, 64, 64, (1, 3, 3), pad=(0, 1, 1), groups=64, dtype="f16", seed=21)
        assert C.plan(wl.N, wl.D, wl.H, wl.W, wl.C, wl.O, wl.k, wl.stride, wl.pad, wl.dil, wl.groups, "f16",
                      v)[0] == v
    else:
        wl = WL.case(2, 1, 20, 20, 64, O, (1, 3, 3), pad=(0, 1, 1), dtype="f16", seed=21)
    x, w = WL.make_inputs(wl)
    xd, wd = x.cuda(), w.cuda()
    dims = C.out_dims(wl.D, wl.H, wl.W, *wl.k, wl.stride, wl.pad, wl.dil)
    y = torch.zeros((wl.N, *dims, O), dtype=torch.float16, device="cuda")
    assert C.last_status() == 0
    C.inject_stall(50_000_000)  # 50 ms
    t0 = time.perf_counter()
    rc = C.conv_fwd_raw(xd.data_ptr(), wd.data_ptr(), y.data_ptr(), _geom(wl), 1, v,
                        torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert C.last_status() == ETIMEOUT
    assert C.last_status() == 0          # read-and-clear
    assert elapsed < 10.0, f"the stalled kernel took {elapsed:.1f} s to give up"
    # the context is still usable: a normal launch gives the right answer
    rc = C.conv_fwd_raw(xd.data_ptr(), wd.data_ptr(), y.data_ptr(), _geom(wl), 1, v,
                        torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert C.last_status() == 0
    y_ref, s_ref = oracle.conv_fwd(x, w, wl.stride, wl.pad, wl.dil, wl.groups)
    assert_parity(y.cpu(), y_ref, s_ref, "f16", f"after stall/{variant}")


def test_inject_rejects_bad_limits():
    with pytest.raises(C.ConvError):
        C.inject_stall(0)
    with pytest.raises(C.ConvError):
        C.inject_stall(20_000_000_000)


def test_injected_stall_in_the_tensor_core_weight_gradient():
    """The same hook in the tensor-core weight-gradient kernel (CTA pairs):
    the stalled launch gives up and the status word reads CONV_ETIMEOUT; the
    next call matches the oracle."""
    gen = torch.Generator().manual_seed(23)
    x = (torch.rand((2, 1, 12, 12, 64), generator=gen) * 2 - 1).to(torch.bfloat16)
    dy = (torch.rand((2, 1, 12, 12, 256), generator=gen) * 2 - 1).to(torch.bfloat16)
    xd, dyd = x.cuda(), dy.cuda()
    assert C.last_status() == 0
    C.inject_stall(50_000_000)
    t0 = time.perf_counter()
    C.conv_wgrad(xd, dyd, (1, 3, 3), padding=(0, 1, 1))
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 10.0
    assert C.last_status() == ETIMEOUT
    assert C.last_status() == 0
    g = C.conv_wgrad(xd, dyd, (1, 3, 3), padding=(0, 1, 1))
    torch.cuda.synchronize()
    assert C.last_status() == 0
    g_ref, s_ref = oracle.conv_wgrad(x, dy, (1, 3, 3), (1, 1, 1), (0, 1, 1))
    assert_parity(g.cpu(), g_ref, s_ref, "bf16", "wgrad after stall")


def test_host_buffer_path_reports_a_timeout():
    """conv_fwd_host waits for its result and then reads the status word: a
    kernel that gave up on a pipeline wait (the injected stall) makes the call
    fail with CONV_ETIMEOUT instead of returning a partial y; the word is then
    clear and the next call is exact."""
    wl = WL.case(2, 1, 20, 20, 64, 64, (1, 3, 3), pad=(0, 1, 1), dtype="f16", seed=24)
    x, w = WL.make_inputs(wl)
    xh, wh = x[:, 0].contiguous().pin_memory(), w[:, 0].contiguous().pin_memory()
    yh = torch.zeros((2, 20, 20, 64), dtype=torch.float16).pin_memory()
    xd, wd = torch.empty_like(xh, device="cuda"), torch.empty_like(wh, device="cuda")
    yd = torch.empty(yh.shape, dtype=torch.float16, device="cuda")
    assert C.last_status() == 0
    C.inject_stall(50_000_000)
    with pytest.raises(C.ConvError) as e:
        C.conv_fwd_host(xh, wh, yh, xd, wd, yd, stride=1, padding=1)
    assert e.value.code == ETIMEOUT
    assert C.last_status() == 0
    C.conv_fwd_host(xh, wh, yh, xd, wd, yd, stride=1, padding=1)
    y_ref, s_ref = oracle.conv_fwd(x, w, wl.stride, wl.pad, wl.dil, wl.groups)
    assert_parity(yh.unsqueeze(1), y_ref, s_ref, "f16", "host path after a timeout")
