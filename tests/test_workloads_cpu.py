"""The input recipe (workloads.py) against the published workload table: the
shapes, strides, paddings, types and seeds of the tutorial's and the MLX
conv3d pull request's layers, the weights' fan-in scaling, the draw order and
the value ranges.  Every parity test and the benchmark take their inputs from
here, so a wrong shape or seed would silently change what is measured."""
from __future__ import annotations

import math

import pytest
import torch

import workloads as WL

# name: (N, D, H, W, C, O, k, stride, pad, dtype, seed, fan_in)
PUBLISHED = {
    "conv2d_f16_n1_56x56_c64_o64_k3": (1, 1, 56, 56, 64, 64, (1, 3, 3), (1, 1, 1), (0, 1, 1), "f16", 0, 576),
    "stem_bf16_n32_224x224_c3_o64_k7s2": (32, 1, 224, 224, 3, 64, (1, 7, 7), (1, 2, 2), (0, 3, 3), "bf16", 1, 147),
    "conv2d_bf16_n64_56x56_c256_o256_k3": (64, 1, 56, 56, 256, 256, (1, 3, 3), (1, 1, 1), (0, 1, 1), "bf16", 2,
                                           2304),
    "conv3d_f16_n4_32c_c64_o128_k333s1": (4, 32, 32, 32, 64, 128, (3, 3, 3), (1, 1, 1), (1, 1, 1), "f16", 3, 1728),
    "conv3d_f16_n4_32c_c64_o128_k333s2": (4, 32, 32, 32, 64, 128, (3, 3, 3), (2, 2, 2), (1, 1, 1), "f16", 3, 1728),
    "conv3d_f16_n4_32c_c64_o128_k311": (4, 32, 32, 32, 64, 128, (3, 1, 1), (1, 1, 1), (1, 0, 0), "f16", 3, 192),
    "conv3d_f16_n4_32c_c64_o128_k133": (4, 32, 32, 32, 64, 128, (1, 3, 3), (1, 1, 1), (0, 1, 1), "f16", 3, 576),
    "conv3d_f16_n2_64c_c32_o64_k333": (2, 64, 64, 64, 32, 64, (3, 3, 3), (1, 1, 1), (1, 1, 1), "f16", 3, 864),
    "conv3d_f16_n1_64c_c64_o128_k333": (1, 64, 64, 64, 64, 128, (3, 3, 3), (1, 1, 1), (1, 1, 1), "f16", 3, 1728),
}
for _dt in ("f16", "f32"):
    for (_S, _C, _O, _fan) in ((16, 21, 21, 567), (16, 65, 65, 1755), (32, 65, 65, 1755), (16, 3, 32, 81)):
        PUBLISHED[f"conv3d_{_dt}_n4_{_S}c_c{_C}_o{_O}_k333"] = (4, _S, _S, _S, _C, _O, (3, 3, 3), (1, 1, 1),
                                                                 (1, 1, 1), _dt, 4, _fan)


@pytest.mark.parametrize("name", sorted(PUBLISHED))
def test_workload_matches_the_published_layer(name):
    N, D, H, W, C, O, k, s, p, dt, seed, fan = PUBLISHED[name]
    wl = WL.WORKLOADS[name]
    assert (wl.N, wl.D, wl.H, wl.W, wl.C, wl.O) == (N, D, H, W, C, O)
    assert (wl.k, wl.stride, wl.pad, wl.dil, wl.groups) == (k, s, p, (1, 1, 1), 1)
    assert (wl.dtype, wl.seed, wl.transpose, wl.wgrad) == (dt, seed, False, False)
    assert WL.fan_in(wl) == fan
    assert wl.x_shape == (N, D, H, W, C) and wl.w_shape == (O, *k, C)


def test_every_forward_workload_is_published_and_the_headline_is_the_3x3_layer():
    fwd = {n for n, wl in WL.WORKLOADS.items() if not (wl.transpose or wl.wgrad or wl.groups > 1)}
    assert fwd == set(PUBLISHED)
    assert WL.HEADLINE == "conv2d_bf16_n64_56x56_c256_o256_k3"


def test_extra_workloads_fan_in():
    dw = WL.WORKLOADS["dwconv_f16_n32_112x112_c128_k3"]
    assert dw.groups == dw.C == dw.O == 128 and WL.fan_in(dw) == 9 and dw.w_shape == (128, 1, 3, 3, 1)
    ct = WL.WORKLOADS["convT_bf16_n16_56x56_c256_o128_k4s2"]
    # a 4x4 filter at stride 2 reaches each output through 2 x 2 taps
    assert ct.transpose and WL.fan_in(ct) == 256 * 4 and ct.w_shape == (256, 1, 4, 4, 128)


@pytest.mark.parametrize("name", ["conv2d_bf16_n64_56x56_c256_o256_k3", "conv3d_f32_n4_16c_c65_o65_k333",
                                  "stem_bf16_n32_224x224_c3_o64_k7s2"])
def test_recipe_draws(name):
    wl = WL.WORKLOADS[name].with_(N=1)
    x, w = WL.make_inputs(wl)
    assert x.dtype == WL.TORCH_DTYPE[wl.dtype] and x.is_contiguous() and tuple(x.shape) == wl.x_shape
    assert w.dtype == x.dtype and w.is_contiguous() and tuple(w.shape) == wl.w_shape
    xf, wf = x.double(), w.double()
    assert xf.min() >= -1.0 and xf.max() <= 1.0
    assert abs(float(xf.mean())) < 0.02 and abs(float(xf.var()) - 1 / 3) < 0.01  # U[-1, 1): variance 1/3
    sigma = 1.0 / math.sqrt(WL.fan_in(wl))
    assert abs(float(wf.std()) / sigma - 1.0) < 0.06 and abs(float(wf.mean())) < 0.1 * sigma
    # x first, then w, from one generator seeded with the workload's seed
    g = torch.Generator().manual_seed(wl.seed)
    x32 = torch.rand(wl.x_shape, generator=g) * 2.0 - 1.0
    w32 = torch.randn(wl.w_shape, generator=g) * sigma
    assert torch.equal(x, x32.to(x.dtype)) and torch.equal(w, w32.to(w.dtype))


def test_recipe_is_deterministic_and_seed_dependent():
    wl = WL.case(2, 3, 5, 6, 7, 9, (1, 3, 3), pad=(0, 1, 1), dtype="bf16", seed=11)
    a = WL.make_inputs(wl)
    b = WL.make_inputs(wl)
    c = WL.make_inputs(wl, seed=12)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert not torch.equal(a[0], c[0]) and not torch.equal(a[1], c[1])
