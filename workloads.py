"""Seeded synthetic inputs for the convolution forward pass.

This module is shared by the CUDA path's callers (bench, smoke check) and by
the tests that feed the oracle.  It holds NO convolution arithmetic: only the
workload shapes and a seeded random generator.

Recipe (one reading, applied everywhere): a fresh ``torch.Generator`` seeded
with the workload's seed draws x first, then w, in float32, directly in their
storage shapes (x NDHWC [N, D, H, W, C]; w [O, kD, kH, kW, C/groups]):
x = U[-1, 1) as ``rand * 2 - 1``; w = N(0, sigma^2) as ``randn * sigma`` with
sigma^2 = 1 / fan_in, fan_in = (C/groups) * kD * kH * kW.  The float32 draws
are then rounded to nearest-even in the workload's dtype (or kept for f32).

The shapes are those of the "Convolutions" tutorial (ResNet-50 stem,
3x3 256->256 layer at 56x56) and of the MLX conv3d pull request's benchmark
tables (the 3-D shapes and the unaligned-channel shapes).  No dataset is used:
uniform random activations stand in for images.
"""
from __future__ import annotations

import dataclasses
import math

import torch

TORCH_DTYPE = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int
    D: int
    H: int
    W: int
    C: int
    O: int
    k: tuple            # (kD, kH, kW)
    stride: tuple       # (sd, sh, sw)
    pad: tuple          # (pd, ph, pw)
    dil: tuple = (1, 1, 1)
    groups: int = 1
    dtype: str = "f16"
    seed: int = 0
    transpose: bool = False      # transposed ("upsampling") convolution: x has C channels, y has O
    out_pad: tuple = (0, 0, 0)   # its output padding
    wgrad: bool = False          # the weight gradient of the forward pass (inputs x and dy)

    @property
    def x_shape(self):
        return (self.N, self.D, self.H, self.W, self.C)

    @property
    def w_shape(self):
        # forward: [O, k, C/groups]; transposed: [C, k, O/groups] (the forward layout with O = C)
        if self.transpose:
            return (self.C, *self.k, self.O // self.groups)
        return (self.O, *self.k, self.C // self.groups)

    def with_(self, **kw):
        return dataclasses.replace(self, **kw)


def _c3(name, N, D, H, W, C, O, k, s, p, dtype, seed):
    return Workload(name, N, D, H, W, C, O, tuple(k), tuple(s), tuple(p), dtype=dtype, seed=seed)


# The five workload families, in order.  2-D convolutions are D = kD = 1.
WORKLOADS = {
    # small 2-D case: N=1, 56x56, 64->64, 3x3/1/1, fp16, seed 0
    "conv2d_f16_n1_56x56_c64_o64_k3": _c3("conv2d_f16_n1_56x56_c64_o64_k3",
                                          1, 1, 56, 56, 64, 64, (1, 3, 3), (1, 1, 1), (0, 1, 1), "f16", 0),
    # ResNet-50 stem: N=32, 224x224, 3->64, 7x7/2/3 -> 112x112, bf16, seed 1
    "stem_bf16_n32_224x224_c3_o64_k7s2": _c3("stem_bf16_n32_224x224_c3_o64_k7s2",
                                             32, 1, 224, 224, 3, 64, (1, 7, 7), (1, 2, 2), (0, 3, 3), "bf16", 1),
    # 3x3 256->256 at 56x56, N=64, bf16, seed 2 (3.7 GFLOP per image)
    "conv2d_bf16_n64_56x56_c256_o256_k3": _c3("conv2d_bf16_n64_56x56_c256_o256_k3",
                                              64, 1, 56, 56, 256, 256, (1, 3, 3), (1, 1, 1), (0, 1, 1), "bf16", 2),
    # conv3d fp16 sweep, seed 3
    "conv3d_f16_n4_32c_c64_o128_k333s1": _c3("conv3d_f16_n4_32c_c64_o128_k333s1",
                                             4, 32, 32, 32, 64, 128, (3, 3, 3), (1, 1, 1), (1, 1, 1), "f16", 3),
    "conv3d_f16_n4_32c_c64_o128_k333s2": _c3("conv3d_f16_n4_32c_c64_o128_k333s2",
                                             4, 32, 32, 32, 64, 128, (3, 3, 3), (2, 2, 2), (1, 1, 1), "f16", 3),
    "conv3d_f16_n4_32c_c64_o128_k311": _c3("conv3d_f16_n4_32c_c64_o128_k311",
                                           4, 32, 32, 32, 64, 128, (3, 1, 1), (1, 1, 1), (1, 0, 0), "f16", 3),
    "conv3d_f16_n4_32c_c64_o128_k133": _c3("conv3d_f16_n4_32c_c64_o128_k133",
                                           4, 32, 32, 32, 64, 128, (1, 3, 3), (1, 1, 1), (0, 1, 1), "f16", 3),
    "conv3d_f16_n2_64c_c32_o64_k333": _c3("conv3d_f16_n2_64c_c32_o64_k333",
                                          2, 64, 64, 64, 32, 64, (3, 3, 3), (1, 1, 1), (1, 1, 1), "f16", 3),
    "conv3d_f16_n1_64c_c64_o128_k333": _c3("conv3d_f16_n1_64c_c64_o128_k333",
                                           1, 64, 64, 64, 64, 128, (3, 3, 3), (1, 1, 1), (1, 1, 1), "f16", 3),
}
# conv3d with unaligned channel counts, fp16 and fp32, 3x3x3/1/1, seed 4
for _dt in ("f16", "f32"):
    for (_N, _S, _C, _O) in ((4, 16, 21, 21), (4, 16, 65, 65), (4, 32, 65, 65), (4, 16, 3, 32)):
        _n = f"conv3d_{_dt}_n{_N}_{_S}c_c{_C}_o{_O}_k333"
        WORKLOADS[_n] = _c3(_n, _N, _S, _S, _S, _C, _O, (3, 3, 3), (1, 1, 1), (1, 1, 1), _dt, 4)

# Depthwise 3x3/1/1 (groups = C = O = 128) at 112x112, N=32, fp16, seed 5: the
# tutorial's variants table lists depthwise layers as memory-bound work for
# direct kernels; MobileNet-style block shape.
WORKLOADS["dwconv_f16_n32_112x112_c128_k3"] = Workload(
    "dwconv_f16_n32_112x112_c128_k3", 32, 1, 112, 112, 128, 128, (1, 3, 3), (1, 1, 1), (0, 1, 1),
    groups=128, dtype="f16", seed=5)

# Transposed convolution 4x4/2/1 (a decoder's 2x upsampling layer), 256 -> 128
# channels, 56x56 -> 112x112, N=16, bf16, seed 6: the tutorial's variants
# table names transposed convolutions for decoders and diffusion models.
WORKLOADS["convT_bf16_n16_56x56_c256_o128_k4s2"] = Workload(
    "convT_bf16_n16_56x56_c256_o128_k4s2", 16, 1, 56, 56, 256, 128, (1, 4, 4), (1, 2, 2), (0, 1, 1),
    dtype="bf16", seed=6, transpose=True)

# Weight gradient of the 3x3 256->256 layer at 56x56, N=64, bf16, seed 7 (the
# headline forward layer's third pass).
WORKLOADS["wgrad_bf16_n64_56x56_c256_o256_k3"] = Workload(
    "wgrad_bf16_n64_56x56_c256_o256_k3", 64, 1, 56, 56, 256, 256, (1, 3, 3), (1, 1, 1), (0, 1, 1),
    dtype="bf16", seed=7, wgrad=True)

# Name of the workload the benchmark times by default: the tutorial's
# arithmetic-intensity example (3x3, 256->256, 56x56) at batch 64.
HEADLINE = "conv2d_bf16_n64_56x56_c256_o256_k3"


def fan_in(wl: Workload) -> int:
    """Inputs summed into one output: C/groups x taps (forward), or the
    transposed pass's input channels per group x the taps that reach an
    output (taps / stride per dimension, rounded up)."""
    if wl.transpose:
        reach = 1
        for k, s in zip(wl.k, wl.stride):
            reach *= -(-k // s)
        return (wl.C // wl.groups) * reach
    return (wl.C // wl.groups) * wl.k[0] * wl.k[1] * wl.k[2]


def make_inputs(wl: Workload, seed: int | None = None):
    """Seeded host tensors (x, w) in the workload's dtype, contiguous NDHWC / O kD kH kW Cg."""
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed if seed is None else seed)
    x = torch.rand(wl.x_shape, generator=g, dtype=torch.float32) * 2.0 - 1.0
    sigma = 1.0 / math.sqrt(fan_in(wl))
    w = torch.randn(wl.w_shape, generator=g, dtype=torch.float32) * sigma
    dt = TORCH_DTYPE[wl.dtype]
    return x.to(dt).contiguous(), w.to(dt).contiguous()


def make_wgrad_inputs(wl: Workload, dy_shape, seed: int | None = None):
    """Seeded host tensors (x, dy) for a weight-gradient workload: x as above,
    then dy = U[-1, 1) in the forward output's shape `dy_shape` (computed by
    the caller), both rounded to the workload's dtype."""
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed if seed is None else seed)
    x = torch.rand(wl.x_shape, generator=g, dtype=torch.float32) * 2.0 - 1.0
    dy = torch.rand(tuple(dy_shape), generator=g, dtype=torch.float32) * 2.0 - 1.0
    dt = TORCH_DTYPE[wl.dtype]
    return x.to(dt).contiguous(), dy.to(dt).contiguous()


def case(N, D, H, W, C, O, k, stride=(1, 1, 1), pad=(0, 0, 0), dil=(1, 1, 1), groups=1,
         dtype="f16", seed=0, name="case") -> Workload:
    """An ad-hoc workload (tests): same recipe, any geometry."""
    return Workload(name, N, D, H, W, C, O, tuple(k), tuple(stride), tuple(pad), tuple(dil),
                    groups, dtype, seed)
