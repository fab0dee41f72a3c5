"""The C ABI's host side (no GPU needed): symbols, extents, argument checks, planning."""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "conv_fwd.h")


@pytest.fixture(scope="module")
def C():
    from implicit_gemm_convolution_conv2d_b200 import _build
    _build.build()
    import implicit_gemm_convolution_conv2d_b200 as mod
    mod.lib()
    return mod


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(conv_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("conv_fwd", "conv_fwd_variant", "conv_fwd_host", "conv_out_dims", "conv_plan",
              "conv_last_status", "conv_strerror", "conv_version", "conv_fwd_ex", "conv_out_dims_ex",
              "conv_plan_ex"):
        assert n in names, n


def test_library_exports_every_declared_symbol(C):
    nm = subprocess.run(["nm", "-D", "--defined-only", C.LIB_PATH], capture_output=True, text=True, check=True)
    exported = {ln.split()[-1] for ln in nm.stdout.splitlines() if ln.strip()}
    for n in declared_functions():
        assert n in exported, f"{n} declared in conv_fwd.h but not exported"
        assert hasattr(C.lib(), n)


def test_out_dims_match_oracle(C):
    rng = np.random.default_rng(0)
    n = 0
    while n < 400:
        dims = rng.integers(1, 40, 3)
        k = rng.integers(1, 8, 3)
        s = rng.integers(1, 4, 3)
        p = rng.integers(0, 4, 3)
        d = rng.integers(1, 4, 3)
        try:
            ref = oracle.out_dims(*dims, *k, s, p, d)
        except ValueError:
            with pytest.raises(C.ConvError):
                C.out_dims(*dims, *k, s, p, d)
            continue
        assert C.out_dims(*dims, *k, s, p, d) == ref
        n += 1


def test_side_padding_out_dims_match_oracle(C):
    rng = np.random.default_rng(1)
    n = 0
    while n < 300:
        dims = rng.integers(1, 30, 3)
        k = rng.integers(1, 6, 3)
        s = rng.integers(1, 4, 3)
        pl = rng.integers(0, 4, 3)
        ph = rng.integers(0, 4, 3)
        d = rng.integers(1, 3, 3)
        try:
            ref = oracle.out_dims(*dims, *k, s, pl, d, pad_hi=ph)
        except ValueError:
            with pytest.raises(C.ConvError):
                C.out_dims(*dims, *k, s, pl, d, ph)
            continue
        assert C.out_dims(*dims, *k, s, pl, d, ph) == ref
        n += 1


def test_flip_and_side_padding_arguments(C):
    L = C.lib()
    i3 = lambda *v: (ctypes.c_int * 3)(*v)
    s, p, d = i3(1, 1, 1), i3(0, 1, 1), i3(1, 1, 1)
    X, Wt, Y = 0x10000, 0x20000, 0x40000       # never dereferenced: checks come first
    ex = lambda ph, flip, dt=1, v=-1: L.conv_fwd_ex(X, Wt, Y, 1, 1, 4, 4, 16, 16, 1, 3, 3, s, p, ph, d, 1, flip,
                                                    dt, v, None)
    assert ex(i3(0, -1, 0), 0) == -1           # negative high-side pad
    assert ex(i3(0, 1, 1), 2) == -1            # flip is 0 or 1
    assert ex(i3(0, 1, 1), 0, 9) == -2         # dtype
    assert ex(i3(0, 1, 1), 0, 1, 14) == -1     # unknown variant
    assert ex(i3(0, 1, 1), 0, 1, 12) == -7     # the transposed-convolution phase kernel: not a forward variant
    # flip keeps the phase-packed kernel (its B rows are built from the mirrored filter)
    stem = (2, 1, 32, 32, 3, 64, (1, 7, 7), (1, 2, 2), (0, 3, 3), (1, 1, 1), 1, "bf16")
    assert C.plan(*stem)[0] == C.VARIANT_TC_PHASE
    assert C.plan(*stem, flip=1)[0] == C.VARIANT_TC_PHASE
    # depth padding on one side makes a 2-D-looking problem 3-D (Do = 2)
    assert C.out_dims(1, 8, 8, 1, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1), (1, 1, 1)) == (2, 8, 8)


def test_out_dims_pinned_values(C):
    # tutorial: 224x224, 7x7, stride 2 -> 112x112 (pad 3)
    assert C.out_dims(1, 224, 224, 1, 7, 7, (1, 2, 2), (0, 3, 3), (1, 1, 1)) == (1, 112, 112)


def test_invalid_arguments_rejected_on_host(C):
    L = C.lib()
    i3 = lambda *v: (ctypes.c_int * 3)(*v)
    s, p, d = i3(1, 1, 1), i3(0, 1, 1), i3(1, 1, 1)
    X, Wt, Y = 0x10000, 0x20000, 0x40000       # never dereferenced: checks come first
    call = lambda *a: L.conv_fwd(*a)
    # non-positive sizes, empty batch
    assert call(X, Wt, Y, 0, 1, 4, 4, 16, 16, 1, 3, 3, s, p, d, 1, 1, None) == -1
    assert call(X, Wt, Y, 1, 1, 4, 4, 0, 16, 1, 3, 3, s, p, d, 1, 1, None) == -1
    # C % groups, O % groups
    assert call(X, Wt, Y, 1, 1, 4, 4, 16, 16, 1, 3, 3, s, p, d, 3, 1, None) == -1
    assert call(X, Wt, Y, 1, 1, 4, 4, 16, 18, 1, 3, 3, s, p, d, 4, 1, None) == -1
    # empty output (kernel larger than padded input)
    assert call(X, Wt, Y, 1, 1, 2, 2, 16, 16, 1, 5, 5, s, i3(0, 0, 0), d, 1, 1, None) == -1
    # bad stride / dilation / pad
    assert call(X, Wt, Y, 1, 1, 4, 4, 16, 16, 1, 3, 3, i3(1, 0, 1), p, d, 1, 1, None) == -1
    assert call(X, Wt, Y, 1, 1, 4, 4, 16, 16, 1, 3, 3, s, i3(0, -1, 1), d, 1, 1, None) == -1
    assert call(X, Wt, Y, 1, 1, 4, 4, 16, 16, 1, 3, 3, s, p, i3(1, 1, 0), 1, 1, None) == -1
    # dtype
    assert call(X, Wt, Y, 1, 1, 4, 4, 16, 16, 1, 3, 3, s, p, d, 1, 9, None) == -2
    # NULL, misaligned, aliasing
    assert call(0, Wt, Y, 1, 1, 4, 4, 16, 16, 1, 3, 3, s, p, d, 1, 1, None) == -1
    assert call(X + 8, Wt, Y, 1, 1, 4, 4, 16, 16, 1, 3, 3, s, p, d, 1, 1, None) == -3
    assert call(X, Wt, X + 16, 1, 1, 4, 4, 16, 16, 1, 3, 3, s, p, d, 1, 1, None) == -4
    assert call(X, Wt, Wt, 1, 1, 4, 4, 16, 16, 1, 3, 3, s, p, d, 1, 1, None) == -4
    # overflow of the element count
    big = 1 << 30
    assert call(X, Wt, Y, big, big, 4, 4, 16, 16, 1, 3, 3, s, p, d, 1, 1, None) == -1
    # unknown variant
    assert L.conv_fwd_variant(X, Wt, Y, 1, 1, 4, 4, 16, 16, 1, 3, 3, s, p, d, 1, 1, 14, None) == -1
    assert L.conv_fwd_variant(X, Wt, Y, 1, 1, 4, 4, 16, 16, 1, 3, 3, s, p, d, 1, 1, -2, None) == -1


def test_strerror_covers_codes(C):
    for code in range(0, -9, -1):
        assert C.strerror(code) and C.strerror(code) != "unknown error"
    assert C.strerror(-99) == "unknown error"


def test_variant_plan(C):
    plan = lambda *a, **k: C.plan(*a, **k)
    v, bn, st, _ = plan(64, 1, 56, 56, 256, 256, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 1, "bf16")
    assert v == C.VARIANT_TC_TMA_PAIR and bn == 256 and st >= 2
    v, bn, _, _ = plan(1, 1, 56, 56, 64, 64, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 1, "f16")
    assert v == C.VARIANT_TC_TMA and bn == 64
    v, bn, _, _ = plan(4, 32, 32, 32, 64, 128, (3, 3, 3), (2, 2, 2), (1, 1, 1), (1, 1, 1), 1, "f16")
    assert v in (C.VARIANT_TC_TMA, C.VARIANT_TC_TMA_PAIR) and bn == 128
    # 128 output channels, stride 1, 64-channel chunks, kH >= 2: the transposed halo kernel
    v, bn, st, _ = plan(4, 32, 32, 32, 64, 128, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), 1, "f16")
    assert v == C.VARIANT_TC_HALO_T and bn == 256 and st >= 2
    # 64 output channels, 32-channel chunks: the transposed halo kernel with M = 64,
    # all weights resident in shared memory (a single pipeline stage)
    v, bn, st, _ = plan(2, 64, 64, 64, 32, 64, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), 1, "f16")
    assert v == C.VARIANT_TC_HALO_T and bn == 256 and st == 1
    # 1x3x3 64 -> 128: resident weights too; two groups: streamed weights
    assert plan(4, 32, 32, 32, 64, 128, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 1, "f16")[2] == 1
    assert plan(2, 1, 9, 9, 128, 256, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 2, "f16",
                C.VARIANT_TC_HALO_T)[2] >= 2
    # ... with kH = 1 (no strip reuse) and a short reduction (K = 192): the plain
    # single-CTA im2col kernel; with a longer one (K = 5 x 128): the transposed im2col kernel
    v, bn, _, _ = plan(4, 32, 32, 32, 64, 128, (3, 1, 1), (1, 1, 1), (1, 0, 0), (1, 1, 1), 1, "f16")
    assert v == C.VARIANT_TC_TMA and bn == 128
    v, bn, _, _ = plan(4, 32, 32, 32, 128, 128, (5, 1, 1), (1, 1, 1), (2, 0, 0), (1, 1, 1), 1, "f16")
    assert v == C.VARIANT_TC_TMA_T and bn == 256
    # block height adapts to Ho: 56 rows -> blocks of 28 (MMA N = 224)
    v, bn, _, _ = plan(64, 1, 56, 56, 256, 256, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 1, "bf16",
                       C.VARIANT_TC_HALO_T_PAIR)
    assert v == C.VARIANT_TC_HALO_T_PAIR and bn == 224
    # the stem: 3 input channels -> phase packing, 4 pixels x 64 channels per GEMM row
    v, bn, st, _ = plan(32, 1, 224, 224, 3, 64, (1, 7, 7), (1, 2, 2), (0, 3, 3), (1, 1, 1), 1, "bf16")
    assert v == C.VARIANT_TC_PHASE and bn == 256 and st >= 2
    # ... unless a condition fails (W*C*2 not a multiple of 16; Wo not a multiple of P)
    assert plan(2, 1, 16, 15, 3, 64, (1, 7, 7), (1, 2, 2), (0, 3, 3), (1, 1, 1), 1, "bf16")[0] == C.VARIANT_TC_GATHER
    assert plan(2, 1, 16, 24, 3, 64, (1, 7, 7), (1, 3, 3), (0, 3, 3), (1, 1, 1), 1, "bf16")[0] == C.VARIANT_TC_GATHER
    # unaligned channels at stride 1: the staged kernel, 16 x 8 output blocks (Ho = 16)
    v, bn, st, _ = plan(4, 16, 16, 16, 65, 65, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), 1, "f16")
    assert v == C.VARIANT_TC_STAGED and bn == 128 and st >= 2
    # (4,32^3,65)->65: 32 x 8 blocks, two slots beside the staged input and weight rows
    v, bn, st, ct = plan(4, 32, 32, 32, 65, 65, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), 1, "f16")
    assert v == C.VARIANT_TC_STAGED and bn == 256 and st == 2 and ct == 148
    # 21 channels: the staged kernel too; 3 channels: the gather kernel (faster there)
    assert plan(4, 16, 16, 16, 21, 21, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), 1, "f16")[0] == C.VARIANT_TC_STAGED
    assert plan(4, 16, 16, 16, 3, 32, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), 1, "f16")[0] == C.VARIANT_TC_GATHER
    # the staged kernel on request: Ho = 9 takes 12-row blocks (the fewest padded rows, ties to
    # the taller block); stride 2, O > 128 and two groups are refused
    assert plan(1, 1, 9, 9, 3, 8, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 1, "bf16",
                C.VARIANT_TC_STAGED)[:2] == (C.VARIANT_TC_STAGED, 96)
    for args in [(1, 1, 16, 16, 21, 21, (1, 3, 3), (1, 2, 2), (0, 1, 1), (1, 1, 1), 1, "f16"),
                 (1, 1, 16, 16, 21, 130, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 1, "f16"),
                 (1, 1, 16, 16, 42, 42, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 2, "f16")]:
        with pytest.raises(C.ConvError) as e:
            plan(*args, C.VARIANT_TC_STAGED)
        assert e.value.code == -7
    # ... but the gather kernel past its conditions (O > 128; groups; flip)
    v, bn, _, _ = plan(4, 16, 16, 16, 65, 130, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), 1, "f16")
    assert v == C.VARIANT_TC_GATHER
    assert plan(2, 4, 8, 8, 42, 42, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), 2, "f16")[0] == C.VARIANT_TC_GATHER
    assert plan(2, 4, 8, 8, 21, 21, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), 1, "f16",
                flip=1)[0] == C.VARIANT_TC_GATHER
    v, _, _, _ = plan(4, 16, 16, 16, 65, 65, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), 1, "f32")
    assert v == C.VARIANT_SIMT
    # 3-D with pad beyond the rank-5 im2col corner range goes to the staged kernel
    v, _, _, _ = plan(1, 40, 8, 8, 64, 64, (3, 3, 3), (1, 1, 1), (17, 1, 1), (1, 1, 1), 1, "f16")
    assert v == C.VARIANT_TC_STAGED
    # channel chunks of 32 and 16
    assert plan(2, 64, 64, 64, 32, 256, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), 1, "f16")[0] == C.VARIANT_TC_TMA_PAIR
    assert plan(2, 64, 64, 64, 32, 384, (1, 1, 1), (1, 1, 1), (0, 0, 0), (1, 1, 1), 1, "f16")[0] == C.VARIANT_TC_TMA
    assert plan(2, 64, 64, 64, 128, 384, (3, 1, 1), (1, 1, 1), (1, 0, 0), (1, 1, 1), 1, "f16")[0] == \
        C.VARIANT_TC_TMA_T
    assert plan(1, 1, 9, 9, 48, 96, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 3, "f16")[0] == C.VARIANT_TC_TMA
    assert plan(1, 1, 9, 9, 128, 64, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 2, "f16")[0] == C.VARIANT_TC_TMA


def test_explicit_variant_plan(C):
    """conv_plan_variant resolves an explicit variant or refuses it by the
    same rule conv_fwd_variant applies."""
    g3 = (64, 1, 56, 56, 256, 256, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 1)
    for name in ("TC_TMA", "TC_TMA_PAIR", "TC_GATHER", "TC_HALO", "TC_HALO_PAIR", "TC_TMA_T", "TC_HALO_T",
                 "TC_HALO_T_PAIR", "SIMT"):
        v = getattr(C, "VARIANT_" + name)
        assert C.plan(*g3, "bf16", v)[0] == v
    assert C.plan(*g3, "bf16", C.VARIANT_AUTO) == C.plan(*g3, "bf16")
    # C = 3: no im2col tensor map, no halo
    stem = (32, 1, 224, 224, 3, 64, (1, 7, 7), (1, 2, 2), (0, 3, 3), (1, 1, 1), 1)
    for name in ("TC_TMA", "TC_TMA_PAIR", "TC_HALO", "TC_HALO_PAIR"):
        with pytest.raises(C.ConvError) as e:
            C.plan(*stem, "bf16", getattr(C, "VARIANT_" + name))
        assert e.value.code == -7
    assert C.plan(*stem, "bf16", C.VARIANT_TC_PHASE)[0] == C.VARIANT_TC_PHASE
    # phase packing needs C small enough that P*O <= 256
    with pytest.raises(C.ConvError) as e:
        C.plan(*g3, "bf16", C.VARIANT_TC_PHASE)
    assert e.value.code == -7
    # tensor-core variants need f16/bf16
    with pytest.raises(C.ConvError) as e:
        C.plan(*g3, "f32", C.VARIANT_TC_TMA)
    assert e.value.code == -7
    # depthwise (groups = C = O) with 16-byte channel vectors, any type.  The
    # direct form computes 8 channels per thread for 16-bit types, 4 for
    # f32; the TMA-staged form 4 channels of several pixels.  The TMA-staged form
    # runs persistent CTAs (at most two per SM for each channel tile, the
    # planner assumes 148 SMs without a device) over a ring of 2-4 slabs; the
    # direct form launches one block per 256 (channel vector, pixel group) tasks
    dw = (32, 1, 112, 112, 128, 128, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 128)
    for dt, vec in (("f16", 8), ("bf16", 8), ("f32", 4)):
        v, bn, stages, ctas = C.plan(*dw, dt)
        assert (v, bn) == (C.VARIANT_DEPTHWISE, 4) and 2 <= stages <= 4 and ctas <= 2 * 148
        v, bn, stages, ctas = C.plan(*dw, dt, C.VARIANT_DEPTHWISE_DIRECT)
        assert (v, bn, stages) == (C.VARIANT_DEPTHWISE_DIRECT, vec, 1)
        assert ctas == -(-32 * 112 * 28 * (128 // vec) // 256)
    dw4 = (2, 1, 7, 9, 4, 4, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 4)
    assert C.plan(*dw4, "f32")[0] == C.VARIANT_DEPTHWISE
    assert C.plan(*dw4, "f16")[0] != C.VARIANT_DEPTHWISE
    for args in ((*dw4, "f16"), (*g3, "bf16")):
        for v in (C.VARIANT_DEPTHWISE, C.VARIANT_DEPTHWISE_DIRECT):
            with pytest.raises(C.ConvError) as e:
                C.plan(*args, v)
            assert e.value.code == -7
    # a slab taller than one TMA box allows (5 rows at height dilation 70 span
    # 281 > 256 input rows): DEPTHWISE runs the direct form, one stage
    tall = (1, 1, 200, 32, 16, 16, (1, 5, 3), (1, 1, 1), (0, 140, 1), (1, 70, 1), 16)
    assert C.plan(*tall, "f16")[:3] == (C.VARIANT_DEPTHWISE, 8, 1)  # the direct form's 8 channels
    with pytest.raises(C.ConvError) as e:
        C.plan(*g3, "bf16", 14)
    assert e.value.code == -1
    with pytest.raises(C.ConvError) as e:   # the transposed-convolution phase kernel
        C.plan(*g3, "bf16", C.VARIANT_TC_TMA_PHASES)
    assert e.value.code == -7


def test_transpose_extents_and_plans(C):
    """Transposed-convolution extents agree with the oracle's; the planner runs
    it on the TMA-fed phase kernel where that fits (16-bit, dilation 1,
    64-/128-channel multiples), else the gather kernel (16-bit) or the FP32
    kernel, and refuses the forward-only variants."""
    import oracle
    for D, H, W, k, s, p, op, d in ((3, 4, 5, (1, 3, 3), (1, 2, 2), (0, 1, 1), (0, 1, 1), (1, 1, 1)),
                                    (5, 6, 7, (3, 3, 3), (2, 1, 2), (1, 1, 0), (1, 0, 1), (1, 2, 1)),
                                    (1, 28, 28, (1, 4, 4), (1, 2, 2), (0, 1, 1), (0, 0, 0), (1, 1, 1))):
        assert C.transpose_out_dims(D, H, W, *k, s, p, op, d) == oracle.convT_out_dims(D, H, W, *k, s, p, op, d)
    g = (2, 1, 28, 28, 256, 128, (1, 4, 4), (1, 2, 2), (0, 1, 1), (0, 0, 0), (1, 1, 1), 1)
    assert C.transpose_plan(*g, "f16")[0] == C.VARIANT_TC_TMA_PHASES
    assert C.transpose_plan(*g, "f16", C.VARIANT_TC_GATHER)[0] == C.VARIANT_TC_GATHER
    assert C.transpose_plan(*g, "f32")[0] == C.VARIANT_SIMT
    # dilation 2, or 32 input channels, or 64 output channels: the gather kernel
    g_dil = (2, 1, 28, 28, 256, 128, (1, 3, 3), (1, 2, 2), (0, 1, 1), (0, 1, 1), (1, 2, 2), 1)
    g_c32 = (2, 1, 28, 28, 32, 128, (1, 4, 4), (1, 2, 2), (0, 1, 1), (0, 0, 0), (1, 1, 1), 1)
    g_o64 = (2, 1, 28, 28, 256, 64, (1, 4, 4), (1, 2, 2), (0, 1, 1), (0, 0, 0), (1, 1, 1), 1)
    for gg in (g_dil, g_c32, g_o64):
        assert C.transpose_plan(*gg, "f16")[0] == C.VARIANT_TC_GATHER
        with pytest.raises(C.ConvError) as e:
            C.transpose_plan(*gg, "f16", C.VARIANT_TC_TMA_PHASES)
        assert e.value.code == -7
    for v in (C.VARIANT_TC_TMA, C.VARIANT_TC_TMA_PAIR, C.VARIANT_TC_HALO_T, C.VARIANT_TC_PHASE, C.VARIANT_DEPTHWISE):
        with pytest.raises(C.ConvError) as e:
            C.transpose_plan(*g, "f16", v)
        assert e.value.code == -7
    # padding beyond d*(k-1) (a crop of the dilated sum) is not supported
    with pytest.raises(C.ConvError) as e:
        C.transpose_plan(1, 1, 8, 8, 16, 16, (1, 3, 3), (1, 2, 2), (0, 3, 3), (0, 0, 0), (1, 1, 1), 1, "f16")
    assert e.value.code == -7
    # output padding must stay below max(stride, dilation)
    with pytest.raises(C.ConvError):
        C.transpose_out_dims(1, 8, 8, 1, 3, 3, (1, 2, 2), (0, 1, 1), (0, 2, 2), (1, 1, 1))


def test_wgrad_workspace_and_arguments(C):
    """The weight gradient's fp32 workspace: one slice of O x taps x C/G floats
    per range of the split pixel reduction, for every type; the split depends
    on the shape alone; bad shapes are refused on the host."""
    g = (2, 1, 9, 8, 16, 24, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 1)
    # 144 pixels: too few for a second range
    for dt in ("bf16", "f16", "f32"):
        assert C.wgrad_workspace_size(*g, dt) == 24 * 9 * 16 * 4
    assert C.wgrad_workspace_size(2, 1, 9, 8, 16, 24, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 4, "bf16") == \
        24 * 9 * 4 * 4
    # the 3x3 256->256 layer at batch 64.  16-bit: the tensor-core path, 9 tiles of 256 x 256
    # columns, so 8 ranges for the 74 CTA pairs of a 148-SM B200; f32: the FP32 path, 144 tiles
    # of 64 x 64, so 3 ranges for ~296 blocks
    geo = (64, 1, 56, 56, 256, 256, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 1)
    slice_bytes = 256 * 9 * 256 * 4
    assert C.wgrad_workspace_size(*geo, "bf16") == 8 * slice_bytes
    assert C.wgrad_workspace_size(*geo, "f32") == 3 * slice_bytes
    with pytest.raises(C.ConvError) as e:   # C not divisible by groups
        C.wgrad_workspace_size(2, 1, 9, 8, 16, 24, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 5, "bf16")
    assert e.value.code == -1
    with pytest.raises(C.ConvError) as e:   # a kernel larger than the padded input
        C.wgrad_workspace_size(1, 1, 2, 2, 8, 8, (1, 5, 5), (1, 1, 1), (0, 0, 0), (1, 1, 1), 1, "f32")
    assert e.value.code == -1


def test_planner_on_random_geometries(C):
    """The planners answer every geometry with a variant or a clean error code
    (seeded random forward, depthwise and transposed shapes, all types)."""
    import random
    rng = random.Random(7)
    valid_codes = {-1, -7}
    for _ in range(300):
        G = rng.choice([1, 1, 2, 4])
        dw = rng.random() < 0.3
        Cc = rng.choice([3, 4, 8, 16, 24, 32, 64, 128, 200, 256]) * (1 if dw else G)
        O = Cc if dw else rng.choice([8, 16, 32, 64, 96, 128, 256]) * G
        if dw:
            G = Cc
        two_d = rng.random() < 0.6
        D = 1 if two_d else rng.randint(1, 12)
        H, W = rng.randint(1, 40), rng.randint(1, 40)
        k = (1 if two_d else rng.randint(1, 3), rng.randint(1, 7), rng.randint(1, 7))
        s = (1 if two_d else rng.randint(1, 2), rng.randint(1, 3), rng.randint(1, 3))
        d = (1, rng.randint(1, 2), rng.randint(1, 2))
        p = tuple(rng.randint(0, (k[i] - 1) * d[i]) for i in range(3))
        dt = rng.choice(["f16", "bf16", "f32"])
        try:
            v, bn, st, ct = C.plan(rng.randint(1, 4), D, H, W, Cc, O, k, s, p, d, G, dt)
            assert v in C.VARIANT_NAMES and bn > 0 and st >= 1 and ct >= 1, (v, bn, st, ct)
        except C.ConvError as e:
            assert e.code in valid_codes, e.code
        op = tuple(rng.randint(0, max(s[i], d[i]) - 1) for i in range(3))
        try:
            v, bn, st, ct = C.transpose_plan(rng.randint(1, 4), D, H, W, Cc, O, k, s, p, op, d, G, dt)
            assert v in (C.VARIANT_TC_GATHER, C.VARIANT_SIMT, C.VARIANT_TC_TMA_PHASES) and ct >= 1, (v, ct)
            if v == C.VARIANT_TC_TMA_PHASES:   # its conditions, as the header states them
                assert dt != "f32" and d == (1, 1, 1) and (Cc // G) % 64 == 0 and (O // G) % 128 == 0
        except C.ConvError as e:
            assert e.code in valid_codes, e.code
