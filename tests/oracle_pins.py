"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with what the pages or the mathematics fix.  The
same battery runs on the real oracle (every pin must hold) and on copies of
the oracle's C source with a deliberately planted mistake (at least one pin
must fail), see ``test_oracle_pins.py``.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _t(a, dtype=torch.float32):
    return torch.as_tensor(np.asarray(a), dtype=dtype).contiguous()


def _torch_conv_f64(x, w, stride, pad, dil, groups):
    """torch's CPU float64 convolution (an independent witness) on NDHWC data."""
    xt = torch.as_tensor(x, dtype=torch.float64).permute(0, 4, 1, 2, 3)
    wt = torch.as_tensor(w, dtype=torch.float64).permute(0, 4, 1, 2, 3)
    yt = torch.nn.functional.conv3d(xt, wt, stride=tuple(stride), padding=tuple(pad),
                                    dilation=tuple(dil), groups=groups)
    return yt.permute(0, 2, 3, 4, 1).contiguous().numpy()


def _grid_values(rng, shape, bits=8):
    """Random values on a coarse binary grid: exact in binary16 and in sums."""
    return (rng.integers(-(1 << bits), (1 << bits) + 1, size=shape) / float(1 << bits)).astype(np.float32)


# ---------------------------------------------------------------------------
# Pages' worked example and printed values
# ---------------------------------------------------------------------------

def pin_tutorial_example(orc):
    """Tutorial section 4: 3x3 input 1..9, kernel [[1,0],[0,-1]] -> [[-4,-4],[-4,-4]] exactly.

    The printed result also fixes cross-correlation (no flip): the flipped
    kernel [[-1,0],[0,1]] would give +4.
    """
    g = json.load(open(os.path.join(GOLDEN, "tutorial_tiny_example.json")))
    x = _t(g["x_hw"]).reshape(1, 1, 3, 3, 1)
    w = _t(g["k_hw"]).reshape(1, 1, 2, 2, 1)
    y, s = orc.conv_fwd(x, w, (1, 1, 1), (0, 0, 0), (1, 1, 1), 1)
    assert np.array_equal(y.reshape(2, 2), np.array(g["y_hw"], dtype=np.float64)), y.reshape(2, 2)
    # each printed term pair is (x*1, x*(-1)): |terms| sum to S
    terms = np.array(g["terms_hw"], dtype=np.float64)
    assert np.array_equal(s.reshape(2, 2), terms.sum(-1)), s.reshape(2, 2)
    # the same data in half precision and bfloat16 (all values exact there)
    for dt in (torch.float16, torch.bfloat16):
        y2, _ = orc.conv_fwd(x.to(dt), w.to(dt))
        assert np.array_equal(y2, y)


def pin_output_extent(orc):
    """Tutorial section 4: the ResNet-50 stem (224x224, 7x7, stride 2) has a 112x112 output
    (its FLOP formula multiplies by 112 x 112); with pad 3 the floor formula gives that.
    Other extents are checked against torch's convolution output shape."""
    assert orc.out_dims(1, 224, 224, 1, 7, 7, (1, 2, 2), (0, 3, 3), (1, 1, 1)) == (1, 112, 112)
    rng = np.random.default_rng(7)
    for _ in range(60):
        I = int(rng.integers(1, 20)); k = int(rng.integers(1, 6)); s = int(rng.integers(1, 4))
        d = int(rng.integers(1, 4)); p = int(rng.integers(0, 4))
        if I + 2 * p - d * (k - 1) - 1 < 0:
            continue
        xt = torch.zeros(1, 1, 1, 1, I, dtype=torch.float64)
        wt = torch.zeros(1, 1, 1, 1, k, dtype=torch.float64)
        ref = torch.nn.functional.conv3d(xt, wt, stride=(1, 1, s), padding=(0, 0, p), dilation=(1, 1, d)).shape[-1]
        assert orc.out_dims(1, 1, I, 1, 1, k, (1, 1, s), (0, 0, p), (1, 1, d))[2] == ref


# ---------------------------------------------------------------------------
# Closed forms
# ---------------------------------------------------------------------------

def pin_constant_input(orc):
    """x == 1, w == 1: every output counts its in-range taps times C/groups.

    Without padding every window is full, so y = kD*kH*kW*C/groups
    = FLOPs / (2 * number of outputs) -- the tutorial's FLOP formula read per output.
    With padding, a border output counts only the taps that land inside."""
    N, D, H, W, C, O = 2, 3, 7, 6, 4, 3
    for k, s, p, dl in (((1, 3, 3), (1, 1, 1), (0, 0, 0), (1, 1, 1)),
                        ((3, 2, 3), (1, 2, 1), (0, 0, 0), (1, 1, 2)),
                        ((3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1)),
                        ((1, 3, 2), (1, 2, 3), (0, 2, 1), (1, 2, 1))):
        x = torch.ones(N, D, H, W, C)
        w = torch.ones(O, *k, C)
        y, s_ = orc.conv_fwd(x, w, s, p, dl, 1)
        Do, Ho, Wo = y.shape[1:4]
        for od in range(Do):
            for oh in range(Ho):
                for ow in range(Wo):
                    cnt = 0
                    for kd in range(k[0]):
                        for kh in range(k[1]):
                            for kw in range(k[2]):
                                i = (od * s[0] - p[0] + kd * dl[0], oh * s[1] - p[1] + kh * dl[1],
                                     ow * s[2] - p[2] + kw * dl[2])
                                cnt += all(0 <= a < b for a, b in zip(i, (D, H, W)))
                    assert np.all(y[:, od, oh, ow, :] == cnt * C), (k, s, p, od, oh, ow)
        if p == (0, 0, 0):
            assert np.all(y == k[0] * k[1] * k[2] * C)
        assert np.array_equal(y, s_)


def pin_delta_kernel(orc):
    """Identity (delta) kernels: w[o, centre, c] = [o == c].

    With pad = dil*(k-1)/2 and stride 1 the output is the input exactly; with
    stride s it is the input subsampled by s; an off-centre delta shifts the
    input with zeros entering from the padding."""
    rng = np.random.default_rng(1)
    N, D, H, W, C = 2, 5, 9, 8, 5
    x = _t(_grid_values(rng, (N, D, H, W, C)))
    for dil in (1, 2):
        k = 3
        w = torch.zeros(C, k, k, k, C)
        for c in range(C):
            w[c, 1, 1, 1, c] = 1.0
        p = dil
        y, _ = orc.conv_fwd(x, w, (1, 1, 1), (p, p, p), (dil, dil, dil), 1)
        assert np.array_equal(y, x.double().numpy())
        for st in ((2, 2, 2), (1, 3, 2)):
            y, _ = orc.conv_fwd(x, w, st, (p, p, p), (dil, dil, dil), 1)
            ref = x.double().numpy()[:, ::st[0], ::st[1], ::st[2], :]
            assert y.shape == ref.shape and np.array_equal(y, ref)
    # off-centre: tap (kd,kh,kw) = (0, 2, 0) of a 3x3x3 kernel at pad 1 reads x[d-1, h+1, w-1]
    w = torch.zeros(C, 3, 3, 3, C)
    for c in range(C):
        w[c, 0, 2, 0, c] = 1.0
    y, _ = orc.conv_fwd(x, w, (1, 1, 1), (1, 1, 1), (1, 1, 1), 1)
    xs = np.zeros((N, D + 2, H + 2, W + 2, C))
    xs[:, 1:-1, 1:-1, 1:-1, :] = x.double().numpy()
    ref = xs[:, 0:D, 2:H + 2, 0:W, :]
    assert np.array_equal(y, ref)


def pin_pointwise_is_matmul(orc):
    """Tutorial section 5 variants table: a 1x1 convolution is exactly a GEMM over
    channels: y[m, o] = sum_c x[m, c] w[o, c]."""
    rng = np.random.default_rng(2)
    N, D, H, W, C, O = 2, 2, 5, 7, 16, 12
    x = _t(rng.standard_normal((N, D, H, W, C)))
    w = _t(rng.standard_normal((O, 1, 1, 1, C)))
    y, _ = orc.conv_fwd(x, w)
    ref = x.double().reshape(-1, C).numpy() @ w.double().reshape(O, C).numpy().T
    assert np.allclose(y.reshape(-1, O), ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# Independent witnesses
# ---------------------------------------------------------------------------

def _im2col_matmul(x, w, stride, pad, dil, groups):
    """Tutorial section 5 ("How convolution becomes GEMM") and exercise A: build the
    patch matrix explicitly (zero-padded input, one row per output position, one
    column per (tap, channel)), then one matmul per group with the reshaped weights."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    N, D, H, W, C = x.shape
    O, kD, kH, kW, Cg = w.shape
    Og = O // groups
    pd, ph, pw = pad
    xp = np.zeros((N, D + 2 * pd, H + 2 * ph, W + 2 * pw, C))
    xp[:, pd:pd + D, ph:ph + H, pw:pw + W, :] = x
    Do = (D + 2 * pd - dil[0] * (kD - 1) - 1) // stride[0] + 1
    Ho = (H + 2 * ph - dil[1] * (kH - 1) - 1) // stride[1] + 1
    Wo = (W + 2 * pw - dil[2] * (kW - 1) - 1) // stride[2] + 1
    cols = np.zeros((N, Do, Ho, Wo, kD, kH, kW, C))
    for kd in range(kD):
        for kh in range(kH):
            for kw in range(kW):
                d0, h0, w0 = kd * dil[0], kh * dil[1], kw * dil[2]
                cols[:, :, :, :, kd, kh, kw, :] = xp[:, d0:d0 + (Do - 1) * stride[0] + 1:stride[0],
                                                     h0:h0 + (Ho - 1) * stride[1] + 1:stride[1],
                                                     w0:w0 + (Wo - 1) * stride[2] + 1:stride[2], :]
    y = np.zeros((N * Do * Ho * Wo, O))
    for g in range(groups):
        a = cols[..., g * Cg:(g + 1) * Cg].reshape(N * Do * Ho * Wo, kD * kH * kW * Cg)
        b = w[g * Og:(g + 1) * Og].reshape(Og, kD * kH * kW * Cg)
        y[:, g * Og:(g + 1) * Og] = a @ b.T
    return y.reshape(N, Do, Ho, Wo, O)


_GEOMS = [
    # N, D, H, W, C, O, k, stride, pad, dil, groups
    (1, 1, 3, 3, 1, 1, (1, 2, 2), (1, 1, 1), (0, 0, 0), (1, 1, 1), 1),
    (2, 1, 9, 7, 6, 4, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 1),
    (2, 1, 11, 10, 3, 5, (1, 7, 7), (1, 2, 2), (0, 3, 3), (1, 1, 1), 1),
    (1, 1, 12, 9, 8, 6, (1, 3, 2), (1, 2, 3), (0, 2, 1), (1, 2, 3), 2),
    (2, 5, 6, 7, 4, 8, (3, 3, 3), (1, 1, 1), (1, 1, 1), (1, 1, 1), 1),
    (1, 6, 7, 5, 6, 6, (3, 1, 1), (2, 1, 1), (1, 0, 0), (1, 1, 1), 3),
    (1, 4, 8, 8, 4, 4, (1, 3, 3), (1, 1, 1), (0, 1, 1), (1, 1, 1), 4),   # depthwise
    (2, 7, 6, 9, 6, 4, (2, 3, 2), (2, 2, 1), (1, 0, 2), (2, 1, 3), 2),
]


def pin_im2col_equivalence(orc):
    """The oracle's direct sum equals an explicit im2col matrix times the reshaped
    weights (a separate construction) on tiny shapes, to fp64 rounding."""
    rng = np.random.default_rng(3)
    for (N, D, H, W, C, O, k, s, p, dl, G) in _GEOMS:
        x = _t(rng.uniform(-1, 1, (N, D, H, W, C)))
        w = _t(rng.standard_normal((O, *k, C // G)))
        y, _ = orc.conv_fwd(x, w, s, p, dl, G)
        ref = _im2col_matmul(x.numpy(), w.numpy(), s, p, dl, G)
        assert y.shape == ref.shape, (y.shape, ref.shape)
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-12), np.abs(y - ref).max()


def pin_torch_witness(orc):
    """torch.nn.functional.conv3d in CPU float64 (NCDHW after a permute) agrees,
    for every stride / pad / dilation / groups combination, on y and on
    S = conv(|x|, |w|)."""
    rng = np.random.default_rng(4)
    for (N, D, H, W, C, O, k, s, p, dl, G) in _GEOMS:
        x = _t(rng.uniform(-1, 1, (N, D, H, W, C))).to(torch.float16)
        w = _t(rng.standard_normal((O, *k, C // G))).to(torch.float16)
        y, S = orc.conv_fwd(x, w, s, p, dl, G)
        ref = _torch_conv_f64(x.double(), w.double(), s, p, dl, G)
        refS = _torch_conv_f64(x.double().abs(), w.double().abs(), s, p, dl, G)
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-12), np.abs(y - ref).max()
        assert np.allclose(S, refS, rtol=1e-12, atol=1e-12), np.abs(S - refS).max()


# ---------------------------------------------------------------------------
# Invariants
# ---------------------------------------------------------------------------

def pin_linearity(orc):
    """conv(a*x1 + b*x2, w) = a*conv(x1, w) + b*conv(x2, w), and likewise in w.
    Inputs on a coarse grid keep every combination exact in float32."""
    rng = np.random.default_rng(5)
    N, D, H, W, C, O = 2, 3, 6, 7, 5, 4
    k, s, p, dl = (3, 2, 3), (1, 2, 1), (1, 1, 1), (1, 1, 2)
    x1, x2 = _grid_values(rng, (N, D, H, W, C)), _grid_values(rng, (N, D, H, W, C))
    w1, w2 = _grid_values(rng, (O, *k, C)), _grid_values(rng, (O, *k, C))
    a, b = 3.0, -2.0
    y1, _ = orc.conv_fwd(_t(x1), _t(w1), s, p, dl)
    y2, _ = orc.conv_fwd(_t(x2), _t(w1), s, p, dl)
    yc, _ = orc.conv_fwd(_t(a * x1 + b * x2), _t(w1), s, p, dl)
    assert np.allclose(yc, a * y1 + b * y2, rtol=0, atol=1e-9)
    z2, _ = orc.conv_fwd(_t(x1), _t(w2), s, p, dl)
    zc, _ = orc.conv_fwd(_t(x1), _t(a * w1 + b * w2), s, p, dl)
    assert np.allclose(zc, a * y1 + b * z2, rtol=0, atol=1e-9)


def pin_translation(orc):
    """Weight sharing (tutorial section 1): shifting the input by stride*delta shifts
    the output by delta, away from the borders."""
    rng = np.random.default_rng(6)
    N, D, H, W, C, O = 1, 1, 14, 13, 3, 2
    k, s = (1, 3, 3), (1, 2, 2)
    x = _grid_values(rng, (N, D, H, W, C))
    w = _t(_grid_values(rng, (O, *k, C)))
    y, _ = orc.conv_fwd(_t(x), w, s, (0, 0, 0))
    dh, dw = 1, 2
    xs = np.zeros_like(x)
    xs[:, :, s[1] * dh:, s[2] * dw:, :] = x[:, :, :H - s[1] * dh, :W - s[2] * dw, :]
    ys, _ = orc.conv_fwd(_t(xs), w, s, (0, 0, 0))
    assert np.array_equal(ys[:, :, dh:, dw:, :], y[:, :, :y.shape[2] - dh, :y.shape[3] - dw, :])


def pin_groups_split(orc):
    """Tutorial variants table: grouped convolution splits the channels into G groups --
    the result equals G independent convolutions concatenated along C and O;
    depthwise is G = C (one filter per channel)."""
    rng = np.random.default_rng(8)
    N, D, H, W = 2, 3, 6, 5
    for C, O, G in ((6, 9, 3), (4, 8, 2), (5, 5, 5), (4, 12, 4)):
        x = _t(rng.uniform(-1, 1, (N, D, H, W, C)))
        w = _t(rng.standard_normal((O, 3, 3, 3, C // G)))
        y, _ = orc.conv_fwd(x, w, (1, 1, 1), (1, 1, 1), (1, 1, 1), G)
        Cg, Og = C // G, O // G
        for g in range(G):
            yg, _ = orc.conv_fwd(x[..., g * Cg:(g + 1) * Cg].contiguous(), w[g * Og:(g + 1) * Og].contiguous(),
                                 (1, 1, 1), (1, 1, 1), (1, 1, 1), 1)
            assert np.array_equal(y[..., g * Og:(g + 1) * Og], yg)


def pin_points_match_full(orc):
    """The sampled-output entry point returns the same values as the full pass."""
    rng = np.random.default_rng(9)
    N, D, H, W, C, O, k, s, p, dl, G = _GEOMS[-1]
    for dt in (torch.float32, torch.float16, torch.bfloat16):
        x = _t(rng.uniform(-1, 1, (N, D, H, W, C))).to(dt)
        w = _t(rng.standard_normal((O, *k, C // G))).to(dt)
        y, S = orc.conv_fwd(x, w, s, p, dl, G)
        idx = rng.integers(0, y.size, 200)
        yp, Sp = orc.conv_fwd_points(x, w, idx, s, p, dl, G)
        assert np.array_equal(yp, y.ravel()[idx]) and np.array_equal(Sp, S.ravel()[idx])


# ---------------------------------------------------------------------------
# The two options of the MLX pull request's discussion: flip and per-side padding
# ---------------------------------------------------------------------------

def pin_flip_tutorial_example(orc):
    """The tutorial's worked example with the filter flipped: the kernel acts as
    [[-1,0],[0,1]], each output is x[i+1][j+1] - x[i][j] = 4 for the input 1..9,
    exactly; flipping a filter that is its own reversal changes nothing."""
    g = json.load(open(os.path.join(GOLDEN, "tutorial_tiny_example.json")))
    x = _t(g["x_hw"]).reshape(1, 1, 3, 3, 1)
    w = _t(g["k_hw"]).reshape(1, 1, 2, 2, 1)
    y, _ = orc.conv_fwd(x, w, flip=True)
    assert np.array_equal(y.reshape(2, 2), np.full((2, 2), 4.0)), y.reshape(2, 2)
    sym = _t([[1.0, 2.0], [2.0, 1.0]]).reshape(1, 1, 2, 2, 1)
    assert np.array_equal(orc.conv_fwd(x, sym, flip=True)[0], orc.conv_fwd(x, sym)[0])


_GEOMS_EX = [
    # (N, D, H, W, C, O, k, stride, pad_lo, pad_hi, dil, groups)
    (1, 1, 7, 9, 3, 4, (1, 3, 3), (1, 1, 1), (0, 1, 2), (0, 2, 0), (1, 1, 1), 1),
    (2, 5, 6, 7, 4, 6, (3, 2, 3), (2, 1, 2), (1, 0, 2), (0, 1, 1), (1, 2, 1), 2),
    (1, 1, 9, 8, 2, 3, (1, 4, 3), (1, 2, 1), (0, 3, 0), (0, 0, 2), (1, 1, 2), 1),
]


def pin_flip_and_side_padding_torch_witness(orc):
    """torch float64 convolution of the explicitly zero-padded input (F.pad with
    the two sides' amounts, then no padding), with the filter reversed by torch
    in its spatial dimensions for flip, agrees on y and on S."""
    rng = np.random.default_rng(21)
    for (N, D, H, W, C, O, k, s, pl, ph, dl, G) in _GEOMS_EX:
        x = _t(rng.uniform(-1, 1, (N, D, H, W, C))).to(torch.float16)
        w = _t(rng.standard_normal((O, *k, C // G))).to(torch.float16)
        xp = torch.nn.functional.pad(x.double(), (0, 0, pl[2], ph[2], pl[1], ph[1], pl[0], ph[0]))
        for flip in (False, True):
            wr = w.double().flip(dims=(1, 2, 3)) if flip else w.double()
            y, S = orc.conv_fwd(x, w, s, pl, dl, G, pad_hi=ph, flip=flip)
            ref = _torch_conv_f64(xp, wr, s, (0, 0, 0), dl, G)
            refS = _torch_conv_f64(xp.abs(), wr.abs(), s, (0, 0, 0), dl, G)
            assert y.shape == ref.shape, (y.shape, ref.shape)
            assert np.allclose(y, ref, rtol=1e-12, atol=1e-12), np.abs(y - ref).max()
            assert np.allclose(S, refS, rtol=1e-12, atol=1e-12), np.abs(S - refS).max()


def pin_side_padding_is_a_crop(orc):
    """At stride 1, padding (p, q) below/above equals padding (p, p) with the last
    p - q outputs of that dimension dropped (q <= p), or the first q - p of the
    (q, q) result dropped (q >= p): the index origin moves only with the low side."""
    rng = np.random.default_rng(22)
    x = _t(_grid_values(rng, (1, 1, 8, 9, 3)))
    w = _t(_grid_values(rng, (5, 1, 3, 3, 3)))
    y_lo, _ = orc.conv_fwd(x, w, (1, 1, 1), (0, 2, 1), (1, 1, 1), 1, pad_hi=(0, 0, 1))
    y_sym, _ = orc.conv_fwd(x, w, (1, 1, 1), (0, 2, 1), (1, 1, 1), 1)
    assert np.array_equal(y_lo, y_sym[:, :, :-2, :, :])
    y_hi, _ = orc.conv_fwd(x, w, (1, 1, 1), (0, 0, 1), (1, 1, 1), 1, pad_hi=(0, 2, 1))
    y_sym2, _ = orc.conv_fwd(x, w, (1, 1, 1), (0, 2, 1), (1, 1, 1), 1)
    assert np.array_equal(y_hi, y_sym2[:, :, 2:, :, :])
    assert orc.out_dims(1, 8, 9, 1, 3, 3, (1, 1, 1), (0, 2, 1), (1, 1, 1), pad_hi=(0, 0, 1)) == (1, 8, 9)


# ---------------------------------------------------------------------------
# Transposed ("upsampling") convolution (tutorial variants table)
# ---------------------------------------------------------------------------

_T_GEOMS = [
    # (N, D, H, W, C, O, k, stride, pad, dil, groups) of the forward pass
    (2, 1, 7, 6, 3, 4, (1, 3, 3), (1, 2, 2), (0, 1, 1), (1, 1, 1), 1),
    (1, 5, 6, 7, 4, 6, (3, 3, 3), (2, 1, 2), (1, 1, 0), (1, 2, 1), 2),
    (1, 1, 9, 8, 6, 3, (1, 4, 4), (1, 2, 3), (0, 1, 2), (1, 1, 1), 3),
    (2, 1, 5, 5, 2, 2, (1, 2, 2), (1, 2, 2), (0, 0, 0), (1, 1, 1), 1),
    (1, 4, 6, 9, 4, 4, (2, 2, 3), (1, 2, 1), (1, 0, 2), (2, 1, 2), 2),
]


def _t_out_pad(I, k, s, p, d):
    """Output padding that makes the transposed pass return the forward input's extent."""
    return tuple((I[i] + 2 * p[i] - d[i] * (k[i] - 1) - 1) % s[i] for i in range(3))


def pin_transpose_adjoint(orc):
    """The transposed convolution is the adjoint of the forward pass with the
    same weights: sum(conv(a, w) * b) == sum(a * convT(b, w)) exactly, for
    integer-valued a, w, b (every product and sum exact in binary64).  This
    ties the transposed pass to the forward oracle, which the other pins fix."""
    rng = np.random.default_rng(21)
    for N, D, H, W, C, O, k, s, p, d, G in _T_GEOMS:
        a = _t(rng.integers(-4, 5, (N, D, H, W, C)))
        w = _t(rng.integers(-4, 5, (O, *k, C // G)))
        f, _ = orc.conv_fwd(a, w, s, p, d, G)
        b = _t(rng.integers(-4, 5, f.shape))
        op = _t_out_pad((D, H, W), k, s, p, d)
        t, _ = orc.conv_transpose(b, w, s, p, op, d, G)
        assert t.shape == tuple(a.shape)
        assert float(np.sum(f * b.double().numpy())) == float(np.sum(a.double().numpy() * t))


def pin_transpose_torch_witness(orc):
    """torch's CPU float64 conv_transpose3d (NCDHW; weight [Cin, Cout/G, k...])
    agrees with the oracle's transposed pass, y and the magnitude sum S."""
    rng = np.random.default_rng(22)
    for N, D, H, W, C, O, k, s, p, d, G in _T_GEOMS:
        Do, Ho, Wo = orc.out_dims(D, H, W, *k, s, p, d)
        x = _t(rng.uniform(-1, 1, (N, Do, Ho, Wo, O)))
        w = _t(rng.standard_normal((O, *k, C // G)))
        op = _t_out_pad((D, H, W), k, s, p, d)
        y, S = orc.conv_transpose(x, w, s, p, op, d, G)
        xt = x.double().permute(0, 4, 1, 2, 3)
        wt = w.double().permute(0, 4, 1, 2, 3)
        yt = torch.nn.functional.conv_transpose3d(xt, wt, stride=s, padding=p, output_padding=op, groups=G,
                                                  dilation=d).permute(0, 2, 3, 4, 1).numpy()
        st = torch.nn.functional.conv_transpose3d(xt.abs(), wt.abs(), stride=s, padding=p, output_padding=op,
                                                  groups=G, dilation=d).permute(0, 2, 3, 4, 1).numpy()
        assert y.shape == yt.shape
        assert np.allclose(y, yt, rtol=1e-12, atol=1e-12) and np.allclose(S, st, rtol=1e-12, atol=1e-12)


def pin_transpose_delta_upsamples(orc):
    """Closed form: a one-tap filter (1 at kh = kw = 0) with stride 2 and no
    padding inserts zeros: y[2i, 2j] = x[i, j], every other output 0; a centre
    tap with padding 1 does the same shifted into place."""
    x = _t(np.arange(1, 13, dtype=np.float32).reshape(1, 1, 3, 4, 1))
    w = torch.zeros(1, 1, 3, 3, 1)
    w[0, 0, 0, 0, 0] = 1.0
    y, _ = orc.conv_transpose(x, w, (1, 2, 2), (0, 0, 0), (0, 0, 0))
    assert y.shape == (1, 1, 7, 9, 1)
    ref = np.zeros((7, 9))
    ref[0:6:2, 0:8:2] = x.numpy().reshape(3, 4)
    assert np.array_equal(y.reshape(7, 9), ref)
    wc = torch.zeros(1, 1, 3, 3, 1)
    wc[0, 0, 1, 1, 0] = 1.0
    y2, _ = orc.conv_transpose(x, wc, (1, 2, 2), (0, 1, 1), (0, 1, 1))
    assert y2.shape == (1, 1, 6, 8, 1)
    ref2 = np.zeros((6, 8))
    ref2[0:6:2, 0:8:2] = x.numpy().reshape(3, 4)
    assert np.array_equal(y2.reshape(6, 8), ref2)


# ---------------------------------------------------------------------------
# Weight gradient of the forward pass
# ---------------------------------------------------------------------------

_W_GEOMS = [
    # (N, D, H, W, C, O, k, stride, pad_lo, pad_hi, dil, groups)
    (2, 1, 7, 6, 3, 4, (1, 3, 3), (1, 2, 2), (0, 1, 1), (0, 1, 1), (1, 1, 1), 1),
    (1, 4, 5, 6, 4, 6, (3, 3, 2), (2, 1, 1), (1, 0, 1), (0, 2, 0), (1, 2, 1), 2),
    (2, 1, 8, 7, 6, 3, (1, 2, 3), (1, 1, 2), (0, 1, 0), (0, 0, 2), (1, 2, 1), 3),
]


def pin_transpose_points_match_full(orc):
    """The transposed sampled-output entry point returns the same values as the
    full transposed pass (itself tied to the forward oracle by the adjoint pin),
    on odd extents (Qh != Qw, so a swapped index decode shows), strides, output
    padding and groups, in every storage type."""
    rng = np.random.default_rng(23)
    geoms = [
        # (N, D, H, W, Cin, Cout, k, stride, pad, out_pad, dil, groups) of the transposed pass
        (2, 1, 5, 7, 6, 9, (1, 3, 3), (1, 2, 2), (0, 1, 1), (0, 1, 0), (1, 1, 1), 3),
        (1, 3, 4, 6, 4, 6, (2, 3, 3), (2, 1, 3), (0, 1, 1), (1, 0, 2), (1, 1, 1), 2),
        (3, 1, 6, 5, 5, 7, (1, 4, 2), (1, 2, 1), (0, 1, 0), (0, 1, 0), (1, 1, 2), 1),
    ]
    for N, D, H, W, Ci, Co, k, s, p, op, d, G in geoms:
        for dt in (torch.float32, torch.float16, torch.bfloat16):
            x = _t(rng.uniform(-1, 1, (N, D, H, W, Ci))).to(dt)
            w = _t(rng.standard_normal((Ci, *k, Co // G))).to(dt)
            y, S = orc.conv_transpose(x, w, s, p, op, d, G)
            idx = np.concatenate([rng.integers(0, y.size, 300), [0, y.size - 1]])
            yp, Sp = orc.conv_transpose_points(x, w, idx, s, p, op, d, G)
            assert np.array_equal(yp, y.ravel()[idx]) and np.array_equal(Sp, S.ravel()[idx])


def pin_wgrad_adjoint(orc):
    """The weight gradient is the adjoint of the forward pass in w:
    sum(conv(x, w) * dy) == sum(w * wgrad(x, dy)) exactly for integer data."""
    rng = np.random.default_rng(31)
    for N, D, H, W, C, O, k, s, p, ph, d, G in _W_GEOMS:
        x = _t(rng.integers(-4, 5, (N, D, H, W, C)))
        w = _t(rng.integers(-4, 5, (O, *k, C // G)))
        y, _ = orc.conv_fwd(x, w, s, p, d, G, pad_hi=ph)
        dy = _t(rng.integers(-4, 5, y.shape))
        g, _ = orc.conv_wgrad(x, dy, k, s, p, d, G, pad_hi=ph)
        assert g.shape == tuple(w.shape)
        assert float(np.sum(y * dy.double().numpy())) == float(np.sum(w.double().numpy() * g))


def pin_wgrad_torch_witness(orc):
    """torch's float64 autograd of conv3d with respect to the weight agrees
    (symmetric padding), and so does its magnitude sum with |x|, |dy|."""
    rng = np.random.default_rng(32)
    for N, D, H, W, C, O, k, s, p, _, d, G in _W_GEOMS:
        x = _t(rng.uniform(-1, 1, (N, D, H, W, C)))
        Do, Ho, Wo = orc.out_dims(D, H, W, *k, s, p, d)
        dy = _t(rng.uniform(-1, 1, (N, Do, Ho, Wo, O)))
        g, S = orc.conv_wgrad(x, dy, k, s, p, d, G)

        def torch_grad(xa, dya):
            xt = torch.as_tensor(xa, dtype=torch.float64).permute(0, 4, 1, 2, 3)
            wt = torch.zeros((O, C // G, *k), dtype=torch.float64, requires_grad=True)
            yt = torch.nn.functional.conv3d(xt, wt, stride=s, padding=p, dilation=d, groups=G)
            yt.backward(torch.as_tensor(dya, dtype=torch.float64).permute(0, 4, 1, 2, 3))
            return wt.grad.permute(0, 2, 3, 4, 1).numpy()

        try:
            ref, ref_s = torch_grad(x, dy), torch_grad(x.abs(), dy.abs())
        except RuntimeError as e:  # dy shaped by the oracle's extents does not fit torch's output
            raise AssertionError(f"torch rejects the oracle's output extents: {e}") from None
        assert np.allclose(g, ref, rtol=1e-12, atol=1e-12)
        assert np.allclose(S, ref_s, rtol=1e-12, atol=1e-12)


def pin_wgrad_pointwise_is_matmul(orc):
    """Closed form: for a 1x1 filter at stride 1 the weight gradient is the
    matrix product dy^T x over all pixels (exact on integer data)."""
    rng = np.random.default_rng(33)
    x = rng.integers(-4, 5, (2, 3, 4, 5, 6))
    dy = rng.integers(-4, 5, (2, 3, 4, 5, 7))
    g, _ = orc.conv_wgrad(_t(x), _t(dy), (1, 1, 1))
    ref = dy.reshape(-1, 7).T.astype(np.float64) @ x.reshape(-1, 6).astype(np.float64)
    assert np.array_equal(g.reshape(7, 6), ref)


ALL_PINS = [pin_tutorial_example, pin_output_extent, pin_constant_input, pin_delta_kernel,
            pin_pointwise_is_matmul, pin_im2col_equivalence, pin_torch_witness, pin_linearity,
            pin_translation, pin_groups_split, pin_points_match_full, pin_flip_tutorial_example,
            pin_flip_and_side_padding_torch_witness, pin_side_padding_is_a_crop, pin_transpose_adjoint,
            pin_transpose_torch_witness, pin_transpose_delta_upsamples, pin_transpose_points_match_full,
            pin_wgrad_adjoint, pin_wgrad_torch_witness,
            pin_wgrad_pointwise_is_matmul]
