"""CPU oracle for the convolution forward pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It never calls into the CUDA library and
the CUDA library never calls into it; the two share only the seeded input
generator in ``workloads.py``, which holds no convolution arithmetic.

The arithmetic lives in ``conv_ref.c`` (plain C, fp64, OpenMP over output
rows).  It is the direct sliding-window sum of the "Convolutions" tutorial
(section 1, "What is it?", and the loop of section 4, "Tiny example"), widened
to channels, batch, depth, stride, zero padding, dilation ("gaps in the
kernel", section 5's variants table) and groups (same table), in the
channels-last layouts of section 7 and of the MLX conv3d pull request's
benchmark table: x (N, D, H, W, C), w (O, kD, kH, kW, C/groups).

The same file holds the transposed ("upsampling") convolution of the same
page's variants table, read as the adjoint of the forward pass, and the
weight gradient of the forward pass.

Every function here is pinned by ``tests/test_oracle_pins.py`` against things
other than itself: the tutorial's worked example, its printed FLOP and byte
counts, closed forms (delta kernels, constant inputs), invariants (linearity,
translation, group splitting) and independent witnesses (a NumPy im2col+matmul
on tiny shapes, torch's CPU float64 convolution).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "conv_ref.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

DTYPE_CODE = {"f32": 0, "f16": 1, "bf16": 2}


def build(force: bool = False) -> str:
    """Compile ``conv_ref.c`` into ``liboracle.so`` (gcc, OpenMP, -O2, strict IEEE)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


class Oracle:
    """The C oracle behind a ctypes handle.

    The module-level functions use the library built from ``conv_ref.c``;
    tests may load another build of the same source (for instance one with a
    deliberately planted mistake) as ``Oracle(path)`` and run the same pins.
    """

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        i3 = ctypes.POINTER(ctypes.c_int)
        dp = ctypes.POINTER(ctypes.c_double)
        common = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int] + [ctypes.c_int] * 9 + [i3, i3, i3, ctypes.c_int]
        lib.oracle_conv_fwd.argtypes = common + [dp, dp]
        lib.oracle_conv_fwd.restype = ctypes.c_int
        lib.oracle_conv_fwd_points.argtypes = common + [ctypes.POINTER(ctypes.c_int64), ctypes.c_int64, dp, dp]
        lib.oracle_conv_fwd_points.restype = ctypes.c_int
        lib.oracle_out_dims.argtypes = [ctypes.c_int] * 6 + [i3, i3, i3, i3]
        lib.oracle_out_dims.restype = ctypes.c_int
        # padding below / above and the flip flag (the forms with "_ex")
        common_ex = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int] + [ctypes.c_int] * 9 + \
            [i3, i3, i3, i3, ctypes.c_int, ctypes.c_int]
        lib.oracle_conv_fwd_ex.argtypes = common_ex + [dp, dp]
        lib.oracle_conv_fwd_ex.restype = ctypes.c_int
        lib.oracle_conv_fwd_points_ex.argtypes = common_ex + [ctypes.POINTER(ctypes.c_int64), ctypes.c_int64, dp, dp]
        lib.oracle_conv_fwd_points_ex.restype = ctypes.c_int
        lib.oracle_out_dims_ex.argtypes = [ctypes.c_int] * 6 + [i3, i3, i3, i3, i3]
        lib.oracle_out_dims_ex.restype = ctypes.c_int
        # transposed convolution: ..., stride, pad, out_pad, dil, groups
        common_t = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int] + [ctypes.c_int] * 9 + \
            [i3, i3, i3, i3, ctypes.c_int]
        lib.oracle_conv_transpose.argtypes = common_t + [dp, dp]
        lib.oracle_conv_transpose.restype = ctypes.c_int
        lib.oracle_conv_transpose_points.argtypes = common_t + [ctypes.POINTER(ctypes.c_int64), ctypes.c_int64,
                                                                dp, dp]
        lib.oracle_conv_transpose_points.restype = ctypes.c_int
        lib.oracle_convT_out_dims.argtypes = [ctypes.c_int] * 6 + [i3, i3, i3, i3, i3]
        lib.oracle_convT_out_dims.restype = ctypes.c_int
        # weight gradient: x, dy, dtype, N..kW, stride, pad_lo, pad_hi, dil, groups, dw, s
        lib.oracle_conv_wgrad.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int] + [ctypes.c_int] * 9 + \
            [i3, i3, i3, i3, ctypes.c_int, dp, dp]
        lib.oracle_conv_wgrad.restype = ctypes.c_int
        lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_f64.restype = ctypes.c_double
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_f64_to_f16_rn.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_f16_rn.restype = ctypes.c_uint16
        lib.oracle_f64_to_bf16_rn.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_bf16_rn.restype = ctypes.c_uint16
        lib.oracle_max_threads.restype = ctypes.c_int
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        self.lib = lib
        self.path = path

    def out_dims(self, D, H, W, kD, kH, kW, stride, pad, dil, pad_hi=None):
        """Output extents (Do, Ho, Wo): floor((I + p_lo + p_hi - dil*(k-1) - 1)/s) + 1 per
        dimension; `pad` is the padding below (and above, unless `pad_hi` is given)."""
        out = (ctypes.c_int * 3)()
        rc = self.lib.oracle_out_dims_ex(D, H, W, kD, kH, kW, _i3(stride), _i3(pad),
                                         _i3(pad if pad_hi is None else pad_hi), _i3(dil), out)
        if rc:
            raise ValueError("oracle.out_dims: invalid geometry")
        return tuple(out)

    def conv_fwd(self, x, w, stride=(1, 1, 1), pad=(0, 0, 0), dil=(1, 1, 1), groups=1, pad_hi=None,
                 flip=False):
        """Full output of the direct sum.

        x: [N, D, H, W, C] and w: [O, kD, kH, kW, C/groups] CPU tensors (float32,
        float16 or bfloat16, both the same).  `pad` pads below each dimension
        (and above, unless `pad_hi` is given); `flip` reads the filter reversed
        in every spatial dimension (a true convolution).  Returns (y, S), float64
        NumPy arrays of shape [N, Do, Ho, Wo, O]: y the sum, S = sum |x*w| over
        the same terms.
        """
        px, nx, kx = _raw(x)
        pw, nw, kw_ = _raw(w)
        if nx != nw:
            raise TypeError("oracle: x and w must share a dtype")
        N, D, H, W, C, O, kD, kH, kW = _shape_args(kx, kw_, groups)
        hi = pad if pad_hi is None else pad_hi
        Do, Ho, Wo = self.out_dims(D, H, W, kD, kH, kW, stride, pad, dil, hi)
        y = np.empty((N, Do, Ho, Wo, O), dtype=np.float64)
        s = np.empty_like(y)
        dp = ctypes.POINTER(ctypes.c_double)
        rc = self.lib.oracle_conv_fwd_ex(px, pw, DTYPE_CODE[nx], N, D, H, W, C, O, kD, kH, kW,
                                         _i3(stride), _i3(pad), _i3(hi), _i3(dil), int(groups), int(bool(flip)),
                                         y.ctypes.data_as(dp), s.ctypes.data_as(dp))
        if rc:
            raise ValueError(f"oracle.conv_fwd failed ({rc})")
        return y, s

    def conv_fwd_points(self, x, w, idx, stride=(1, 1, 1), pad=(0, 0, 0), dil=(1, 1, 1), groups=1,
                        pad_hi=None, flip=False):
        """Selected outputs: idx are flat indices into [N, Do, Ho, Wo, O]. Returns (y, S) float64."""
        px, nx, kx = _raw(x)
        pw, nw, kw_ = _raw(w)
        if nx != nw:
            raise TypeError("oracle: x and w must share a dtype")
        N, D, H, W, C, O, kD, kH, kW = _shape_args(kx, kw_, groups)
        hi = pad if pad_hi is None else pad_hi
        idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int64).ravel())
        y = np.empty(idx.shape[0], dtype=np.float64)
        s = np.empty_like(y)
        dp = ctypes.POINTER(ctypes.c_double)
        rc = self.lib.oracle_conv_fwd_points_ex(px, pw, DTYPE_CODE[nx], N, D, H, W, C, O, kD, kH, kW,
                                                _i3(stride), _i3(pad), _i3(hi), _i3(dil), int(groups),
                                                int(bool(flip)),
                                                idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                                idx.shape[0], y.ctypes.data_as(dp), s.ctypes.data_as(dp))
        if rc:
            raise ValueError(f"oracle.conv_fwd_points failed ({rc})")
        return y, s


    def convT_out_dims(self, D, H, W, kD, kH, kW, stride, pad, out_pad, dil):
        """Transposed-convolution extents: (I-1)*s - 2p + d*(k-1) + 1 + op per dimension."""
        out = (ctypes.c_int * 3)()
        rc = self.lib.oracle_convT_out_dims(D, H, W, kD, kH, kW, _i3(stride), _i3(pad), _i3(out_pad), _i3(dil),
                                            out)
        if rc:
            raise ValueError("oracle.convT_out_dims: invalid geometry")
        return tuple(out)

    def conv_transpose(self, x, w, stride=(1, 1, 1), pad=(0, 0, 0), out_pad=(0, 0, 0), dil=(1, 1, 1), groups=1):
        """Full output of the transposed convolution (the adjoint of conv_fwd with
        the same weights).

        x: [N, D, H, W, Cin] and w: [Cin, kD, kH, kW, Cout/groups] CPU tensors of
        one dtype.  Returns (y, S) float64 arrays of shape [N, Qd, Qh, Qw, Cout].
        """
        px, nx, kx = _raw(x)
        pw, nw, kw_ = _raw(w)
        if nx != nw:
            raise TypeError("oracle: x and w must share a dtype")
        N, D, H, W, Cin = (int(v) for v in kx.shape)
        Ci, kD, kH, kW, Cog = (int(v) for v in kw_.shape)
        if Ci != Cin:
            raise ValueError("oracle: w's first dimension must be x's channel count")
        Cout = Cog * groups
        Q = self.convT_out_dims(D, H, W, kD, kH, kW, stride, pad, out_pad, dil)
        y = np.empty((N, *Q, Cout), dtype=np.float64)
        s = np.empty_like(y)
        dp = ctypes.POINTER(ctypes.c_double)
        rc = self.lib.oracle_conv_transpose(px, pw, DTYPE_CODE[nx], N, D, H, W, Cin, Cout, kD, kH, kW,
                                            _i3(stride), _i3(pad), _i3(out_pad), _i3(dil), int(groups),
                                            y.ctypes.data_as(dp), s.ctypes.data_as(dp))
        if rc:
            raise ValueError(f"oracle.conv_transpose failed ({rc})")
        return y, s

    def conv_transpose_points(self, x, w, idx, stride=(1, 1, 1), pad=(0, 0, 0), out_pad=(0, 0, 0),
                              dil=(1, 1, 1), groups=1):
        """Selected outputs of the transposed convolution (flat indices into [N, Qd, Qh, Qw, Cout])."""
        px, nx, kx = _raw(x)
        pw, nw, kw_ = _raw(w)
        if nx != nw:
            raise TypeError("oracle: x and w must share a dtype")
        N, D, H, W, Cin = (int(v) for v in kx.shape)
        _, kD, kH, kW, Cog = (int(v) for v in kw_.shape)
        idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int64).ravel())
        y = np.empty(idx.shape[0], dtype=np.float64)
        s = np.empty_like(y)
        dp = ctypes.POINTER(ctypes.c_double)
        rc = self.lib.oracle_conv_transpose_points(px, pw, DTYPE_CODE[nx], N, D, H, W, Cin, Cog * groups, kD, kH,
                                                   kW, _i3(stride), _i3(pad), _i3(out_pad), _i3(dil), int(groups),
                                                   idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                                   idx.shape[0], y.ctypes.data_as(dp), s.ctypes.data_as(dp))
        if rc:
            raise ValueError(f"oracle.conv_transpose_points failed ({rc})")
        return y, s


    def conv_wgrad(self, x, dy, k, stride=(1, 1, 1), pad=(0, 0, 0), dil=(1, 1, 1), groups=1, pad_hi=None):
        """Weight gradient of conv_fwd: dw[o, k, c] = sum over pixels of dy * x.

        x: [N, D, H, W, C]; dy: [N, Do, Ho, Wo, O] (one dtype); k = (kD, kH, kW).
        Returns (dw, S) float64 arrays of shape [O, kD, kH, kW, C/groups].
        """
        px, nx, kx = _raw(x)
        py, ny, ky = _raw(dy)
        if nx != ny:
            raise TypeError("oracle: x and dy must share a dtype")
        N, D, H, W, C = (int(v) for v in kx.shape)
        O = int(ky.shape[-1])
        hi = pad if pad_hi is None else pad_hi
        if tuple(ky.shape[1:4]) != self.out_dims(D, H, W, *k, stride, pad, dil, hi):
            raise ValueError("oracle: dy's extents do not match the forward pass")
        dw = np.empty((O, *k, C // groups), dtype=np.float64)
        s = np.empty_like(dw)
        dp = ctypes.POINTER(ctypes.c_double)
        rc = self.lib.oracle_conv_wgrad(px, py, DTYPE_CODE[nx], N, D, H, W, C, O, *k, _i3(stride), _i3(pad),
                                        _i3(hi), _i3(dil), int(groups), dw.ctypes.data_as(dp), s.ctypes.data_as(dp))
        if rc:
            raise ValueError(f"oracle.conv_wgrad failed ({rc})")
        return dw, s


_default = None


def _load():
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default.lib


def default() -> Oracle:
    _load()
    return _default


def _i3(v):
    return (ctypes.c_int * 3)(*[int(a) for a in v])


def _raw(t):
    """(pointer, dtype name, keep-alive) for a contiguous CPU tensor/array."""
    import torch
    if isinstance(t, np.ndarray):
        t = torch.from_numpy(np.ascontiguousarray(t))
    t = t.detach().cpu().contiguous()
    name = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}.get(t.dtype)
    if name is None:
        raise TypeError(f"oracle: unsupported dtype {t.dtype}")
    return ctypes.c_void_p(t.data_ptr()), name, t


def _shape_args(x, w, groups):
    N, D, H, W, C = (int(v) for v in x.shape)
    O, kD, kH, kW, Cg = (int(v) for v in w.shape)
    if Cg * groups != C:
        raise ValueError(f"oracle: weight channels {Cg} x groups {groups} != C {C}")
    return N, D, H, W, C, O, kD, kH, kW


def out_dims(D, H, W, kD, kH, kW, stride, pad, dil, pad_hi=None):
    return default().out_dims(D, H, W, kD, kH, kW, stride, pad, dil, pad_hi)


def conv_fwd(x, w, stride=(1, 1, 1), pad=(0, 0, 0), dil=(1, 1, 1), groups=1, pad_hi=None, flip=False):
    return default().conv_fwd(x, w, stride, pad, dil, groups, pad_hi, flip)


def conv_fwd_points(x, w, idx, stride=(1, 1, 1), pad=(0, 0, 0), dil=(1, 1, 1), groups=1, pad_hi=None,
                    flip=False):
    return default().conv_fwd_points(x, w, idx, stride, pad, dil, groups, pad_hi, flip)


def convT_out_dims(D, H, W, kD, kH, kW, stride, pad, out_pad, dil):
    return default().convT_out_dims(D, H, W, kD, kH, kW, stride, pad, out_pad, dil)


def conv_transpose(x, w, stride=(1, 1, 1), pad=(0, 0, 0), out_pad=(0, 0, 0), dil=(1, 1, 1), groups=1):
    return default().conv_transpose(x, w, stride, pad, out_pad, dil, groups)


def conv_transpose_points(x, w, idx, stride=(1, 1, 1), pad=(0, 0, 0), out_pad=(0, 0, 0), dil=(1, 1, 1),
                          groups=1):
    return default().conv_transpose_points(x, w, idx, stride, pad, out_pad, dil, groups)


def conv_wgrad(x, dy, k, stride=(1, 1, 1), pad=(0, 0, 0), dil=(1, 1, 1), groups=1, pad_hi=None):
    return default().conv_wgrad(x, dy, k, stride, pad, dil, groups, pad_hi)


conv_wgrad.__doc__ = Oracle.conv_wgrad.__doc__
conv_transpose.__doc__ = Oracle.conv_transpose.__doc__
conv_fwd.__doc__ = Oracle.conv_fwd.__doc__
conv_fwd_points.__doc__ = Oracle.conv_fwd_points.__doc__
out_dims.__doc__ = Oracle.out_dims.__doc__


def decode(bits, dtype):
    """float64 values of raw binary16 / bfloat16 bit patterns (uint16 array)."""
    f = _load().oracle_f16_to_f64 if dtype == "f16" else _load().oracle_bf16_to_f64
    b = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([f(int(v)) for v in b], dtype=np.float64)


def round_bits(values, dtype):
    """Correctly rounded (nearest, ties to even) binary16/bfloat16 bit patterns of float64 values."""
    f = _load().oracle_f64_to_f16_rn if dtype == "f16" else _load().oracle_f64_to_bf16_rn
    v = np.asarray(values, dtype=np.float64).ravel()
    return np.array([f(float(a)) for a in v], dtype=np.uint16)


def round_to(values, dtype):
    """float64 value of the correctly rounded `dtype` neighbour of each float64 value."""
    v = np.asarray(values, dtype=np.float64)
    if dtype == "f32":
        return v.astype(np.float32).astype(np.float64)
    if dtype == "f16":
        # binary16 has few enough values that rounding through the C encoder per
        # element is affordable only for small arrays; NumPy's float64->float16
        # cast is itself correctly rounded and is pinned against the encoder.
        return v.astype(np.float16).astype(np.float64)
    bits = round_bits(v, "bf16") if v.size <= 200_000 else _bf16_rn_vector(v)
    return decode_bf16_vector(bits).reshape(v.shape)


def decode_bf16_vector(bits):
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def _bf16_rn_vector(v):
    """Vector form of the bfloat16 encoder: float64 -> nearest-even bfloat16 bits.

    Rounds the float64 value once, at the bfloat16 quantum of its binade (found
    exactly with frexp), so there is no double rounding through float32.
    """
    v = np.asarray(v, dtype=np.float64).ravel()
    a = np.abs(v)
    sign = np.signbit(v).astype(np.uint16) << 15
    _, e = np.frexp(a)                       # a = m * 2^e, m in [0.5, 1)
    E = np.maximum(e.astype(np.float64) - 1.0, -126.0)
    q = np.exp2(E - 7.0)
    r = np.rint(a / q) * q
    _, e2 = np.frexp(r)
    E2 = e2.astype(np.float64) - 1.0
    sub = E2 < -126
    mant_n = r / np.exp2(E2 - 7.0) - 128.0
    mant_s = r / np.exp2(-133.0)
    bits = np.where(sub, mant_s, (E2 + 127.0) * 128.0 + mant_n)
    bits = np.where(r == 0, 0.0, bits)
    bits = np.where(r >= 2.0 ** 128, float(0x7F80), bits)
    bits = np.where(np.isinf(a), float(0x7F80), bits)
    out = bits.astype(np.uint32).astype(np.uint16) | sign
    out[np.isnan(v)] = 0x7FC0
    return out


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))
