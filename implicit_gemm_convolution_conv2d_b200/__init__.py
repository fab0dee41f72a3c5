"""Implicit-GEMM convolution forward for NVIDIA B200 (sm_100a).

A thin ctypes binding over the C ABI in ``include/conv_fwd.h``
(``libconvfwd.so``, built in-tree from ``csrc/``).  This module only marshals
arguments: shapes, pointers and the current CUDA stream.  Every step of the
convolution runs in the library's CUDA kernels; there is no CPU path, and the
module raises if the library is missing or the tensors are not on a CUDA
device.

Layouts are channels-last: x [N, D, H, W, C] (or [N, H, W, C] for 2-D),
w [O, kD, kH, kW, C/groups] (or [O, kH, kW, C/groups]), y [N, Do, Ho, Wo, O].
"""
from __future__ import annotations

import ctypes
import os

__all__ = ["conv_fwd", "conv_fwd_host", "out_dims", "plan", "conv_transpose", "transpose_out_dims",
           "transpose_plan", "conv_wgrad", "wgrad_workspace_size", "wgrad_plan", "last_status", "strerror", "lib",
           "CONV_F32", "CONV_F16", "CONV_BF16", "VARIANT_AUTO", "VARIANT_SIMT", "VARIANT_TC_TMA",
           "VARIANT_TC_GATHER", "VARIANT_TC_TMA_PAIR", "VARIANT_TC_HALO", "VARIANT_TC_HALO_PAIR",
           "VARIANT_TC_TMA_T", "VARIANT_TC_HALO_T", "VARIANT_TC_HALO_T_PAIR", "VARIANT_TC_PHASE", "VARIANT_DEPTHWISE", "VARIANT_DEPTHWISE_DIRECT",
           "VARIANT_TC_TMA_PHASES", "VARIANT_TC_STAGED", "ConvError"]

CONV_F32, CONV_F16, CONV_BF16 = 0, 1, 2
VARIANT_AUTO, VARIANT_SIMT, VARIANT_TC_TMA, VARIANT_TC_GATHER, VARIANT_TC_TMA_PAIR = -1, 0, 1, 2, 3
VARIANT_TC_HALO, VARIANT_TC_HALO_PAIR, VARIANT_TC_TMA_T, VARIANT_TC_HALO_T, VARIANT_TC_HALO_T_PAIR = 4, 5, 6, 7, 8
VARIANT_TC_PHASE = 9
VARIANT_DEPTHWISE = 10
VARIANT_DEPTHWISE_DIRECT = 11
VARIANT_TC_TMA_PHASES = 12       # conv_transpose only: sub-pixel phases fed by TMA, CTA pairs
VARIANT_TC_STAGED = 13           # any channel count: realigned input regions read as per-tap views
VARIANT_NAMES = {VARIANT_SIMT: "simt_ffma", VARIANT_TC_TMA: "tcgen05_tma_im2col",
                 VARIANT_TC_GATHER: "tcgen05_gather", VARIANT_TC_TMA_PAIR: "tcgen05_tma_im2col_pair",
                 VARIANT_TC_HALO: "tcgen05_tma_halo", VARIANT_TC_HALO_PAIR: "tcgen05_tma_halo_pair",
                 VARIANT_TC_TMA_T: "tcgen05_tma_im2col_t", VARIANT_TC_HALO_T: "tcgen05_tma_halo_t",
                 VARIANT_TC_HALO_T_PAIR: "tcgen05_tma_halo_t_pair", VARIANT_TC_PHASE: "tcgen05_tma_phase",
                 VARIANT_DEPTHWISE: "depthwise_tma", VARIANT_DEPTHWISE_DIRECT: "depthwise_direct",
                 VARIANT_TC_TMA_PHASES: "tcgen05_tma_phases_pair", VARIANT_TC_STAGED: "tcgen05_staged_t"}

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libconvfwd.so")
_lib = None


class ConvError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} ({code})" if what else f"{strerror(code)} ({code})")


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m implicit_gemm_convolution_conv2d_b200._build`")
        L = ctypes.CDLL(LIB_PATH)
        i3 = ctypes.POINTER(ctypes.c_int)
        vp, ci = ctypes.c_void_p, ctypes.c_int
        geo = [ci] * 9 + [i3, i3, i3, ci, ci]
        L.conv_out_dims.argtypes = [ci] * 6 + [i3, i3, i3, i3]
        L.conv_fwd.argtypes = [vp, vp, vp] + geo + [vp]
        L.conv_fwd_variant.argtypes = [vp, vp, vp] + geo + [ci, vp]
        L.conv_fwd_host.argtypes = [vp] * 6 + geo + [vp]
        L.conv_plan.argtypes = geo + [i3, i3, i3]
        L.conv_plan_variant.argtypes = geo + [ci, i3, i3, i3]
        # the general forms: per-side padding and flip (geo_ex: ..., stride, pad_lo, pad_hi, dil, groups, flip, dtype)
        geo_ex = [ci] * 9 + [i3, i3, i3, i3, ci, ci, ci]
        L.conv_out_dims_ex.argtypes = [ci] * 6 + [i3, i3, i3, i3, i3]
        L.conv_fwd_ex.argtypes = [vp, vp, vp] + geo_ex + [ci, vp]
        L.conv_plan_ex.argtypes = geo_ex + [ci, i3, i3, i3]
        # transposed convolution: ..., stride, pad, out_pad, dil, groups, dtype
        geo_t = [ci] * 9 + [i3, i3, i3, i3, ci, ci]
        L.conv_transpose_out_dims.argtypes = [ci] * 6 + [i3, i3, i3, i3, i3]
        L.conv_transpose.argtypes = [vp, vp, vp] + geo_t + [ci, vp]
        L.conv_transpose_plan.argtypes = geo_t + [ci, i3, i3, i3]
        # weight gradient: ..., stride, pad_lo, pad_hi, dil, groups, dtype
        L.conv_wgrad_workspace_size.argtypes = geo_ex[:-2] + [ci, ctypes.POINTER(ctypes.c_ulonglong)]
        L.conv_wgrad.argtypes = [vp, vp, vp] + geo_ex[:-2] + [ci, vp, ctypes.c_ulonglong, vp]
        L.conv_wgrad_noalloc.argtypes = [vp, vp, vp] + geo_ex[:-2] + [ci, vp]
        L.conv_wgrad_plan.argtypes = geo_ex[:-2] + [ci, i3, i3]
        L.conv_last_status.argtypes = [vp]
        L.conv_debug_inject_stall.argtypes = [ctypes.c_ulonglong]
        L.conv_strerror.argtypes = [ci]
        L.conv_strerror.restype = ctypes.c_char_p
        for f in ("conv_out_dims", "conv_fwd", "conv_fwd_variant", "conv_fwd_host", "conv_plan",
                  "conv_plan_variant", "conv_last_status", "conv_version", "conv_debug_inject_stall",
                  "conv_out_dims_ex", "conv_fwd_ex", "conv_plan_ex"):
            getattr(L, f).restype = ci
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().conv_strerror(int(code)).decode()


def _i3(v):
    return (ctypes.c_int * 3)(*[int(a) for a in v])


def _triple(v, name, spatial_default=None):
    if isinstance(v, int):
        return (v, v, v) if spatial_default is None else (spatial_default, v, v)
    v = tuple(int(a) for a in v)
    if len(v) == 2:
        return (spatial_default if spatial_default is not None else 1,) + v
    if len(v) != 3:
        raise ValueError(f"{name} must have 2 or 3 entries")
    return v


def _dtype_code(t):
    import torch
    code = {torch.float32: CONV_F32, torch.float16: CONV_F16, torch.bfloat16: CONV_BF16}.get(t.dtype)
    if code is None:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return code


def out_dims(D, H, W, kD, kH, kW, stride, pad, dil, pad_hi=None):
    """(Do, Ho, Wo) as computed by the library (host only); `pad` pads below each
    dimension, and above unless `pad_hi` is given."""
    out = (ctypes.c_int * 3)()
    rc = lib().conv_out_dims_ex(D, H, W, kD, kH, kW, _i3(stride), _i3(pad),
                                _i3(pad if pad_hi is None else pad_hi), _i3(dil), out)
    if rc:
        raise ConvError(rc, "conv_out_dims")
    return tuple(out)


def _geometry(x, w, stride, padding, dilation):
    two_d = x.dim() == 4
    if two_d:
        if w.dim() != 4:
            raise ValueError("2-D input needs a [O, kH, kW, C/groups] weight")
        N, H, W, C = x.shape
        D = 1
        O, kH, kW, Cg = w.shape
        kD = 1
        s = _triple(stride, "stride", 1)
        p = _triple(padding, "padding", 0)
        d = _triple(dilation, "dilation", 1)
        if isinstance(stride, int):
            s = (1, stride, stride)
        if isinstance(padding, int):
            p = (0, padding, padding)
        if isinstance(dilation, int):
            d = (1, dilation, dilation)
    else:
        if x.dim() != 5 or w.dim() != 5:
            raise ValueError("x must be [N,D,H,W,C] and w [O,kD,kH,kW,C/groups]")
        N, D, H, W, C = x.shape
        O, kD, kH, kW, Cg = w.shape
        s, p, d = _triple(stride, "stride"), _triple(padding, "padding"), _triple(dilation, "dilation")
    return two_d, (int(N), int(D), int(H), int(W), int(C), int(O), int(kD), int(kH), int(kW), int(Cg)), s, p, d


def conv_fwd(x, w, stride=1, padding=0, dilation=1, groups=1, *, out=None, variant=VARIANT_AUTO, stream=None,
             padding_hi=None, flip=False):
    """y = conv(x, w) on the current CUDA stream (or `stream`).  Returns y.

    x, w: contiguous CUDA tensors of one dtype (float16, bfloat16 or float32).
    `out` may supply a preallocated contiguous y.  `variant` forces a kernel
    (VARIANT_*); the default lets the library choose.  `padding` pads below
    each spatial dimension and, unless `padding_hi` is given, above it too;
    `flip` reads the filter reversed in every spatial dimension.

    The call only queues the kernel.  A kernel that gives up on a pipeline
    wait (after 2 s) writes no further output and records it in the device
    status word: check ``last_status()`` (it waits for the stream) before
    trusting y.
    """
    import torch
    if not (x.is_cuda and w.is_cuda):
        raise ValueError("conv_fwd runs on CUDA tensors only")
    if x.dtype != w.dtype:
        raise TypeError("x and w must share a dtype")
    two_d, (N, D, H, W, C, O, kD, kH, kW, Cg), s, p, d = _geometry(x, w, stride, padding, dilation)
    if Cg * groups != C:
        raise ValueError(f"weight has {Cg} channels per group but C={C}, groups={groups}")
    ph = p if padding_hi is None else _geometry(x, w, stride, padding_hi, dilation)[3]
    Do, Ho, Wo = out_dims(D, H, W, kD, kH, kW, s, p, d, ph)
    shape = (N, Ho, Wo, O) if two_d else (N, Do, Ho, Wo, O)
    if out is None:
        out = torch.empty(shape, dtype=x.dtype, device=x.device)
    elif tuple(out.shape) != shape or out.dtype != x.dtype or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous {x.dtype} tensor of shape {shape}")
    x = x.contiguous()
    w = w.contiguous()
    st = stream if stream is not None else torch.cuda.current_stream(x.device)
    with torch.cuda.device(x.device):
        rc = lib().conv_fwd_ex(x.data_ptr(), w.data_ptr(), out.data_ptr(), N, D, H, W, C, O, kD, kH, kW,
                               _i3(s), _i3(p), _i3(ph), _i3(d), int(groups), int(bool(flip)), _dtype_code(x),
                               int(variant), st.cuda_stream)
    if rc:
        raise ConvError(rc, "conv_fwd")
    return out


def wgrad_workspace_size(N, D, H, W, C, O, k, stride, pad, dil, groups, dtype, pad_hi=None):
    """Bytes of fp32 workspace conv_wgrad needs for these shapes (one slice of
    partial sums per range of the split pixel reduction)."""
    code = {"f32": CONV_F32, "f16": CONV_F16, "bf16": CONV_BF16}[dtype]
    out = ctypes.c_ulonglong()
    rc = lib().conv_wgrad_workspace_size(N, D, H, W, C, O, *k, _i3(stride), _i3(pad),
                                         _i3(pad if pad_hi is None else pad_hi), _i3(dil), int(groups), code,
                                         ctypes.byref(out))
    if rc:
        raise ConvError(rc, "conv_wgrad_workspace_size")
    return out.value


WGRAD_FP32, WGRAD_TENSOR_CORES = 0, 1
WGRAD_PATH_NAMES = {WGRAD_FP32: "simt_wgrad", WGRAD_TENSOR_CORES: "tcgen05_wgrad_pair"}


def wgrad_plan(N, D, H, W, C, O, k, stride, pad, dil, groups, dtype, pad_hi=None):
    """(path, ranges) conv_wgrad takes for these shapes: WGRAD_FP32 or
    WGRAD_TENSOR_CORES, and the number of ranges of its split pixel reduction."""
    code = {"f32": CONV_F32, "f16": CONV_F16, "bf16": CONV_BF16}[dtype]
    path, ns = (ctypes.c_int * 1)(), (ctypes.c_int * 1)()
    rc = lib().conv_wgrad_plan(N, D, H, W, C, O, *k, _i3(stride), _i3(pad), _i3(pad if pad_hi is None else pad_hi),
                               _i3(dil), int(groups), code, path, ns)
    if rc:
        raise ConvError(rc, "conv_wgrad_plan")
    return path[0], ns[0]


def conv_wgrad(x, dy, kernel_size, stride=1, padding=0, dilation=1, groups=1, *, padding_hi=None, out=None,
               workspace=None, stream=None):
    """Weight gradient of conv_fwd: dw[o, k, c] = sum over output pixels of dy * x.

    x: [N, (D,) H, W, C]; dy: [N, (Do,) Ho, Wo, O]; kernel_size: (kD,) kH, kW.
    Returns dw [O, (kD,) kH, kW, C/groups] in x's dtype.  The call needs an
    fp32 workspace of wgrad_workspace_size bytes; one is allocated with torch
    when `workspace` is None.
    """
    import torch
    if not (x.is_cuda and dy.is_cuda):
        raise ValueError("conv_wgrad runs on CUDA tensors only")
    if x.dtype != dy.dtype:
        raise TypeError("x and dy must share a dtype")
    two_d = x.dim() == 4
    k = tuple(kernel_size) if not isinstance(kernel_size, int) else (kernel_size,) * (2 if two_d else 3)
    if two_d:
        k = (1, *k)
        N, H, W, C = x.shape
        D = 1
        s = (1, stride, stride) if isinstance(stride, int) else (1, *stride)
        p = (0, padding, padding) if isinstance(padding, int) else (0, *padding)
        d = (1, dilation, dilation) if isinstance(dilation, int) else (1, *dilation)
        ph = p if padding_hi is None else ((0, padding_hi, padding_hi) if isinstance(padding_hi, int)
                                           else (0, *padding_hi))
    else:
        N, D, H, W, C = x.shape
        s, p, d = _triple(stride, "stride"), _triple(padding, "padding"), _triple(dilation, "dilation")
        ph = p if padding_hi is None else _triple(padding_hi, "padding_hi")
    O = int(dy.shape[-1])
    N, D, H, W, C = int(N), int(D), int(H), int(W), int(C)
    Do, Ho, Wo = out_dims(D, H, W, *k, s, p, d, ph)
    if (dy.shape[1:-1] if not two_d else (1, *dy.shape[1:-1])) != ((Do, Ho, Wo) if not two_d else (1, Ho, Wo)):
        raise ValueError("dy's extents do not match the forward pass")
    shape = (O, *k[1:], C // groups) if two_d else (O, *k, C // groups)
    if out is None:
        out = torch.empty(shape, dtype=x.dtype, device=x.device)
    code = _dtype_code(x)
    need = wgrad_workspace_size(N, D, H, W, C, O, k, s, p, d, groups,
                                {CONV_F32: "f32", CONV_F16: "f16", CONV_BF16: "bf16"}[code], ph)
    if need and workspace is None:
        workspace = torch.empty(need // 4, dtype=torch.float32, device=x.device)
    x = x.contiguous()
    dy = dy.contiguous()
    st = stream if stream is not None else torch.cuda.current_stream(x.device)
    with torch.cuda.device(x.device):
        rc = lib().conv_wgrad(x.data_ptr(), dy.data_ptr(), out.data_ptr(), N, D, H, W, C, O, *k, _i3(s), _i3(p),
                              _i3(ph), _i3(d), int(groups), code, workspace.data_ptr() if need else None,
                              int(workspace.numel() * workspace.element_size()) if need else 0, st.cuda_stream)
    if rc:
        raise ConvError(rc, "conv_wgrad")
    return out


def conv_wgrad_raw(x_ptr, dy_ptr, dw_ptr, geom, dtype, ws_ptr=None, ws_bytes=0, stream_handle=0):
    """The C entry point on raw device pointers: geom = (N,D,H,W,C,O,kD,kH,kW,stride,pad_lo,pad_hi,dil,groups)."""
    N, D, H, W, Cc, O, kD, kH, kW, s, p, ph, d, g = geom
    return lib().conv_wgrad(x_ptr, dy_ptr, dw_ptr, N, D, H, W, Cc, O, kD, kH, kW, _i3(s), _i3(p), _i3(ph), _i3(d),
                            int(g), int(dtype), ws_ptr, int(ws_bytes), stream_handle)


def conv_wgrad_noalloc_raw(x_ptr, dy_ptr, dw_ptr, geom, dtype, stream_handle=0):
    """conv_wgrad_noalloc on raw device pointers (no workspace: the library's
    static scratch array); geom as for conv_wgrad_raw."""
    N, D, H, W, Cc, O, kD, kH, kW, s, p, ph, d, g = geom
    return lib().conv_wgrad_noalloc(x_ptr, dy_ptr, dw_ptr, N, D, H, W, Cc, O, kD, kH, kW, _i3(s), _i3(p), _i3(ph),
                                    _i3(d), int(g), int(dtype), stream_handle)


def transpose_out_dims(D, H, W, kD, kH, kW, stride, pad, out_pad, dil):
    """(Qd, Qh, Qw) of the transposed convolution, as computed by the library (host only)."""
    out = (ctypes.c_int * 3)()
    rc = lib().conv_transpose_out_dims(D, H, W, kD, kH, kW, _i3(stride), _i3(pad), _i3(out_pad), _i3(dil), out)
    if rc:
        raise ConvError(rc, "conv_transpose_out_dims")
    return tuple(out)


def conv_transpose(x, w, stride=1, padding=0, output_padding=0, dilation=1, groups=1, *, out=None,
                   variant=VARIANT_AUTO, stream=None):
    """Transposed ("upsampling") convolution on the current CUDA stream (or
    `stream`): the adjoint of conv_fwd with the same weights.  Returns y.

    x: [N, (D,) H, W, Cin]; w: [Cin, (kD,) kH, kW, Cout/groups] (conv_fwd's
    weight layout with O = Cin); y: [N, (Qd,) Qh, Qw, Cout] with
    Q = (I-1)*s - 2p + d*(k-1) + 1 + output_padding per dimension.
    """
    import torch
    if not (x.is_cuda and w.is_cuda):
        raise ValueError("conv_transpose runs on CUDA tensors only")
    if x.dtype != w.dtype:
        raise TypeError("x and w must share a dtype")
    two_d, (N, D, H, W, Cin, Ci, kD, kH, kW, Cog), s, p, d = _geometry(x, w, stride, padding, dilation)
    op = _geometry(x, w, stride, output_padding, dilation)[3]
    if Ci != Cin:
        raise ValueError(f"weight's first dimension {Ci} must equal the input channels {Cin}")
    Cout = Cog * groups
    Qd, Qh, Qw = transpose_out_dims(D, H, W, kD, kH, kW, s, p, op, d)
    shape = (N, Qh, Qw, Cout) if two_d else (N, Qd, Qh, Qw, Cout)
    if out is None:
        out = torch.empty(shape, dtype=x.dtype, device=x.device)
    elif tuple(out.shape) != shape or out.dtype != x.dtype or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous {x.dtype} tensor of shape {shape}")
    x = x.contiguous()
    w = w.contiguous()
    st = stream if stream is not None else torch.cuda.current_stream(x.device)
    with torch.cuda.device(x.device):
        rc = lib().conv_transpose(x.data_ptr(), w.data_ptr(), out.data_ptr(), N, D, H, W, Cin, Cout, kD, kH, kW,
                                  _i3(s), _i3(p), _i3(op), _i3(d), int(groups), _dtype_code(x), int(variant),
                                  st.cuda_stream)
    if rc:
        raise ConvError(rc, "conv_transpose")
    return out


def conv_transpose_raw(x_ptr, w_ptr, y_ptr, geom, dtype, variant=VARIANT_AUTO, stream_handle=0):
    """The C entry point on raw device pointers: geom = (N,D,H,W,Cin,Cout,kD,kH,kW,stride,pad,out_pad,dil,groups)."""
    N, D, H, W, Ci, Co, kD, kH, kW, s, p, op, d, g = geom
    return lib().conv_transpose(x_ptr, w_ptr, y_ptr, N, D, H, W, Ci, Co, kD, kH, kW, _i3(s), _i3(p), _i3(op),
                                _i3(d), int(g), int(dtype), int(variant), stream_handle)


def transpose_plan(N, D, H, W, Cin, Cout, k, stride, pad, out_pad, dil, groups, dtype, variant=VARIANT_AUTO):
    """(variant, BN, stages, CTAs) the library would use for a transposed convolution."""
    bn, st, ct = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    code = {"f32": CONV_F32, "f16": CONV_F16, "bf16": CONV_BF16}[dtype]
    rc = lib().conv_transpose_plan(N, D, H, W, Cin, Cout, *k, _i3(stride), _i3(pad), _i3(out_pad), _i3(dil),
                                   int(groups), code, int(variant), ctypes.byref(bn), ctypes.byref(st),
                                   ctypes.byref(ct))
    if rc < 0:
        raise ConvError(rc, "conv_transpose_plan")
    return rc, bn.value, st.value, ct.value


def conv_fwd_raw(x_ptr, w_ptr, y_ptr, geom, dtype, variant=VARIANT_AUTO, stream_handle=0, pad_hi=None, flip=0):
    """The C entry point on raw device pointers: geom = (N,D,H,W,C,O,kD,kH,kW,stride,pad,dil,groups)
    (conv_fwd_variant; conv_fwd_ex when `pad_hi` or `flip` is given)."""
    N, D, H, W, C, O, kD, kH, kW, s, p, d, g = geom
    if pad_hi is None and not flip:
        return lib().conv_fwd_variant(x_ptr, w_ptr, y_ptr, N, D, H, W, C, O, kD, kH, kW, _i3(s), _i3(p), _i3(d),
                                      int(g), int(dtype), int(variant), stream_handle)
    return lib().conv_fwd_ex(x_ptr, w_ptr, y_ptr, N, D, H, W, C, O, kD, kH, kW, _i3(s), _i3(p),
                             _i3(p if pad_hi is None else pad_hi), _i3(d), int(g), int(flip), int(dtype),
                             int(variant), stream_handle)


def conv_fwd_host(x_host, w_host, y_host, x_dev, w_dev, y_dev, stride=1, padding=0, dilation=1, groups=1,
                  stream=None):
    """Host-buffer entry point: copies x, w in, runs, copies y out, waits
    (chunks of the batch overlap their copies with the kernels).  Raises
    ConvError, code -6, when a kernel gave up on a pipeline wait.

    x_host/w_host/y_host: CPU tensors (pinned for asynchronous copies);
    x_dev/w_dev/y_dev: CUDA tensors of the same shapes (caller-owned scratch).
    """
    import torch
    two_d, (N, D, H, W, C, O, kD, kH, kW, Cg), s, p, d = _geometry(x_host, w_host, stride, padding, dilation)
    st = stream if stream is not None else torch.cuda.current_stream(x_dev.device)
    with torch.cuda.device(x_dev.device):
        rc = lib().conv_fwd_host(x_host.data_ptr(), w_host.data_ptr(), y_host.data_ptr(), x_dev.data_ptr(),
                                 w_dev.data_ptr(), y_dev.data_ptr(), N, D, H, W, C, O, kD, kH, kW, _i3(s), _i3(p),
                                 _i3(d), int(groups), _dtype_code(x_host), st.cuda_stream)
    if rc:
        raise ConvError(rc, "conv_fwd_host")
    return y_host


def plan(N, D, H, W, C, O, k, stride, pad, dil, groups, dtype, variant=VARIANT_AUTO, pad_hi=None, flip=0):
    """(variant, BN, stages, ctas) the library would use; dtype is 'f32' | 'f16' | 'bf16'.
    With an explicit `variant`, the plan of that variant (ConvError if it cannot run)."""
    code = {"f32": CONV_F32, "f16": CONV_F16, "bf16": CONV_BF16}[dtype]
    bn, st, ct = (ctypes.c_int * 1)(), (ctypes.c_int * 1)(), (ctypes.c_int * 1)()
    v = lib().conv_plan_ex(N, D, H, W, C, O, *k, _i3(stride), _i3(pad), _i3(pad if pad_hi is None else pad_hi),
                           _i3(dil), int(groups), int(flip), code, int(variant), bn, st, ct)
    if v < 0:
        raise ConvError(v, "conv_plan_variant")
    return v, bn[0], st[0], ct[0]


def inject_stall(timeout_ns: int) -> None:
    """Test hook: the next tensor-core launch times out after `timeout_ns` on purpose."""
    rc = lib().conv_debug_inject_stall(int(timeout_ns))
    if rc:
        raise ConvError(rc, "conv_debug_inject_stall")


def last_status(stream=None) -> int:
    """Wait for the stream, then read and clear the device status word (0 = ok)."""
    import torch
    st = stream if stream is not None else torch.cuda.current_stream()
    return int(lib().conv_last_status(st.cuda_stream))
