"""The product path's boundary on the CPU: no fallback, no shared code with the oracle.

The library and its binding must fail loudly rather than compute anywhere but in
the CUDA kernels, and the checker (oracle/) must stay independent of what it
checks: neither side imports, includes or links the other.
"""
from __future__ import annotations

import os
import re
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "implicit_gemm_convolution_conv2d_b200")
PKG_NAME = "implicit_gemm_convolution_conv2d_b200"


def _files(top, exts):
    for d, _, names in os.walk(top):
        if "__pycache__" in d:
            continue
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def test_tensor_entry_points_refuse_cpu_tensors():
    import implicit_gemm_convolution_conv2d_b200 as cf
    x = torch.zeros(1, 4, 4, 4, 8, dtype=torch.float16)
    w = torch.zeros(8, 3, 3, 3, 8, dtype=torch.float16)
    with pytest.raises(ValueError, match="CUDA"):
        cf.conv_fwd(x, w, padding=1)
    with pytest.raises(ValueError, match="CUDA"):
        cf.conv_transpose(x, w.transpose(0, 4).contiguous(), padding=1)
    with pytest.raises(ValueError, match="CUDA"):
        cf.conv_wgrad(x, x, (3, 3, 3), padding=1)


def test_missing_library_raises():
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "import implicit_gemm_convolution_conv2d_b200 as cf\n"
        "cf.LIB_PATH = '/nonexistent/libconvfwd.so'; cf._lib = None\n"
        "try:\n"
        "    cf.out_dims(1, 8, 8, 1, 3, 3, 1, 1, 1)\n"
        "except ImportError as e:\n"
        "    print('raised', 'libconvfwd.so' in str(e))\n"
        "else:\n"
        "    print('returned')\n" % ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert out.stdout.strip() == "raised True", out.stdout + out.stderr


def test_product_sources_never_reach_the_oracle():
    pat = re.compile(r"^\s*(import\s+oracle|from\s+oracle|#\s*include\s+[<\"][^>\"]*(oracle|conv_ref))", re.M)
    for path in list(_files(PKG, (".py", ".cu", ".cuh", ".h", ".c"))) + list(_files(os.path.join(ROOT, "include"),
                                                                                  (".h",))):
        with open(path) as f:
            assert not pat.search(f.read()), path


def test_oracle_never_reaches_the_product():
    pat = re.compile(r"(%s|libconvfwd|conv_fwd\.h|csrc)" % PKG_NAME)
    for path in _files(os.path.join(ROOT, "oracle"), (".py", ".c", ".h")):
        with open(path) as f:
            assert not pat.search(f.read()), path
