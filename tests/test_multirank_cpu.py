"""The benchmark's multi-rank plumbing on CPU (gloo, world size 2).

The forward convolution shards over independent batches with no data-path
collective; what ranks share is only the timing: a barrier around the timed
region and the maximum of the per-rank device times.  This checks that logic
with two gloo processes.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    ws, r, local = bench.dist_env()
    assert (ws, r, local) == (world, rank, rank)
    d = bench.init_dist(ws, "gloo")
    bench.barrier(d)
    local_ms = 10.0 * (rank + 1)                 # rank 1 is the slow one
    ms, n = bench.aggregate(d, local_ms)
    out[rank] = (ms, n)
    d.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_max_time_gloo():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(100)
        assert p.exitcode == 0
    assert out[0] == (20.0, 2) and out[1] == (20.0, 2)


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.init_dist(1, "gloo") is None
    assert bench.aggregate(None, 3.5) == (3.5, 1)


def test_flop_and_byte_counters_match_the_tutorial():
    """The bench's FLOP and byte counters against the printed figures of the
    "Convolutions" tutorial (golden fixture): 236 MFLOP for the ResNet-50 stem,
    3.7 GFLOP / 4.4 MB / 841 FLOP per byte for the 3x3 256->256 layer."""
    import json
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import workloads as WL
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "tutorial_counts.json")))
    st = g["stem"]
    wl = WL.case(1, 1, st["H"], st["W"], st["C"], st["O"], (1, st["k"], st["k"]), (1, st["stride"], st["stride"]),
                 (0, st["pad"], st["pad"]), dtype="bf16")
    dims = (1, st["H_out"], st["W_out"])
    f = bench.conv_flops(wl, dims)
    assert f == 2 * 112 * 112 * 3 * 64 * 7 * 7
    assert abs(f / st["flops_printed"] - 1) < st["flops_rel_tol"]
    c3 = g["conv3x3_256"]
    wl = WL.case(1, 1, c3["H"], c3["W"], c3["C"], c3["O"], (1, 3, 3), pad=(0, 1, 1), dtype="bf16")
    dims = (1, 56, 56)
    f = bench.conv_flops(wl, dims)
    xb, wb, yb = bench.conv_bytes(wl, dims)
    assert abs(f / c3["flops_printed"] - 1) < c3["flops_rel_tol"]
    for got, key in ((xb, "x_bytes_printed"), (wb, "w_bytes_printed"), (yb, "y_bytes_printed"),
                     (xb + wb + yb, "bytes_printed")):
        assert abs(got / c3[key] - 1) < c3["bytes_rel_tol"], (key, got)
    assert abs(f / (xb + wb + yb) / c3["intensity_printed"] - 1) < c3["intensity_rel_tol"]


def test_kernel_source_sets_cover_every_kernel():
    """Every kernel name a bench line can report has the list of source files
    its traffic record is keyed on, and those files exist."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import implicit_gemm_convolution_conv2d_b200 as C
    names = set(C.VARIANT_NAMES.values()) | set(C.WGRAD_PATH_NAMES.values())
    csrc = os.path.join(ROOT, "implicit_gemm_convolution_conv2d_b200", "csrc")
    for name in names:
        assert name in bench.KERNEL_SOURCES, name
        for f in bench.KERNEL_SOURCES[name]:
            assert os.path.exists(os.path.join(csrc, f)), (name, f)
        assert len(bench.kernel_source_hash(name)) == 12


def test_kernel_source_sets_are_closed_under_includes():
    """A kernel's traffic record must go stale when any header its code pulls in
    changes: every local header included by a header of the set is in the set
    (the two .cu files, which include every kernel, are the host side and are
    not followed)."""
    import re
    import sys
    sys.path.insert(0, ROOT)
    import bench
    csrc = os.path.join(ROOT, "implicit_gemm_convolution_conv2d_b200", "csrc")
    for name, files in bench.KERNEL_SOURCES.items():
        for f in files:
            if not f.endswith(".cuh"):
                continue
            with open(os.path.join(csrc, f)) as fh:
                for inc in re.findall(r'^#include "([^"]+\.cuh)"', fh.read(), re.M):
                    assert inc in files, (name, f, inc)


def test_transposed_and_weight_gradient_counters():
    """A transposed convolution counts the FLOPs of the forward pass it is the
    adjoint of (2 x its input pixels x Cin x taps x Cout/G); the weight
    gradient counts those of the forward pass."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import workloads as WL
    t = WL.WORKLOADS["convT_bf16_n16_56x56_c256_o128_k4s2"]
    assert bench.conv_flops(t) == 2 * 16 * 56 * 56 * 256 * 16 * 128
    g = WL.WORKLOADS["wgrad_bf16_n64_56x56_c256_o256_k3"]
    assert bench.conv_flops(g, (1, 56, 56)) == 2 * 64 * 56 * 56 * 256 * 9 * 256


@pytest.mark.timeout(300)
def test_reference_arm_loads_only_the_oracle():
    """`bench.py --impl reference` times the oracle and must not map the CUDA
    library into its process: after a short run, /proc/self/maps holds
    liboracle.so and no libconvfwd.so; its line carries the CPU model."""
    import json
    import subprocess
    import sys
    code = ("import sys, json; sys.argv = ['bench.py', '--impl', 'reference', '--steps', '1', '--warmup', '3', "
            "'--workload', 'conv2d_f16_n1_56x56_c64_o64_k3']; sys.path.insert(0, %r); import bench; bench.main(); "
            "m = open('/proc/self/maps').read(); "
            "print(json.dumps({'oracle': 'liboracle.so' in m, 'product': 'libconvfwd.so' in m}))" % ROOT)
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=280)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(ln) for ln in r.stdout.splitlines() if ln.startswith("{")]
    line, maps = lines[0], lines[-1]
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert "cpu_model" in line["cpu_baseline"]
    assert maps == {"oracle": True, "product": False}
    # the rest of the line's contract
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "e2e", "cpu_baseline"):
        assert key in line, key
    assert line["value"] > 0 and line["ms_per_step"] > 0 and line["steps"] == 1 and line["warmup"] >= 3
    assert line["higher_is_better"] is True and line["unit"] == "TFLOP/s" and line["vs_baseline"] is None
    assert line["config"]["workload"] == "conv2d_f16_n1_56x56_c64_o64_k3" and "sample" in line["config"]
    cb = line["cpu_baseline"]
    assert cb["value"] == line["value"] and cb["unit"] == line["unit"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
