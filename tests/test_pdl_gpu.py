"""Back-to-back dependent launches (needs a B200).

Every kernel of the library is launched with programmatic stream
serialization: it may start its setup while the kernel before it on the
stream is still running, and waits for that kernel's writes before it reads
or writes global memory.  These tests run chains of convolutions where each
layer reads the output of the one before, queued back to back on one stream
and captured in a CUDA graph, and require the results to be bit-identical to
the same chain run one launch at a time with the device synchronised between
launches (every kernel here sums in a fixed order, so the results are
deterministic).  The parity of each kernel against the oracle is covered by
the other GPU tests.
"""
from __future__ import annotations

import pytest
import torch

pytestmark = pytest.mark.gpu

C = pytest.importorskip("implicit_gemm_convolution_conv2d_b200")

DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert C.last_status() == 0


# name: (x shape NDHWC, dtype, layers); a layer is (O, kernel, stride, pad, groups, variant name)
CHAINS = {
    "pair_2d_256": ((2, 1, 20, 20, 256), "bf16",
                    [(256, (1, 3, 3), 1, (0, 1, 1), 1, "TC_TMA_PAIR")] * 3),
    "tma_single_2d": ((2, 1, 18, 18, 64), "f16",
                      [(64, (1, 3, 3), 1, (0, 1, 1), 1, "TC_TMA"), (128, (1, 3, 3), 2, (0, 1, 1), 1, "TC_TMA"),
                       (128, (1, 1, 1), 1, (0, 0, 0), 1, "TC_TMA")]),
    "halo_t_3d": ((2, 6, 12, 16, 128), "f16",
                  [(128, (3, 3, 3), 1, (1, 1, 1), 1, "TC_HALO_T")] * 3),
    "halo_plain_2d": ((2, 1, 24, 16, 64), "bf16",
                      [(64, (1, 3, 3), 1, (0, 1, 1), 1, "TC_HALO")] * 3),
    "tma_t_3d": ((2, 4, 16, 16, 64), "f16",
                 [(128, (3, 3, 3), 1, (1, 1, 1), 1, "TC_TMA_T"), (128, (1, 1, 1), 1, (0, 0, 0), 1, "TC_TMA_T")]),
    "gather_unaligned": ((2, 6, 8, 8, 21), "f16",
                         [(21, (3, 3, 3), 1, (1, 1, 1), 1, "TC_GATHER")] * 3),
    "stem_then_tma": ((2, 1, 32, 32, 3), "bf16",
                      [(64, (1, 7, 7), 2, (0, 3, 3), 1, "TC_PHASE"), (64, (1, 3, 3), 1, (0, 1, 1), 1, "TC_TMA")]),
    "simt_f32": ((2, 4, 10, 10, 24), "f32",
                 [(24, (3, 3, 3), 1, (1, 1, 1), 1, "SIMT")] * 3),
    "depthwise": ((2, 1, 28, 28, 64), "f16",
                  [(64, (1, 3, 3), 1, (0, 1, 1), 64, "DEPTHWISE")] * 3),
}


def _weights(x_ch, layers, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    ws, c = [], x_ch
    for O, k, _s, _p, G, _v in layers:
        fan = (c // G) * k[0] * k[1] * k[2]
        ws.append((torch.randn((O, *k, c // G), generator=g) / fan ** 0.5).to(DT[dtype]).cuda())
        c = O
    return ws


def _layer(h, w, layer, out=None):
    O, k, s, p, G, v = layer
    return C.conv_fwd(h, w, stride=s, padding=p, groups=G, variant=getattr(C, "VARIANT_" + v), out=out)


@pytest.mark.parametrize("name", sorted(CHAINS))
def test_dependent_chain_matches_synchronised_launches(name):
    shape, dtype, layers = CHAINS[name]
    g = torch.Generator().manual_seed(11)
    x = ((torch.rand(shape, generator=g) * 2 - 1).to(DT[dtype])).cuda()
    ws = _weights(shape[-1], layers, dtype, 12)
    # one launch at a time, the device synchronised after each
    ref, h = [], x
    for w, layer in zip(ws, layers):
        h = _layer(h, w, layer)
        torch.cuda.synchronize()
        ref.append(h.clone())
    assert C.last_status() == 0
    outs = [torch.empty_like(r) for r in ref]

    def chain():
        h = x
        for w, layer, o in zip(ws, layers, outs):
            o.zero_()
            h = _layer(h, w, layer, out=o)

    # back to back on one stream
    for _ in range(2):
        chain()
    torch.cuda.synchronize()
    for i, (o, r) in enumerate(zip(outs, ref)):
        assert torch.equal(o, r), f"{name}: layer {i} differs when queued back to back"
    # captured in a CUDA graph and replayed
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        chain()
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(3):
            chain()
    for _ in range(2):
        for o in outs:
            o.fill_(0)
        graph.replay()
        torch.cuda.synchronize()
        for i, (o, r) in enumerate(zip(outs, ref)):
            assert torch.equal(o, r), f"{name}: layer {i} differs in a graph replay"
    del graph
    assert C.last_status() == 0


def test_weight_gradient_after_forward_in_one_graph():
    """The weight gradient (range kernel, then ordered sum) consumes a forward
    output produced by the launch just before it."""
    g = torch.Generator().manual_seed(5)
    x = ((torch.rand((2, 1, 16, 16, 256), generator=g) * 2 - 1).bfloat16()).cuda()
    w = (torch.randn((256, 1, 3, 3, 256), generator=g) / 48).bfloat16().cuda()
    y = C.conv_fwd(x, w, padding=(0, 1, 1))
    dw_ref = C.conv_wgrad(x, y, (1, 3, 3), padding=(0, 1, 1))
    torch.cuda.synchronize()
    dw = torch.empty_like(dw_ref)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        y2 = C.conv_fwd(x, w, padding=(0, 1, 1))
        C.conv_wgrad(x, y2, (1, 3, 3), padding=(0, 1, 1), out=dw)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        y2.zero_()
        C.conv_fwd(x, w, padding=(0, 1, 1), out=y2)
        C.conv_wgrad(x, y2, (1, 3, 3), padding=(0, 1, 1), out=dw)
    dw.fill_(0)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(dw, dw_ref)
    del graph
    assert C.last_status() == 0
