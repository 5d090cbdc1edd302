"""dB and dA beside the dX GEMM (qlora_set_side_overlap), against the serial path and the oracle.

When the dX GEMM runs whole tiles, the backward can run dB = s dY^T XA and dA = s dYB^T X on
a few SMs taken from it (qlora_backward_side_sms) while it runs on the rest, from a stream the
library forks after dY B and joins before the call returns.  The side kernel sums every reduction in the cluster kernels' step ranges and order,
so checked here through the C ABI:
* mode 2 (beside the GEMM whenever it runs whole tiles) gives the bits of mode 0 (serial) for dX, dA and dB,
  single adapter (dB and dA in one side launch) and packed adapters (two side launches, dB with
  r columns per adapter, dA with n r), ragged token counts and ranks 16 to 64;
* the outputs meet the parity bar against the oracle (max|err| / max|ref| <= 2e-2);
* the shapes do take the side path on this device (qlora_backward_side_sms > 0 in mode 2);
* a CUDA-graph capture of the backward (fork and join captured as graph edges) replays to the
  same bits, twice.
"""

import numpy as np
import pytest
import torch

import parity
from nf4_base_lora_blockwise_b200 import abi, linear, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    prev = abi.qlora_set_side_overlap(1)
    yield
    abi.qlora_set_side_overlap(prev)


def _spare(M, K, N, R):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return abi.qlora_backward_side_sms(M, N, K, R, sms, 2)


def _bwd(mode, dY, X, w, A, B, XA, alpha, Ns=None):
    abi.qlora_set_side_overlap(mode)
    if Ns is None:
        out = linear.backward(dY, X, w, A, B, XA, alpha)
    else:
        out = linear.grouped_backward(dY, X, w, A, B, XA, list(Ns), alpha)
    torch.cuda.synchronize()
    assert linear.device_error() == 0
    return out


def _same(a, b):
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("M,K,N,r", [
    (4096, 4096, 1024, 16),
    (3000, 4096, 1024, 16),   # ragged last token tile
    (3000, 4096, 1024, 64),
])
def test_side_matches_serial(M, K, N, r):
    if _spare(M, K, N, r) == 0:
        pytest.skip("the dX GEMM does not run whole tiles for this shape on this device")
    inp, L = parity.make(M, K, N, r, seed=M + r, dy_std=1.0)
    lin = inp["linears"][0]
    X, dY = inp["X"].cuda(), inp["dY"].cuda()
    A, B = lin["A"].cuda(), lin["B"].cuda()
    w = linear.nf4_pack(lin["W0"].cuda())
    H, XA = linear.forward(X, w, A, B, L.alpha)
    serial = _bwd(0, dY, X, w, A, B, XA, L.alpha)
    side = _bwd(2, dY, X, w, A, B, XA, L.alpha)
    _same(serial, side)
    rows = np.concatenate([np.arange(0, M, 97), [M - 1]])
    parity.check_linear(inp, L, {"H": H, "XA": XA, "dX": side[0], "dA": side[1], "dB": side[2]},
                        rows=rows)


def test_side_packed_adapters():
    Ns, r, M, K = (2048, 1024), 16, 4096, 4096
    if _spare(M, K, sum(Ns), len(Ns) * r) == 0:
        pytest.skip("the dX GEMM does not run whole tiles for this shape on this device")
    inp = synth.make_grouped(M, K, list(Ns), r, seed=7, dy_std=1.0)
    alpha = 2.0 * r
    W0, A, B = parity.stacked(inp)
    X, dY = inp["X"].cuda(), inp["dY"].cuda()
    A, B = A.cuda(), B.cuda()
    w = linear.nf4_pack(W0.cuda())
    H, XA = linear.grouped_forward(X, w, A, B, list(Ns), alpha)
    serial = _bwd(0, dY, X, w, A, B, XA, alpha, Ns)
    side = _bwd(2, dY, X, w, A, B, XA, alpha, Ns)
    _same(serial, side)
    rows = np.concatenate([np.arange(0, M, 127), [M - 1]])
    parity.check_grouped(inp, Ns, alpha,
                         {"H": H, "XA": XA, "dX": side[0], "dA": side[1], "dB": side[2]},
                         rows=rows)


def test_side_in_a_graph():
    M, K, N, r = 4096, 4096, 1024, 16
    if _spare(M, K, N, r) == 0:
        pytest.skip("the dX GEMM does not run whole tiles for this shape on this device")
    inp, L = parity.make(M, K, N, r, seed=11, dy_std=1.0)
    lin = inp["linears"][0]
    X, dY = inp["X"].cuda(), inp["dY"].cuda()
    A, B = lin["A"].cuda(), lin["B"].cuda()
    w = linear.nf4_pack(lin["W0"].cuda())
    H, XA = linear.forward(X, w, A, B, L.alpha)
    ref = _bwd(0, dY, X, w, A, B, XA, L.alpha)
    abi.qlora_set_side_overlap(2)
    dX = torch.empty_like(ref[0])
    dA = torch.empty_like(ref[1])
    dB = torch.empty_like(ref[2])
    ws = linear.alloc_workspace(M, N, K, r, "cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):  # eager once on the capture stream (creates the side stream)
        linear.backward(dY, X, w, A, B, XA, L.alpha, dX=dX, dA=dA, dB=dB, ws=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s, capture_error_mode="relaxed"):
        linear.backward(dY, X, w, A, B, XA, L.alpha, dX=dX, dA=dA, dB=dB, ws=ws)
    for _ in range(2):
        dX.fill_(float("nan"))
        dA.fill_(float("nan"))
        dB.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert linear.device_error() == 0
        _same(ref, (dX, dA, dB))
    del g
