"""The rank-r down-projections computed inside the dequant GEMM launches, against the oracle.

With qlora_set_rank_fusion(1), when a GEMM runs whole tiles of two halves of 144..240 tokens and the packed rank n r is at most
32 (dX: r = 16 or 32), the forward launch computes X A^T and the dX launch computes dY B_bd on
the tensor cores, from the activation tiles it streams anyway: each token tile's first tiles add
M = 128 MMAs for one 128-token window each, the epilogue publishes the window per token tile, and
every tile's extension step waits for its token tile's windows.  Checked here, through the C
ABI, with the same bar as every parity test (max|err| / max|ref| <= 2e-2 for h, XA, dX, dA, dB):
* that the fused launch ran (one kernel for the forward instead of two);
* 144- and 176-token halves (overlapping windows) and a ragged last token tile whose second
  half holds fewer than 128 tokens (one window);
* ranks 8, 16, 24, 32 in the forward (rank tile zero-filled to 16 or 32 rows), 16 and 32 in dX
  (the MN-major rank-operand tile);
* packed adapters in the forward (dense [M, n r]) and in dX (block-diagonal B);
* repeat calls bit for bit.
"""

import pytest
import torch

import parity
from nf4_base_lora_blockwise_b200 import abi, linear, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    prev = abi.qlora_set_rank_fusion(True)  # opt-in; restored after each test
    yield
    abi.qlora_set_rank_fusion(prev)


def _fused(M, rows_w, steps, R, r, trans):
    """Whether this GEMM launch fuses its down-projection on this device."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return abi.qlora_gemm_rank_fusable(M, rows_w, steps, sms, R, r, trans) > 0


def _fwd_launches(X, w, A, B, alpha, group_rows=None):
    torch.cuda.synchronize()
    n0 = abi.qlora_launch_counter()
    if group_rows is None:
        H, XA = linear.forward(X, w, A, B, alpha)
    else:
        H, XA = linear.grouped_forward(X, w, A, B, list(group_rows), alpha)
    torch.cuda.synchronize()
    return H, XA, abi.qlora_launch_counter() - n0


@pytest.mark.parametrize("M,K,N,r", [
    (774, 768, 10240, 16),   # 144-token halves, 80 row tiles x 3 token tiles, the last 198 tokens
    (774, 768, 10240, 8),    # rank tile zero-filled from 8 to 16 rows
    (774, 768, 10240, 24),   # ... from 24 to 32
    (774, 768, 10240, 32),
    (1300, 1024, 8192, 16),  # 176-token halves
])
def test_fused_forward(M, K, N, r):
    assert _fused(M, N, K // 64 + 1, r, r, False)
    inp, L = parity.make(M, K, N, r, seed=M + r, dy_std=1.0)
    lin = inp["linears"][0]
    X, A, B = inp["X"].cuda(), lin["A"].cuda(), lin["B"].cuda()
    w = linear.nf4_pack(lin["W0"].cuda())
    H, XA, n = _fwd_launches(X, w, A, B, L.alpha)
    assert n == 1, "the forward should run as one fused launch"
    assert linear.device_error() == 0
    H2, XA2, _ = _fwd_launches(X, w, A, B, L.alpha)
    assert torch.equal(H, H2) and torch.equal(XA, XA2)
    dX, dA, dB = linear.backward(inp["dY"].cuda(), X, w, A, B, XA, L.alpha)
    torch.cuda.synchronize()
    assert linear.device_error() == 0
    got = {"H": H, "XA": XA, "dX": dX, "dA": dA, "dB": dB}
    parity.check_linear(inp, L, got)


@pytest.mark.parametrize("M,K,N,r", [
    (774, 10240, 768, 16),   # dX: 80 row tiles (input features) x 3 token tiles
    (774, 10240, 768, 32),
    (1300, 8192, 1024, 16),
])
def test_fused_dx(M, K, N, r):
    assert _fused(M, K, N // 64 + 1, r, r, True)
    inp, L = parity.make(M, K, N, r, seed=M + K + r, dy_std=1.0)
    got = parity.run_linear(inp, L)
    parity.check_linear(inp, L, got)
    # Repeat the backward: bit for bit.
    lin = inp["linears"][0]
    X, dY = inp["X"].cuda(), inp["dY"].cuda()
    A, B = lin["A"].cuda(), lin["B"].cuda()
    XA = got["XA"].cuda()
    a = linear.backward(dY, X, got["w"], A, B, XA, L.alpha)
    b = linear.backward(dY, X, got["w"], A, B, XA, L.alpha)
    torch.cuda.synchronize()
    assert linear.device_error() == 0
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_fused_grouped_forward():
    """Two adapters (packed rank 32) on 10240 rows: the fused forward computes the dense
    [M, 2 r] XA for both."""
    M, K, Ns, r = 774, 768, (5120, 5120), 16
    inp = synth.make_grouped(M, K, Ns, r, seed=5, dy_std=1.0)
    W0, A, B = parity.stacked(inp)
    X = inp["X"].cuda()
    w = linear.nf4_pack(W0.cuda())
    H, XA, n = _fwd_launches(X, w, A.cuda(), B.cuda(), 2.0 * r, group_rows=Ns)
    assert n == 1
    dX, dA, dB = linear.grouped_backward(inp["dY"].cuda(), X, w, A.cuda(), B.cuda(), XA,
                                         list(Ns), 2.0 * r)
    torch.cuda.synchronize()
    assert linear.device_error() == 0
    parity.check_grouped(inp, Ns, 2.0 * r, {"H": H, "XA": XA, "dX": dX, "dA": dA, "dB": dB})


@pytest.mark.parametrize("Ns,r", [((384, 384), 16)])
def test_fused_grouped_dx(Ns, r):
    """dX with adapters along N: dY B_bd takes, for each 64-column step of dY, only its
    adapter's r columns of the output (TMEM columns g r .. g r + r - 1 of the window)."""
    M, K = 774, 10240
    assert _fused(M, K, sum(Ns) // 64 + 1, len(Ns) * r, r, True)
    inp = synth.make_grouped(M, K, Ns, r, seed=6, dy_std=1.0)
    got = parity.run_grouped(inp, Ns, 2.0 * r)
    parity.check_grouped(inp, Ns, 2.0 * r, got)


def test_separate_by_default():
    """Off (the default), the same forward runs the down-projection as a launch of its own."""
    abi.qlora_set_rank_fusion(False)
    M, K, N, r = 774, 768, 10240, 16
    inp, L = parity.make(M, K, N, r, seed=3, dy_std=1.0)
    lin = inp["linears"][0]
    X, A, B = inp["X"].cuda(), lin["A"].cuda(), lin["B"].cuda()
    w = linear.nf4_pack(lin["W0"].cuda())
    H, XA, n = _fwd_launches(X, w, A, B, L.alpha)
    assert n == 2
    abi.qlora_set_rank_fusion(True)
    H2, XA2, n2 = _fwd_launches(X, w, A, B, L.alpha)
    assert n2 == 1
    assert linear.device_error() == 0
    # Same inputs, other summation order: within a few bf16 ulps of each other.
    assert (H.float() - H2.float()).abs().max().item() <= 2e-2 * H.float().abs().max().item()
    assert (XA.float() - XA2.float()).abs().max().item() <= 2e-2 * XA.float().abs().max().item()
