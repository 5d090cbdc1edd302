"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the same seeded inputs.

Bit-exact for the packed codes, absmax (and double-quant codes / scales) and the dequantised
weight; max|err| / max|ref| <= 2e-2 for h, XA, dX, dA and dB.  Shapes span several tiles in
every dimension plus ragged token tails and the degenerate cases of the method.
"""

import numpy as np
import pytest
import torch

import parity
from nf4_base_lora_blockwise_b200 import linear, synth
from oracle import nf4, qlora

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


# ------------------------------------------------------------------------------------------
# NF4 pack / dequant: bit-exact
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("dq", [False, True])
@pytest.mark.parametrize("N,K", [(512, 256), (384, 640), (64, 64 * 41)])
def test_pack_and_dequant_bit_exact(N, K, dq):
    inp, _ = parity.make(4, K, N, 8, seed=N + K)
    W = inp["linears"][0]["W0"]
    wg = parity.gpu_pack(W, dq)
    parity.check_pack(wg, parity.oracle_pack(W, dq), dq)


def test_pack_degenerate_blocks():
    """All-zero blocks (code 7, +0.0), constant blocks (all 0 or all 15), exact midpoints,
    and the codebook round trip, through the GPU quantiser."""
    c32 = nf4.codebook_f32()
    m32 = nf4.midpoints_f32()
    W = np.zeros((64, 256), np.float32)
    W[1, :64] = 0.25
    W[2, 64:128] = -0.5
    W[3, :16] = c32 * np.float32(0.125)     # exact in bf16 after scaling? rounded below
    W[3, 16] = 0.125
    W[4, :15] = m32                           # x exactly on midpoints (absmax 1 below)
    W[4, 15] = 1.0
    Wt = torch.from_numpy(W).to(torch.bfloat16)
    for dq in (False, True):
        wg = parity.gpu_pack(Wt, dq)
        ref = parity.oracle_pack(Wt, dq)
        parity.check_pack(wg, ref, dq)
        codes = nf4.unpack_codes(wg.q.cpu().numpy())
        assert np.all(codes[0] == 7)
        assert np.all(codes[1, :64] == 15) and np.all(codes[2, 64:128] == 0)


# ------------------------------------------------------------------------------------------
# Forward + backward: tolerance
# ------------------------------------------------------------------------------------------
def test_tiny_workload_all_rows():
    """The tiny single-layer workload: in 256, out 512, r 8, alpha 16, 64 tokens."""
    w = synth.workload("tiny")
    inp = synth.make_inputs(w, seed=0)
    L = w.linears[0]
    got = parity.run_linear(inp, L)
    parity.check_pack(got["w"], parity.oracle_pack(inp["linears"][0]["W0"], False), False)
    parity.check_linear(inp, L, got)


@pytest.mark.parametrize(
    "M,K,N,r,dq",
    [
        (300, 512, 384, 16, False),   # 2 token tiles (ragged), 3 row tiles, 8 k-steps
        (1, 256, 256, 16, False),     # single token
        (17, 384, 640, 8, False),     # ragged small M, r padded to 16 in the MMA
        (200, 320, 192, 64, True),    # double-quant absmax, odd K/64 and N/64 tile tails
        (96, 256, 128, 128, False),   # r = 128: two extension chunks
        (40, 192, 320, 72, False),    # r = 72: odd rank tile count, 80-wide extension
        (512, 1024, 512, 32, False),  # 2 full token tiles
    ],
)
def test_linear_parity(M, K, N, r, dq):
    inp, L = parity.make(M, K, N, r, seed=M * 7 + K, dy_std=1.0)
    got = parity.run_linear(inp, L, dq=dq)
    parity.check_linear(inp, L, got, dq=dq)


def test_no_dx_path():
    inp, L = parity.make(64, 256, 512, 16, seed=3)
    got = parity.run_linear(inp, L, need_dx=False)
    assert got["dX"] is None
    parity.check_linear(inp, L, got)


def test_B_zero_gives_base_product():
    inp, L = parity.make(130, 256, 256, 16, seed=5)
    inp["linears"][0]["B"].zero_()
    got = parity.run_linear(inp, L)
    _, Wd = parity.oracle_deq(inp["linears"][0]["W0"], False)
    ref = parity.f32(inp["X"]).astype(np.float64) @ Wd.T.astype(np.float64)
    assert qlora.rel_err(parity.f32(got["H"]), ref) <= parity.TOL
    assert np.all(parity.f32(got["dA"]) == 0)


def test_W0_zero_gives_lora_only():
    inp, L = parity.make(70, 256, 192, 16, seed=6)
    inp["linears"][0]["W0"].zero_()
    got = parity.run_linear(inp, L)
    codes = nf4.unpack_codes(got["w"].q.cpu().numpy())
    assert np.all(codes == 7)
    X, A, B = (parity.f32(inp["X"]).astype(np.float64), parity.f32(inp["linears"][0]["A"]),
               parity.f32(inp["linears"][0]["B"]))
    ref = (L.alpha / L.r) * (X @ A.T.astype(np.float64)) @ B.T.astype(np.float64)
    assert qlora.rel_err(parity.f32(got["H"]), ref) <= parity.TOL


def test_repeat_calls_deterministic():
    inp, L = parity.make(257, 512, 256, 16, seed=9)
    a = parity.run_linear(inp, L)
    b = parity.run_linear(inp, L)
    for k in ("H", "XA", "dX", "dA", "dB"):
        assert torch.equal(a[k], b[k]), k


def test_swiglu_parity():
    g = torch.randn(3, 1000, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    u = torch.randn(3, 1000, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    da = torch.randn(3, 1000, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    a = linear.swiglu_forward(g.cuda(), u.cuda())
    dg, du = linear.swiglu_backward(g.cuda(), u.cuda(), da.cuda())
    torch.cuda.synchronize()
    fg, fu, fd = parity.f32(g), parity.f32(u), parity.f32(da)
    assert qlora.rel_err(parity.f32(a), qlora.swiglu_forward(fg, fu)) <= 1e-2
    rg, ru = qlora.swiglu_backward(fg, fu, fd)
    assert qlora.rel_err(parity.f32(dg), rg) <= 1e-2
    assert qlora.rel_err(parity.f32(du), ru) <= 1e-2


@pytest.mark.parametrize("M,K,N,r", [(300, 512, 384, 16), (9, 256, 256, 16), (2048, 256, 2048, 16)])
def test_recompute_xa_is_bit_identical(M, K, N, r):
    """Recompute instead of store: with no saved XA the backward recomputes X A^T with the
    forward's own kernel, so every gradient equals the saving path's bit for bit."""
    inp, L = parity.make(M, K, N, r, seed=M + 5, dy_std=1.0)
    lin = inp["linears"][0]
    X, dY, A, B = (inp["X"].cuda(), inp["dY"].cuda(), lin["A"].cuda(), lin["B"].cuda())
    w = linear.nf4_pack(lin["W0"].cuda())
    H, XA = linear.forward(X, w, A, B, L.alpha)
    H2, none = linear.forward(X, w, A, B, L.alpha, save_xa=False)
    assert none is None
    saved = linear.backward(dY, X, w, A, B, XA, L.alpha)
    recomputed = linear.backward(dY, X, w, A, B, None, L.alpha)
    torch.cuda.synchronize()
    assert linear.device_error() == 0
    assert torch.equal(H, H2)
    for a, b, k in zip(saved, recomputed, ("dX", "dA", "dB")):
        assert torch.equal(a, b), k


@pytest.mark.parametrize(
    "M,K,N,r,dq",
    [
        (64, 256, 512, 1, False),      # r = 1: padded to 8
        (17, 384, 640, 4, False),      # few-token forward and dX
        (300, 512, 384, 12, True),     # stream-K, double-quant
        (2048, 256, 2048, 100, False), # whole tiles, r = 100 -> 104
        (96, 256, 128, 127, False),    # r = 127 -> 128: two extension chunks
    ],
)
def test_linear_parity_any_rank(M, K, N, r, dq):
    """Ranks that are not multiples of 8 (the C ABI takes 1 <= r <= 128): the layer runs at r
    rounded up to 8 on zero-padded copies of A, B and XA, and hands back [M, r] / [r, K] /
    [N, r] results; same bar against the oracle."""
    inp, L = parity.make(M, K, N, r, seed=M * 5 + r, dy_std=1.0)
    got = parity.run_linear(inp, L, dq=dq)
    assert got["XA"].shape == (M, r) and got["dA"].shape == (r, K) and got["dB"].shape == (N, r)
    parity.check_linear(inp, L, got, dq=dq)


def test_any_rank_recompute_matches_saved():
    """r = 12 with XA_saved NULL: the backward recomputes X A^T (into the padded copy) and gives
    the same gradients bit for bit."""
    inp, L = parity.make(200, 256, 384, 12, seed=77, dy_std=1.0)
    lin = inp["linears"][0]
    X, dY, A, B = inp["X"].cuda(), inp["dY"].cuda(), lin["A"].cuda(), lin["B"].cuda()
    w = linear.nf4_pack(lin["W0"].cuda())
    H, XA = linear.forward(X, w, A, B, L.alpha)
    saved = linear.backward(dY, X, w, A, B, XA, L.alpha)
    H2, none = linear.forward(X, w, A, B, L.alpha, save_xa=False)
    recomputed = linear.backward(dY, X, w, A, B, None, L.alpha)
    torch.cuda.synchronize()
    assert none is None and torch.equal(H, H2)
    for a, b in zip(saved, recomputed):
        assert torch.equal(a, b)
