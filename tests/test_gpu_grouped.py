"""GPU parity of the packed-adapter layer (several LoRA adapters along the rows of one stacked
NF4 weight, sharing X) against the oracle, through the C ABI.

Same bar as the single layer: max|err| / max|ref| <= 2e-2 for h, XA, dX, dA and dB, checked
over the whole packed output and per adapter.  Cases cover:
* stream-K and whole-tile forward schedules;
* the few-token forward (M <= 32);
* ragged token tails;
* double-quantised absmax;
* ranks that are not multiples of 16;
* a packed rank of 128 (two dX extension chunks);
* eight adapters.
"""

import numpy as np
import pytest
import torch

import parity
from nf4_base_lora_blockwise_b200 import linear, synth
from oracle import qlora

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize(
    "M,K,Ns,r,dq",
    [
        (300, 512, (256, 128, 128), 16, False),   # q/k/v-like, stream-K, ragged tokens
        (5, 256, (256, 128, 128), 16, False),     # few-token forward
        (32, 384, (384, 256), 16, False),         # few-token forward at its largest M
        (200, 384, (384, 256), 64, True),         # double-quant; packed rank 128: 2 dX chunks
        (130, 256, (128,) * 8, 8, False),         # eight adapters
        (96, 320, (128, 256, 128), 24, False),    # r = 24: columns not on 16-element bounds
        (2048, 256, (2048, 1536, 1536), 16, False),  # 160 tiles: whole-tile forward schedule
    ],
)
def test_grouped_parity(M, K, Ns, r, dq):
    inp = synth.make_grouped(M, K, Ns, r, seed=M + K + len(Ns), dy_std=1.0)
    alpha = 2.0 * r
    got = parity.run_grouped(inp, Ns, alpha, dq=dq)
    parity.check_grouped(inp, Ns, alpha, got, dq=dq)


def test_grouped_one_adapter_matches_single_layer_bitwise():
    """One adapter through the packed entry points runs the single layer's launches."""
    inp = synth.make_grouped(257, 512, (384,), 16, seed=11)
    got = parity.run_grouped(inp, (384,), 32.0)
    lin = inp["linears"][0]
    X, dY = inp["X"].cuda(), inp["dY"].cuda()
    A, B = lin["A"].cuda(), lin["B"].cuda()
    w = linear.nf4_pack(lin["W0"].cuda())
    H, XA = linear.forward(X, w, A, B, 32.0)
    dX, dA, dB = linear.backward(dY, X, w, A, B, XA, 32.0)
    torch.cuda.synchronize()
    for k, v in (("H", H), ("XA", XA), ("dX", dX), ("dA", dA), ("dB", dB)):
        assert torch.equal(got[k].cpu(), v.cpu()), k


def test_grouped_zero_adapter_leaves_others():
    """B and A of the middle adapter zero: its outputs are the base product alone, its dA and
    dB are zero, and the other adapters' results stay within the bar."""
    Ns = (256, 128, 256)
    inp = synth.make_grouped(150, 256, Ns, 16, seed=12, dy_std=1.0)
    inp["linears"][1]["A"].zero_()
    inp["linears"][1]["B"].zero_()
    got = parity.run_grouped(inp, Ns, 32.0)
    parity.check_grouped(inp, Ns, 32.0, got)
    assert torch.count_nonzero(got["dA"][16:32]) == 0
    assert torch.count_nonzero(got["dB"][256:384]) == 0


def test_grouped_no_dx_and_deterministic():
    Ns = (256, 128, 128)
    inp = synth.make_grouped(300, 512, Ns, 16, seed=13, dy_std=1.0)
    a = parity.run_grouped(inp, Ns, 32.0)
    b = parity.run_grouped(inp, Ns, 32.0)
    for k in ("H", "XA", "dX", "dA", "dB"):
        assert torch.equal(a[k], b[k]), k
    c = parity.run_grouped(inp, Ns, 32.0, need_dx=False)
    assert c["dX"] is None
    for k in ("H", "XA", "dA", "dB"):
        assert torch.equal(a[k], c[k]), k


def test_grouped_recompute_xa_is_bit_identical():
    Ns = (256, 128, 128)
    inp = synth.make_grouped(300, 512, Ns, 16, seed=14, dy_std=1.0)
    W0, A, B = parity.stacked(inp)
    X, dY, A, B = inp["X"].cuda(), inp["dY"].cuda(), A.cuda(), B.cuda()
    w = linear.nf4_pack(W0.cuda())
    H, XA = linear.grouped_forward(X, w, A, B, list(Ns), 32.0)
    H2, none = linear.grouped_forward(X, w, A, B, list(Ns), 32.0, save_xa=False)
    assert none is None
    saved = linear.grouped_backward(dY, X, w, A, B, XA, list(Ns), 32.0)
    recomputed = linear.grouped_backward(dY, X, w, A, B, None, list(Ns), 32.0)
    torch.cuda.synchronize()
    assert linear.device_error() == 0
    assert torch.equal(H, H2)
    for a, b, k in zip(saved, recomputed, ("dX", "dA", "dB")):
        assert torch.equal(a, b), k


@pytest.mark.parametrize("M,I", [(3, 1000), (64, 14336 // 8)])
def test_swiglu_packed_parity(M, I):
    """SwiGLU on a packed gate/up output [M, 2I] against the oracle on its column blocks."""
    gen = torch.Generator().manual_seed(M + I)
    gu = torch.randn(M, 2 * I, generator=gen).to(torch.bfloat16)
    da = torch.randn(M, I, generator=gen).to(torch.bfloat16)
    a = linear.swiglu_packed_forward(gu.cuda())
    dgu = linear.swiglu_packed_backward(gu.cuda(), da.cuda())
    torch.cuda.synchronize()
    g, u = qlora.split_cols(parity.f32(gu), [I, I])
    assert qlora.rel_err(parity.f32(a), qlora.swiglu_forward(g, u)) <= 1e-2
    rg, ru = qlora.swiglu_backward(g, u, parity.f32(da))
    dg, du = qlora.split_cols(parity.f32(dgu), [I, I])
    assert qlora.rel_err(dg, rg) <= 1e-2
    assert qlora.rel_err(du, ru) <= 1e-2
