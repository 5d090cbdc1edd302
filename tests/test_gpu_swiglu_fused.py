"""The packed gate/up forward with its SwiGLU in the GEMM epilogue (qlora_grouped_fwd_swiglu),
through the C ABI.

Where the dequant GEMM runs whole tiles, each CTA computes a gate tile and then the up tile of
the same rows and tokens, and the up tile's epilogue writes act = silu(g) u from the g it has
just written.  Checked here:
* GU, the saved XA and act have the bits of qlora_grouped_fwd followed by
  qlora_swiglu_packed_fwd (the path the call falls back to), on whole-tile shapes with ragged
  token tails, at the MLP workload's full size, and on a double-quantised weight;
* the fused shapes take one launch fewer than that sequence (no SwiGLU launch), and shapes the
  epilogue cannot serve (stream-K, few tokens) fall back to it;
* act meets the oracle's SwiGLU on the GPU's own g and u (max|err| / max|ref| <= 1e-2), and the
  packed layer's GU meets the oracle's forward per adapter (the parity bar, 2e-2).
"""

import numpy as np
import pytest
import torch

import parity
from nf4_base_lora_blockwise_b200 import abi, linear, synth
from oracle import qlora

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _inputs(M, K, I, r, seed, dq=False):
    g = torch.Generator().manual_seed(seed)
    X = torch.randn((M, K), generator=g).to(torch.bfloat16)
    W0 = (torch.randn((2 * I, K), generator=g) * 0.02).to(torch.bfloat16)
    A = ((torch.rand((2 * r, K), generator=g) * 2 - 1) / 64).to(torch.bfloat16)
    B = (torch.randn((2 * I, r), generator=g) * 0.02).to(torch.bfloat16)
    w = linear.nf4_pack(W0.cuda(), double_quant=dq)
    return X.cuda(), w, A.cuda(), B.cuda(), W0


def _launches(fn):
    torch.cuda.synchronize()
    n0 = abi.qlora_launch_counter()
    out = fn()
    torch.cuda.synchronize()
    assert linear.device_error() == 0
    return out, abi.qlora_launch_counter() - n0


def _both(M, K, I, r, seed, dq=False):
    X, w, A, B, W0 = _inputs(M, K, I, r, seed, dq)
    alpha = 2.0 * r

    def unfused():
        GU, XA = linear.grouped_forward(X, w, A, B, [I, I], alpha)
        return GU, XA, linear.swiglu_packed_forward(GU)

    ref, n_ref = _launches(unfused)
    got, n_got = _launches(lambda: linear.gate_up_swiglu_forward(X, w, A, B, alpha))
    for a, b, name in zip(ref, got, ("GU", "XA", "act")):
        assert torch.equal(a, b), name
    return ref, n_ref, n_got, (X, w, A, B, W0, alpha)


@pytest.mark.parametrize("M,K,I,r,dq", [
    (2048, 1024, 4096, 16, False),   # whole tiles, 480-token tiles
    (1900, 512, 4096, 16, False),    # ragged last token tile
    (2304, 768, 3072, 32, True),     # double-quantised absmax, r = 32
])
def test_fused_equals_layer_then_swiglu(M, K, I, r, dq):
    _, n_ref, n_got, _ = _both(M, K, I, r, seed=M + I, dq=dq)
    assert n_got == n_ref - 1, "the SwiGLU is in the GEMM epilogue, not a launch of its own"


@pytest.mark.parametrize("M,K,I,r", [
    (300, 512, 1024, 16),   # few tiles: stream-K, so the call falls back
    (16, 512, 1024, 16),    # few tokens
])
def test_fallback_equals_layer_then_swiglu(M, K, I, r):
    _, n_ref, n_got, _ = _both(M, K, I, r, seed=7 * M + r)
    assert n_got == n_ref


def test_fused_meets_the_oracle():
    M, K, I, r = 2048, 512, 2048 + 2048, 16
    (GU, XA, act), _, n_got, (X, w, A, B, W0, alpha) = _both(M, K, I, r, seed=3)
    rows = np.concatenate([np.arange(0, M, 61), [M - 1]])
    g, u = qlora.split_cols(parity.f32(GU)[rows], [I, I])
    assert qlora.rel_err(parity.f32(act)[rows], qlora.swiglu_forward(g, u)) <= 1e-2
    _, Wd = parity.oracle_deq(W0, False)
    Xr = parity.f32(X)[rows].astype(np.float64)
    Af = parity.f32(A).astype(np.float64)
    Bf = parity.f32(B).astype(np.float64)
    s = alpha / r
    for gi in range(2):
        rs = slice(gi * I, (gi + 1) * I)
        ref = Xr @ Wd[rs].astype(np.float64).T + s * (Xr @ Af[gi * r:(gi + 1) * r].T) @ Bf[rs].T
        assert qlora.rel_err(parity.f32(GU)[rows][:, rs], ref) <= parity.TOL


def test_full_size_mlp_gate_up():
    """The MLP workload's packed gate/up layer (4096 -> 2 x 14336, 8192 tokens, r = 16)."""
    w = synth.workload("mlp_8b")
    gate = w.linears[0]
    _, n_ref, n_got, _ = _both(w.M, gate.K, gate.N, gate.r, seed=11)
    assert n_got == n_ref - 1
