"""The rank-r products through the C ABI, element by element against the fp64 oracle.

qlora_lora_grad (s dY^T XA, s dYB^T X), and qlora_lora_down (X A^T, dY B with the
block-diagonal B of packed adapters) when tokens are few or the rank wide, split their
reduction over the CTAs of a cluster and sum the partials in a fixed order in distributed
shared memory; qlora_lora_down with many tokens and r <= 32 gives each warp whole token rows
(shapes with M >= 4096 below), including a reduction that is not a multiple of 256.  Covered here: every small-tile layout the
kernels use (8, 16, 32, 64 and 128 columns, swizzled; 24, 40, 48, 72, 120, unswizzled rows),
ragged token counts (M not a multiple of 64 or 128), column counts that leave half a 128-wide
tile, cluster sizes 1 to 8, repeat calls bit for bit, and no scratch passed at all.
"""

import numpy as np
import pytest
import torch

from nf4_base_lora_blockwise_b200 import abi, linear
from oracle import qlora

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _rand(shape, std, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


def _f64(t):
    return t.detach().cpu().float().numpy().astype(np.float64)


def _down(inp, w, w_rc, R, groups=None, scale=2.0):
    M, C = inp.shape
    saved = torch.empty((M, R), dtype=torch.bfloat16, device="cuda")
    scaled = torch.empty((M, R), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    abi.qlora_lora_down(inp.data_ptr(), M, C, w.data_ptr(), 1 if w_rc else 0, R, groups, scale,
                        saved.data_ptr(), scaled.data_ptr(), None, 0, s)
    torch.cuda.synchronize()
    assert linear.device_error() == 0
    return saved, scaled


def _grad(big, small, R, out_cr, groups=None, scale=0.5):
    M, C = big.shape
    out = torch.full((C, R) if out_cr else (R, C), float("nan"), dtype=torch.float32,
                     device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    abi.qlora_lora_grad(big.data_ptr(), M, C, small.data_ptr(), R, groups, scale,
                        out.data_ptr(), 0 if out_cr else 1, None, 0, s)
    torch.cuda.synchronize()
    assert linear.device_error() == 0
    return out


@pytest.mark.parametrize("M,C,R", [
    (1, 256, 16), (77, 192, 8), (300, 512, 24), (130, 1024, 32), (4096, 4096, 16),
    (4500, 320, 24), (8192, 640, 32), (4096, 256, 8),
    (257, 640, 40), (64, 256, 48), (513, 448, 64), (100, 320, 72), (33, 256, 120),
    (200, 512, 128),
])
def test_down_A_form(M, C, R):
    X = _rand((M, C), 1.0, M + C).cuda()
    A = _rand((R, C), 0.05, R).cuda()
    saved, scaled = _down(X, A, True, R, scale=2.0)
    ref = qlora.lora_down(_f64(X), _f64(A))
    assert qlora.rel_err(_f64(saved), ref) <= TOL
    assert qlora.rel_err(_f64(scaled), 2.0 * ref) <= TOL
    # scaled is bf16(s * v) of the same fp32 sum; with s = 2 it is exactly 2 * saved
    assert torch.equal(scaled.float(), 2.0 * saved.float())
    again, _ = _down(X, A, True, R, scale=2.0)
    assert torch.equal(saved, again)


@pytest.mark.parametrize("M,C,R", [(300, 512, 16), (65, 1024, 8), (129, 384, 24), (64, 512, 64),
                                   (31, 256, 128), (4096, 1024, 16), (4100, 448, 32),
                                   (6000, 256, 8)])
def test_down_B_form(M, C, R):
    dY = _rand((M, C), 1.0, 7 * M).cuda()
    B = _rand((C, R), 0.05, C).cuda()
    saved, _ = _down(dY, B, False, R)
    ref = _f64(dY) @ _f64(B)
    assert qlora.rel_err(_f64(saved), ref) <= TOL


@pytest.mark.parametrize("M,Ns,r", [(200, [256, 128, 128], 16), (200, [128, 384], 24),
                                    (200, [128] * 8, 8), (4096, [256, 128, 128], 16),
                                    (4096, [128, 384], 8)])
def test_down_block_diagonal(M, Ns, r):
    """dY B_bd: adapter g's columns of dY feed output columns g r .. g r + r - 1 only."""
    C = sum(Ns)
    dY = _rand((M, C), 1.0, 11).cuda()
    B = _rand((C, r), 0.05, 12).cuda()
    saved, _ = _down(dY, B, False, r * len(Ns), groups=Ns)
    ref = np.zeros((M, r * len(Ns)))
    edges = np.cumsum([0] + Ns)
    for g in range(len(Ns)):
        ref[:, g * r:(g + 1) * r] = _f64(dY)[:, edges[g]:edges[g + 1]] @ _f64(B)[edges[g]:edges[g + 1]]
    assert qlora.rel_err(_f64(saved), ref) <= TOL


@pytest.mark.parametrize("out_cr", [True, False])
@pytest.mark.parametrize("M,C,R", [(1, 256, 16), (77, 192, 8), (300, 512, 24), (4096, 4096, 16),
                                   (1000, 640, 64), (129, 320, 72), (64, 256, 128),
                                   (513, 1024, 40)])
def test_grad(M, C, R, out_cr):
    big = _rand((M, C), 0.1, M).cuda()
    small = _rand((M, R), 1.0, R + 1).cuda()
    out = _grad(big, small, R, out_cr, scale=0.5)
    ref = 0.5 * _f64(big).T @ _f64(small)
    got = _f64(out) if out_cr else _f64(out).T
    assert np.isfinite(got).all()
    assert qlora.rel_err(got, ref) <= TOL
    again = _grad(big, small, R, out_cr, scale=0.5)
    assert torch.equal(out, again)


@pytest.mark.parametrize("Ns,r", [([256, 128, 128], 16), ([128, 384], 24)])
def test_grad_per_adapter_columns(Ns, r):
    """dB of packed adapters: column c of adapter g takes small's columns g r .. g r + r - 1."""
    M, C = 333, sum(Ns)
    big = _rand((M, C), 0.1, 21).cuda()
    small = _rand((M, r * len(Ns)), 1.0, 22).cuda()
    out = _grad(big, small, r, True, groups=Ns, scale=2.0)
    edges = np.cumsum([0] + Ns)
    ref = np.zeros((C, r))
    for g in range(len(Ns)):
        ref[edges[g]:edges[g + 1]] = 2.0 * _f64(big)[:, edges[g]:edges[g + 1]].T @ \
            _f64(small)[:, g * r:(g + 1) * r]
    assert qlora.rel_err(_f64(out), ref) <= TOL


@pytest.mark.parametrize("M,C,R,w_rc", [(16, 14336, 16, False), (1, 14336, 16, False),
                                        (100, 4096, 16, True), (16, 4096, 32, True),
                                        (128, 14336, 24, False)])
def test_down_few_tokens_split(M, C, R, w_rc):
    """With workspace, few tokens split the reduction over several clusters: their fp32 partials
    go to ws and a second launch adds them in cluster order.  Same bar against the oracle, within
    a few bf16 ulps of the single-cluster result, and bit for bit on repeat."""
    inp = _rand((M, C), 1.0, M + C + R)
    w = _rand((R, C) if w_rc else (C, R), 0.05, R + 3)
    inp, w = inp.cuda(), w.cuda()
    ws = torch.empty(8 << 20, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream

    def run(with_ws):
        saved = torch.empty((M, R), dtype=torch.bfloat16, device="cuda")
        scaled = torch.empty((M, R), dtype=torch.bfloat16, device="cuda")
        n0 = abi.qlora_launch_counter()
        abi.qlora_lora_down(inp.data_ptr(), M, C, w.data_ptr(), 1 if w_rc else 0, R, None, 2.0,
                            saved.data_ptr(), scaled.data_ptr(),
                            ws.data_ptr() if with_ws else None, ws.numel() if with_ws else 0, s)
        torch.cuda.synchronize()
        assert linear.device_error() == 0
        return saved, scaled, abi.qlora_launch_counter() - n0

    saved, scaled, n = run(True)
    assert n == 2, "few tokens with workspace: the split reduction and its finalize"
    ref = _f64(inp) @ (_f64(w).T if w_rc else _f64(w))
    assert qlora.rel_err(_f64(saved), ref) <= TOL
    assert qlora.rel_err(_f64(scaled), 2.0 * ref) <= TOL
    one, _, n1 = run(False)
    assert n1 == 1
    assert (one.float() - saved.float()).abs().max() <= 2e-2 * saved.float().abs().max()
    again, _, _ = run(True)
    assert torch.equal(saved, again)
