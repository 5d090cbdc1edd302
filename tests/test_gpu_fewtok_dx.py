"""The few-token dX kernel (M <= 32) through the C ABI, against the oracle.

qlora_nf4_gemm with transpose_w = 1 (and so the layer's backward) runs dX for at most 32 tokens
as weight panels: each CTA decodes 64 rows x 256 columns of deq(W0) at a time into shared memory
and multiplies by dY with mma.sync, a finalize adding the row splits in order and the LoRA term
(s dYB) A.  Checked here (max|err| / max|ref| <= 2e-2, the parity bar):
* one and two 16-token blocks (M = 1, 5, 16, 17, 32);
* output-column bands that are not a multiple of 256 (K = 320, 448: a last band of 64 or 192
  columns, the rest zero-filled by TMA and never written);
* weights of a single 64-row step (N = 64) and many steps split over many CTAs;
* double-quantised absmax; ranks 8 to 64 in the LoRA term;
* that the launch is the few-token kernel and its finalize (two launches), and repeats bit for bit.
"""

import numpy as np
import pytest
import torch

import parity
from nf4_base_lora_blockwise_b200 import abi, linear
from oracle import qlora

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("M,K,N,r,dq", [
    (1, 256, 512, 16, False),
    (5, 320, 192, 8, True),
    (16, 4096, 1024, 16, False),
    (17, 448, 640, 24, False),
    (32, 2048, 256, 64, True),
    (16, 256, 64, 16, False),
])
def test_fewtok_dx(M, K, N, r, dq):
    inp, L = parity.make(M, K, N, r, seed=3 * M + K + N, dy_std=1.0)
    lin = inp["linears"][0]
    w = linear.nf4_pack(lin["W0"].cuda(), double_quant=dq)
    dY = inp["dY"].cuda()
    A = lin["A"].cuda()
    g = torch.Generator().manual_seed(M + r)
    sdYB = (torch.randn((M, r), generator=g) * 0.5).to(torch.bfloat16).cuda()
    ws = linear.alloc_workspace(M, N, K, r, "cuda")
    s = torch.cuda.current_stream().cuda_stream

    def run():
        dX = torch.full((M, K), float("nan"), dtype=torch.bfloat16, device="cuda")
        torch.cuda.synchronize()
        n0 = abi.qlora_launch_counter()
        abi.qlora_nf4_gemm(dY.data_ptr(), w.c_struct(), 1, A.data_ptr(), sdYB.data_ptr(), M, r,
                           None, dX.data_ptr(), ws.data_ptr(), ws.numel(), s)
        torch.cuda.synchronize()
        assert linear.device_error() == 0
        return dX, abi.qlora_launch_counter() - n0

    dX, n = run()
    assert n == 2, "the few-token dX kernel and its finalize"
    _, Wd = parity.oracle_deq(lin["W0"], dq)
    ref = parity.f32(dY).astype(np.float64) @ Wd.astype(np.float64) + \
        parity.f32(sdYB).astype(np.float64) @ parity.f32(A).astype(np.float64)
    got = parity.f32(dX)
    assert np.isfinite(got).all()
    assert qlora.rel_err(got, ref) <= parity.TOL
    again, _ = run()
    assert torch.equal(dX, again)


def test_fewtok_dx_in_the_layer():
    """The layer's backward at 16 tokens takes the few-token dX; all gradients at the bar."""
    inp, L = parity.make(16, 1024, 2048, 16, seed=41, dy_std=1.0)
    got = parity.run_linear(inp, L)
    parity.check_linear(inp, L, got)
