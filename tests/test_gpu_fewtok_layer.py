"""The few-token layer (M <= 32) in three launches per direction, through the C ABI.

At a few tokens the rank-r down-projection splits its reduction over several clusters and
leaves fp32 partials; instead of a finalize launch of its own, the few-token kernels' last
launch adds them:
* forward: the down-projection, the few-token product, and its finalize, which sums X A^T
  from the partials (writing the saved XA) and adds the LoRA term;
* backward: dY B's partials, the few-token dX kernel, and one last launch that sums dY B and
  computes dX, dA = s dYB^T X and dB = s dY^T XA.
Checked here:
* the launch counts (3 and 3, instead of 4 and 5);
* h and the saved XA have the bits of the stage entry points run one after another
  (qlora_lora_down with its own finalize, then qlora_nf4_gemm): the sums run in the same order;
* dX, dA, dB meet the parity bar against the oracle (max|err| / max|ref| <= 2e-2), single
  adapter and packed adapters, ranks 16 and 64;
* the recomputing backward (no saved XA) gives the saving backward's bits.
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


def _launches(fn):
    torch.cuda.synchronize()
    n0 = abi.qlora_launch_counter()
    out = fn()
    torch.cuda.synchronize()
    assert linear.device_error() == 0
    return out, abi.qlora_launch_counter() - n0


@pytest.mark.parametrize("M,r", [(1, 16), (16, 16), (32, 16), (16, 64)])
def test_fewtok_forward_folds_the_down_projection(M, r):
    K, N = 4096, 2048
    inp, L = parity.make(M, K, N, r, seed=5 * M + r, dy_std=1.0)
    lin = inp["linears"][0]
    X, A, B = inp["X"].cuda(), lin["A"].cuda(), lin["B"].cuda()
    w = linear.nf4_pack(lin["W0"].cuda())
    (H, XA), n = _launches(lambda: linear.forward(X, w, A, B, L.alpha))
    assert n == 3, "down-projection, few-token kernel, its finalize"
    s = torch.cuda.current_stream().cuda_stream
    ws = torch.empty(64 << 20, dtype=torch.uint8, device="cuda")
    saved = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    scaled = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    H2 = torch.empty_like(H)

    def stages():
        abi.qlora_lora_down(X.data_ptr(), M, K, A.data_ptr(), 1, r, None, L.alpha / r,
                            saved.data_ptr(), scaled.data_ptr(), ws.data_ptr(), ws.numel(), s)
        abi.qlora_nf4_gemm(X.data_ptr(), w.c_struct(), 0, B.data_ptr(), scaled.data_ptr(), M, r,
                           None, H2.data_ptr(), ws.data_ptr(), ws.numel(), s)

    _, n2 = _launches(stages)
    assert n2 == 4
    assert torch.equal(XA, saved)
    assert torch.equal(H, H2)


@pytest.mark.parametrize("M,r", [(1, 16), (9, 16), (16, 16), (32, 16), (16, 64)])
def test_fewtok_backward_in_three_launches(M, r):
    K, N = 4096, 2048
    inp, L = parity.make(M, K, N, r, seed=7 * M + r, dy_std=1.0)
    lin = inp["linears"][0]
    X, dY, A, B = (inp["X"].cuda(), inp["dY"].cuda(), lin["A"].cuda(), lin["B"].cuda())
    w = linear.nf4_pack(lin["W0"].cuda())
    H, XA = linear.forward(X, w, A, B, L.alpha)
    (dX, dA, dB), n = _launches(lambda: linear.backward(dY, X, w, A, B, XA, L.alpha))
    assert n == 3, "dY B partials, few-token dX kernel, the last launch"
    again, _ = _launches(lambda: linear.backward(dY, X, w, A, B, None, L.alpha))
    for a, b, k in zip((dX, dA, dB), again, ("dX", "dA", "dB")):
        assert torch.equal(a, b), k
    (_, dA2, dB2), n2 = _launches(lambda: linear.backward(dY, X, w, A, B, XA, L.alpha,
                                                         need_dx=False))
    assert n2 == 2
    assert torch.equal(dA, dA2) and torch.equal(dB, dB2)
    parity.check_linear(inp, L, {"H": H, "XA": XA, "dX": dX, "dA": dA, "dB": dB})


def test_fewtok_packed_adapters():
    Ns, r, M, K = (2048, 1024, 1024), 16, 16, 4096
    inp = synth.make_grouped(M, K, list(Ns), r, seed=19, dy_std=1.0)
    got, n = _launches(lambda: parity.run_grouped(inp, Ns, 2.0 * r))
    parity.check_grouped(inp, Ns, 2.0 * r, got)
