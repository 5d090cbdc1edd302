"""The allocation-free forward entry point (qlora_linear_fwd_noalloc).

Some callers cannot allocate device memory at all -- a host framework that owns every device
allocation and hands out no workspace, or a host linking the C ABI without a device allocator
of its own -- so they cannot pass the workspace qlora_linear_fwd needs.  This entry point keeps
its scratch in a fixed array inside the library instead.  Here it is called through the C ABI,
twice in a row on the same inputs, and each result is checked against qlora_linear_fwd's within
the tolerance the parity tests use; a problem too large for the fixed scratch must be refused
before anything is enqueued.  This file is named to be collected last.
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


@pytest.mark.parametrize("M,K,N,r", [
    (16, 512, 384, 16),      # few tokens: the register-direct kernel's slots in the scratch
    (300, 512, 384, 16),     # stream-K tcgen05 GEMM whose partials fit beside s*XA
    (16384, 4096, 384, 16),  # stream-K partials too large for what is left: whole tiles
])
def test_noalloc_forward_matches_workspace_forward_twice(M, K, N, r):
    inp, L = parity.make(M, K, N, r, seed=21)
    lin = inp["linears"][0]
    X, A, B = inp["X"].cuda(), lin["A"].cuda(), lin["B"].cuda()
    w = linear.nf4_pack(lin["W0"].cuda())
    H_ref, XA_ref = linear.forward(X, w, A, B, L.alpha)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        H = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        XA = torch.full((M, r), float("nan"), dtype=torch.bfloat16, device="cuda")
        abi.qlora_linear_fwd_noalloc(X.data_ptr(), w.c_struct(), A.data_ptr(), B.data_ptr(), M,
                                     r, L.alpha, H.data_ptr(), XA.data_ptr(), stream)
        torch.cuda.synchronize()
        assert linear.device_error() == 0
        assert qlora.rel_err(parity.f32(H), parity.f32(H_ref)) <= parity.TOL
        assert qlora.rel_err(parity.f32(XA), parity.f32(XA_ref)) <= parity.TOL
        assert np.isfinite(parity.f32(H)).all()


def test_noalloc_refuses_problems_beyond_its_scratch():
    inp, L = parity.make(64, 256, 128, 128, seed=22)
    lin = inp["linears"][0]
    w = linear.nf4_pack(lin["W0"].cuda())
    M = abi.qlora_noalloc_scratch_bytes() // (2 * 128) + 1   # s*XA alone exceeds the scratch
    code = abi._lib().qlora_linear_fwd_noalloc(1 << 20, w.c_struct(), 1 << 20, 1 << 20, M, 128,
                                              256.0, 1 << 20, 1 << 20, None)
    assert code == 5   # QLORA_ERR_WORKSPACE, nothing enqueued
