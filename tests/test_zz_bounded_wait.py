"""Failure detection on the GPU, without a fault: a wait that nothing completes runs out.

The self-test kernel waits, through the kernels' own bounded wait, on a shared-memory barrier
that nothing arrives on.  The wait must give up after its limit (2 s), record its site in the
device error word and let the kernel end, so the host reads QLORA_ERR_TIMEOUT with code 6 and
the context keeps working: a layer run afterwards still matches the oracle.
"""

import time

import pytest
import torch

import parity
from nf4_base_lora_blockwise_b200 import abi, linear

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.synchronize()
    assert linear.device_error() == 0            # the word starts clear
    abi.qlora_selftest_bounded_wait(torch.cuda.current_stream().cuda_stream)
    t0 = time.time()
    code = linear.device_error()                 # synchronises: returns once the wait gave up
    waited = time.time() - t0
    assert code == 6                             # site 6, CTA 0, tag 0
    assert 1.5 < waited < 60
    assert linear.device_error() == 0            # reading cleared it
    inp, L = parity.make(130, 256, 256, 16, seed=21)
    got = parity.run_linear(inp, L)
    parity.check_linear(inp, L, got)
