"""GPU parity of the chunked LM head + cross-entropy (qlora_lm_head_ce) against the oracle.

Token losses and the loss within 1e-2 relative (max|err| / max|ref|); dX within the layer's
2e-2.  The logits pass through bf16 between the GEMM and the cross-entropy, which moves each
by at most 2^-8 of its size: for these inputs that is well under 1 % of a token's loss.
Cases cover:
* several chunks with a ragged last one;
* a last chunk of at most 32 tokens (the few-token forward kernel with no adapter);
* one chunk for the whole batch;
* ignored labels (-100 and V), and a batch with every label ignored;
* loss only (no dX);
* the full-size workload on sampled rows.
"""

import numpy as np
import pytest
import torch

import parity
from nf4_base_lora_blockwise_b200 import linear, synth
from oracle import lm_head, qlora

pytestmark = pytest.mark.gpu
TOL_LOSS = 1e-2


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _run(inp, chunk, need_dx=True):
    X = inp["X"].cuda()
    labels = inp["labels"].cuda()
    w = linear.nf4_pack(inp["linears"][0]["W0"].cuda())
    loss, tl, dX = linear.lm_head_ce(X, w, labels, chunk=chunk, need_dx=need_dx)
    torch.cuda.synchronize()
    assert linear.device_error() == 0
    return loss.cpu(), tl.cpu(), (dX.cpu() if dX is not None else None)


def _oracle(inp):
    _, Wd = parity.oracle_deq(inp["linears"][0]["W0"], False)
    return lm_head.lm_head_ce(parity.f32(inp["X"]), Wd, inp["labels"].numpy())


@pytest.mark.parametrize("M,K,V,chunk,ignore", [
    (300, 256, 1024, 128, 0.0),     # 3 chunks, the last 44 tokens
    (150, 384, 640, 64, 0.1),       # last chunk 22 tokens: few-token forward; some ignored
    (200, 256, 1088, 0, 0.0),       # one chunk for the whole batch; V not a multiple of 128
    (64, 128, 512, 16, 0.25),       # chunks of 16 tokens, K = 128 (two reduction steps)
])
def test_lm_head_ce_parity(M, K, V, chunk, ignore):
    inp = synth.make_lm_head(M, K, V, seed=M + V, ignore_frac=ignore, w_std=0.05)
    loss, tl, dX = _run(inp, chunk)
    ref = _oracle(inp)
    assert qlora.rel_err(tl.numpy(), ref["token_loss"]) <= TOL_LOSS
    assert abs(float(loss[0]) - ref["loss"]) <= TOL_LOSS * abs(ref["loss"])
    assert qlora.rel_err(parity.f32(dX), ref["dX"]) <= parity.TOL
    ignored = ~((inp["labels"] >= 0) & (inp["labels"] < V)).numpy()
    assert np.all(tl.numpy()[ignored] == 0) and np.all(parity.f32(dX)[ignored] == 0)


def test_lm_head_ce_labels_out_of_range_and_all_ignored():
    inp = synth.make_lm_head(40, 128, 256, seed=3, w_std=0.05)
    inp["labels"][::3] = 256          # == V: ignored
    inp["labels"][1::7] = -100
    loss, tl, dX = _run(inp, 16)
    ref = _oracle(inp)
    assert qlora.rel_err(tl.numpy(), ref["token_loss"]) <= TOL_LOSS
    assert abs(float(loss[0]) - ref["loss"]) <= TOL_LOSS * abs(ref["loss"])
    assert qlora.rel_err(parity.f32(dX), ref["dX"]) <= parity.TOL
    inp["labels"][:] = -100
    loss, tl, dX = _run(inp, 16)
    assert float(loss[0]) == 0.0 and torch.count_nonzero(tl) == 0
    assert torch.count_nonzero(dX.float()) == 0


def test_lm_head_ce_loss_only_matches():
    inp = synth.make_lm_head(100, 256, 512, seed=4, w_std=0.05)
    a = _run(inp, 32)
    b = _run(inp, 32, need_dx=False)
    assert b[2] is None
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_lm_head_ce_full_size_sampled():
    """Llama-3-8B head 4096 -> 128256 on 4096 tokens, chunks of 1024 (the bench's
    configuration): token losses and dX on 32 sampled rows; the loss against the mean of the
    GPU's own token losses."""
    w = synth.workload("lm_head_ce_8b")
    inp = synth.make_inputs(w, seed=0)
    loss, tl, dX = _run(inp, synth.CE_CHUNK)
    L = w.linears[0]
    full = parity.oracle_pack(inp["linears"][0]["W0"], False)
    Wd = parity.oracle_dequant(full)
    del full
    rows = synth.sample_rows(w.M, count=32).numpy()
    n = lm_head.valid_count(inp["labels"].numpy(), L.N)
    ref_tl, ref_dx = lm_head.lm_head_ce_rows(parity.f32(inp["X"]), Wd, inp["labels"].numpy(),
                                             rows, n)
    assert qlora.rel_err(tl.numpy()[rows], ref_tl) <= TOL_LOSS
    assert qlora.rel_err(parity.f32(dX)[rows], ref_dx) <= parity.TOL
    mean = float(np.sum(tl.numpy().astype(np.float64)) / n)
    assert abs(float(loss[0]) - mean) <= 1e-5 * mean
