"""Pins for the packed-adapter oracle (CPU only).

Packed adapters are n independent LoRA layers on one input: outputs side by side, input
gradients added, adapter weights and their gradients stacked by rows.  The oracle computes
that as a loop over adapters.  The pins check it against constructions other than that loop:
* the one-matmul block-diagonal form of the packed layer;
* float64 autograd of that form;
* central finite differences on the packed tensors;
* the relabelling symmetry (permuting adapters permutes the blocks);
* the single-layer oracle for one adapter.
"""

import numpy as np
import torch

from oracle import nf4, qlora


def _deq(N, K, rng):
    W0 = rng.standard_normal((N, K)) * 0.02
    w32 = nf4.bf16_bits_to_f32(nf4.f32_to_bf16_bits(W0.astype(np.float32)))
    p = nf4.quantize(w32)
    return nf4.dequantize(p["q"], p["absmax_eff"], N, K).astype(np.float64)


def _case(M=5, K=128, Ns=(8, 4, 6), r=3, seed=0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    Wds = [_deq(N, K, rng) for N in Ns]
    As = [rng.standard_normal((r, K)) * 0.1 for _ in Ns]
    Bs = [rng.standard_normal((N, r)) * 0.1 for N in Ns]
    dY = rng.standard_normal((M, sum(Ns)))
    return X, Wds, As, Bs, dY


def _block_diagonal(Bs):
    """B_bd [sum N, n r]: adapter g's B in rows of g, columns g r .. g r + r - 1, zero elsewhere."""
    r = Bs[0].shape[1]
    Ns = [B.shape[0] for B in Bs]
    out = np.zeros((sum(Ns), r * len(Bs)))
    row = 0
    for g, B in enumerate(Bs):
        for i in range(B.shape[0]):
            for j in range(r):
                out[row + i, g * r + j] = B[i, j]
        row += B.shape[0]
    return out


def test_one_adapter_is_the_single_layer():
    X, Wds, As, Bs, dY = _case(Ns=(12,), seed=1)
    h, xa = qlora.grouped_forward(X, Wds, As, Bs, 6.0)
    h1, xa1 = qlora.forward(X, Wds[0], As[0], Bs[0], 6.0)
    assert np.array_equal(h, h1) and np.array_equal(xa, xa1)
    g = qlora.grouped_backward(dY, X, Wds, As, Bs, 6.0)
    g1 = qlora.backward(dY, X, Wds[0], As[0], Bs[0], 6.0)
    for k in ("dA", "dB"):
        assert np.array_equal(g[k], g1[k]), k
    assert np.allclose(g["dX"], g1["dX"], rtol=1e-13, atol=1e-13)


def test_block_diagonal_form_and_autograd():
    """H = X W_cat^T + s (X A_cat^T) B_bd^T; gradients by float64 autograd of that form: dX
    directly, dA as A_cat's gradient, dB as the diagonal blocks of B_bd's gradient."""
    M, K, Ns, r, alpha = 6, 192, (8, 4, 6), 3, 9.0
    X, Wds, As, Bs, dY = _case(M, K, Ns, r, seed=2)
    s = alpha / r
    tX = torch.tensor(X, requires_grad=True)
    tA = torch.tensor(np.concatenate(As, axis=0), requires_grad=True)
    tBbd = torch.tensor(_block_diagonal(Bs), requires_grad=True)
    tW = torch.tensor(np.concatenate(Wds, axis=0))
    H = tX @ tW.T + s * (tX @ tA.T) @ tBbd.T
    H.backward(torch.tensor(dY))

    h, xa = qlora.grouped_forward(X, Wds, As, Bs, alpha)
    assert np.allclose(h, H.detach().numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(xa, (tX @ tA.T).detach().numpy(), rtol=1e-12, atol=1e-12)
    g = qlora.grouped_backward(dY, X, Wds, As, Bs, alpha)
    assert np.allclose(g["dX"], tX.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(g["dA"], tA.grad.numpy(), rtol=1e-12, atol=1e-12)
    gbd = tBbd.grad.numpy()
    row = 0
    for i, N in enumerate(Ns):
        blk = gbd[row:row + N, i * r:(i + 1) * r]
        assert np.allclose(g["dB"][row:row + N], blk, rtol=1e-12, atol=1e-12)
        row += N
    assert g["dA"].shape == (len(Ns) * r, K) and g["dB"].shape == (sum(Ns), r)


def test_finite_differences_on_packed_tensors():
    """L = <dY, H> is linear in each of X, A_cat, B_cat: a central difference with step 1 is
    the exact directional derivative (up to float64 rounding)."""
    M, K, Ns, r, alpha = 4, 128, (6, 10), 2, 4.0
    X, Wds, As, Bs, dY = _case(M, K, Ns, r, seed=3)
    g = qlora.grouped_backward(dY, X, Wds, As, Bs, alpha)

    def loss(X_, As_, Bs_):
        return float(np.sum(dY * qlora.grouped_forward(X_, Wds, As_, Bs_, alpha)[0]))

    rng = np.random.default_rng(30)
    Acat = np.concatenate(As, axis=0)
    Bcat = np.concatenate(Bs, axis=0)
    for _ in range(6):
        i, j = rng.integers(len(Ns) * r), rng.integers(K)
        E = np.zeros_like(Acat)
        E[i, j] = 1.0
        pa = np.split(Acat + E, len(Ns))
        ma = np.split(Acat - E, len(Ns))
        fd = (loss(X, pa, Bs) - loss(X, ma, Bs)) / 2.0
        assert abs(fd - g["dA"][i, j]) <= 1e-9 * max(1.0, abs(fd))
        i, j = rng.integers(sum(Ns)), rng.integers(r)
        E = np.zeros_like(Bcat)
        E[i, j] = 1.0
        pb = np.split(Bcat + E, np.cumsum(Ns)[:-1])
        mb = np.split(Bcat - E, np.cumsum(Ns)[:-1])
        fd = (loss(X, As, pb) - loss(X, As, mb)) / 2.0
        assert abs(fd - g["dB"][i, j]) <= 1e-9 * max(1.0, abs(fd))
        i, j = rng.integers(M), rng.integers(K)
        E = np.zeros_like(X)
        E[i, j] = 1.0
        fd = (loss(X + E, As, Bs) - loss(X - E, As, Bs)) / 2.0
        assert abs(fd - g["dX"][i, j]) <= 1e-9 * max(1.0, abs(fd))


def test_adapter_permutation():
    M, K, Ns, r, alpha = 5, 128, (8, 4, 6), 2, 3.0
    X, Wds, As, Bs, dY = _case(M, K, Ns, r, seed=4)
    perm = [2, 0, 1]
    h, xa = qlora.grouped_forward(X, Wds, As, Bs, alpha)
    hp, xap = qlora.grouped_forward(X, [Wds[p] for p in perm], [As[p] for p in perm],
                                    [Bs[p] for p in perm], alpha)
    hb = qlora.split_cols(h, Ns)
    xb = qlora.split_cols(xa, [r] * 3)
    assert np.array_equal(hp, np.concatenate([hb[p] for p in perm], axis=1))
    assert np.array_equal(xap, np.concatenate([xb[p] for p in perm], axis=1))
    dYb = qlora.split_cols(dY, Ns)
    dYp = np.concatenate([dYb[p] for p in perm], axis=1)
    g = qlora.grouped_backward(dY, X, Wds, As, Bs, alpha)
    gp = qlora.grouped_backward(dYp, X, [Wds[p] for p in perm], [As[p] for p in perm],
                                [Bs[p] for p in perm], alpha)
    dA = np.split(g["dA"], 3)
    dB = np.split(g["dB"], np.cumsum(Ns)[:-1])
    assert np.array_equal(gp["dA"], np.concatenate([dA[p] for p in perm]))
    assert np.array_equal(gp["dB"], np.concatenate([dB[p] for p in perm]))
    assert np.allclose(gp["dX"], g["dX"], rtol=1e-12, atol=1e-12)


def test_row_variants_match_full():
    X, Wds, As, Bs, dY = _case(7, 128, (4, 8), 2, seed=5)
    rows = [0, 3, 6]
    h, _ = qlora.grouped_forward(X, Wds, As, Bs, 2.0)
    assert np.allclose(qlora.grouped_forward_rows(X, Wds, As, Bs, 2.0, rows), h[rows],
                       rtol=1e-13, atol=1e-13)
    g = qlora.grouped_backward(dY, X, Wds, As, Bs, 2.0)
    assert np.allclose(qlora.grouped_backward_dx_rows(dY, Wds, As, Bs, 2.0, rows), g["dX"][rows],
                       rtol=1e-13, atol=1e-13)
