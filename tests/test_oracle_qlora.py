"""Pins for the LoRA-linear oracle (CPU only).

The oracle's forward/backward are checked against: a pure-Python triple-loop GEMM, central
finite differences of L = <dY, h> in float64, torch float64 autograd of the forward formula
(the yardstick the pages name: gradients equal plain autograd up to rounding), linearity, and
closed forms for B = 0, A = 0 and W0 = 0.
"""

import numpy as np
import pytest
import torch

from oracle import nf4, qlora


def _rand(shape, rng, scale=1.0):
    return rng.standard_normal(shape) * scale


def _case(M=4, K=64, N=8, r=2, seed=0):
    rng = np.random.default_rng(seed)
    X = _rand((M, K), rng)
    W0 = _rand((N, K), rng, 0.02)
    w32 = nf4.bf16_bits_to_f32(nf4.f32_to_bf16_bits(W0.astype(np.float32)))
    packed = nf4.quantize(w32)
    Wd = nf4.dequantize(packed["q"], packed["absmax_eff"], N, K).astype(np.float64)
    A = _rand((r, K), rng, 0.1)
    B = _rand((N, r), rng, 0.1)
    dY = _rand((M, N), rng)
    return X, Wd, A, B, dY


def _matmul_loops(P, Q):
    """Triple loop, pure Python."""
    m, k = len(P), len(P[0])
    n = len(Q[0])
    out = [[0.0] * n for _ in range(m)]
    for i in range(m):
        for j in range(n):
            acc = 0.0
            for t in range(k):
                acc += P[i][t] * Q[t][j]
            out[i][j] = acc
    return np.array(out)


def test_forward_backward_vs_triple_loop():
    M, K, N, r = 3, 64, 5, 2
    X, Wd, A, B, dY = _case(M, K, N, r, seed=7)
    alpha = 3.0
    s = alpha / r
    XA = _matmul_loops(X.tolist(), A.T.tolist())
    base = _matmul_loops(X.tolist(), Wd.T.tolist())
    lora = _matmul_loops(XA.tolist(), B.T.tolist())
    h_ref = base + s * lora
    h, XA_o = qlora.forward(X, Wd, A, B, alpha)
    assert np.allclose(h, h_ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(XA_o, XA, rtol=1e-12, atol=1e-12)
    dYB = _matmul_loops(dY.tolist(), B.tolist())
    dX_ref = _matmul_loops(dY.tolist(), Wd.tolist()) + s * _matmul_loops(dYB.tolist(), A.tolist())
    dB_ref = s * _matmul_loops(dY.T.tolist(), XA.tolist())
    dA_ref = s * _matmul_loops(dYB.T.tolist(), X.tolist())
    g = qlora.backward(dY, X, Wd, A, B, alpha)
    for key, ref in (("dX", dX_ref), ("dB", dB_ref), ("dA", dA_ref), ("dYB", dYB)):
        assert np.allclose(g[key], ref, rtol=1e-12, atol=1e-12), key


def test_finite_differences():
    M, K, N, r = 4, 64, 8, 2
    X, Wd, A, B, dY = _case(M, K, N, r, seed=1)
    alpha = 4.0

    def loss(X_, A_, B_):
        return float(np.sum(dY * qlora.forward(X_, Wd, A_, B_, alpha)[0]))

    g = qlora.backward(dY, X, Wd, A, B, alpha)
    eps = 1e-6
    rng = np.random.default_rng(11)
    for name, arr, grad in (("X", X, g["dX"]), ("A", A, g["dA"]), ("B", B, g["dB"])):
        for _ in range(12):
            idx = tuple(rng.integers(0, d) for d in arr.shape)
            plus = arr.copy()
            minus = arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args_p = {"X": X, "A": A, "B": B}
            args_m = dict(args_p)
            args_p[name] = plus
            args_m[name] = minus
            fd = (loss(args_p["X"], args_p["A"], args_p["B"])
                  - loss(args_m["X"], args_m["A"], args_m["B"])) / (2 * eps)
            scale = max(1.0, np.max(np.abs(grad)))
            assert abs(fd - grad[idx]) <= 1e-7 * scale, (name, idx, fd, grad[idx])


def test_autograd_float64_crosscheck():
    M, K, N, r = 5, 128, 16, 4
    X, Wd, A, B, dY = _case(M, K, N, r, seed=2)
    alpha = 8.0
    tX = torch.tensor(X, dtype=torch.float64, requires_grad=True)
    tA = torch.tensor(A, dtype=torch.float64, requires_grad=True)
    tB = torch.tensor(B, dtype=torch.float64, requires_grad=True)
    tW = torch.tensor(Wd, dtype=torch.float64)
    h = torch.nn.functional.linear(tX, tW) + (alpha / r) * torch.nn.functional.linear(
        torch.nn.functional.linear(tX, tA), tB)
    h.backward(torch.tensor(dY, dtype=torch.float64))
    g = qlora.backward(dY, X, Wd, A, B, alpha)
    assert np.allclose(h.detach().numpy(), qlora.forward(X, Wd, A, B, alpha)[0], rtol=1e-12, atol=1e-12)
    assert np.allclose(tX.grad.numpy(), g["dX"], rtol=1e-12, atol=1e-12)
    assert np.allclose(tA.grad.numpy(), g["dA"], rtol=1e-12, atol=1e-12)
    assert np.allclose(tB.grad.numpy(), g["dB"], rtol=1e-12, atol=1e-12)


def test_B_zero_and_A_zero():
    X, Wd, A, B, dY = _case(6, 128, 12, 4, seed=3)
    h, _ = qlora.forward(X, Wd, A, np.zeros_like(B), 8.0)
    assert np.array_equal(h, X @ Wd.T)
    g = qlora.backward(dY, X, Wd, np.zeros_like(A), B, 8.0)
    assert np.array_equal(g["dB"], np.zeros_like(B))
    assert np.array_equal(g["dX"], dY @ Wd)


def test_W0_zero_closed_form():
    rng = np.random.default_rng(4)
    M, K, N, r = 3, 128, 6, 2
    packed = nf4.quantize(np.zeros((N, K), np.float32))
    assert np.all(nf4.unpack_codes(packed["q"]) == 7) and np.all(packed["absmax"] == 0)
    Wd = nf4.dequantize(packed["q"], packed["absmax_eff"], N, K)
    assert np.all(Wd == 0)
    X = rng.standard_normal((M, K))
    A = rng.standard_normal((r, K))
    B = rng.standard_normal((N, r))
    h, _ = qlora.forward(X, Wd, A, B, 6.0)
    assert np.allclose(h, 3.0 * X @ A.T @ B.T, rtol=1e-13, atol=1e-13)


def test_linearity_in_X():
    X, Wd, A, B, _ = _case(4, 64, 8, 2, seed=5)
    X2 = np.random.default_rng(6).standard_normal(X.shape)
    h1 = qlora.forward(X, Wd, A, B, 2.0)[0]
    h2 = qlora.forward(X2, Wd, A, B, 2.0)[0]
    h12 = qlora.forward(X + X2, Wd, A, B, 2.0)[0]
    assert np.allclose(h12, h1 + h2, rtol=1e-12, atol=1e-12)


def test_row_variants_match_full():
    X, Wd, A, B, dY = _case(9, 128, 16, 4, seed=8)
    rows = np.array([0, 3, 8])
    h = qlora.forward(X, Wd, A, B, 5.0)[0]
    assert np.allclose(qlora.forward_rows(X, Wd, A, B, 5.0, rows), h[rows], rtol=1e-13, atol=1e-13)
    g = qlora.backward(dY, X, Wd, A, B, 5.0)
    assert np.allclose(qlora.backward_dx_rows(dY, Wd, A, B, 5.0, rows), g["dX"][rows],
                       rtol=1e-13, atol=1e-13)
    w = qlora.backward_weights(dY, X, A, B, 5.0)
    assert np.allclose(w["dA"], g["dA"]) and np.allclose(w["dB"], g["dB"])


def test_swiglu_closed_forms_and_finite_differences():
    # closed forms: silu(0) = 0, d silu/dg (0) = 1/2, silu(g) -> g for large g
    a = qlora.swiglu_forward(np.array([0.0, 40.0]), np.array([3.0, 2.0]))
    assert a[0] == 0.0 and a[1] == pytest.approx(80.0, rel=1e-15)
    dg, du = qlora.swiglu_backward(np.array([0.0]), np.array([2.0]), np.array([1.0]))
    assert dg[0] == pytest.approx(1.0) and du[0] == 0.0
    rng = np.random.default_rng(9)
    g = rng.standard_normal(50) * 3
    u = rng.standard_normal(50)
    da = rng.standard_normal(50)
    dg, du = qlora.swiglu_backward(g, u, da)
    eps = 1e-6
    fd_g = (qlora.swiglu_forward(g + eps, u) - qlora.swiglu_forward(g - eps, u)) / (2 * eps) * da
    fd_u = (qlora.swiglu_forward(g, u + eps) - qlora.swiglu_forward(g, u - eps)) / (2 * eps) * da
    assert np.allclose(dg, fd_g, rtol=1e-7, atol=1e-8)
    assert np.allclose(du, fd_u, rtol=1e-7, atol=1e-8)


def test_rel_err_metric():
    ref = np.array([1.0, -4.0, 2.0])
    got = np.array([1.1, -4.0, 2.0])
    assert qlora.rel_err(got, ref) == pytest.approx(0.1 / 4.0)
