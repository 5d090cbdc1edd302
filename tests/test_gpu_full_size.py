"""GPU parity at the benchmark's full sizes, in the launch configuration bench.py times.

Every workload the benchmark runs is checked here on the same seeded inputs:

* NF4 codes, absmax (and the double-quant codes / scales) and the dequantised weight:
  bit-exact, on a fixed sample of weight rows (absmax and the double-quant groups are checked in
  full).
* h and dX: on a fixed seeded sample of 512 token rows plus the first and last, every column.
* XA, dA and dB: in full.

The floating-point bar is max|err| / max|ref| <= 2e-2.  The oracle computes the sampled rows in
float64 (its products are chunked over output columns only to bound host memory).
"""

import numpy as np
import pytest
import torch

import parity
from nf4_base_lora_blockwise_b200 import linear, synth
from oracle import nf4, qlora

pytestmark = pytest.mark.gpu

W_ROWS = 96  # weight rows whose codes / dequantised values are compared bit for bit


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _weight_rows(N, seed=7):
    g = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, N - 1], g.choice(N, W_ROWS, replace=False)]))
    return rows


def _rows_matmul(Xr, Wd_f32, chunk=2048):
    """Xr [m, K] float64 times Wd^T (Wd [N, K] float32, bf16-exact) -> [m, N] float64."""
    N = Wd_f32.shape[0]
    out = np.empty((Xr.shape[0], N))
    for c in range(0, N, chunk):
        out[:, c:c + chunk] = Xr @ Wd_f32[c:c + chunk].astype(np.float64).T
    return out


def _rows_matmul_t(Yr, Wd_f32, chunk=2048):
    """Yr [m, N] float64 times Wd (Wd [N, K]) -> [m, K] float64."""
    K = Wd_f32.shape[1]
    out = np.empty((Yr.shape[0], K))
    for c in range(0, K, chunk):
        out[:, c:c + chunk] = Yr @ Wd_f32[:, c:c + chunk].astype(np.float64)
    return out


def check_one_linear(X_cpu, dY_cpu, lin, L, tag):
    X, dY = X_cpu.cuda(), dY_cpu.cuda()
    A, B = lin["A"].cuda(), lin["B"].cuda()
    w = linear.nf4_pack(lin["W0"].cuda(), double_quant=L.double_quant)
    H, XA = linear.forward(X, w, A, B, L.alpha)
    dX, dA, dB = linear.backward(dY, X, w, A, B, XA, L.alpha)
    torch.cuda.synchronize()
    assert linear.device_error() == 0

    # --- NF4 storage: bit-exact on sampled weight rows, absmax / DQ arrays in full.
    full = parity.oracle_pack(lin["W0"], L.double_quant)
    parity.check_pack(w, parity.subset(full, _weight_rows(L.N)), L.double_quant)
    del w

    # --- Oracle on sampled token rows, in float64.
    M = X_cpu.shape[0]
    rows = synth.sample_rows(M).numpy()
    Wd = parity.oracle_dequant(full)          # float32, bf16-exact, all rows
    del full
    Xf = parity.f32(X_cpu)
    dYf = parity.f32(dY_cpu)
    Af = parity.f32(lin["A"]).astype(np.float64)
    Bf = parity.f32(lin["B"]).astype(np.float64)
    s = L.alpha / L.r
    Xr = Xf[rows].astype(np.float64)
    dYr = dYf[rows].astype(np.float64)
    h_ref = _rows_matmul(Xr, Wd) + s * ((Xr @ Af.T) @ Bf.T)
    dx_ref = _rows_matmul_t(dYr, Wd) + s * ((dYr @ Bf) @ Af)
    wts = qlora.backward_weights(dYf, Xf, Af, Bf, L.alpha)
    errs = {
        "h": qlora.rel_err(parity.f32(H)[rows], h_ref),
        "dX": qlora.rel_err(parity.f32(dX)[rows], dx_ref),
        "XA": qlora.rel_err(parity.f32(XA), wts["XA"]),
        "dA": qlora.rel_err(parity.f32(dA), wts["dA"]),
        "dB": qlora.rel_err(parity.f32(dB), wts["dB"]),
    }
    for k, v in errs.items():
        assert v <= parity.TOL, f"{tag} {k}: {v:.3e}"
    return errs, H, dX


@pytest.mark.parametrize("name", ["q_proj_8b", "proj_70b_dq", "sweep_m1", "sweep_m16",
                                  "sweep_m128", "sweep_m1024", "sweep_m16384"])
def test_full_size_workload(name):
    w = synth.workload(name)
    inp = synth.make_inputs(w, seed=0)
    for L, lin in zip(w.linears, inp["linears"]):
        check_one_linear(lin["X"], lin["dY"], lin, L, f"{name}/{L.name}")


def check_packed(X_cpu, dY_cpu, lins, Ls, tag):
    """Adapters sharing X packed into one layer, at full size: codes and absmax of the stacked
    weight bit-exact on sampled rows; h and dX on the sampled token rows, h per adapter; XA, dA
    and dB in full, per adapter.  Returns the GPU's packed output H."""
    Ns = [L.N for L in Ls]
    L0 = Ls[0]
    W0 = torch.cat([d["W0"] for d in lins])
    A = torch.cat([d["A"] for d in lins])
    B = torch.cat([d["B"] for d in lins])
    X, dY = X_cpu.cuda(), dY_cpu.cuda()
    wg = linear.nf4_pack(W0.cuda())
    H, XA = linear.grouped_forward(X, wg, A.cuda(), B.cuda(), Ns, L0.alpha)
    dX, dA, dB = linear.grouped_backward(dY, X, wg, A.cuda(), B.cuda(), XA, Ns, L0.alpha)
    torch.cuda.synchronize()
    assert linear.device_error() == 0
    full = parity.oracle_pack(W0, False)
    parity.check_pack(wg, parity.subset(full, _weight_rows(sum(Ns))), False)
    del wg
    Wd = parity.oracle_dequant(full)
    del full
    M = X_cpu.shape[0]
    rows = synth.sample_rows(M).numpy()
    Xf, dYf = parity.f32(X_cpu), parity.f32(dY_cpu)
    Xr, dYr = Xf[rows].astype(np.float64), dYf[rows].astype(np.float64)
    s = L0.alpha / L0.r
    edges = np.cumsum([0] + Ns)
    r = L0.r
    dx_ref = np.zeros((len(rows), L0.K))
    Hr = parity.f32(H)[rows]
    XAf, dAf, dBf = parity.f32(XA), parity.f32(dA), parity.f32(dB)
    errs = {}
    for g, d in enumerate(lins):
        a, b = edges[g], edges[g + 1]
        Ag = parity.f32(d["A"]).astype(np.float64)
        Bg = parity.f32(d["B"]).astype(np.float64)
        h_ref = _rows_matmul(Xr, Wd[a:b]) + s * ((Xr @ Ag.T) @ Bg.T)
        errs[f"h{g}"] = qlora.rel_err(Hr[:, a:b], h_ref)
        dx_ref += _rows_matmul_t(dYr[:, a:b], Wd[a:b]) + s * ((dYr[:, a:b] @ Bg) @ Ag)
        wts = qlora.backward_weights(dYf[:, a:b], Xf, Ag, Bg, L0.alpha)
        errs[f"XA{g}"] = qlora.rel_err(XAf[:, g * r:(g + 1) * r], wts["XA"])
        errs[f"dA{g}"] = qlora.rel_err(dAf[g * r:(g + 1) * r], wts["dA"])
        errs[f"dB{g}"] = qlora.rel_err(dBf[a:b], wts["dB"])
    errs["dX"] = qlora.rel_err(parity.f32(dX)[rows], dx_ref)
    for k, v in errs.items():
        assert v <= parity.TOL, f"{tag} {k}: {v:.3e}"
    return H


def test_full_size_mlp():
    """The MLP workload in the bench's launch configuration: gate and up 4096->14336 packed
    into one layer on 8192 tokens, the packed SwiGLU, down 14336->4096.  The packed layer is
    checked per adapter with a seeded upstream gradient; down is checked on its actual input
    (the GPU's SwiGLU output), and the SwiGLU elementwise on the sampled rows."""
    w = synth.workload("mlp_8b")
    inp = synth.make_inputs(w, seed=0)
    gate, up, down = w.linears
    lg, lu, ld = inp["linears"]
    rows = synth.sample_rows(w.M).numpy()
    H = check_packed(inp["X"], _grad_like(w.M, 2 * gate.N, 1), [lg, lu], [gate, up],
                     "mlp/gate+up")
    a = linear.swiglu_packed_forward(H)
    torch.cuda.synchronize()
    g, u = qlora.split_cols(parity.f32(H)[rows], [gate.N, up.N])
    assert qlora.rel_err(parity.f32(a)[rows], qlora.swiglu_forward(g, u)) <= 1e-2
    del H
    check_one_linear(a.cpu(), inp["dY"], ld, down, "mlp/down")


def test_full_size_packed_qkv():
    """The packed-adapter workload: q 4096->4096, k and v 4096->1024 on one stacked NF4 weight
    with their own r 16 adapters, sharing 4096 tokens, in the grouped launch sequence."""
    w = synth.workload("qkv_8b")
    inp = synth.make_inputs(w, seed=0)
    check_packed(inp["X"], inp["dY"], inp["linears"], list(w.linears), "qkv_8b")


def _grad_like(M, N, seed):
    g = torch.Generator().manual_seed(1000 + seed)
    return (torch.randn((M, N), generator=g) * 1e-2).to(torch.bfloat16)


@pytest.mark.parametrize("K,N,M", [(4096, 4096, None), (4096, 14336, None), (14336, 4096, None),
                                   (4096, 14336, 16), (4096, 14336, 1024)])
def test_one_hot_products_reproduce_the_weight(K, N, M):
    """With one-hot activations each output row of the dequant GEMM is one row (dX) or one
    column (forward) of deq(W0), exactly: one product by 1.0 accumulated in fp32 and rounded to
    bf16 is the bf16 weight itself, so every element must equal the oracle's dequantised weight
    exactly (compared as values: the sign of a zero is left to the tensor core's adder).
    Three repeats at a full grid: every pipeline slot is reused many times, so a slot refilled
    before its reads finished shows up as wrong values here (the LoRA extension input is zero
    and contributes nothing).  M = None takes every row / column of the weight (whole-tile
    schedule); M = 16 and 1024 tokens give fewer tiles than SMs, i.e. the stream-K schedule,
    whose cut tiles are summed from partials (exact too: all but one partial are zero).  The
    forward at M = 16 runs the few-token kernel, exact up to the weight's bf16 rounding."""
    from nf4_base_lora_blockwise_b200 import abi

    inp, L = parity.make(4, K, N, 16, seed=K + 3 * N)
    W0 = inp["linears"][0]["W0"]
    ref = parity.oracle_pack(W0, False)
    ref_w = nf4.dequantize(ref["q"], ref["absmax_eff"], N, K)      # [N, K] float32, bf16 values
    w = linear.nf4_pack(W0.cuda())
    cw = w.c_struct()
    r = 16
    A = torch.zeros((r, K), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((N, r), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    Md, Mf = (N, K) if M is None else (M, M)
    ws = linear.alloc_workspace(max(Md, Mf), N, K, r, "cuda")

    def one_hot(m, C):
        t = torch.zeros((m, C), dtype=torch.bfloat16, device="cuda")
        i = torch.arange(m, device="cuda")
        t[i, i % C] = 1.0
        return t

    # dX[m, :] = deq(W0)[m % N, :]
    dY = one_hot(Md, N)
    zero = torch.zeros((Md, r), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        dX = torch.full((Md, K), float("nan"), dtype=torch.bfloat16, device="cuda")
        abi.qlora_nf4_gemm(dY.data_ptr(), cw, 1, A.data_ptr(), zero.data_ptr(), Md, r, None,
                           dX.data_ptr(), ws.data_ptr(), ws.numel(), stream)
        torch.cuda.synchronize()
        assert linear.device_error() == 0
        bad = int((parity.f32(dX) != ref_w[np.arange(Md) % N]).sum())
        assert bad == 0, f"dX: {bad} elements differ from deq(W0) rows"
    # h[m, :] = deq(W0)[:, m % K]
    X = one_hot(Mf, K)
    zero = torch.zeros((Mf, r), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        H = torch.full((Mf, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        abi.qlora_nf4_gemm(X.data_ptr(), cw, 0, B.data_ptr(), zero.data_ptr(), Mf, r, None,
                           H.data_ptr(), ws.data_ptr(), ws.numel(), stream)
        torch.cuda.synchronize()
        assert linear.device_error() == 0
        ref_h = ref_w.T[np.arange(Mf) % K]
        if M is not None and M <= 32:
            # The few-token forward applies the block scale after the products: the weight
            # enters as bf16(c) * absmax, rounded once more to bf16 here, instead of
            # bf16(c * absmax).  bf16 rounds within 2^-8 relative, so the two paths agree
            # within 3 * 2^-8 relative (exact zeros stay zero).
            err = np.abs(parity.f32(H) - ref_h)
            bound = 3.0 * 2.0 ** -8 * np.abs(ref_h)
            bad = int((err > bound).sum())
        else:
            bad = int((parity.f32(H) != ref_h).sum())
        assert bad == 0, f"h: {bad} elements differ from deq(W0) columns"
