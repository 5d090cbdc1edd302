"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and the CPU
oracle on the same seeded inputs, and compare (bit-exact for codes, absmax and dequantised
weights; max|err| / max|ref| <= TOL for the floating-point outputs)."""

import numpy as np
import torch

from nf4_base_lora_blockwise_b200 import linear, synth
from oracle import nf4, qlora

# Tolerance stated for the bf16-in / fp32-accumulate outputs h, dX, dA, dB.
TOL = 2e-2


def f32(t):
    """bf16/fp32 torch tensor (any device) -> float32 numpy (exact for bf16 values)."""
    return t.detach().to("cpu").float().numpy()


def bits(t):
    """bf16 torch tensor -> uint16 numpy bit patterns."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_pack(W_bf16_cpu, dq, rows=None, chunk=2048):
    """Oracle quantisation of W0.  With ``rows``, codes are produced for those rows only
    (absmax and the double-quant groups always cover the whole weight).  Rows are independent
    once the effective absmax is known, so codes are computed ``chunk`` rows at a time to bound
    host memory (the arithmetic is unchanged)."""
    w = f32(W_bf16_cpu)
    N, K = w.shape
    am = nf4.block_absmax(w)
    out = {"absmax": am.reshape(-1)}
    if dq:
        q8, sc = nf4.double_quant(am.reshape(-1))
        eff = nf4.dq_effective_absmax(q8, sc).reshape(N, K // 64)
        out["absmax_q8"], out["absmax_scale"] = q8, sc
    else:
        eff = am
    out["absmax_eff"] = eff
    sel = np.arange(N) if rows is None else np.asarray(rows)
    out["rows"] = sel
    q = np.empty((len(sel), K // 2), np.uint8)
    for c in range(0, len(sel), chunk):
        r = sel[c:c + chunk]
        q[c:c + chunk] = nf4.pack_codes(nf4.choose_codes(w[r], eff[r]))
    out["q"] = q
    return out


def oracle_dequant(ref, chunk=2048):
    """deq(W0) as float32 (bf16-exact) for the rows in ``ref`` (row chunks bound memory)."""
    q, eff, rows = ref["q"], ref["absmax_eff"], ref["rows"]
    K = q.shape[1] * 2
    out = np.empty((len(rows), K), np.float32)
    for c in range(0, len(rows), chunk):
        r = rows[c:c + chunk]
        out[c:c + chunk] = nf4.dequantize(q[c:c + chunk], eff[r], len(r), K)
    return out


def subset(ref, rows):
    """A copy of a full-weight oracle pack restricted to the given weight rows."""
    out = dict(ref)
    out["rows"] = np.asarray(rows)
    out["q"] = ref["q"][np.asarray(rows)]
    return out


def gpu_pack(W_bf16_cpu, dq):
    W = W_bf16_cpu.cuda()
    w = linear.nf4_pack(W, double_quant=dq)
    torch.cuda.synchronize()
    return w


def check_pack(wg, ref, dq):
    """Bit-exact: codes, absmax (and q8 / scale), and the dequantised weight."""
    rows = ref["rows"]
    q = wg.q.cpu().numpy()[rows]
    assert np.array_equal(q, ref["q"]), "packed codes differ"
    assert np.array_equal(wg.absmax.cpu().numpy().view(np.uint32),
                          ref["absmax"].view(np.uint32)), "absmax differs"
    if dq:
        assert np.array_equal(wg.absmax_q8.cpu().numpy(), ref["absmax_q8"]), "q8 differs"
        assert np.array_equal(wg.absmax_scale.cpu().numpy().view(np.uint32),
                              ref["absmax_scale"].view(np.uint32)), "scale differs"
    deq = bits(linear.nf4_dequant(wg))[rows]
    N, K = wg.N, wg.K
    ref_deq = nf4.dequantize_bits(ref["q"], ref["absmax_eff"][rows], len(rows), K)
    assert np.array_equal(deq, ref_deq), "dequantised weight differs"


def oracle_deq(W_bf16_cpu, dq):
    ref = oracle_pack(W_bf16_cpu, dq)
    N, K = W_bf16_cpu.shape
    return ref, nf4.dequantize(ref["q"], ref["absmax_eff"], N, K)


def run_linear(inp, L, dq=None, need_dx=True):
    """GPU pack + forward + backward of one linear; returns a dict of CPU tensors."""
    dq = L.double_quant if dq is None else dq
    lin = inp["linears"][0]
    X, dY = inp["X"].cuda(), inp["dY"].cuda()
    A, B = lin["A"].cuda(), lin["B"].cuda()
    w = linear.nf4_pack(lin["W0"].cuda(), double_quant=dq)
    H, XA = linear.forward(X, w, A, B, L.alpha)
    dX, dA, dB = linear.backward(dY, X, w, A, B, XA, L.alpha, need_dx=need_dx)
    torch.cuda.synchronize()
    code = linear.device_error()
    assert code == 0, f"device error word set: {code}"
    return {"w": w, "H": H, "XA": XA, "dX": dX, "dA": dA, "dB": dB}


def check_linear(inp, L, got, rows=None, dq=None):
    """Compare the GPU outputs with the oracle (all rows, or the sampled ``rows``)."""
    dq = L.double_quant if dq is None else dq
    lin = inp["linears"][0]
    ref, Wd = oracle_deq(lin["W0"], dq)
    X, dY, A, B = (f32(inp["X"]), f32(inp["dY"]), f32(lin["A"]), f32(lin["B"]))
    M = X.shape[0]
    rows = np.arange(M) if rows is None else np.asarray(rows)
    errs = {}
    h_ref = qlora.forward_rows(X, Wd, A, B, L.alpha, rows)
    errs["h"] = qlora.rel_err(f32(got["H"])[rows], h_ref)
    errs["XA"] = qlora.rel_err(f32(got["XA"]), qlora.lora_down(X, A))
    wts = qlora.backward_weights(dY, X, A, B, L.alpha)
    errs["dA"] = qlora.rel_err(f32(got["dA"]), wts["dA"])
    errs["dB"] = qlora.rel_err(f32(got["dB"]), wts["dB"])
    if got["dX"] is not None:
        dx_ref = qlora.backward_dx_rows(dY, Wd, A, B, L.alpha, rows)
        errs["dX"] = qlora.rel_err(f32(got["dX"])[rows], dx_ref)
    for k, v in errs.items():
        assert v <= TOL, f"{k}: max|err|/max|ref| = {v:.3e} > {TOL}"
    return errs, ref


def make(M, K, N, r, alpha=None, seed=0, **kw):
    inp = synth.make_linear(M, K, N, r, alpha=alpha, seed=seed, **kw)
    L = synth.LinearShape("linear", K, N, r, alpha if alpha else 2.0 * r)
    return inp, L


# ------------------------------------------------------------------------------------------
# Packed adapters (one stacked NF4 weight, adapters along its rows, sharing X)
# ------------------------------------------------------------------------------------------
def stacked(inp):
    """W0, A, B of every adapter stacked by rows (CPU bf16)."""
    lins = inp["linears"]
    return (torch.cat([l["W0"] for l in lins]), torch.cat([l["A"] for l in lins]),
            torch.cat([l["B"] for l in lins]))


def run_grouped(inp, Ns, alpha, dq=False, need_dx=True):
    """GPU pack of the stacked weight + grouped forward + backward; CPU tensors out."""
    W0, A, B = stacked(inp)
    X, dY = inp["X"].cuda(), inp["dY"].cuda()
    A, B = A.cuda(), B.cuda()
    w = linear.nf4_pack(W0.cuda(), double_quant=dq)
    H, XA = linear.grouped_forward(X, w, A, B, list(Ns), alpha)
    dX, dA, dB = linear.grouped_backward(dY, X, w, A, B, XA, list(Ns), alpha, need_dx=need_dx)
    torch.cuda.synchronize()
    code = linear.device_error()
    assert code == 0, f"device error word set: {code}"
    return {"w": w, "H": H, "XA": XA, "dX": dX, "dA": dA, "dB": dB}


def check_grouped(inp, Ns, alpha, got, rows=None, dq=False):
    """The packed layer against the oracle: the stacked weight is quantised as one tensor and
    its dequantised rows split by adapter.  Returns the error dict."""
    W0, _, _ = stacked(inp)
    ref, Wd = oracle_deq(W0, dq)
    edges = np.cumsum([0] + list(Ns))
    Wds = [Wd[edges[i]:edges[i + 1]] for i in range(len(Ns))]
    As = [f32(l["A"]) for l in inp["linears"]]
    Bs = [f32(l["B"]) for l in inp["linears"]]
    X, dY = f32(inp["X"]), f32(inp["dY"])
    M = X.shape[0]
    rows = np.arange(M) if rows is None else np.asarray(rows)
    errs = {}
    errs["h"] = qlora.rel_err(f32(got["H"])[rows],
                              qlora.grouped_forward_rows(X, Wds, As, Bs, alpha, rows))
    errs["XA"] = qlora.rel_err(f32(got["XA"]), np.concatenate([qlora.lora_down(X, A) for A in As],
                                                              axis=1))
    wts = qlora.grouped_backward_weights(dY, X, As, Bs, alpha)
    errs["dA"] = qlora.rel_err(f32(got["dA"]), wts["dA"])
    errs["dB"] = qlora.rel_err(f32(got["dB"]), wts["dB"])
    # Per adapter too: a small adapter's error must not hide under a large one's scale.
    r = As[0].shape[0]
    for i in range(len(Ns)):
        errs[f"dA{i}"] = qlora.rel_err(f32(got["dA"])[i * r:(i + 1) * r],
                                       wts["dA"][i * r:(i + 1) * r])
        errs[f"dB{i}"] = qlora.rel_err(f32(got["dB"])[edges[i]:edges[i + 1]],
                                       wts["dB"][edges[i]:edges[i + 1]])
        errs[f"h{i}"] = qlora.rel_err(
            f32(got["H"])[rows][:, edges[i]:edges[i + 1]],
            qlora.forward_rows(X, Wds[i], As[i], Bs[i], alpha, rows))
    if got["dX"] is not None:
        errs["dX"] = qlora.rel_err(f32(got["dX"])[rows],
                                   qlora.grouped_backward_dx_rows(dY, Wds, As, Bs, alpha, rows))
    for k, v in errs.items():
        assert v <= TOL, f"{k}: max|err|/max|ref| = {v:.3e} > {TOL}"
    return errs
