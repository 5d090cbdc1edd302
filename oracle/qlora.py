"""LoRA-adapted linear over a frozen NF4 base -- oracle, TEST INFRASTRUCTURE ONLY.

Forward (from "Unsloth vs QLoRA vs Liger-Kernel", section 1 "The Bottlenecks in Standard
PyTorch Fine-Tuning", which writes h = W0 x + (alpha/r) B A x for one column x; here rows of X
are tokens, so the same map reads)::

    XA = X A^T                          [M, r]
    h  = X deq(W0)^T + s * XA B^T       [M, N],   s = alpha / r

Backward.  The pages say the gradients are derived by hand and equal plain autograd up to
rounding ("Unsloth vs QLoRA vs Liger-Kernel", FAQ "Does Unsloth cause accuracy degradation?";
"FTDD-03" teaching script, [SLIDE 3], decisions one and two) but print no formula.  The
formulas are the exact gradients of the forward above for an upstream gradient dY = dL/dh,
with W0 frozen (no weight gradient for it)::

    dYB = dY B                          [M, r]
    dX  = dY deq(W0) + s * dYB A        [M, K]
    dB  = s * dY^T XA                   [N, r]
    dA  = s * dYB^T X                   [r, K]

Everything is float64 on the bf16-valued inputs and on the bf16-valued deq(W0) produced by
``oracle.nf4``; XA and dYB stay unrounded float64 here (the GPU keeps them in bf16; the
difference sits inside the stated tolerance).  Matrix products use NumPy's BLAS matmul.

``*_rows`` variants evaluate h and dX on a subset of token rows only -- each row of h and dX
depends on that row of X / dY alone -- so large workloads can be checked on sampled rows while
dA and dB are still computed over all tokens.
"""

import numpy as np


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def scale(alpha, r):
    """s = alpha / r in float64."""
    return float(alpha) / float(r)


def forward(X, Wdeq, A, B, alpha):
    """Return (h, XA) for X [M,K], Wdeq [N,K], A [r,K], B [N,r]."""
    X, Wdeq, A, B = _f64(X), _f64(Wdeq), _f64(A), _f64(B)
    s = scale(alpha, A.shape[0])
    XA = X @ A.T
    h = X @ Wdeq.T + s * (XA @ B.T)
    return h, XA


def forward_rows(X, Wdeq, A, B, alpha, rows):
    """h restricted to the given token rows: X[rows] deq^T + s X[rows] A^T B^T."""
    Xr = _f64(X)[np.asarray(rows)]
    return forward(Xr, Wdeq, A, B, alpha)[0]


def lora_down(X, A):
    """XA = X A^T in float64 (the saved rank-r activation)."""
    return _f64(X) @ _f64(A).T


def backward(dY, X, Wdeq, A, B, alpha):
    """Return dict(dX, dA, dB, dYB, XA) -- the hand-derived gradients in float64."""
    dY, X, Wdeq, A, B = _f64(dY), _f64(X), _f64(Wdeq), _f64(A), _f64(B)
    s = scale(alpha, A.shape[0])
    XA = X @ A.T
    dYB = dY @ B
    dX = dY @ Wdeq + s * (dYB @ A)
    dB = s * (dY.T @ XA)
    dA = s * (dYB.T @ X)
    return {"dX": dX, "dA": dA, "dB": dB, "dYB": dYB, "XA": XA}


def backward_weights(dY, X, A, B, alpha):
    """dA and dB over all tokens (O(M r (K+N)) work) plus dYB and XA."""
    dY, X, A, B = _f64(dY), _f64(X), _f64(A), _f64(B)
    s = scale(alpha, A.shape[0])
    XA = X @ A.T
    dYB = dY @ B
    return {"dA": s * (dYB.T @ X), "dB": s * (dY.T @ XA), "dYB": dYB, "XA": XA}


def backward_dx_rows(dY, Wdeq, A, B, alpha, rows):
    """dX restricted to the given token rows."""
    dYr = _f64(dY)[np.asarray(rows)]
    A, B = _f64(A), _f64(B)
    s = scale(alpha, A.shape[0])
    return dYr @ _f64(Wdeq) + s * ((dYr @ B) @ A)


# --------------------------------------------------------------------------------------
# Several adapters packed into one layer ("Speed Up Fine-Tuning 2x with Unsloth on Llama and
# Mistral", "How it works internally", item 3: several LoRA adapters packed into one tensor;
# "Unsloth vs QLoRA vs Liger-Kernel", section 5, step 2: adapters on q/k/v and gate/up, which
# read the same input).  The pages give no formula beyond the single layer, so the packed
# layer is read as exactly that: n independent layers (W0_g, A_g, B_g) on one X, each with
# s = alpha / r, whose outputs sit side by side in columns and whose input gradients add.
# The lists below hold the adapters in order; packed tensors stack them (H, dY, XA_saved by
# columns; A, dA, B, dB by rows).
# --------------------------------------------------------------------------------------
def split_cols(T, widths):
    """Column blocks of T of the given widths, in order."""
    T = _f64(T)
    edges = np.cumsum([0] + list(widths))
    assert edges[-1] == T.shape[1]
    return [T[:, edges[i]:edges[i + 1]] for i in range(len(widths))]


def grouped_forward(X, Wdeqs, As, Bs, alpha):
    """Return (H, XA_saved): each adapter's forward, outputs placed side by side."""
    outs = [forward(X, Wd, A, B, alpha) for Wd, A, B in zip(Wdeqs, As, Bs)]
    return (np.concatenate([h for h, _ in outs], axis=1),
            np.concatenate([xa for _, xa in outs], axis=1))


def grouped_forward_rows(X, Wdeqs, As, Bs, alpha, rows):
    return grouped_forward(_f64(X)[np.asarray(rows)], Wdeqs, As, Bs, alpha)[0]


def grouped_backward_weights(dY, X, As, Bs, alpha):
    """dA (adapters' dA_g stacked by rows) and dB (dB_g stacked by rows); adapter g takes its
    own column block of dY."""
    dYs = split_cols(dY, [B.shape[0] for B in Bs])
    parts = [backward_weights(dYg, X, A, B, alpha) for dYg, A, B in zip(dYs, As, Bs)]
    return {"dA": np.concatenate([p["dA"] for p in parts], axis=0),
            "dB": np.concatenate([p["dB"] for p in parts], axis=0)}


def grouped_backward_dx_rows(dY, Wdeqs, As, Bs, alpha, rows):
    """dX on the given rows: the sum over adapters of each one's input gradient."""
    dYs = split_cols(dY, [B.shape[0] for B in Bs])
    return sum(backward_dx_rows(dYg, Wd, A, B, alpha, rows)
               for dYg, Wd, A, B in zip(dYs, Wdeqs, As, Bs))


def grouped_backward(dY, X, Wdeqs, As, Bs, alpha):
    """All gradients of the packed layer over every row: dict(dX, dA, dB)."""
    out = grouped_backward_weights(dY, X, As, Bs, alpha)
    out["dX"] = grouped_backward_dx_rows(dY, Wdeqs, As, Bs, alpha, np.arange(_f64(X).shape[0]))
    return out


# --------------------------------------------------------------------------------------
# SwiGLU glue between gate/up and down in the MLP workload ("Unsloth vs QLoRA vs
# Liger-Kernel", section 2 names the MLP SwiGLU among the hand-differentiated ops; the pages
# print no formula).  a = silu(g) * u with silu(g) = g * sigmoid(g).
# --------------------------------------------------------------------------------------
def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def swiglu_forward(g, u):
    g, u = _f64(g), _f64(u)
    return g * _sigmoid(g) * u


def swiglu_backward(g, u, da):
    """Exact derivatives of a = g sigmoid(g) u: returns (dg, du)."""
    g, u, da = _f64(g), _f64(u), _f64(da)
    sg = _sigmoid(g)
    dg = da * u * sg * (1.0 + g * (1.0 - sg))
    du = da * g * sg
    return dg, du


def rel_err(got, ref):
    """The tolerance metric: max |got - ref| / max |ref|."""
    got, ref = _f64(got), _f64(ref)
    den = np.max(np.abs(ref))
    num = np.max(np.abs(got - ref))
    return float(num / den) if den > 0 else float(num)
