"""LM head + cross-entropy over a frozen NF4 head -- oracle, TEST INFRASTRUCTURE ONLY.

"Unsloth vs QLoRA vs Liger-Kernel", section 3 (Liger-Kernel fused cross-entropy): the last
layer projects hidden states to the vocabulary and takes the cross-entropy loss; the fused
kernel computes it in chunks instead of holding all logits.  Chunking changes only where the
logits live, not what is computed, so the oracle is the plain definition::

    z      = X deq(W)^T                           [M, V]   (W frozen, no adapter)
    l_m    = logsumexp(z_m) - z_m[y_m]            for labels y_m in [0, V), else 0
    loss   = sum_m l_m / n,   n = #{m : 0 <= y_m < V}      (0 when n = 0)
    dz     = (softmax(z) - onehot(y)) / n         on counted rows, 0 elsewhere
    dX     = dz deq(W)                            [M, K]

Labels outside [0, V) (such as -100) are read as "ignore this token", the usual convention of
the cross-entropy loss the pages name; W gets no gradient.  Everything is float64 on the
bf16-valued inputs and the bf16-valued deq(W) from ``oracle.nf4``.  ``*_rows`` variants take a
subset of token rows plus the batch's count n (each row's loss and dX row depend on that row
alone, and on n), so full-size checks can sample rows.
"""

import numpy as np


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def valid_count(labels, V):
    y = np.asarray(labels)
    return int(np.sum((y >= 0) & (y < V)))


def logsumexp_rows(z):
    """Stable row-wise log(sum(exp(z))): the row maximum is taken out first."""
    z = _f64(z)
    mx = np.max(z, axis=1)
    return mx + np.log(np.sum(np.exp(z - mx[:, None]), axis=1))


def ce_from_logits(z, labels, n):
    """(token losses [m], dz [m, V]) of logits z [m, V], labels [m], batch count n."""
    z = _f64(z)
    y = np.asarray(labels)
    m, V = z.shape
    ok = (y >= 0) & (y < V)
    lse = logsumexp_rows(z)
    yy = np.where(ok, y, 0)
    picked = z[np.arange(m), yy]
    loss = np.where(ok, lse - picked, 0.0)
    dz = np.exp(z - lse[:, None])
    dz[np.arange(m), yy] -= 1.0
    dz[~ok] = 0.0
    dz = dz / n if n > 0 else np.zeros_like(dz)
    return loss, dz


def lm_head_ce(X, Wdeq, labels):
    """dict(loss, token_loss [M], dX [M, K]) for X [M, K], Wdeq [V, K], labels [M]."""
    X, Wdeq = _f64(X), _f64(Wdeq)
    n = valid_count(labels, Wdeq.shape[0])
    tl, dz = ce_from_logits(X @ Wdeq.T, labels, n)
    return {"loss": float(np.sum(tl) / n) if n > 0 else 0.0, "token_loss": tl, "dX": dz @ Wdeq,
            "count": n}


def lm_head_ce_rows(X, Wdeq, labels, rows, n):
    """(token losses, dX rows) on the given token rows, with the batch's count n."""
    rows = np.asarray(rows)
    Xr, Wdeq = _f64(X)[rows], _f64(Wdeq)
    tl, dz = ce_from_logits(Xr @ Wdeq.T, np.asarray(labels)[rows], n)
    return tl, dz @ Wdeq
