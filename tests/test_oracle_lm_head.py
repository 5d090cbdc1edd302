"""Pins for the LM head + cross-entropy oracle (CPU only).

Checked against:
* closed forms: W = 0 gives loss log V and dX = 0; a two-word vocabulary gives the logistic
  loss;
* a pure-Python brute force of softmax and log on a tiny case;
* central finite differences of the loss in X;
* ignored tokens (labels outside [0, V)) and the all-ignored batch;
* stability and shift invariance of the logits' cross-entropy at large magnitude;
* zero row sums of the logits' gradient;
* chunking over tokens, which changes nothing.
"""

import math

import numpy as np

from oracle import lm_head, nf4


def _deq(V, K, rng, std=0.05):
    W0 = rng.standard_normal((V, K)) * std
    w32 = nf4.bf16_bits_to_f32(nf4.f32_to_bf16_bits(W0.astype(np.float32)))
    p = nf4.quantize(w32)
    return nf4.dequantize(p["q"], p["absmax_eff"], V, K).astype(np.float64)


def test_zero_head_gives_log_v():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((5, 128))
    V = 192
    out = lm_head.lm_head_ce(X, np.zeros((V, 128)), np.array([0, 3, 191, 7, 50]))
    assert np.allclose(out["token_loss"], math.log(V), rtol=0, atol=1e-13)
    assert abs(out["loss"] - math.log(V)) < 1e-13
    assert np.all(out["dX"] == 0)


def test_two_word_vocabulary_is_the_logistic_loss():
    rng = np.random.default_rng(1)
    z = rng.standard_normal((6, 2)) * 3
    y = np.array([0, 1, 1, 0, 1, 0])
    loss, dz = lm_head.ce_from_logits(z, y, 6)
    other = z[np.arange(6), 1 - y]
    mine = z[np.arange(6), y]
    assert np.allclose(loss, np.log1p(np.exp(other - mine)), rtol=1e-13, atol=1e-14)
    # d loss / d z_y = -(1 - sigmoid(z_y - z_other)), shared by the batch of 6
    sig = 1.0 / (1.0 + np.exp(-(mine - other)))
    assert np.allclose(dz[np.arange(6), y], -(1.0 - sig) / 6, rtol=1e-12, atol=1e-15)


def test_brute_force_tiny():
    z = [[0.5, -1.0, 2.0, 0.0, 0.25], [3.0, 3.0, -2.0, 1.0, 0.5], [-0.5, 0.0, 0.0, 0.0, 4.0]]
    y = [2, 0, 4]
    n = 3
    loss, dz = lm_head.ce_from_logits(np.array(z), np.array(y), n)
    for i, row in enumerate(z):
        den = sum(math.exp(v) for v in row)
        assert abs(loss[i] - (math.log(den) - row[y[i]])) < 1e-13
        for j, v in enumerate(row):
            want = (math.exp(v) / den - (1.0 if j == y[i] else 0.0)) / n
            assert abs(dz[i, j] - want) < 1e-15


def test_finite_differences_in_x():
    rng = np.random.default_rng(2)
    M, K, V = 4, 128, 64
    X = rng.standard_normal((M, K))
    Wd = _deq(V, K, rng)
    y = np.array([1, 63, -100, 20])
    out = lm_head.lm_head_ce(X, Wd, y)
    h = 1e-5
    for _ in range(8):
        i, j = rng.integers(M), rng.integers(K)
        E = np.zeros_like(X)
        E[i, j] = h
        fd = (lm_head.lm_head_ce(X + E, Wd, y)["loss"] - lm_head.lm_head_ce(X - E, Wd, y)["loss"]) / (2 * h)
        assert abs(fd - out["dX"][i, j]) <= 1e-7 * max(1.0, abs(fd))


def test_ignored_tokens():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((5, 128))
    Wd = _deq(64, 128, rng)
    y = np.array([5, -100, 64, 0, -1])       # 64 == V and negatives are ignored
    out = lm_head.lm_head_ce(X, Wd, y)
    assert out["count"] == 2
    assert np.all(out["token_loss"][[1, 2, 4]] == 0) and np.all(out["dX"][[1, 2, 4]] == 0)
    kept = lm_head.lm_head_ce(X[[0, 3]], Wd, y[[0, 3]])
    assert abs(out["loss"] - kept["loss"]) < 1e-13
    assert np.allclose(out["dX"][[0, 3]], kept["dX"], rtol=1e-13, atol=1e-15)
    none = lm_head.lm_head_ce(X, Wd, np.full(5, -100))
    assert none["loss"] == 0.0 and np.all(none["dX"] == 0)


def test_stability_and_shift_invariance():
    rng = np.random.default_rng(4)
    z = rng.standard_normal((3, 100)) * 5
    y = np.array([0, 50, 99])
    a, da = lm_head.ce_from_logits(z, y, 3)
    b, db = lm_head.ce_from_logits(z + 1000.0, y, 3)
    assert np.all(np.isfinite(b)) and np.allclose(a, b, rtol=1e-10, atol=1e-10)
    assert np.allclose(da, db, rtol=1e-9, atol=1e-15)
    assert np.allclose(da.sum(axis=1), 0.0, atol=1e-15)


def test_rows_variant_matches_full():
    rng = np.random.default_rng(5)
    X = rng.standard_normal((9, 128))
    Wd = _deq(128, 128, rng)
    y = rng.integers(0, 128, 9)
    out = lm_head.lm_head_ce(X, Wd, y)
    tl, dx = lm_head.lm_head_ce_rows(X, Wd, y, [0, 4, 8], out["count"])
    assert np.allclose(tl, out["token_loss"][[0, 4, 8]], rtol=1e-13, atol=1e-13)
    assert np.allclose(dx, out["dX"][[0, 4, 8]], rtol=1e-12, atol=1e-15)


def test_chunking_changes_nothing():
    """The fused loss is read as chunks of tokens: each chunk's logits, its rows' losses and its
    gradient scaled by the whole batch's count.  That gives the unchunked losses, loss and dX
    for any chunk size, including a ragged last chunk."""
    rng = np.random.default_rng(6)
    M, K, V = 23, 128, 96
    X = rng.standard_normal((M, K))
    Wd = _deq(V, K, rng)
    y = rng.integers(0, V, M)
    y[[2, 9]] = -100
    full = lm_head.lm_head_ce(X, Wd, y)
    n = lm_head.valid_count(y, V)
    for c in (1, 5, 8, 23, 64):
        tl, dx = [], []
        for m0 in range(0, M, c):
            t, d = lm_head.ce_from_logits(X[m0:m0 + c] @ Wd.T, y[m0:m0 + c], n)
            tl.append(t)
            dx.append(d @ Wd)
        tl, dx = np.concatenate(tl), np.concatenate(dx)
        assert np.allclose(tl, full["token_loss"], rtol=1e-13, atol=1e-13)
        assert abs(tl.sum() / n - full["loss"]) < 1e-12
        assert np.allclose(dx, full["dX"], rtol=1e-12, atol=1e-15)
