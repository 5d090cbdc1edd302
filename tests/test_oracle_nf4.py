"""Pins for the NF4 oracle (CPU only).

Each test checks ``oracle.nf4`` against something other than itself: closed forms of the
4-bit NormalFloat construction evaluated through the normal CDF (the inverse of the map the
oracle uses), brute-force nearest-level search, torch's own bf16 rounding, hand-worked
packing, and the invariants the blockwise absmax scheme must satisfy.
"""

import math
import os

import numpy as np
import pytest
import torch

from oracle import nf4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _phi(x):
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def _phi_inv_bisect(p):
    lo, hi = -10.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if _phi(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def test_offset_closed_form():
    assert nf4.OFFSET == pytest.approx(1.0 - (1.0 / 32 + 1.0 / 30) / 2, abs=0)
    assert abs(nf4.OFFSET - 0.96770833333333333) < 1e-15


def test_codebook_invariants():
    c = nf4.codebook_f64()
    assert c.shape == (16,)
    assert np.all(np.diff(c) > 0)
    assert c[0] == -1.0 and c[7] == 0.0 and c[15] == 1.0
    assert np.sum(c < 0) == 7 and np.sum(c > 0) == 8
    c32 = nf4.codebook_f32()
    assert c32.dtype == np.float32 and c32[0] == -1 and c32[7] == 0 and c32[15] == 1


def test_codebook_equal_probability_spacing():
    """Through the CDF: the positive levels sit at 8 equally spaced probabilities ending at
    OFFSET, the negative ones at 7, once scaled back by the normalising quantile."""
    c = nf4.codebook_f64()
    z = _phi_inv_bisect(nf4.OFFSET)
    step_pos = (nf4.OFFSET - 0.5) / 8
    step_neg = (nf4.OFFSET - 0.5) / 7
    pos = c[8:]                         # ascending, 8 values
    for j, v in enumerate(pos):         # j = 0 is the smallest positive level
        p_expected = 0.5 + (j + 1) * step_pos
        assert abs(_phi(v * z) - p_expected) < 1e-12
    neg = c[:7][::-1]                   # -0.09.. first
    for j, v in enumerate(neg):
        p_expected = 0.5 + (j + 1) * step_neg
        assert abs(_phi(-v * z) - p_expected) < 1e-12


def test_codebook_matches_golden_fixture():
    """Regression pin against the committed fp32 table (written by make_golden.py)."""
    path = os.path.join(GOLDEN, "nf4_codebook_f32.txt")
    vals = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            vals.append(int(line.split()[0], 16))
    got = nf4.codebook_f32().view(np.uint32)
    assert [int(v) for v in got] == vals


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(100000).astype(np.float32) * np.float32(3.0)
    # exact ties: low 16 bits == 0x8000, both parities of the kept lsb
    hi = rng.integers(0x3000, 0x4F00, 4000).astype(np.uint32)
    ties = ((hi << np.uint32(16)) | np.uint32(0x8000)).view(np.float32)
    allx = np.concatenate([x, ties, -ties, np.array([0.0, -0.0, 1e-30, -65504.0], np.float32)])
    ours = nf4.f32_to_bf16_bits(allx)
    ref = torch.from_numpy(allx).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = nf4.bf16_bits_to_f32(ref)
    assert np.array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def _bf16_exact(a):
    return nf4.bf16_bits_to_f32(nf4.f32_to_bf16_bits(np.asarray(a, np.float32)))


@pytest.mark.parametrize("s", [1.0, 0.5, 2.0 ** -7, 0.0371, 3.3])
def test_codebook_roundtrip(s):
    """A block holding (bf16-rounded) c_i * s and +-s quantises back to code i, and
    dequantises to RN_bf16(RN_fp32(c_i * absmax))."""
    c32 = nf4.codebook_f32()
    s_bf = _bf16_exact(s)[()]
    row = np.zeros(64, np.float32)
    row[:16] = _bf16_exact(c32.astype(np.float64) * s_bf)
    row[16] = s_bf
    row[17] = -s_bf
    w = row.reshape(1, 64)
    out = nf4.quantize(w)
    assert out["absmax"][0] == s_bf
    codes = nf4.unpack_codes(out["q"])[0]
    assert list(codes[:16]) == list(range(16))
    assert codes[16] == 15 and codes[17] == 0
    deq = nf4.dequantize_bits(out["q"], out["absmax_eff"], 1, 64)[0]
    expect = nf4.f32_to_bf16_bits((c32.astype(np.float64) * np.float64(s_bf)).astype(np.float32))
    assert np.array_equal(deq[:16], expect)


def test_absmax_element_maps_to_extreme_code():
    rng = np.random.default_rng(1)
    w = _bf16_exact(rng.standard_normal((16, 256)) * 0.02)
    out = nf4.quantize(w)
    codes = nf4.unpack_codes(out["q"])
    for n in range(16):
        for kb in range(4):
            blk = w[n, kb * 64:(kb + 1) * 64]
            j = int(np.argmax(np.abs(blk)))
            assert out["absmax"][n * 4 + kb] == np.abs(blk[j])
            assert codes[n, kb * 64 + j] == (15 if blk[j] > 0 else 0)


def test_degenerate_blocks():
    w = np.zeros((2, 128), np.float32)
    w[0, 64:] = 0.25          # constant positive block
    w[1, :64] = -0.75         # constant negative block
    out = nf4.quantize(w)
    codes = nf4.unpack_codes(out["q"])
    assert np.all(codes[0, :64] == 7)       # all-zero block -> the exact zero
    assert np.all(codes[0, 64:] == 15)
    assert np.all(codes[1, :64] == 0)
    assert np.all(codes[1, 64:] == 7)
    deq = nf4.dequantize_bits(out["q"], out["absmax_eff"], 2, 128)
    assert np.all(deq[0, :64] == 0) and np.all(deq[1, 64:] == 0)   # +0.0, not -0.0
    assert np.all(nf4.bf16_bits_to_f32(deq[0, 64:]) == 0.25)
    assert np.all(nf4.bf16_bits_to_f32(deq[1, :64]) == -0.75)


def test_midpoint_rule_equals_brute_force_nearest_level():
    rng = np.random.default_rng(2)
    x = rng.uniform(-1.3, 1.3, 100000).astype(np.float32)
    c64 = nf4.codebook_f32().astype(np.float64)
    exact_mid = (c64[:-1] + c64[1:]) / 2
    keep = np.min(np.abs(x[:, None].astype(np.float64) - exact_mid[None, :]), axis=1) > 1e-6
    x = x[keep]
    w = x.reshape(-1, 64) if x.size % 64 == 0 else x[: x.size // 64 * 64].reshape(-1, 64)
    codes = nf4.choose_codes(w, np.ones((w.shape[0], 1), np.float32)).reshape(-1)
    brute = np.argmin(np.abs(w.reshape(-1)[:, None].astype(np.float64) - c64[None, :]), axis=1)
    assert np.array_equal(codes, brute)


def test_exact_midpoint_goes_to_lower_code():
    m = nf4.midpoints_f32()
    w = np.zeros((1, 64), np.float32)
    w[0, :15] = m
    codes = nf4.choose_codes(w, np.ones((1, 1), np.float32))[0]
    assert list(codes[:15]) == list(range(15))
    # one ulp above the midpoint goes up
    w[0, :15] = np.nextafter(m, np.float32(2))
    codes = nf4.choose_codes(w, np.ones((1, 1), np.float32))[0]
    assert list(codes[:15]) == list(range(1, 16))


def test_pack_nibble_order_hand_worked():
    codes = np.array([[1, 2, 3, 4, 15, 0, 7, 9]], np.uint8)
    q = nf4.pack_codes(codes)
    assert list(q[0]) == [0x12, 0x34, 0xF0, 0x79]
    assert np.array_equal(nf4.unpack_codes(q), codes)


def test_double_quant_invariants():
    rng = np.random.default_rng(3)
    w = _bf16_exact(rng.standard_normal((8, 64 * 100)) * 0.015)   # 800 blocks: 3 full groups + 32
    am = nf4.block_absmax(w).reshape(-1)
    q8, sc = nf4.double_quant(am)
    assert q8.dtype == np.uint8 and sc.shape == (4,)
    for g in range(4):
        seg = am[g * 256:(g + 1) * 256]
        qs = q8[g * 256:(g + 1) * 256]
        assert qs[int(np.argmax(seg))] == 255
        assert sc[g] == np.float32(np.float64(seg.max()) / 255.0)
        eff = nf4.dq_effective_absmax(qs, np.array([sc[g]], np.float32)[np.zeros(1, int)])
        # effective absmax within half a step (plus fp32 rounding) of the true absmax
        assert np.all(np.abs(eff.astype(np.float64) - seg) <= sc[g] * (0.5 + 1e-5))
    out = nf4.quantize(w, double_quant_absmax=True)
    assert np.array_equal(out["absmax_q8"], q8)
    eff = nf4.dq_effective_absmax(q8, sc)
    assert np.array_equal(out["absmax_eff"], eff)
    # codes are chosen with the effective absmax
    ref_codes = nf4.choose_codes(w, eff.reshape(8, 100))
    assert np.array_equal(nf4.unpack_codes(out["q"]), ref_codes)


def test_double_quant_zero_group_and_tiny_absmax():
    am = np.zeros(300, np.float32)
    am[256] = 1.0
    am[257] = 1e-3      # rounds to q8 = 0 -> effective absmax 0 -> codes 7
    q8, sc = nf4.double_quant(am)
    assert sc[0] == 0 and np.all(q8[:256] == 0)
    assert q8[256] == 255 and q8[257] == 0
    w = np.zeros((1, 64 * 300), np.float32)
    w[0, 257 * 64:258 * 64] = np.float32(1e-3)
    w[0, 256 * 64] = 1.0
    out = nf4.quantize(w, double_quant_absmax=True)
    codes = nf4.unpack_codes(out["q"])[0]
    assert np.all(codes[257 * 64:258 * 64] == 7)
