"""NF4 (4-bit NormalFloat) blockwise quantisation -- oracle, TEST INFRASTRUCTURE ONLY.

What the pages fix: the frozen base weight W0 is stored as 4-bit NormalFloat (NF4), a 75 %
cut of base-weight memory against FP16 ("Unsloth vs QLoRA vs Liger-Kernel", FAQ "What is the
difference between LoRA and QLoRA?"; "Speed up fine-tuning 2x", "How it works internally",
item 1 "4-bit Quantization").  Everything below that the pages leave open is a stated
reading:

R1  Codebook.  The 4-bit NormalFloat construction: quantiles of N(0, 1) taken at evenly
    spaced probabilities, asymmetric so that zero is exact -- 8 strictly positive levels,
    7 strictly negative levels and an exact 0 -- then divided by the largest magnitude so the
    set spans exactly [-1, 1].  The probabilities run from ``OFFSET`` down to 1/2: the
    positive half takes 9 evenly spaced points on [1/2, OFFSET] and drops the one at 1/2,
    the negative half takes 8 evenly spaced points and drops the one at 1/2 (negated).
    ``OFFSET = 1 - (1/32 + 1/30)/2`` is the mean of the outermost bin-centre probabilities
    of a 16-level and a 15-level equal-probability partition (the two halves hold 16 and 15
    bins' worth of levels once mirrored), which keeps Q(OFFSET) finite.  The GPU uses the
    fp32 rounding of each value (``codebook_f32``).
R2  Blocks.  64 consecutive elements of the row-major W0 [N, K] form one block; K % 64 == 0,
    so a block never straddles rows.  absmax[n, kb] = max |W0[n, 64 kb : 64 kb + 64]|,
    stored fp32 in row-major [N, K/64] order (block index = n * K/64 + kb).
R3  Code choice.  x = RN_fp32(w / absmax); code = #{i in 0..14 : x > m_i} with midpoints
    m_i = RN_fp32((c_i + c_{i+1}) / 2) of the fp32 codebook.  A value exactly on a
    midpoint takes the lower code.  A block whose (effective) absmax is 0 gets code 7 (the
    exact zero) everywhere.
R4  Packing.  Two codes per byte, row-major: element 2j of a row goes to the HIGH nibble
    (bits 7..4) of byte j, element 2j+1 to the low nibble.  Q has shape [N, K/2].
R5  Double-quantised absmax (8-bit absmax per 64-block, fp32 second-level scale per 256
    absmax values).  Groups are 256 consecutive absmax values in block order (the last group
    may be partial).  S_g = RN_fp32(max(absmax in g) / 255);
    q8 = clamp(rint_half_even(RN_fp32(absmax / S_g)), 0, 255) (q8 = 0 when S_g == 0);
    the effective absmax is absmax' = RN_fp32(q8 * S_g) and W0 is quantised with absmax'.
R6  Dequantisation.  deq = RN_bf16(RN_fp32(c_fp32[code] * absmax)) -- an fp32 product
    rounded once to fp32 and then once to bf16 (round to nearest, ties to even).

Precision: every fp32 result above is computed in float64 and rounded once to float32.  For a
single +, *, / of float32 operands this equals the correctly rounded float32 result, because
float64 carries more than 2*24+2 significand bits.
"""

import numpy as np
from scipy.special import ndtri

BLOCK = 64          # R2
GROUP = 256         # R5
OFFSET = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)   # R1


# --------------------------------------------------------------------------------------
# bf16 helpers (bit-level, NumPy has no bf16 type)
# --------------------------------------------------------------------------------------
def bf16_bits_to_f32(bits):
    """uint16 bf16 bit patterns -> the float32 values they encode (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def f32_to_bf16_bits(x):
    """Round float32 values to bf16, round-to-nearest, ties-to-even; returns uint16 bits.

    The 16 dropped bits are compared against one half ulp of bf16: add 0x7FFF plus the lowest
    kept bit and truncate.  Inputs here are finite (no NaN handling needed).
    """
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def round_f32(x64):
    """Round float64 values once to float32 (IEEE round to nearest even)."""
    return np.asarray(x64, dtype=np.float64).astype(np.float32)


# --------------------------------------------------------------------------------------
# R1: the codebook
# --------------------------------------------------------------------------------------
def codebook_f64():
    """The 16 NF4 levels in float64, ascending; c[0] = -1, c[7] = 0, c[15] = +1 (R1)."""
    pos_p = np.linspace(OFFSET, 0.5, 9)[:-1]    # 8 probabilities in (1/2, OFFSET]
    neg_p = np.linspace(OFFSET, 0.5, 8)[:-1]    # 7 probabilities in (1/2, OFFSET]
    pos = ndtri(pos_p)
    neg = -ndtri(neg_p)
    levels = np.concatenate([neg, [0.0], pos])
    levels = np.sort(levels)
    return levels / np.max(np.abs(levels))


def codebook_f32():
    """fp32 rounding of the codebook -- the table both quantiser and dequantiser use."""
    return round_f32(codebook_f64())


def midpoints_f32(c32=None):
    """m_i = RN_fp32((c_i + c_{i+1}) / 2) for i = 0..14 (R3)."""
    c = codebook_f32() if c32 is None else np.asarray(c32, np.float32)
    c64 = c.astype(np.float64)
    return round_f32((c64[:-1] + c64[1:]) / 2.0)


# --------------------------------------------------------------------------------------
# R2, R3: absmax and code choice
# --------------------------------------------------------------------------------------
def block_absmax(w_f32):
    """absmax per 64-block of row-major W0 [N, K] (values bf16-exact in float32) -> [N, K/64]."""
    w = np.asarray(w_f32, dtype=np.float32)
    n, k = w.shape
    assert k % BLOCK == 0
    return np.abs(w).reshape(n, k // BLOCK, BLOCK).max(axis=2).astype(np.float32)


def choose_codes(w_f32, absmax_f32):
    """Code per element (uint8 in 0..15) given the effective fp32 absmax per block (R3)."""
    w = np.asarray(w_f32, dtype=np.float32)
    n, k = w.shape
    a = np.asarray(absmax_f32, dtype=np.float32).reshape(n, k // BLOCK)
    a_full = np.repeat(a, BLOCK, axis=1)
    zero = a_full == 0
    safe = np.where(zero, np.float32(1), a_full).astype(np.float64)
    x = round_f32(w.astype(np.float64) / safe)
    m = midpoints_f32()
    codes = np.zeros(w.shape, dtype=np.uint8)
    for mi in m:                       # count midpoints strictly below x
        codes += (x > mi).astype(np.uint8)
    codes[zero] = 7
    return codes


def pack_codes(codes):
    """R4: [N, K] codes -> [N, K/2] bytes, even element in the high nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    hi = c[:, 0::2]
    lo = c[:, 1::2]
    return ((hi << 4) | lo).astype(np.uint8)


def unpack_codes(q):
    """Inverse of ``pack_codes``."""
    q = np.asarray(q, dtype=np.uint8)
    n, kh = q.shape
    out = np.empty((n, 2 * kh), dtype=np.uint8)
    out[:, 0::2] = q >> 4
    out[:, 1::2] = q & 0x0F
    return out


# --------------------------------------------------------------------------------------
# R5: double-quantised absmax
# --------------------------------------------------------------------------------------
def double_quant(absmax_f32):
    """absmax [nblocks] -> (q8 uint8 [nblocks], scale fp32 [ceil(nblocks/256)]) (R5)."""
    a = np.asarray(absmax_f32, dtype=np.float32).reshape(-1)
    nb = a.size
    ng = (nb + GROUP - 1) // GROUP
    scale = np.zeros(ng, dtype=np.float32)
    q8 = np.zeros(nb, dtype=np.uint8)
    for g in range(ng):
        seg = a[g * GROUP:(g + 1) * GROUP]
        s = round_f32(np.float64(seg.max()) / 255.0)
        scale[g] = s
        if s == 0:
            continue
        t = round_f32(seg.astype(np.float64) / np.float64(s))
        q8[g * GROUP:(g + 1) * GROUP] = np.clip(np.rint(t), 0, 255).astype(np.uint8)
    return q8, scale


def dq_effective_absmax(q8, scale):
    """absmax' = RN_fp32(q8 * S_g) per block (R5)."""
    q = np.asarray(q8, dtype=np.uint8).reshape(-1).astype(np.float64)
    g = np.arange(q.size) // GROUP
    return round_f32(q * np.asarray(scale, np.float32)[g].astype(np.float64))


# --------------------------------------------------------------------------------------
# Whole pack and dequant
# --------------------------------------------------------------------------------------
def quantize(w_f32, double_quant_absmax=False):
    """Quantise bf16-valued W0 [N, K] (given as float32).

    Returns a dict with ``q`` [N, K/2] uint8, ``absmax`` [N*K/64] fp32 (first-level absmax),
    and, when ``double_quant_absmax``, ``absmax_q8`` [N*K/64] uint8 and ``absmax_scale``
    [ceil(N*K/64/256)] fp32.  ``absmax_eff`` is the absmax the codes were chosen with.
    """
    w = np.asarray(w_f32, dtype=np.float32)
    n, k = w.shape
    am = block_absmax(w).reshape(-1)
    out = {"absmax": am}
    if double_quant_absmax:
        q8, sc = double_quant(am)
        eff = dq_effective_absmax(q8, sc)
        out["absmax_q8"] = q8
        out["absmax_scale"] = sc
    else:
        eff = am
    out["absmax_eff"] = eff
    out["q"] = pack_codes(choose_codes(w, eff.reshape(n, k // BLOCK)))
    return out


def dequantize_bits(q, absmax_eff, n, k):
    """R6: packed codes + effective absmax -> deq(W0) as bf16 bit patterns [N, K] (uint16)."""
    codes = unpack_codes(np.asarray(q, np.uint8).reshape(n, k // 2))
    c64 = codebook_f32().astype(np.float64)
    a = np.repeat(np.asarray(absmax_eff, np.float32).reshape(n, k // BLOCK), BLOCK, axis=1)
    prod = round_f32(c64[codes] * a.astype(np.float64))
    return f32_to_bf16_bits(prod)


def dequantize(q, absmax_eff, n, k):
    """deq(W0) as float32 (bf16-exact values) [N, K]."""
    return bf16_bits_to_f32(dequantize_bits(q, absmax_eff, n, k))
