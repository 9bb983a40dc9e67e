"""Blockwise 4-bit quantization with other 16-level code books, with or without double
quantization, and the merge of trained adapters back into a re-quantized base.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): the CUDA path never imports this.

Sources (page title, section):

* "QLoRA Paper Breakdown: 4-Bit NormalFloat (NF4), Double Quantization, and Paged
  Optimizers" (fullstackaihub teardown): section 1 (standard INT4 divides [-c, +c] into 16
  equally spaced bins), section 3 (single blockwise quantization, 4 + 32/64 = 4.5 bits per
  parameter), "Engineering Limitations" (full-rank updates need the adapters dequantized and
  merged into 16-bit precision).
* dmarx anthology, sota-230 (the data-type comparison: Int4, Float4 (E2M1), Float4 (E3M0),
  NF4 + double quantization).
* "QLoRA Explained: What Actually Trains in 4 Bits? | Part 2/6" (video description): adapter
  merging / re-quantization is a deployment step.

Pins (``tests/test_oracle_variants.py``):

====================  ========================================================
function              pinned by
====================  ========================================================
fp4_e2m1_codebook     the E2M1 values rebuilt from the format's bit fields
int4_codebook         16 equally spaced rationals, endpoints -1 and +1
nearest_midpoint      brute-force argmin (ties to the lower index) on strictly
                      increasing tables; the signed zeros of E2M1 in closed form
quantize_blockwise    equals ``nf4.quantize_nf4_dq`` for NF4 + DQ; exact-rational
                      brute force on tiny tensors for E2M1 and INT4; storage
                      4.5 bits per weight without DQ (teardown section 3)
dequant_blockwise     exact-rational recomputation over many blocks
merge_requantize      B = 0 returns the base's own bf16 values; an exact-rational
                      recomputation of the float64 sum and its one bf16 rounding
                      on small shapes; the sum order (index order) against a
                      reordered sum that differs in float64
====================  ========================================================
"""

from __future__ import annotations

from fractions import Fraction

import numpy as np

from . import nf4

B1 = nf4.B1
B2 = nf4.B2


# ----------------------------------------------------------------------------------------
# code books
# ----------------------------------------------------------------------------------------

def fp4_e2m1_codebook() -> np.ndarray:
    """The 16 values of the 4-bit float E2M1 (1 sign, 2 exponent bits with bias 1, 1 mantissa
    bit: 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives), divided by 6 so that they span
    [-1, 1], sorted, each rounded to the nearest fp32.  Both zeros are kept (-0 below +0).

    Reading: the pages name the data type (sota-230) without a normalisation; absmax scaling
    maps the block onto the type's largest magnitude, 6.  Codes index this sorted table; they
    are not the E2M1 bit patterns."""
    mags = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
            Fraction(4), Fraction(6)]
    neg = [-m for m in reversed(mags)]                 # -6 .. -0
    vals = [nf4.f32_from_rational(v / 6) for v in neg + mags]
    out = np.array(vals, dtype=np.float32)
    out[7] = np.float32(-0.0)                           # the negative zero
    return out


def int4_codebook() -> np.ndarray:
    """16 equally spaced levels over [-1, 1], both ends included: q_i = -1 + 2 i / 15.

    Reading: the teardown (section 1) describes standard INT4 as 16 equally spaced bins over
    [-c, +c]; with absmax scaling the block's largest weight maps exactly to an end level, as
    with NF4."""
    return np.array([nf4.f32_from_rational(Fraction(2 * i - 15, 15)) for i in range(16)], dtype=np.float32)


CODEBOOKS = {"nf4": nf4.nf4_codebook, "fp4_e2m1": fp4_e2m1_codebook, "int4": int4_codebook}


def codebook(name: str) -> np.ndarray:
    return CODEBOOKS[name]()


# ----------------------------------------------------------------------------------------
# nearest level by the midpoint rule
# ----------------------------------------------------------------------------------------

def nearest_midpoint(n, table: np.ndarray) -> np.ndarray:
    """code = #{j : n > (q_j + q_{j+1}) / 2}: the nearest level, an exact tie going to the lower
    index.  For a strictly increasing table this is argmin |n - q_j|; for E2M1's two zeros
    (whose midpoint is 0) it gives -0 for n <= 0 and +0 for small n > 0, keeping the sign.
    Midpoints are exact in float64 for fp32 levels."""
    q = np.asarray(table, np.float32).astype(np.float64)
    mids = 0.5 * (q[:-1] + q[1:])
    n = np.asarray(n, np.float32).astype(np.float64).ravel()
    return np.searchsorted(mids, n, side="left").astype(np.uint8)


# ----------------------------------------------------------------------------------------
# blockwise quantize / dequantize with a code book, with or without double quantization
# ----------------------------------------------------------------------------------------

def quantize_blockwise(w, table: np.ndarray, double_quant: bool) -> dict:
    """Flat blocks of 64, absmax per block, n = fp32(w / absmax) (correctly rounded), the code
    of the nearest level (``nearest_midpoint``), two codes per byte (element 2i in the low
    nibble).  An all-zero block codes to the level-7 slot (zero in every table here).  With
    double quantization the absmax values are coded exactly as ``nf4.double_quantize`` does;
    without it they are kept as fp32 (teardown section 3, single blockwise quantization)."""
    w = np.asarray(w, dtype=np.float32).ravel()
    nb = -(-w.size // B1)
    wp = np.zeros(nb * B1, dtype=np.float32)
    wp[:w.size] = w
    blocks = wp.reshape(nb, B1)
    absmax = np.max(np.abs(blocks), axis=1).astype(np.float32)
    safe = np.where(absmax > 0, absmax, np.float32(1)).astype(np.float64)
    n = (blocks.astype(np.float64) / safe[:, None]).astype(np.float32)
    codes = nearest_midpoint(n, table).reshape(nb, B1)
    codes[absmax == 0, :] = 7
    flat = codes.ravel()
    packed = (flat[0::2] | (flat[1::2] << 4)).astype(np.uint8)
    out = {"codes": packed, "absmax": absmax, "numel": w.size}
    if double_quant:
        out.update(nf4.double_quantize(absmax))
    return out


def dequant_blockwise(packed, table: np.ndarray, numel: int, scale_codes=None, c2=None, mean=None,
                      absmax=None) -> np.ndarray:
    """W'_e = bf16(fp32(q[code_e] * s_b)), s_b the block's scale: the fmaf of its double-quantized
    code (``nf4.block_scales``) or, without double quantization, its fp32 absmax."""
    q = np.asarray(table, np.float32)
    codes = nf4.unpack_codes(packed, numel)
    if absmax is not None:
        s = np.asarray(absmax, np.float32)
    else:
        s = nf4.block_scales(scale_codes, c2, mean)
    sb = s[np.arange(numel) // B1]
    prod = (q[codes].astype(np.float64) * sb.astype(np.float64)).astype(np.float32)
    return nf4.bf16_rn_bits(prod)


def storage_bits(numel: int, double_quant: bool) -> float:
    """Bits per weight of the stored parts (codes and scales, without the per-tensor mean)."""
    nb = -(-numel // B1)
    if double_quant:
        ng = -(-nb // B2)
        return (nb * B1 * 4 + nb * 8 + ng * 32) / numel
    return (nb * B1 * 4 + nb * 32) / numel


# ----------------------------------------------------------------------------------------
# adapter merge + re-quantization
# ----------------------------------------------------------------------------------------

def bf16_rn_from_f64(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (nearest, ties to even), once: the float64 significand
    keeps its top 8 bits (7 stored), the dropped 45 bits decide the rounding.  Returns the
    16-bit patterns.  Magnitudes below 2^-126 (bf16 subnormals) take the exact-rational path."""
    x = np.asarray(x, np.float64).ravel()
    b = x.view(np.uint64)
    lsb = (b >> np.uint64(45)) & np.uint64(1)
    rb = (b + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    y = rb.view(np.float64).astype(np.float32)          # exact: 8 significant bits
    out = (y.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    small = (np.abs(x) < 2.0 ** -126) & (x != 0)
    for i in np.flatnonzero(small):
        out[i] = _bf16_rn_scalar(float(x[i]))
    out[x == 0] = np.where(np.signbit(x[x == 0]), 0x8000, 0).astype(np.uint16)
    return out


def _bf16_rn_scalar(v: float) -> int:
    if v == 0.0:
        return 0x8000 if np.signbit(v) else 0
    r = Fraction(v)
    sign = 0x8000 if r < 0 else 0
    a = abs(r)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    e = max(e, -126)
    scaled = abs(r) / Fraction(2) ** (e - 7)
    lo = scaled.numerator // scaled.denominator
    rem = scaled - lo
    up = rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1)
    mant = lo + (1 if up else 0)
    if mant >= 256:
        mant //= 2
        e += 1
    if mant < 128:
        return sign | mant
    return sign | ((e + 127) << 7) | (mant - 128)


def merge_requantize(w_deq_bits: np.ndarray, A: np.ndarray, B: np.ndarray, s: float, table: np.ndarray,
                     double_quant: bool = True) -> dict:
    """Fold the adapters into the frozen base and quantize the result again.

    W''[n, k] = bf16( W'[n, k] + s * sum_j B[n, j] A[j, k] ), then ``quantize_blockwise`` of W''.

    Steps (teardown, "Engineering Limitations": full-rank updates need the adapters merged into
    16-bit precision; video description: merging / re-quantization at deployment):
    1. The rank-r sum is formed in float64, term by term in index order j = 0 .. r-1 (each
       product of two bf16 values is exact in float64).
    2. t = float64(s * sum); v = float64(W' + t).
    3. W'' = bf16 of v, one rounding to nearest even.
    Reading: the pages fix no precision or order for the merge; float64 in index order is a
    determinism choice, and the bf16 result is the adapters' dtype.  W' is the exact bf16
    dequantized base (``dequant_blockwise``), given as bit patterns [N, K]."""
    Wd = nf4.bf16_bits_to_f32(np.asarray(w_deq_bits, np.uint16)).astype(np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    N, K = Wd.shape
    r = A.shape[0]
    acc = np.zeros((N, K), np.float64)
    for j in range(r):
        acc = acc + B[:, j:j + 1] * A[j:j + 1, :]
    v = Wd + float(s) * acc
    merged = bf16_rn_from_f64(v).reshape(N, K)
    q = quantize_blockwise(nf4.bf16_bits_to_f32(merged).ravel(), table, double_quant)
    q["merged_bits"] = merged
    return q
