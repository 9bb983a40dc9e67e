"""NF4 blockwise quantization with double quantization (DQ), and its dequantization.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): the CUDA path never imports this.

Every function restates one step of the method in the order the pages give it.
Where the pages leave a step open, the reading taken is stated in the docstring
("Reading: ...").  Pins (the independent checks in ``tests/test_oracle_*.py``):

=====================  ======================================================
function               pinned by
=====================  ======================================================
nf4_codebook           printed table (fixture), the 10-digit level of the
                       video page's worked lookup, structure (7 neg / 0 /
                       8 pos, endpoints +-1), quantile construction
nf4_construct          reproduces the printed table to 3e-7
nearest_level          exact-rational brute force over every fp32 value
                       within +-64 ulp of each midpoint; the worked lookup
e4m3_decode/encode     closed form of all 256 codes; round trip of every
                       finite code; exact-rational nearest search on
                       midpoints; saturation
tree_sum_f64           equals exact rational sums on dyadic inputs;
                       permutation / padding invariants
quantize_nf4_dq        brute-force exact-rational recomputation on tiny
                       tensors; storage arithmetic of the pages; exact-zero
                       blocks; reconstruction error bound of the scales
dequant_nf4_dq         worked lookup (reconstruction 0.3218604028); exact
                       zeros; closed-form single-block cases; 600 blocks of
                       distinct scales (3 groups) against exact rationals
bf16_rn_bits           torch's fp32 -> bf16 cast on every tie pattern (both
                       parities of the kept bit) and neighbours; exact
                       rational nearest-even rounding on random patterns
=====================  ======================================================
"""

from __future__ import annotations

from fractions import Fraction
from statistics import NormalDist

import numpy as np

# Block sizes: B1 = 64 weights share one absmax; B2 = 256 absmax values share one
# FP32 second-level constant ("QLoRA Paper Breakdown", section 3; "QLoRA, explained.",
# method steps 2 and 3).
B1 = 64
B2 = 256

# The NF4 code book as printed with 8 decimals in "QLoRA Paper Breakdown", section 2,
# the 16-entry lookup table of "Step-by-Step Construction of the 16 NF4 Codebook Values".
NF4_PRINTED = (
    "-1.00000000", "-0.69619280", "-0.52507305", "-0.39491749",
    "-0.28444138", "-0.18477343", "-0.09105004", "0.00000000",
    "0.07958030", "0.16093020", "0.24611230", "0.33791524",
    "0.44070983", "0.56261700", "0.72295684", "1.00000000",
)


# ----------------------------------------------------------------------------------------
# exact rounding helpers (definitions of round-to-nearest-even onto fp32 / bf16)
# ----------------------------------------------------------------------------------------

def f32_from_rational(x: Fraction) -> np.float32:
    """fp32 value nearest to the exact rational ``x``; ties go to the even significand."""
    guess = np.float32(float(x))          # within one ulp of the answer
    cands = [np.nextafter(guess, np.float32(-np.inf)), guess,
             np.nextafter(guess, np.float32(np.inf))]
    def key(c):
        bits = int(np.array(c, dtype=np.float32).view(np.uint32))
        return (abs(Fraction(float(c)) - x), bits & 1)
    return np.float32(min(cands, key=key))


def bf16_rn_bits(x32: np.ndarray) -> np.ndarray:
    """Round fp32 values to bfloat16 (nearest, ties to even); returns the 16-bit patterns.

    bfloat16 keeps the top 16 bits of the fp32 pattern; rounding to nearest-even adds
    half of the dropped range (0x7FFF) plus the kept LSB before truncating.
    """
    b = np.asarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    return ((b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------------------
# step 1: the code book
# ----------------------------------------------------------------------------------------

def nf4_codebook() -> np.ndarray:
    """The 16 NF4 levels as fp32: each printed decimal rounded to the nearest fp32.

    Reading: the printed 8-decimal table is normative.  The level printed as
    -0.09105004 lies almost exactly between two fp32 values; the nearest one is taken.
    """
    return np.array([f32_from_rational(Fraction(s)) for s in NF4_PRINTED], dtype=np.float32)


def nf4_construct(k: int = 4) -> np.ndarray:
    """Build the k-bit NormalFloat levels from standard-normal quantiles (float64).

    "QLoRA, explained.", method step 1, and "QLoRA Paper Breakdown", section 2: the two
    halves are estimated separately so that zero is exact -- 2^(k-1) quantiles for the
    negative side and 2^(k-1)+1 for the positive side, each half including zero; one
    duplicate zero is dropped (7 negative, 0, 8 positive for k=4); the set is normalised
    into [-1, 1].

    Reading (the pages do not state the probability range): the quantiles are taken at
    evenly spaced probabilities from 1/2 up to an endpoint p_max, and p_max is the average
    of the two usual endpoint choices 1 - 1/(2*15) and 1 - 1/(2*16) (the pages speak of
    averaging neighbouring quantiles).  With it the construction reproduces the printed
    table to within 2e-7; the printed table stays normative for every other use.
    """
    nd = NormalDist()
    n_pos = 2 ** (k - 1) + 1            # 9 quantile points on [0, 1], including 0
    n_neg = 2 ** (k - 1)                # 8 quantile points on [-1, 0], including 0
    p_max = 0.5 * ((1.0 - 1.0 / (2 * 15)) + (1.0 - 1.0 / (2 * 16)))
    pos = [nd.inv_cdf(0.5 + j * (p_max - 0.5) / (n_pos - 1)) for j in range(1, n_pos)]
    neg = [-nd.inv_cdf(0.5 + j * (p_max - 0.5) / (n_neg - 1)) for j in range(1, n_neg)]
    levels = np.array(sorted(neg + [0.0] + pos), dtype=np.float64)
    return levels / np.max(np.abs(levels))


# ----------------------------------------------------------------------------------------
# step 2: nearest level
# ----------------------------------------------------------------------------------------

def nearest_level(n: np.ndarray, table: np.ndarray | None = None) -> np.ndarray:
    """Index of the nearest NF4 level to each fp32 value: argmin_j |n - q_j|.

    "QLoRA Paper Breakdown", section 3, level-1 formula (argmin over the code book);
    "QLoRA, explained.", method step 2 (each weight is stored as the index of its closest level).
    Reading: the pages are silent on ties; an exact tie goes to the lower index
    (toward -1), which is what ``np.argmin`` returns.  Distances are float64; for fp32
    inputs in [-1, 1] every distance that can decide a tie is exact in float64.
    """
    q = (nf4_codebook() if table is None else table).astype(np.float64)
    n = np.asarray(n, dtype=np.float32).astype(np.float64).ravel()
    out = np.empty(n.size, dtype=np.uint8)
    step = 1 << 20
    for lo in range(0, n.size, step):
        d = np.abs(n[lo:lo + step, None] - q[None, :])
        out[lo:lo + step] = np.argmin(d, axis=1)
    return out


# ----------------------------------------------------------------------------------------
# 8-bit float (E4M3) codes for the double-quantised scales
# ----------------------------------------------------------------------------------------

def e4m3_decode(code) -> np.ndarray:
    """Value of each E4M3 byte (OCP 8-bit float "E4M3FN": 1 sign, 4 exponent bits with
    bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN, largest finite 448).

    Exponent field 0 is subnormal: m * 2^-9.  Otherwise (8 + m) * 2^(e - 10).
    """
    c = np.asarray(code, dtype=np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e == 0, m * 2.0 ** -9, (8 + m) * np.exp2(e - 10.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


_E4M3_POS = e4m3_decode(np.arange(127))      # codes 0x00..0x7E, strictly increasing


def e4m3_encode_rn(v: np.ndarray) -> np.ndarray:
    """E4M3 code of each fp32 value: the nearest finite E4M3 value, ties to the even code,
    magnitudes beyond 448 saturate to 448, the sign bit is kept (so -0.0 and negative
    values that round to zero give 0x80), NaN gives 0x7F.

    Reading: "QLoRA, explained." step 3 and the level-2 formula of "QLoRA Paper
    Breakdown" section 3 ask for an 8-bit float code without naming the format.  E4M3
    is taken: the 8-bit float with the most mantissa bits.  Rounding is to nearest even.
    """
    v = np.asarray(v, dtype=np.float32).ravel()
    a = np.abs(v.astype(np.float64))
    neg = np.signbit(v)
    a_c = np.minimum(a, 448.0)
    hi = np.searchsorted(_E4M3_POS, a_c, side="left")          # first value >= a
    hi = np.clip(hi, 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_lo = np.abs(a_c - _E4M3_POS[lo])
    d_hi = np.abs(_E4M3_POS[hi] - a_c)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(neg, code | np.uint8(0x80), code).astype(np.uint8)
    code = np.where(np.isnan(a), np.uint8(0x7F), code).astype(np.uint8)
    return code


# ----------------------------------------------------------------------------------------
# double quantization helpers
# ----------------------------------------------------------------------------------------

def tree_sum_f64(c: np.ndarray) -> float:
    """Sum in float64 by a perfect binary tree over adjacent pairs ((c0+c1)+(c2+c3))+...,
    the input zero-padded to the next power of two.

    Reading: "QLoRA, explained." step 3 and the level-2 formula of "QLoRA Paper
    Breakdown" section 3 centre the scales by their mean but fix no summation order; this
    fixed order makes the mean bit-reproducible.
    """
    c = np.asarray(c, dtype=np.float64).ravel()
    size = 1
    while size < c.size:
        size *= 2
    s = np.zeros(size, dtype=np.float64)
    s[:c.size] = c
    while s.size > 1:
        s = s[0::2] + s[1::2]
    return float(s[0])


def _fmaf(a: np.ndarray, b: np.ndarray, c: np.ndarray) -> np.ndarray:
    """fp32 fused multiply-add with a single rounding: fp32(a*b + c) computed exactly.

    a must carry at most 29 significant bits (here: E4M3 values, 4 bits), so a*b is exact
    in float64.  The float64 sum is checked for exactness (two-sum error term); inexact
    elements are recomputed with exact rationals.
    """
    a64 = np.asarray(a, np.float64); b64 = np.asarray(b, np.float64); c64 = np.asarray(c, np.float64)
    a64, b64, c64 = np.broadcast_arrays(a64, b64, c64)
    p = a64 * b64
    s = p + c64
    bb = s - p
    err = (p - (s - bb)) + (c64 - bb)
    out = s.astype(np.float32)
    for i in np.flatnonzero(err != 0):
        out.flat[i] = f32_from_rational(Fraction(float(p.flat[i])) + Fraction(float(c64.flat[i])))
    return out


# ----------------------------------------------------------------------------------------
# quantize: steps 2 and 3 of the method
# ----------------------------------------------------------------------------------------

def block_absmax(w) -> np.ndarray:
    """Step 1-2 of ``quantize_nf4_dq``: absmax of each flat block of 64 (zero-padded tail)."""
    w = np.asarray(w, dtype=np.float32).ravel()
    nb = -(-w.size // B1)
    wp = np.zeros(nb * B1, dtype=np.float32)
    wp[:w.size] = w
    return np.max(np.abs(wp.reshape(nb, B1)), axis=1).astype(np.float32)


def level1_codes(w) -> tuple:
    """Steps 1-4 of ``quantize_nf4_dq``: per-block absmax and the packed NF4 codes."""
    w = np.asarray(w, dtype=np.float32).ravel()
    nb = -(-w.size // B1)
    wp = np.zeros(nb * B1, dtype=np.float32)
    wp[:w.size] = w
    blocks = wp.reshape(nb, B1)
    absmax = np.max(np.abs(blocks), axis=1).astype(np.float32)
    safe = np.where(absmax > 0, absmax, np.float32(1)).astype(np.float64)
    n = (blocks.astype(np.float64) / safe[:, None]).astype(np.float32)
    codes = nearest_level(n).reshape(nb, B1)
    codes[absmax == 0, :] = 7
    flat_codes = codes.ravel()
    packed = (flat_codes[0::2] | (flat_codes[1::2] << 4)).astype(np.uint8)
    return absmax, packed


def double_quantize(absmax) -> dict:
    """Step 5 of ``quantize_nf4_dq``: mean, group constants c2 and E4M3 scale codes."""
    absmax = np.asarray(absmax, dtype=np.float32)
    nb = absmax.size
    mean = np.float32(np.float64(tree_sum_f64(absmax)) / np.float64(nb))
    d = (absmax.astype(np.float64) - np.float64(mean)).astype(np.float32)
    ng = -(-nb // B2)
    c2 = np.zeros(ng, dtype=np.float32)
    scale_codes = np.zeros(nb, dtype=np.uint8)
    for g in range(ng):
        dg = d[g * B2:(g + 1) * B2]
        m = np.float32(np.max(np.abs(dg)))
        c2[g] = m
        if m > 0:
            v = (dg.astype(np.float64) / np.float64(m)).astype(np.float32)
            scale_codes[g * B2:(g + 1) * B2] = e4m3_encode_rn(v)
    return {"scale_codes": scale_codes, "c2": c2, "mean": np.float32(mean)}


def quantize_nf4_dq(w) -> dict:
    """Quantize a weight tensor (given as bf16-exact values) to NF4 codes plus DQ scales.

    Steps, in the pages' order ("QLoRA, explained." method steps 2-3; "QLoRA Paper
    Breakdown" section 3, level-1 and level-2 formulas):

    1. Cut the tensor, flattened row-major, into contiguous blocks of 64.  Reading: blocks
       are flat runs of the whole tensor (the pages block the tensor, not its rows), so
       when a row length is not a multiple of 64 a block spans two rows; the last block is
       zero-padded and its pad does not count toward any output.
    2. absmax c_b = max |w| over the block (exact in fp32).
    3. n = fp32(w / c_b) (correctly rounded division), code = nearest level.  Reading: an
       all-zero block (c_b = 0) encodes every weight as the exact-zero level 7.
    4. Pack two codes per byte: element 2i in the low nibble of byte i, 2i+1 in the high
       nibble.  Reading: the pages do not fix the nibble order.
    5. Double quantization: mean = fp32(tree_sum_f64(c) / nb); d_b = fp32(c_b - mean);
       per group of 256 scales c2_g = max |d_b|; scale code e_b = E4M3(fp32(d_b / c2_g)).
       Reading: a group whose c2_g is 0 stores c2 = 0 and codes 0x00.

    Returns a dict with ``codes`` (uint8, 32 bytes per block including the padded tail),
    ``scale_codes`` (uint8, nb), ``c2`` (float32, ng), ``mean`` (float32 scalar) and the
    intermediate ``absmax`` (float32, nb) for inspection.
    """
    w = np.asarray(w, dtype=np.float32).ravel()
    if w.size == 0:
        raise ValueError("empty tensor")
    absmax, packed = level1_codes(w)
    dq = double_quantize(absmax)
    return {"codes": packed, "scale_codes": dq["scale_codes"], "c2": dq["c2"],
            "mean": dq["mean"], "absmax": absmax, "numel": w.size}


def unpack_codes(packed: np.ndarray, numel: int) -> np.ndarray:
    """Inverse of the nibble packing: element 2i from the low nibble of byte i."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p & 0x0F
    out[1::2] = p >> 4
    return out[:numel]


def block_scales(scale_codes: np.ndarray, c2: np.ndarray, mean) -> np.ndarray:
    """Dequantized fp32 block scale s_b = fmaf(e4m3(e_b), c2_g, mean), one rounding.

    "QLoRA Paper Breakdown" section 4, dequantization helper: the inner dequant of the
    scale code undoes the level-2 formula of section 3 (scale the code by the group
    constant, add back the mean).  Reading: a single fp32 rounding (fused multiply-add); no clamp, so a
    tiny block's scale may come out slightly negative or zero.
    """
    e = np.asarray(scale_codes, dtype=np.uint8)
    g = np.arange(e.size) // B2
    return _fmaf(e4m3_decode(e), np.asarray(c2, np.float32)[g], np.float32(mean))


def dequant_nf4_dq(packed, scale_codes, c2, mean, numel: int) -> np.ndarray:
    """NF4 + DQ -> bf16 bit patterns (uint16), one per weight, in the original order.

    "QLoRA Paper Breakdown" section 4, dequantization helper: a weight is the code-book
    level of its code times its block's dequantized scale; "QLoRA, explained." step 4: the
    compute type is BFloat16.  Reading: W' = bf16(fp32(q[code] * s_b)) -- the product is
    rounded to fp32, then to bf16 (both nearest-even).
    """
    q = nf4_codebook()
    codes = unpack_codes(packed, numel)
    s = block_scales(scale_codes, c2, mean)
    sb = s[np.arange(numel) // B1]
    prod = (q[codes].astype(np.float64) * sb.astype(np.float64)).astype(np.float32)
    return bf16_rn_bits(prod)


def storage_bytes(numel: int) -> dict:
    """Bytes of each stored part of an NF4 + DQ tensor of ``numel`` weights."""
    nb = -(-numel // B1)
    ng = -(-nb // B2)
    return {"codes": nb * B1 // 2, "scale_codes": nb, "c2": 4 * ng, "mean": 4}
