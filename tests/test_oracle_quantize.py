"""Pins of the oracle's quantize (absmax, nearest level, packing, double quantization),
dequantize and storage arithmetic.

Independent checks: an exact-rational brute-force recomputation on tiny tensors, the
storage arithmetic printed on the pages (tests/golden/storage_bits.txt), exact zeros,
closed-form special cases and the reconstruction bound of 8-bit scale codes.
"""

from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4


def _bf16_exact(a):
    return nf4.bf16_bits_to_f32(nf4.bf16_rn_bits(np.asarray(a, np.float32)))


def _rat_f32(x: Fraction) -> np.float32:
    return nf4.f32_from_rational(x)


def _exact_e4m3(x: Fraction, neg: bool) -> int:
    best = None
    for c in range(127):
        v = Fraction(float(nf4.e4m3_decode(c)))
        key = (abs(abs(x) - v), c & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1] | (0x80 if neg else 0)


def _bruteforce(w: np.ndarray):
    """Exact-rational restatement used only as an independent check of the oracle."""
    q = [Fraction(float(v)) for v in nf4.nf4_codebook()]
    numel = w.size
    nb = -(-numel // 64)
    wp = [Fraction(0)] * (nb * 64)
    for i, v in enumerate(w):
        wp[i] = Fraction(float(v))
    codes, absmax = [], []
    for b in range(nb):
        blk = wp[b * 64:(b + 1) * 64]
        c = max(abs(v) for v in blk)
        absmax.append(c)
        for v in blk:
            if c == 0:
                codes.append(7)
                continue
            n = Fraction(float(_rat_f32(v / c)))
            best, bestd = 0, None
            for j, qj in enumerate(q):
                d = abs(n - qj)
                if bestd is None or d < bestd:
                    best, bestd = j, d
            codes.append(best)
    mean = _rat_f32(sum(absmax) / nb)
    m = Fraction(float(mean))
    d = [_rat_f32(c - m) for c in absmax]
    ng = -(-nb // 256)
    e, c2 = [], []
    for g in range(ng):
        dg = d[g * 256:(g + 1) * 256]
        mx = max(abs(Fraction(float(v))) for v in dg)
        c2.append(float(mx))
        for v in dg:
            if mx == 0:
                e.append(0)
            else:
                vv = _rat_f32(Fraction(float(v)) / mx)
                e.append(_exact_e4m3(Fraction(float(vv)), bool(np.signbit(vv))))
    return codes, np.array(e, np.uint8), np.array(c2, np.float32), mean


@pytest.mark.parametrize("numel,seed", [(64 * 3, 0), (64 * 300 + 37, 1), (130, 2)])
def test_quantize_matches_exact_bruteforce(numel, seed):
    rng = np.random.default_rng(seed)
    # bf16-exact Gaussian weights with a few exact zeros and one all-zero block
    w = _bf16_exact(rng.standard_normal(numel).astype(np.float32) * 0.02)
    w[rng.random(numel) < 0.05] = 0.0
    if numel >= 192:
        w[64:128] = 0.0
    qd = nf4.quantize_nf4_dq(w)
    codes, e, c2, mean = _bruteforce(w)
    nb = -(-numel // 64)
    assert np.array_equal(nf4.unpack_codes(qd["codes"], nb * 64), np.array(codes, np.uint8))
    assert qd["mean"] == mean
    assert np.array_equal(qd["c2"], c2)
    assert np.array_equal(qd["scale_codes"], e)


def test_packing_order():
    """Element 2i sits in the low nibble of byte i, element 2i+1 in the high nibble."""
    w = np.zeros(64, np.float32)
    w[0] = -1.0; w[1] = 1.0; w[2] = 0.0; w[3] = -1.0
    qd = nf4.quantize_nf4_dq(w)
    assert qd["codes"][0] == (0 | (15 << 4)) and qd["codes"][1] == (7 | (0 << 4))
    assert qd["codes"].size == 32


def test_storage_arithmetic(golden):
    g = {k: float(v) for k, v in golden("storage_bits.txt")}
    numel = 64 * 256 * 1000
    sb = nf4.storage_bytes(numel)
    bits_codes = sb["codes"] * 8 / numel
    bits_scales = (sb["scale_codes"] * 8 + sb["c2"] * 8) / numel
    assert bits_codes == g["nf4_code_bits"]
    assert bits_scales == g["dq_scale_bits"]
    assert bits_codes + bits_scales == g["dq_total_bits"]
    single = 4 + 32 / 64
    assert single == g["single_level_total_bits"] and 32 / 64 == g["single_level_scale_bits"]
    assert single - (bits_codes + bits_scales) == g["dq_saving_bits"]
    assert round(g["dq_saving_bits"] * 65e9 / 8 / 1e9, 3) == g["dq_saving_gb_at_65b"]
    # the per-tensor mean adds 32 bits on top of the pages' idealised figure
    assert sb["mean"] * 8 == 32


def test_exact_zero_round_trip():
    rng = np.random.default_rng(5)
    w = _bf16_exact(rng.standard_normal(64 * 512).astype(np.float32) * 0.02)
    zero = rng.random(w.size) < 0.05
    w[zero] = 0.0
    w[64 * 7:64 * 8] = 0.0                           # an all-zero block
    qd = nf4.quantize_nf4_dq(w)
    codes = nf4.unpack_codes(qd["codes"], w.size)
    assert np.all(codes[zero] == 7)
    out = nf4.dequant_nf4_dq(qd["codes"], qd["scale_codes"], qd["c2"], qd["mean"], w.size)
    assert np.all((out[zero] & 0x7FFF) == 0)         # +0 or -0
    assert np.all((out[64 * 7:64 * 8] & 0x7FFF) == 0)


def test_constant_scale_tensor_is_exact():
    """All blocks share one absmax: mean = absmax, c2 = 0, every scale is exact."""
    rng = np.random.default_rng(9)
    w = _bf16_exact(rng.uniform(-1, 1, 64 * 600).astype(np.float32) * 0.03)
    w.reshape(-1, 64)[:, 0] = np.float32(0.0625)
    w.reshape(-1, 64)[:, 1:] = np.clip(w.reshape(-1, 64)[:, 1:], -0.0625, 0.0625)
    qd = nf4.quantize_nf4_dq(w)
    assert qd["mean"] == np.float32(0.0625) and np.all(qd["c2"] == 0)
    s = nf4.block_scales(qd["scale_codes"], qd["c2"], qd["mean"])
    assert np.all(s == np.float32(0.0625))
    q = nf4.nf4_codebook()
    codes = nf4.unpack_codes(qd["codes"], w.size)
    want = nf4.bf16_rn_bits((q[codes].astype(np.float64) * 0.0625).astype(np.float32))
    got = nf4.dequant_nf4_dq(qd["codes"], qd["scale_codes"], qd["c2"], qd["mean"], w.size)
    assert np.array_equal(got, want)


def test_scale_reconstruction_bound():
    """|s_b - c_b| <= c2_g * 2^-4 (+ fp32 rounding): E4M3 keeps 3 mantissa bits and codes
    live in [-1, 1]; a wrong centring sign or group index breaks this."""
    rng = np.random.default_rng(4)
    w = _bf16_exact((rng.standard_t(3, 64 * 2000) * 0.02).astype(np.float32))
    qd = nf4.quantize_nf4_dq(w)
    s = nf4.block_scales(qd["scale_codes"], qd["c2"], qd["mean"]).astype(np.float64)
    c = qd["absmax"].astype(np.float64)
    c2 = qd["c2"][np.arange(c.size) // 256].astype(np.float64)
    tol = c2 * 2.0 ** -4 + 4 * np.spacing(np.abs(c).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(s - c) <= tol)
    # the normalised codes stay inside [-1, 1] and at least one per group reaches +-1
    v = nf4.e4m3_decode(qd["scale_codes"])
    assert np.all(np.abs(v) <= 1.0)
    for g in range(qd["c2"].size):
        assert np.max(np.abs(v[g * 256:(g + 1) * 256])) == 1.0


def test_tree_sum_exact_on_dyadic_inputs():
    rng = np.random.default_rng(2)
    for n in (1, 2, 3, 255, 256, 257, 1000):
        c = rng.integers(1, 2 ** 8, n).astype(np.float64) * 2.0 ** -12
        assert nf4.tree_sum_f64(c) == float(sum(Fraction(float(x)) for x in c))


def test_tree_sum_order_and_padding():
    c = np.array([1.0, 2.0 ** -60, -1.0, 2.0 ** -60])
    # adjacent-pair tree: (1 + 2^-60) + (-1 + 2^-60) = 1 + (-1) = 0 in float64
    assert nf4.tree_sum_f64(c) == 0.0
    c2 = np.array([1.0, -1.0, 2.0 ** -60, 2.0 ** -60])
    assert nf4.tree_sum_f64(c2) == 2.0 ** -59
    assert nf4.tree_sum_f64(np.array([3.0, 5.0, 7.0])) == 15.0


def test_dequant_scales_follow_fma_definition():
    """Scale = decode(code) * c2 + mean with one rounding (checked against Fractions)."""
    rng = np.random.default_rng(12)
    codes = rng.integers(0, 256, 3000).astype(np.uint8)
    codes[codes == 0x7F] = 0x7E; codes[codes == 0xFF] = 0xFE
    c2 = (rng.random(-(-3000 // 256)) * 0.01).astype(np.float32)
    mean = np.float32(0.0371)
    s = nf4.block_scales(codes, c2, mean)
    for i in range(0, 3000, 7):
        exact = Fraction(float(nf4.e4m3_decode(codes[i]))) * Fraction(float(c2[i // 256])) \
            + Fraction(float(mean))
        assert s[i] == nf4.f32_from_rational(exact)


# ----------------------------------------------------------------------------------------
# dequant over many blocks with distinct scales, against exact rationals
# ----------------------------------------------------------------------------------------

def _e4m3_value(byte: int) -> Fraction:
    """E4M3 (bias 7) value of a byte from the format's closed form, as an exact rational."""
    sign = -1 if byte & 0x80 else 1
    e, m = (byte >> 3) & 15, byte & 7
    mag = Fraction(m, 512) if e == 0 else Fraction(8 + m, 8) * Fraction(2) ** (e - 7)
    return sign * mag


def _bf16_rn_rational(x: Fraction) -> int:
    """bf16 bit pattern nearest to the exact rational x, ties to the even significand
    (restated from the format: 1 sign, 8 exponent bits, 7 stored mantissa bits)."""
    if x == 0:
        return 0
    sign = 0x8000 if x < 0 else 0
    a = abs(x)
    e = 0
    while a >= 2:
        a /= 2; e += 1
    while a < 1:
        a *= 2; e -= 1
    e = max(e, -126)                       # subnormal range: spacing 2^-133
    scaled = abs(x) / Fraction(2) ** (e - 7)   # significand in units of the last place
    lo = scaled.numerator // scaled.denominator
    rem = scaled - lo
    up = rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1)
    mant = lo + (1 if up else 0)           # 128..256 for normals (256 carries into e + 1)
    if mant >= 256:
        mant //= 2; e += 1
    if mant < 128:                         # subnormal
        return sign | mant
    return sign | ((e + 127) << 7) | (mant - 128)


def _dequant_exact(packed, scale_codes, c2, mean, numel):
    """W'_e = bf16(fp32(q[code_e] * fp32(e4m3(e_b) * c2_g + mean))) with b = e // 64 and
    g = b // 256, every rounding done from exact rationals."""
    q = [Fraction(float(v)) for v in nf4.nf4_codebook()]
    codes = nf4.unpack_codes(packed, numel)
    scales = {}
    out = np.empty(numel, np.uint16)
    for e in range(numel):
        b = e // 64
        if b not in scales:
            exact = _e4m3_value(int(scale_codes[b])) * Fraction(float(c2[b // 256])) + Fraction(float(mean))
            scales[b] = Fraction(float(nf4.f32_from_rational(exact)))
        prod = Fraction(float(nf4.f32_from_rational(q[int(codes[e])] * scales[b])))
        out[e] = _bf16_rn_rational(prod)
    return out


def _multiblock_weight(nblocks, seed):
    """bf16 weights whose blocks have widely different absmax values, so that the 8-bit
    scale codes of neighbouring blocks (and the constants of neighbouring groups) differ."""
    rng = np.random.default_rng(seed)
    std = np.exp(rng.uniform(np.log(1e-3), np.log(0.1), nblocks)).astype(np.float32)
    w = rng.standard_normal((nblocks, 64)).astype(np.float32) * std[:, None]
    return _bf16_exact(w.ravel())


def test_dequant_many_blocks_matches_exact_rationals():
    """600 blocks (3 groups of 256, the last partial) with distinct scales: every weight
    uses its own block's scale and its group's constant.  Pins the per-element block and
    group indexing of the dequant, which single-block or constant-scale cases cannot."""
    w = _multiblock_weight(600, 21)
    qd = nf4.quantize_nf4_dq(w)
    assert len(set(qd["scale_codes"].tolist())) > 50 and qd["c2"].size == 3
    got = nf4.dequant_nf4_dq(qd["codes"], qd["scale_codes"], qd["c2"], qd["mean"], w.size)
    want = _dequant_exact(qd["codes"], qd["scale_codes"], qd["c2"], qd["mean"], w.size)
    assert np.array_equal(got, want)


def test_dequant_pin_rejects_a_planted_block_index_mistake():
    """The exact-rational pin above fails for an oracle dequant that indexes the block
    scale by element // 256 instead of element // 64."""
    w = _multiblock_weight(600, 22)
    qd = nf4.quantize_nf4_dq(w)
    q = nf4.nf4_codebook()
    codes = nf4.unpack_codes(qd["codes"], w.size)
    s = nf4.block_scales(qd["scale_codes"], qd["c2"], qd["mean"])
    planted = nf4.bf16_rn_bits((q[codes].astype(np.float64)
                                * s[np.arange(w.size) // 256].astype(np.float64)).astype(np.float32))
    want = _dequant_exact(qd["codes"], qd["scale_codes"], qd["c2"], qd["mean"], w.size)
    assert not np.array_equal(planted, want)


# ----------------------------------------------------------------------------------------
# fp32 -> bf16 rounding: ties to even
# ----------------------------------------------------------------------------------------

def _tie_patterns():
    """fp32 bit patterns whose dropped low half is exactly 0x8000 (a tie), with both
    parities of the kept last bit, over every exponent and both signs; plus neighbours
    0x7FFF / 0x8001 of each."""
    rng = np.random.default_rng(3)
    hi = np.concatenate([np.arange(0, 0x7F80, dtype=np.uint32),            # finite, +
                         rng.integers(0x8000, 0xFF80, 20000).astype(np.uint32)])
    pats = []
    for low in (0x8000, 0x7FFF, 0x8001, 0x0000, 0xFFFF):
        pats.append((hi << np.uint32(16)) | np.uint32(low))
    return np.concatenate(pats)


def test_bf16_rounding_matches_torch_cast_on_ties():
    import torch
    bits = _tie_patterns()
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    got = nf4.bf16_rn_bits(x)
    want = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)
    # both parities of the kept bit really occur among the ties
    ties = (x.view(np.uint32) & np.uint32(0xFFFF)) == np.uint32(0x8000)
    kept = (x.view(np.uint32) >> np.uint32(16)) & np.uint32(1)
    assert np.any(ties & (kept == 0)) and np.any(ties & (kept == 1))


def test_bf16_rounding_matches_exact_rationals():
    rng = np.random.default_rng(8)
    bits = np.concatenate([
        (rng.integers(0x0080, 0x7F00, 4000).astype(np.uint32) << np.uint32(16)) | np.uint32(0x8000),
        rng.integers(0, 0x7F000000, 4000).astype(np.uint32),
        rng.integers(0x80000000, 0xFF000000, 2000).astype(np.uint32),
        np.array([0x00008000, 0x00018000, 0x80008000, 0x3F808000, 0x3F818000], np.uint32),
    ])
    x = bits.view(np.float32)
    got = nf4.bf16_rn_bits(x)
    for xi, gi in zip(x, got):
        assert int(gi) == _bf16_rn_rational(Fraction(float(xi))), hex(int(np.float32(xi).view(np.uint32)))


def test_bf16_pin_rejects_round_half_up():
    """The pins above fail for a rounding that drops the kept-bit term (round half up)."""
    import torch
    x = _tie_patterns().view(np.float32)
    x = x[np.isfinite(x)]
    b = x.view(np.uint32).astype(np.uint64)
    planted = ((b + np.uint64(0x7FFF) + np.uint64(1)) >> np.uint64(16)).astype(np.uint16)
    want = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert not np.array_equal(planted, want)


def test_normalised_value_is_the_correctly_rounded_quotient():
    """The oracle forms n = fp32(w / c) through a float64 quotient; for every pair of bf16
    significands (and exponent gaps 0, 1, 5) it equals the exact quotient rounded once to
    fp32 (ties to even), computed from rationals."""
    mant = [1 + Fraction(m, 128) for m in range(128)]
    ws, cs, exact = [], [], []
    for gap in (0, 1, 5):
        for mw in mant:
            for mc in mant:
                w = mw * Fraction(1, 2 ** gap)
                if w > mc:
                    continue
                ws.append(float(w)); cs.append(float(mc)); exact.append(w / mc)
    w = np.array(ws, np.float32); c = np.array(cs, np.float32)
    n = (w.astype(np.float64) / c.astype(np.float64)).astype(np.float32)
    rng = np.random.default_rng(0)
    for i in rng.choice(len(exact), 6000, replace=False):
        assert n[i] == nf4.f32_from_rational(exact[i])
