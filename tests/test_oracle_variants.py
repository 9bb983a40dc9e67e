"""Pins of the oracle's code-book variants (FP4 E2M1, INT4), single-level (no double
quantization) blockwise quantization, and the adapter merge + re-quantization.

Independent checks: the E2M1 values rebuilt from the format's bit fields, exact rationals for
INT4, brute-force argmin on tiny tensors, exact-rational recomputation of the merge, the
storage arithmetic of the teardown (4 + 32/64 bits per parameter without double quantization).
"""

from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4, variants


def _bf16_exact(a):
    return nf4.bf16_bits_to_f32(nf4.bf16_rn_bits(np.asarray(a, np.float32)))


def test_e2m1_table_from_bit_fields():
    """E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is subnormal (m * 0.5)."""
    vals = set()
    for bits in range(16):
        sgn = -1 if bits & 8 else 1
        e, m = (bits >> 1) & 3, bits & 1
        mag = Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * Fraction(2) ** (e - 1)
        vals.add(sgn * mag)
    assert max(vals) == 6 and min(vals) == -6 and len(vals) == 15        # +-0 coincide
    want = sorted(nf4.f32_from_rational(v / 6) for v in vals)
    t = variants.fp4_e2m1_codebook()
    assert t.size == 16 and t[0] == -1 and t[15] == 1
    assert [float(x) for x in np.delete(t, 7)] == [float(x) for x in want]
    assert np.signbit(t[7]) and not np.signbit(t[8]) and t[7] == 0 and t[8] == 0


def test_int4_table_equally_spaced():
    t = variants.int4_codebook()
    assert t.size == 16 and t[0] == -1 and t[15] == 1
    for i in range(16):
        assert t[i] == nf4.f32_from_rational(Fraction(2 * i - 15, 15))
    gaps = np.diff(t.astype(np.float64))
    assert np.allclose(gaps, 2 / 15, rtol=0, atol=1e-7)


@pytest.mark.parametrize("name", ["nf4", "int4"])
def test_midpoint_rule_is_argmin_ties_low(name):
    t = variants.codebook(name)
    rng = np.random.default_rng(1)
    mids = (t[:-1].astype(np.float64) + t[1:]) / 2
    near = []
    for m in mids:
        f = np.float32(m)
        near += [np.nextafter(f, np.float32(-2)), f, np.nextafter(f, np.float32(2))]
    near += [np.float32(1e-45), np.float32(-1e-45), np.float32(0.0)]
    n = np.concatenate([np.array(near, np.float32), t])
    got = variants.nearest_midpoint(n, t)
    q = [Fraction(float(v)) for v in t]
    for ni, gi in zip(n, got):                       # exact-rational argmin, ties to the lower index
        d = [abs(Fraction(float(ni)) - qj) for qj in q]
        assert gi == d.index(min(d)), (ni, gi)
    r = rng.uniform(-1, 1, 20000).astype(np.float32)
    d = np.abs(r.astype(np.float64)[:, None] - t.astype(np.float64)[None, :])
    assert np.array_equal(variants.nearest_midpoint(r, t), np.argmin(d, axis=1).astype(np.uint8))


def test_e2m1_zero_keeps_its_sign():
    t = variants.fp4_e2m1_codebook()
    n = np.array([0.0, -0.0, 1e-30, -1e-30, 0.04, -0.04, 1 / 24 - 1e-4, 1 / 24 + 1e-4], np.float32)
    got = variants.nearest_midpoint(n, t)
    assert list(got) == [7, 7, 8, 7, 8, 7, 8, 9]


def _bruteforce(w, table):
    q = [Fraction(float(v)) for v in table]
    nb = -(-w.size // 64)
    wp = [Fraction(0)] * (nb * 64)
    for i, v in enumerate(w):
        wp[i] = Fraction(float(v))
    codes = []
    for b in range(nb):
        blk = wp[b * 64:(b + 1) * 64]
        c = max(abs(v) for v in blk)
        for v in blk:
            if c == 0:
                codes.append(7)
                continue
            n = Fraction(float(nf4.f32_from_rational(v / c)))
            best, bestd = 0, None
            for j, qj in enumerate(q):
                d = abs(n - qj)
                # ties: lower index, except that the two zeros of E2M1 split by the sign of n
                if bestd is None or d < bestd or (d == bestd and qj == 0 and n > 0):
                    best, bestd = j, d
            codes.append(best)
    return np.array(codes, np.uint8)


@pytest.mark.parametrize("name", ["fp4_e2m1", "int4"])
def test_quantize_matches_exact_bruteforce(name):
    rng = np.random.default_rng(7)
    w = _bf16_exact(rng.standard_normal(64 * 5 + 17).astype(np.float32) * 0.03)
    w[rng.random(w.size) < 0.05] = 0.0
    w[3] = -w[3]
    t = variants.codebook(name)
    qd = variants.quantize_blockwise(w, t, double_quant=False)
    nb = -(-w.size // 64)
    assert np.array_equal(nf4.unpack_codes(qd["codes"], nb * 64), _bruteforce(w, t))
    assert np.array_equal(qd["absmax"], nf4.block_absmax(w))


def test_nf4_with_dq_is_the_nf4_oracle():
    rng = np.random.default_rng(3)
    w = _bf16_exact(rng.standard_normal(64 * 700 + 9).astype(np.float32) * 0.02)
    a = variants.quantize_blockwise(w, nf4.nf4_codebook(), double_quant=True)
    b = nf4.quantize_nf4_dq(w)
    for k in ("codes", "scale_codes", "c2"):
        assert np.array_equal(a[k], b[k])
    assert a["mean"] == b["mean"]


def test_single_level_storage_is_4p5_bits(golden):
    g = {k: float(v) for k, v in golden("storage_bits.txt")}
    n = 64 * 256 * 100
    assert variants.storage_bits(n, double_quant=False) == g["single_level_total_bits"]
    assert variants.storage_bits(n, double_quant=True) == g["dq_total_bits"]


def test_dequant_without_dq_over_many_blocks():
    rng = np.random.default_rng(11)
    nb = 300
    std = np.exp(rng.uniform(np.log(1e-3), np.log(0.1), nb)).astype(np.float32)
    w = _bf16_exact((rng.standard_normal((nb, 64)).astype(np.float32) * std[:, None]).ravel())
    for name in ("nf4", "fp4_e2m1", "int4"):
        t = variants.codebook(name)
        qd = variants.quantize_blockwise(w, t, double_quant=False)
        got = variants.dequant_blockwise(qd["codes"], t, w.size, absmax=qd["absmax"])
        codes = nf4.unpack_codes(qd["codes"], w.size)
        for e in range(0, w.size, 7):
            qv, sv = t[codes[e]], qd["absmax"][e // 64]
            if qv == 0 or sv == 0:                      # a signed zero: the sign of the product
                want = 0x8000 if (np.signbit(qv) != np.signbit(sv)) else 0
            else:
                prod = nf4.f32_from_rational(Fraction(float(qv)) * Fraction(float(sv)))
                want = int(nf4.bf16_rn_bits(np.array([prod], np.float32))[0])
            assert got[e] == want


def test_bf16_from_f64_matches_exact_rounding():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(3000) * 0.02, rng.standard_normal(1000) * 1e3,
                        (rng.integers(1, 255, 500) * 2.0 + 1) * 2.0 ** -9,      # ties at the bf16 grid
                        np.array([0.0, -0.0, 1.0, -1.0, 2.0 ** -130, 3 * 2.0 ** -134])])
    got = variants.bf16_rn_from_f64(x)
    for xi, gi in zip(x, got):
        assert int(gi) == variants._bf16_rn_scalar(float(xi)), xi


def _merge_exact(Wd_bits, A, B, s):
    """Exact rationals: the float64 sum in index order and its roundings, restated."""
    Wd = nf4.bf16_bits_to_f32(Wd_bits).astype(np.float64)
    N, K = Wd.shape
    out = np.empty((N, K), np.uint16)
    for n in range(N):
        for k in range(K):
            acc = 0.0
            for j in range(A.shape[0]):
                acc = float(Fraction(acc) + Fraction(float(B[n, j])) * Fraction(float(A[j, k])))  # RN to f64
            t = float(Fraction(float(s)) * Fraction(acc))
            v = float(Fraction(float(Wd[n, k])) + Fraction(t))
            out[n, k] = variants._bf16_rn_scalar(v)
    return out


def test_merge_matches_exact_recomputation():
    rng = np.random.default_rng(9)
    N, K, r = 6, 128, 8
    w = _bf16_exact(rng.standard_normal(N * K).astype(np.float32) * 0.02)
    qd = nf4.quantize_nf4_dq(w)
    Wd = nf4.dequant_nf4_dq(qd["codes"], qd["scale_codes"], qd["c2"], qd["mean"], w.size).reshape(N, K)
    A = _bf16_exact(rng.standard_normal((r, K)).astype(np.float32) / np.sqrt(r)).astype(np.float64)
    B = _bf16_exact(rng.standard_normal((N, r)).astype(np.float32) * 0.01).astype(np.float64)
    m = variants.merge_requantize(Wd, A, B, 0.25, nf4.nf4_codebook())
    assert np.array_equal(m["merged_bits"], _merge_exact(Wd, A, B, 0.25))
    again = variants.quantize_blockwise(nf4.bf16_bits_to_f32(m["merged_bits"]).ravel(), nf4.nf4_codebook(), True)
    assert np.array_equal(m["codes"], again["codes"]) and np.array_equal(m["scale_codes"], again["scale_codes"])


def test_merge_with_zero_adapter_returns_the_base():
    rng = np.random.default_rng(10)
    N, K, r = 32, 256, 16
    w = _bf16_exact(rng.standard_normal(N * K).astype(np.float32) * 0.02)
    qd = nf4.quantize_nf4_dq(w)
    Wd = nf4.dequant_nf4_dq(qd["codes"], qd["scale_codes"], qd["c2"], qd["mean"], w.size).reshape(N, K)
    A = rng.standard_normal((r, K))
    m = variants.merge_requantize(Wd, A, np.zeros((N, r)), 0.25, nf4.nf4_codebook())
    assert np.array_equal(m["merged_bits"], Wd)
    # the base's codes survive: every block's absmax level maps back onto +-1
    assert np.array_equal(m["codes"], qd["codes"])


def test_merge_sum_order_is_index_order():
    """A sum whose float64 value depends on the order: index order j = 0, 1, 2 is the one kept."""
    A = np.array([[1.0], [2.0 ** -60], [-1.0]])
    B = np.array([[1.0, 1.0, 1.0]])
    Wd = nf4.bf16_rn_bits(np.array([[0.0]], np.float32)).reshape(1, 1)
    m = variants.merge_requantize(np.zeros((1, 64), np.uint16), np.repeat(A, 64, axis=1), B, 1.0, nf4.nf4_codebook())
    # (1 + 2^-60) rounds to 1 in float64, then + (-1) = 0: the merged weights are exactly zero
    assert np.all(m["merged_bits"] == 0) and Wd.size == 1
