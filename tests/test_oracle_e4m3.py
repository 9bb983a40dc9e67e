"""Pins of the oracle's 8-bit float (E4M3) scale codes.

Independent checks: named values of the OCP E4M3 ("E4M3FN") format, torch's own
float8_e4m3fn dtype as a library routine, exact-rational nearest search with ties to even,
round trips and saturation.
"""

from fractions import Fraction

import numpy as np
import torch

from oracle import nf4


def test_named_values():
    d = nf4.e4m3_decode(np.arange(256))
    assert d[0x00] == 0.0 and not np.signbit(d[0x00])
    assert d[0x80] == 0.0 and np.signbit(d[0x80])
    assert d[0x01] == 2.0 ** -9            # smallest subnormal
    assert d[0x07] == 7 * 2.0 ** -9        # largest subnormal
    assert d[0x08] == 2.0 ** -6            # smallest normal
    assert d[0x38] == 1.0
    assert d[0x7E] == 448.0 and d[0xFE] == -448.0
    assert np.isnan(d[0x7F]) and np.isnan(d[0xFF])
    assert int(np.isnan(d).sum()) == 2


def test_decode_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = nf4.e4m3_decode(np.arange(256))
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()
    assert np.array_equal(np.signbit(got[~np.isnan(got)]), np.signbit(ref[~np.isnan(ref)]))


def test_round_trip_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)])
    back = nf4.e4m3_encode_rn(nf4.e4m3_decode(codes).astype(np.float32))
    assert np.array_equal(back, codes.astype(np.uint8))


def _exact_e4m3(x: Fraction, neg: bool) -> int:
    vals = [(Fraction(float(v)), c) for c, v in enumerate(nf4.e4m3_decode(np.arange(127)))]
    a = abs(x)
    if a > 448:
        a = Fraction(448)
    best = None
    for v, c in vals:
        key = (abs(a - v), c & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1] | (0x80 if neg else 0)


def test_encode_exact_bruteforce_midpoints_and_random():
    pos = nf4.e4m3_decode(np.arange(127))
    mids = [(Fraction(float(pos[i])) + Fraction(float(pos[i + 1]))) / 2 for i in range(126)]
    vals = []
    for m in mids:
        f = np.float32(float(m))
        vals += [f, np.nextafter(f, np.float32(-1e9)), np.nextafter(f, np.float32(1e9))]
    rng = np.random.default_rng(3)
    vals += list(rng.uniform(-1, 1, 3000).astype(np.float32))
    vals += list((rng.uniform(-1, 1, 1000) * 2.0 ** -8).astype(np.float32))
    vals = np.array(vals + [np.float32(-v) for v in vals], dtype=np.float32)
    got = nf4.e4m3_encode_rn(vals)
    want = np.array([_exact_e4m3(Fraction(float(v)), bool(np.signbit(v))) for v in vals],
                    dtype=np.uint8)
    assert np.array_equal(got, want)


def test_encode_matches_torch_in_range():
    """Inside [-448, 448] torch's fp32 -> float8_e4m3fn cast is round-to-nearest-even."""
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.uniform(-1, 1, 200000), rng.uniform(-448, 448, 20000),
                        rng.uniform(-1, 1, 20000) * 2.0 ** -7]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(nf4.e4m3_encode_rn(v), ref)


def test_saturation_signed_zero_and_ties():
    v = np.array([1000.0, -1000.0, 449.0, 0.0, -0.0, -1e-30, 2.0 ** -10, 3 * 2.0 ** -10],
                 dtype=np.float32)
    c = nf4.e4m3_encode_rn(v)
    assert c[0] == 0x7E and c[1] == 0xFE and c[2] == 0x7E
    assert c[3] == 0x00 and c[4] == 0x80 and c[5] == 0x80
    assert c[6] == 0x00          # half of the smallest subnormal ties to even (zero)
    assert c[7] == 0x02          # 1.5 x smallest subnormal ties to the even code 2
