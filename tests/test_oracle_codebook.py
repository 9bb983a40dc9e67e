"""Pins of the oracle's NF4 code book, nearest-level search and the worked lookup.

Sources: the printed table ("QLoRA Paper Breakdown", section 2, stored in
tests/golden/nf4_table.txt), the video page's worked lookup (tests/golden/worked_lookup.txt),
the structure of the construction ("QLoRA, explained." method step 1).
"""

from fractions import Fraction

import numpy as np

from oracle import nf4


def test_codebook_matches_printed_table(golden):
    rows = golden("nf4_table.txt")
    q = nf4.nf4_codebook()
    assert len(rows) == 16 and q.shape == (16,) and q.dtype == np.float32
    for (idx, text), val in zip(rows, q):
        exact = Fraction(text)
        ulp = abs(float(np.spacing(np.float32(val)))) if val != 0 else 0.0
        assert abs(Fraction(float(val)) - exact) <= Fraction(ulp) / 2, (idx, text, val)


def test_codebook_structure():
    """7 negative levels, an exact zero, 8 positive levels, endpoints -1 and +1."""
    q = nf4.nf4_codebook()
    assert np.all(np.diff(q.astype(np.float64)) > 0)
    assert int((q < 0).sum()) == 7 and int((q > 0).sum()) == 8
    assert q[7] == 0.0 and not np.signbit(q[7])
    assert q[0] == -1.0 and q[15] == 1.0


def test_construction_reproduces_table():
    """Quantile construction ("QLoRA, explained." step 1) vs the printed decimals."""
    built = nf4.nf4_construct(4)
    q = nf4.nf4_codebook().astype(np.float64)
    assert built.shape == (16,)
    assert built[7] == 0.0 and built[0] == -1.0 and built[15] == 1.0
    assert np.max(np.abs(built - q)) < 3e-7
    # a symmetric 16-bin construction (no exact zero) or a mis-counted half fails badly
    assert np.min(np.abs(built)) == 0.0


def test_worked_lookup(golden):
    """0.37 / 2 -> level 0.1609302014 -> 0.3218604028, error -0.0481395972 (video page)."""
    g = {k: v for k, v in golden("worked_lookup.txt")}
    w = np.float32(g["weight"]); c = np.float32(g["absmax"])
    n = np.float32(np.float64(w) / np.float64(c))
    assert abs(float(n) - float(g["normalised"])) < 1e-7
    code = int(nf4.nearest_level(np.array([n]))[0])
    q = nf4.nf4_codebook()
    level = float(q[code])
    assert code == 9
    assert abs(level - float(g["level"])) < 5e-11
    recon = level * float(c)
    assert abs(recon - float(g["reconstruction"])) < 5e-11
    assert abs((recon - float(w)) - float(g["error"])) < 5e-9   # w is 0.37 rounded to fp32


def test_worked_lookup_through_quantize_and_dequant(golden):
    """Same block through the whole codec: a single block has mean = absmax, c2 = 0, so the
    dequantized weight is bf16 of the page's reconstruction."""
    g = {k: v for k, v in golden("worked_lookup.txt")}
    w = np.zeros(64, dtype=np.float32)
    w[0] = np.float32(g["absmax"]); w[1] = np.float32(g["weight"])
    qd = nf4.quantize_nf4_dq(w)
    codes = nf4.unpack_codes(qd["codes"], 64)
    assert codes[0] == 15 and codes[1] == 9 and np.all(codes[2:] == 7)
    assert qd["mean"] == np.float32(2.0) and qd["c2"][0] == 0.0
    out = nf4.bf16_bits_to_f32(nf4.dequant_nf4_dq(qd["codes"], qd["scale_codes"], qd["c2"],
                                                  qd["mean"], 64))
    half_ulp_bf16 = 2.0 ** -10   # 0.32 lies in [0.25, 0.5): bf16 spacing 2^-9
    assert abs(float(out[1]) - float(g["reconstruction"])) <= half_ulp_bf16 + 1e-9
    assert out[0] == 2.0 and np.all(out[2:] == 0.0)


def _exact_nearest(x: Fraction, qf) -> int:
    best, bestd = 0, None
    for j, v in enumerate(qf):
        d = abs(x - v)
        if bestd is None or d < bestd:      # strict: ties keep the lower index
            best, bestd = j, d
    return best


def test_nearest_level_bruteforce_near_every_midpoint():
    """Every fp32 value within +-64 ulp of each midpoint (q_j + q_{j+1})/2, against an
    exact-rational argmin with ties to the lower index."""
    q = nf4.nf4_codebook()
    qf = [Fraction(float(v)) for v in q]
    vals = []
    for j in range(15):
        mid = (qf[j] + qf[j + 1]) / 2
        c = np.float32(float(mid))
        lo = c
        for _ in range(64):
            lo = np.nextafter(lo, np.float32(-2))
        x = lo
        for _ in range(129):
            vals.append(x)
            x = np.nextafter(x, np.float32(2))
    vals = np.array(vals, dtype=np.float32)
    got = nf4.nearest_level(vals)
    want = np.array([_exact_nearest(Fraction(float(v)), qf) for v in vals])
    assert np.array_equal(got, want)


def test_nearest_level_bruteforce_random_and_specials():
    rng = np.random.default_rng(7)
    vals = np.concatenate([rng.uniform(-1, 1, 4000).astype(np.float32),
                           np.array([-1, 1, 0.0, -0.0, 1e-30, -1e-30, 1e-45, -1e-45],
                                    dtype=np.float32)])
    q = nf4.nf4_codebook()
    qf = [Fraction(float(v)) for v in q]
    got = nf4.nearest_level(vals)
    want = np.array([_exact_nearest(Fraction(float(v)), qf) for v in vals])
    assert np.array_equal(got, want)
    assert got[-8] == 0 and got[-7] == 15 and got[-6] == 7 and got[-5] == 7


def test_midpoint_ties_go_to_lower_index():
    """Midpoints that are exact fp32 values tie; the lower index wins."""
    q = nf4.nf4_codebook()
    n_ties = 0
    for j in range(15):
        mid = (Fraction(float(q[j])) + Fraction(float(q[j + 1]))) / 2
        m32 = np.float32(float(mid))
        if Fraction(float(m32)) == mid:
            n_ties += 1
            assert nf4.nearest_level(np.array([m32]))[0] == j
    assert n_ties >= 1
