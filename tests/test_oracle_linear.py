"""Pins of the oracle's QLoRA linear forward / backward.

Independent checks: explicit-loop sums on tiny shapes, exact directional derivatives of
<dY, y> (y is linear in each of x, A and B separately, so a central difference is exact up to
rounding), and special cases (B = 0, A = 0, s = 0, x = I).
"""

import numpy as np

from oracle import linear


def _tiny(seed=0, M=3, N=4, K=5, r=2):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((M, K)), rng.standard_normal((N, K)),
            rng.standard_normal((r, K)), rng.standard_normal((N, r)),
            rng.standard_normal((M, N)))


def test_forward_explicit_loops():
    x, W, A, B, _ = _tiny()
    s = 0.75
    y = linear.qlora_forward(x, W, A, B, s)["y"]
    M, K = x.shape; N = W.shape[0]; r = A.shape[0]
    for m in range(M):
        for n in range(N):
            base = sum(x[m, k] * W[n, k] for k in range(K))
            ad = 0.0
            for j in range(r):
                ad += sum(x[m, k] * A[j, k] for k in range(K)) * B[n, j]
            assert abs(y[m, n] - (base + s * ad)) < 1e-12


def _f(x, W, A, B, s, dY):
    return float(np.sum(dY * linear.qlora_forward(x, W, A, B, s)["y"]))


def test_backward_equals_directional_derivatives():
    x, W, A, B, dY = _tiny(1, M=4, N=6, K=5, r=3)
    s = 0.25
    g = linear.qlora_backward(dY, x, W, A, B, s)
    rng = np.random.default_rng(2)
    h = 0.5        # y is linear in each argument, so any step is exact
    for name, val, grad in (("x", x, g["dX"]), ("A", A, g["dA"]), ("B", B, g["dB"])):
        V = rng.standard_normal(val.shape)
        args = {"x": x, "A": A, "B": B}
        plus = dict(args); plus[name] = val + h * V
        minus = dict(args); minus[name] = val - h * V
        fd = (_f(plus["x"], W, plus["A"], plus["B"], s, dY)
              - _f(minus["x"], W, minus["A"], minus["B"], s, dY)) / (2 * h)
        assert abs(fd - float(np.sum(grad * V))) < 1e-10 * (1 + abs(fd)), name


def test_special_cases():
    x, W, A, B, dY = _tiny(3, M=5, N=4, K=5, r=2)
    y0 = linear.qlora_forward(x, W, A, np.zeros_like(B), 0.5)["y"]
    assert np.allclose(y0, x @ W.T, rtol=0, atol=1e-13)
    g0 = linear.qlora_backward(dY, x, W, A, B, 0.0)
    assert np.all(g0["dA"] == 0) and np.all(g0["dB"] == 0)
    assert np.allclose(g0["dX"], dY @ W, rtol=0, atol=1e-13)
    gA = linear.qlora_backward(dY, x, W, np.zeros_like(A), B, 1.0)
    assert np.all(gA["dB"] == 0)
    eye = np.eye(5)
    yI = linear.qlora_forward(eye, W, A, B, 2.0)["y"]
    assert np.allclose(yI, W.T + 2.0 * A.T @ B.T, rtol=0, atol=1e-13)


def test_sampled_rows_match_full():
    x, W, A, B, dY = _tiny(4, M=9, N=7, K=6, r=3)
    rows = np.array([0, 4, 8])
    full = linear.qlora_forward(x, W, A, B, 0.3)["y"]
    assert np.allclose(linear.forward_rows(x, W, A, B, 0.3, rows), full[rows], atol=1e-13)
    g = linear.qlora_backward(dY, x, W, A, B, 0.3)
    assert np.allclose(linear.dx_rows(dY, W, A, B, 0.3, rows), g["dX"][rows], atol=1e-13)


def test_adapter_grads_match_full_backward():
    x, W, A, B, dY = _tiny(5, M=8, N=6, K=7, r=3)
    g = linear.qlora_backward(dY, x, W, A, B, 0.4)
    a = linear.adapter_grads(dY, x, A, B, 0.4)
    assert np.allclose(a["dA"], g["dA"], atol=1e-13) and np.allclose(a["dB"], g["dB"], atol=1e-13)
    assert np.allclose(a["t"], linear.qlora_forward(x, W, A, B, 0.4)["t"], atol=1e-13)


def test_flop_count():
    assert linear.linear_flops(2, 3, 5, 7) == 4 * 2 * 3 * 5 + 6 * 2 * 5 * 7 + 6 * 2 * 3 * 7
