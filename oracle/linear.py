"""QLoRA linear layer, forward and backward, in float64 on the host.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): the CUDA path never imports this.

Shapes (row-major): x [M, K] tokens x in-features, the frozen base W' [N, K]
(out x in, the dequantized NF4 weight), adapters A [r, K] and B [N, r], the LoRA scale
s = alpha / r, output y [M, N].

"QLoRA Paper Breakdown", section 4 (forward pass): Y = X * dequant(W) + (alpha/r) * X * L1 * L2
with L1 in R^{d x r} and L2 in R^{r x k}.  Reading: with the base stored out x in, the
pages' L1 is A^T and L2 is B^T, so

    y  = x W'^T + s (x A^T) B^T.

Section 4 also states that the backward pass needs dY/dX through the dequantized base and
never forms dL/dW; "QLoRA, explained." step 5 says the adapters are the only trained
tensors.  The gradients of <dY, y> are therefore

    dX = dY W' + s (dY B) A,    dA = s (dY B)^T x,    dB = s dY^T (x A^T).

Reading: "QLoRA, explained." notation list drops the LoRA scale from its equation; the
scale of the teardown's section 4 is kept (s is an explicit argument; s = 1 recovers the
unscaled form).

Every product is a float64 matrix product of the exact inputs (bf16 values and the
exact bf16 W'); nothing is rounded.  Pins: explicit-loop brute force on tiny shapes, exact
directional derivatives of <dY, y> (y is linear in each of x, A, B), and special cases
(B = 0, A = 0, s = 0, x = I) in ``tests/test_oracle_linear.py``.
"""

from __future__ import annotations

import numpy as np


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def qlora_forward(x, w_deq, A, B, s: float) -> dict:
    """y = x W'^T + s (x A^T) B^T; also returns the down-projection t = s x A^T."""
    x = _f64(x); W = _f64(w_deq); A = _f64(A); B = _f64(B)
    t = float(s) * (x @ A.T)
    y = x @ W.T + t @ B.T
    return {"y": y, "t": t}


def qlora_backward(dY, x, w_deq, A, B, s: float) -> dict:
    """Gradients of <dY, y> with respect to x, A and B (the base W' is frozen)."""
    dY = _f64(dY); x = _f64(x); W = _f64(w_deq); A = _f64(A); B = _f64(B)
    s = float(s)
    u = s * (dY @ B)                 # [M, r], the adapter's up-gradient projection
    dX = dY @ W + u @ A
    dA = u.T @ x
    dB = s * (dY.T @ (x @ A.T))
    return {"dX": dX, "dA": dA, "dB": dB, "u": u}


def adapter_grads(dY, x, A, B, s: float) -> dict:
    """dA and dB alone (same definitions as ``qlora_backward``), for shapes where the full
    dX product is too slow on the host; also returns t = s x A^T."""
    dY = _f64(dY); x = _f64(x); A = _f64(A); B = _f64(B)
    s = float(s)
    xa = x @ A.T
    return {"dA": (s * (dY @ B)).T @ x, "dB": s * (dY.T @ xa), "t": s * xa}


def forward_rows(x, w_deq, A, B, s: float, rows) -> np.ndarray:
    """Rows ``rows`` of y only (for sampled checks at sizes where the full product is slow)."""
    rows = np.asarray(rows)
    return qlora_forward(_f64(x)[rows], w_deq, A, B, s)["y"]


def dx_rows(dY, w_deq, A, B, s: float, rows) -> np.ndarray:
    """Rows ``rows`` of dX only."""
    rows = np.asarray(rows)
    dY = _f64(dY)[rows]
    return dY @ _f64(w_deq) + (float(s) * (dY @ _f64(B))) @ _f64(A)


def linear_flops(M: int, N: int, K: int, r: int) -> int:
    """Algorithmic flops of one forward + backward: 4MNK + 6MKr + 6MNr (no dW for the base)."""
    return 4 * M * N * K + 6 * M * K * r + 6 * M * N * r
