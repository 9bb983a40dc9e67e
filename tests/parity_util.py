"""Helpers shared by the GPU parity tests: oracle references and the stated tolerance.

Tolerance for the fused forward / backward outputs (bf16 operands, fp32 accumulation):
elementwise |err| <= 2e-2 * (|ref| + 1e-2) and relative Frobenius error <= 5e-3, with the
reference computed by the oracle in float64 from the same bf16 inputs.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import linear as olin
from oracle import nf4 as onf4

ELEM_RTOL = 2e-2
ELEM_FLOOR = 1e-2
FRO_TOL = 5e-3


def to_np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_within_tolerance(got: torch.Tensor | np.ndarray, ref: np.ndarray, what: str) -> None:
    g = to_np64(got) if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    bound = ELEM_RTOL * (np.abs(ref) + ELEM_FLOOR)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance; worst at {i}: "
                             f"got {g[i]!r} ref {ref[i]!r}")
    nref = np.linalg.norm(ref)
    fro = np.linalg.norm(g - ref) / nref if nref > 0 else np.linalg.norm(g)
    assert fro <= FRO_TOL, f"{what}: relative Frobenius error {fro:.3e}"


_WEIGHT_CACHE: dict = {}


def oracle_weight(w_bf16: torch.Tensor) -> dict:
    """Oracle quantize + dequant of a bf16 weight; W' as float64 [N][K] plus the codec parts
    (memoised on the weight's bytes: several tests share one weight)."""
    import hashlib
    key = (tuple(w_bf16.shape), hashlib.sha1(w_bf16.contiguous().view(torch.int16).numpy().tobytes()).hexdigest())
    if key in _WEIGHT_CACHE:
        return _WEIGHT_CACHE[key]
    w = w_bf16.float().cpu().numpy().ravel()
    qd = onf4.quantize_nf4_dq(w)
    bits = onf4.dequant_nf4_dq(qd["codes"], qd["scale_codes"], qd["c2"], qd["mean"], w.size)
    qd["w_deq_bits"] = bits
    qd["w_deq"] = onf4.bf16_bits_to_f32(bits).astype(np.float64).reshape(tuple(w_bf16.shape))
    if len(_WEIGHT_CACHE) > 4:
        _WEIGHT_CACHE.clear()
    _WEIGHT_CACHE[key] = qd
    return qd


def oracle_linear(x, Wd, A, B, dY, s, rows=None) -> dict:
    """Forward / backward references; y and dX restricted to ``rows`` when given."""
    x64 = to_np64(x)
    A64 = to_np64(A)
    B64 = to_np64(B)
    dY64 = to_np64(dY)
    if rows is None:
        f = olin.qlora_forward(x64, Wd, A64, B64, s)
        b = olin.qlora_backward(dY64, x64, Wd, A64, B64, s)
        return {"y": f["y"], "t": f["t"], "dX": b["dX"], "dA": b["dA"], "dB": b["dB"]}
    g = olin.adapter_grads(dY64, x64, A64, B64, s)
    return {
        "y": olin.forward_rows(x64, Wd, A64, B64, s, rows),
        "t": g["t"],
        "dX": olin.dx_rows(dY64, Wd, A64, B64, s, rows),
        "dA": g["dA"],
        "dB": g["dB"],
    }
