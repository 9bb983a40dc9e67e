"""GPU parity of the QLoRA linear forward / backward (through the C ABI) against the oracle,
within the stated tolerance, plus bit-exact special cases of the fused dequant producer."""

import numpy as np
import pytest
import torch

import synth
import bit_nf4_quantized_dq_b200 as q
from parity_util import assert_within_tolerance, oracle_linear, oracle_weight

pytestmark = pytest.mark.gpu


def _run_gpu(W, x, A, B, dY, s):
    Q = q.nf4_quantize_dq(W.cuda())
    xc, Ac, Bc, dYc = x.cuda(), A.cuda(), B.cuda(), dY.cuda()
    y, t = q.qlora_linear_fwd(xc, Q, Ac, Bc, s)
    dX, dA, dB = q.qlora_linear_bwd(dYc, xc, t, Q, Ac, Bc, s)
    torch.cuda.synchronize()
    assert q.check_device_error() == 0
    return {"y": y.cpu(), "t": t.cpu(), "dX": dX.cpu(), "dA": dA.cpu(), "dB": dB.cpu(), "Q": Q}


def _check(W, x, A, B, dY, s, rows=None, tag=""):
    got = _run_gpu(W, x, A, B, dY, s)
    ow = oracle_weight(W)
    ref = oracle_linear(x, ow["w_deq"], A, B, dY, s, rows=rows)
    sel = (lambda a: a) if rows is None else (lambda a: a[torch.as_tensor(rows)])
    assert_within_tolerance(sel(got["y"]), ref["y"], f"{tag} y")
    assert_within_tolerance(sel(got["dX"]), ref["dX"], f"{tag} dX")
    assert_within_tolerance(got["dA"], ref["dA"], f"{tag} dA")
    assert_within_tolerance(got["dB"], ref["dB"], f"{tag} dB")
    # t = s x A^T: each 64-deep block of exact bf16 products is summed in fp32 by the tensor
    # cores (at most 64 additions, each off by under 2^-23 relative even if the hardware
    # truncates), the block sums are added in float64, and the result is rounded once to
    # fp32.  So |err| <= 128 * 2^-23 * s * sum_k |x_k A_jk| + 2^-24 |t| (a factor 2 of slack).
    x64 = x.float().numpy().astype(np.float64)
    A64 = A.float().numpy().astype(np.float64)
    mag = abs(s) * (np.abs(x64) @ np.abs(A64).T)
    t_err = np.abs(got["t"].numpy().astype(np.float64) - ref["t"])
    assert np.all(t_err <= 128 * 2.0 ** -23 * mag + 2.0 ** -24 * np.abs(ref["t"])), f"{tag} t"
    return got


def test_single_1024_r16():
    W = synth.normal_bf16((1024, 1024), 0.02, synth.seed_for(1, 0))
    inp = synth.linear_inputs(128, 1024, 1024, 16, synth.seed_for(1, 1))
    _check(W, inp["x"], inp["A"], inp["B"], inp["dY"], 16.0 / 16, tag="single")


@pytest.fixture(scope="module")
def robust_weight():
    return synth.robust_weight_bf16(4000, 3000, synth.seed_for(5, 0))


@pytest.mark.parametrize("r", [8, 64, 256])
@pytest.mark.parametrize("M", [1, 16, 512, 16384])
def test_robust_4000x3000(robust_weight, r, M):
    """K = 3000 is not a multiple of 64: blocks span rows and the codes take the no-TMA path."""
    inp = synth.linear_inputs(M, 4000, 3000, r, synth.seed_for(5, 10 + r + M))
    rows = None if M <= 512 else np.sort(np.random.default_rng(M + r).choice(M, 192, replace=False))
    _check(robust_weight, inp["x"], inp["A"], inp["B"], inp["dY"], 16.0 / r, rows=rows,
           tag=f"robust r={r} M={M}")


@pytest.mark.parametrize("name", ["q", "down"])
def test_llama7b_512(name):
    lin = {l.name: l for l in synth.LLAMA7B}[name]
    idx = [l.name for l in synth.LLAMA7B].index(name)
    W = synth.normal_bf16((lin.N, lin.K), 0.02, synth.seed_for(2, idx))
    inp = synth.linear_inputs(512, lin.N, lin.K, 64, synth.seed_for(2, 100 + idx))
    _check(W, inp["x"], inp["A"], inp["B"], inp["dY"], 16.0 / 64, tag=f"7b {name}")


@pytest.mark.parametrize("name", ["q", "gate", "down"])
def test_llama13b_8192_sampled_rows(name):
    """The benchmark's configuration (8192 tokens): sampled rows of y and dX, full dA / dB."""
    lin = {l.name: l for l in synth.LLAMA13B}[name]
    idx = [l.name for l in synth.LLAMA13B].index(name)
    W = synth.normal_bf16((lin.N, lin.K), 0.02, synth.seed_for(3, idx))
    inp = synth.linear_inputs(8192, lin.N, lin.K, 64, synth.seed_for(3, 100 + idx))
    rows = np.sort(np.random.default_rng(idx).choice(8192, 128, replace=False))
    _check(W, inp["x"], inp["A"], inp["B"], inp["dY"], 16.0 / 64, rows=rows, tag=f"13b {name}")


def _bits(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("N,K", [(384, 256), (4000, 3000)])
def test_identity_input_reproduces_dequant_bits(N, K):
    """x = I, B = 0: y = W'^T exactly, bit for bit equal to the standalone dequant."""
    W = synth.normal_bf16((N, K), 0.02, 31)
    Q = q.nf4_quantize_dq(W.cuda())
    Wd = q.nf4_dequant(Q)
    x = torch.eye(K, dtype=torch.bfloat16, device="cuda")
    A = synth.normal_bf16((16, K), 0.25, 32).cuda()
    B = torch.zeros((N, 16), dtype=torch.bfloat16, device="cuda")
    y, _ = q.qlora_linear_fwd(x, Q, A, B, 1.0)
    assert np.array_equal(_bits(y), _bits(Wd.t().contiguous()))
    # dY = I (M = N), A = 0: dX = W' exactly
    dY = torch.eye(N, dtype=torch.bfloat16, device="cuda")
    A0 = torch.zeros((16, K), dtype=torch.bfloat16, device="cuda")
    xN = synth.normal_bf16((N, K), 1.0, 33).cuda()
    _, t = q.qlora_linear_fwd(xN, Q, A0, B, 1.0)
    dX, dA, dB = q.qlora_linear_bwd(dY, xN, t, Q, A0, B, 1.0)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(dX), _bits(Wd))
    assert torch.all(dB.float() == 0)


def test_zero_scale_gives_zero_adapter_grads():
    W = synth.normal_bf16((512, 1024), 0.02, 41)
    inp = synth.linear_inputs(256, 512, 1024, 64, 42)
    got = _run_gpu(W, inp["x"], inp["A"], inp["B"], inp["dY"], 0.0)
    assert torch.all(got["dA"].float() == 0) and torch.all(got["dB"].float() == 0)
    assert torch.all(got["t"] == 0)


def test_zero_adapter_b_gives_base_gemm():
    W = synth.normal_bf16((512, 1024), 0.02, 43)
    inp = synth.linear_inputs(256, 512, 1024, 64, 44)
    B0 = torch.zeros_like(inp["B"])
    got = _run_gpu(W, inp["x"], inp["A"], B0, inp["dY"], 0.25)
    ow = oracle_weight(W)
    ref = oracle_linear(inp["x"], ow["w_deq"], inp["A"], B0, inp["dY"], 0.25)
    assert_within_tolerance(got["y"], ref["y"], "B=0 y")


@pytest.mark.parametrize("M", [24, 48, 100, 200, 300, 520])
def test_token_counts_cover_every_tile_width(M):
    """Token counts that select each token-tile width of the fused GEMMs (16 ... 256) and
    the K-split path, on an aligned and on a K % 64 != 0 weight."""
    for (N, K, seed) in ((640, 1024, 51), (520, 1000, 52)):
        W = synth.normal_bf16((N, K), 0.02, seed)
        inp = synth.linear_inputs(M, N, K, 32, seed + 100)
        _check(W, inp["x"], inp["A"], inp["B"], inp["dY"], 0.5, tag=f"M={M} N={N} K={K}")


@pytest.mark.parametrize("M", [256, 300])
def test_dx_256_token_tiles_on_ragged_edges(M):
    """256-token tiles of the fused dX with K % 128 = 64 (the last row tile's second half lies
    past the weight) and N % 64 != 0 (the last k-block of W rows is partial)."""
    N, K = 200, 192
    W = synth.normal_bf16((N, K), 0.02, 61)
    inp = synth.linear_inputs(M, N, K, 64, 62)
    _check(W, inp["x"], inp["A"], inp["B"], inp["dY"], 0.25, tag=f"ragged dX M={M}")
