"""GPU parity of the code-book variants (FP4 E2M1, INT4) and of single-level quantization
(fp32 block scales, no double quantization) against the oracle: codes, scales and dequantized
bf16 values bit-exact, the QLoRA linear within the stated tolerance."""

import numpy as np
import pytest
import torch

import synth
import bit_nf4_quantized_dq_b200 as q
from oracle import nf4 as onf4
from oracle import variants as ov
from parity_util import assert_within_tolerance, oracle_linear

pytestmark = pytest.mark.gpu

FORMATS = [(cb, dq) for cb in ("nf4", "fp4_e2m1", "int4") for dq in (True, False)]


def _check_codec(w: torch.Tensor, cb: str, dq: bool):
    Q = q.quantize(w.cuda(), codebook=cb, double_quant=dq)
    deq = q.nf4_dequant(Q)
    torch.cuda.synchronize()
    assert q.check_device_error() == 0
    table = ov.codebook(cb)
    ref = ov.quantize_blockwise(w.float().numpy().ravel(), table, dq)
    assert np.array_equal(Q.codes.cpu().numpy(), ref["codes"])
    if dq:
        assert np.array_equal(Q.scale_codes.cpu().numpy(), ref["scale_codes"])
        assert np.array_equal(Q.c2.cpu().numpy().view(np.uint32), ref["c2"].view(np.uint32))
        assert Q.mean.cpu().numpy().view(np.uint32)[0] == np.float32(ref["mean"]).view(np.uint32)
        want = ov.dequant_blockwise(ref["codes"], table, w.numel(), ref["scale_codes"], ref["c2"], ref["mean"])
    else:
        assert Q.scale_codes is None and Q.mean is None
        assert np.array_equal(Q.c2.cpu().numpy().view(np.uint32), ref["absmax"].view(np.uint32))
        want = ov.dequant_blockwise(ref["codes"], table, w.numel(), absmax=ref["absmax"])
    got = deq.cpu().contiguous().view(torch.int16).numpy().view(np.uint16).ravel()
    assert np.array_equal(got, want)
    return Q


@pytest.mark.parametrize("cb,dq", FORMATS)
def test_codec_robust_and_ragged(cb, dq):
    _check_codec(synth.robust_weight_bf16(4000, 3000, synth.seed_for(5, 0)), cb, dq)
    _check_codec(synth.normal_bf16((64 * 1000 + 37,), 0.02, 11), cb, dq)
    zeros = torch.zeros(64 * 10, dtype=torch.bfloat16)
    zeros[5] = -0.0
    _check_codec(zeros, cb, dq)


def _reachable_blocks():
    """Every bf16 absmax significand, every bf16 weight within 10 binades below it (both signs)."""
    blocks = []
    mant = np.arange(128, dtype=np.float64)
    for mc in range(128):
        c = 1.0 + mc / 128.0
        ws = []
        for k in range(11):
            w = (1.0 + mant / 128.0) * 2.0 ** (-k)
            w = w[w <= c]
            ws += [w, -w]
        ws.append(np.zeros(3))
        w = np.concatenate(ws).astype(np.float32)
        w = np.pad(w, (0, (-w.size) % 63))
        lead = np.full((w.size // 63, 1), c if mc % 2 == 0 else -c, np.float32)
        blocks.append(np.concatenate([lead, w.reshape(-1, 63)], axis=1))
    return torch.from_numpy(np.concatenate(blocks).ravel()).to(torch.bfloat16)


@pytest.mark.parametrize("cb", ["fp4_e2m1", "int4"])
def test_nearest_level_exhaustive_for_other_tables(cb):
    Q = _check_codec(_reachable_blocks(), cb, False)
    codes = onf4.unpack_codes(Q.codes.cpu().numpy(), Q.numel)
    assert set(np.unique(codes).tolist()) >= set(range(1, 16))


@pytest.mark.parametrize("cb,dq", [("fp4_e2m1", False), ("int4", True), ("nf4", False), ("fp4_e2m1", True)])
@pytest.mark.parametrize("N,K,M", [(640, 1024, 300), (520, 1000, 24), (1024, 1024, 512)])
def test_linear_fwd_bwd(cb, dq, N, K, M):
    W = synth.normal_bf16((N, K), 0.02, 61 + N)
    inp = synth.linear_inputs(M, N, K, 32, 62 + N)
    Q = q.quantize(W.cuda(), codebook=cb, double_quant=dq)
    x, A, B, dY = (inp[k].cuda() for k in ("x", "A", "B", "dY"))
    s = 0.5
    y, t = q.qlora_linear_fwd(x, Q, A, B, s)
    dX, dA, dB = q.qlora_linear_bwd(dY, x, t, Q, A, B, s)
    torch.cuda.synchronize()
    assert q.check_device_error() == 0
    table = ov.codebook(cb)
    ref = ov.quantize_blockwise(W.float().numpy().ravel(), table, dq)
    if dq:
        bits = ov.dequant_blockwise(ref["codes"], table, W.numel(), ref["scale_codes"], ref["c2"], ref["mean"])
    else:
        bits = ov.dequant_blockwise(ref["codes"], table, W.numel(), absmax=ref["absmax"])
    Wd = onf4.bf16_bits_to_f32(bits).astype(np.float64).reshape(N, K)
    o = oracle_linear(inp["x"], Wd, inp["A"], inp["B"], inp["dY"], s)
    tag = f"{cb} dq={dq} {N}x{K} M={M}"
    assert_within_tolerance(y.cpu(), o["y"], tag + " y")
    assert_within_tolerance(dX.cpu(), o["dX"], tag + " dX")
    assert_within_tolerance(dA.cpu(), o["dA"], tag + " dA")
    assert_within_tolerance(dB.cpu(), o["dB"], tag + " dB")


@pytest.mark.parametrize("cb,dq", [("fp4_e2m1", False), ("int4", True)])
def test_identity_input_reproduces_dequant_bits(cb, dq):
    """x = I, B = 0: the fused forward returns the standalone dequant bit for bit."""
    N, K = 384, 256
    W = synth.normal_bf16((N, K), 0.02, 71)
    Q = q.quantize(W.cuda(), codebook=cb, double_quant=dq)
    Wd = q.nf4_dequant(Q)
    x = torch.eye(K, dtype=torch.bfloat16, device="cuda")
    A = synth.normal_bf16((16, K), 0.25, 72).cuda()
    B = torch.zeros((N, 16), dtype=torch.bfloat16, device="cuda")
    y, _ = q.qlora_linear_fwd(x, Q, A, B, 1.0)
    torch.cuda.synchronize()

    def bits(t):
        # the sum behind y[m][n] adds +0 terms to W'[n][m]: a -0 weight (E2M1 has a -0 level)
        # comes out as +0, so zeros are compared without their sign
        b = t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16).copy()
        b[b == 0x8000] = 0
        return b
    assert np.array_equal(bits(y), bits(Wd.t().contiguous()))


def test_single_level_storage_bytes():
    """Without double quantization a weight costs 4 + 32/64 = 4.5 bits (teardown section 3)."""
    W = synth.normal_bf16((1024, 1024), 0.02, 73)
    Q = q.quantize(W.cuda(), codebook="nf4", double_quant=False)
    assert Q.nbytes() * 8 / W.numel() == 4.5
