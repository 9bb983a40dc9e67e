"""GPU parity of the adapter merge + re-quantization (W'' = bf16(W' + s B A), then quantized
again) against the oracle: the merged bf16 weight and the new codes and scales bit-exact."""

import numpy as np
import pytest
import torch

import synth
import bit_nf4_quantized_dq_b200 as q
from oracle import nf4 as onf4
from oracle import variants as ov

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _oracle_base(W, cb, dq):
    table = ov.codebook(cb)
    ref = ov.quantize_blockwise(W.float().numpy().ravel(), table, dq)
    if dq:
        bits = ov.dequant_blockwise(ref["codes"], table, W.numel(), ref["scale_codes"], ref["c2"], ref["mean"])
    else:
        bits = ov.dequant_blockwise(ref["codes"], table, W.numel(), absmax=ref["absmax"])
    return bits.reshape(W.shape), table


@pytest.mark.parametrize("cb,dq", [("nf4", True), ("fp4_e2m1", False), ("int4", True)])
@pytest.mark.parametrize("N,K,r", [(256, 320, 16), (200, 520, 64), (96, 1024, 8)])
def test_merge_matches_oracle(cb, dq, N, K, r):
    W = synth.normal_bf16((N, K), 0.02, 81 + K)
    inp = synth.linear_inputs(8, N, K, r, 82 + K)
    A, B = inp["A"], inp["B"] * 20            # adapters large enough to move weights across levels
    s = 16.0 / r
    Q = q.quantize(W.cuda(), codebook=cb, double_quant=dq)
    Q2, merged = q.merge_requantize(Q, A.cuda(), B.cuda(), s, return_merged=True)
    torch.cuda.synchronize()
    assert q.check_device_error() == 0
    base_bits, table = _oracle_base(W, cb, dq)
    ref = ov.merge_requantize(base_bits, A.float().numpy(), B.float().numpy(), s, table, dq)
    assert np.array_equal(_bits(merged), ref["merged_bits"])
    assert np.array_equal(Q2.codes.cpu().numpy(), ref["codes"])
    if dq:
        assert np.array_equal(Q2.scale_codes.cpu().numpy(), ref["scale_codes"])
        assert np.array_equal(Q2.c2.cpu().numpy().view(np.uint32), ref["c2"].view(np.uint32))
        assert Q2.mean.cpu().numpy().view(np.uint32)[0] == np.float32(ref["mean"]).view(np.uint32)
    else:
        assert np.array_equal(Q2.c2.cpu().numpy().view(np.uint32), ref["absmax"].view(np.uint32))
    assert not np.array_equal(ref["merged_bits"], base_bits)       # the adapters did change the weights


def test_merge_with_zero_adapter_keeps_the_base():
    N, K, r = 512, 768, 16
    W = synth.normal_bf16((N, K), 0.02, 91)
    Q = q.nf4_quantize_dq(W.cuda())
    A = synth.normal_bf16((r, K), 0.25, 92).cuda()
    B = torch.zeros((N, r), dtype=torch.bfloat16, device="cuda")
    Q2, merged = q.merge_requantize(Q, A, B, 0.25, return_merged=True)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(merged), _bits(q.nf4_dequant(Q)))
    assert torch.equal(Q2.codes, Q.codes)
