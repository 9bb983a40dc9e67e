"""GPU parity of the NF4 + DQ codec (through the C ABI) against the oracle: bit-exact codes,
E4M3 scale codes, group constants, mean and dequantized bf16 values."""

import numpy as np
import pytest
import torch

from oracle import nf4 as onf4
import synth
import bit_nf4_quantized_dq_b200 as q

pytestmark = pytest.mark.gpu


def _gpu_quant(w: torch.Tensor):
    Q = q.nf4_quantize_dq(w.cuda())
    torch.cuda.synchronize()
    assert q.check_device_error() == 0
    return (Q.codes.cpu().numpy(), Q.scale_codes.cpu().numpy(), Q.c2.cpu().numpy(),
            np.float32(Q.mean.cpu().numpy()[0]), Q)


def _assert_codec_equal(w: torch.Tensor):
    codes, e, c2, mean, Q = _gpu_quant(w)
    ref = onf4.quantize_nf4_dq(w.float().numpy().ravel())
    assert mean.view(np.uint32) == np.float32(ref["mean"]).view(np.uint32)
    assert np.array_equal(c2.view(np.uint32), ref["c2"].view(np.uint32))
    assert np.array_equal(e, ref["scale_codes"])
    assert np.array_equal(codes, ref["codes"])
    return ref, Q


def test_quantize_single_1024():
    w = synth.normal_bf16((1024, 1024), 0.02, synth.seed_for(1, 0))
    _assert_codec_equal(w)


def test_quantize_ragged_1d_and_tiny():
    for numel, seed in ((64 * 1000 + 37, 11), (1, 12), (63, 13), (64, 14), (65, 15), (64 * 256 + 1, 16)):
        w = synth.normal_bf16((numel,), 0.02, seed)
        _assert_codec_equal(w)


def test_quantize_robust_4000x3000_padded_final_group():
    w = synth.robust_weight_bf16(4000, 3000, synth.seed_for(5, 0))
    ref, _ = _assert_codec_equal(w)
    assert ref["c2"].size == 733          # 187500 blocks -> last group holds 108 scales


def test_quantize_degenerate_tensors():
    zeros = torch.zeros(64 * 300, dtype=torch.bfloat16)
    ref, _ = _assert_codec_equal(zeros)
    assert np.all(ref["codes"] == 0x77) and np.all(ref["c2"] == 0) and ref["mean"] == 0
    const = torch.full((64 * 300,), 0.03125, dtype=torch.bfloat16)
    _assert_codec_equal(const)
    mixed = synth.normal_bf16((64 * 600,), 0.02, 21)
    mixed[64 * 10:64 * 20] = 0
    mixed[5] = 0
    _assert_codec_equal(mixed)
    big = synth.normal_bf16((64 * 512,), 300.0, 22)        # large magnitudes, exponents > 0
    _assert_codec_equal(big)
    tiny = synth.normal_bf16((64 * 512,), 1e-30, 23)       # tiny magnitudes
    _assert_codec_equal(tiny)


def test_nearest_level_sweep_every_bf16_ratio():
    """Blocks [c, w1..w63]: for 160 absmax values c, every bf16 w in [-c, c] is normalised and
    snapped; this places many fp32 n right next to every midpoint between levels."""
    rng = np.random.default_rng(5)
    all_bf16 = np.arange(0, 1 << 16, dtype=np.uint32) << 16
    vals = all_bf16.view(np.float32)
    vals = vals[np.isfinite(vals)]
    blocks = []
    for c in (rng.uniform(0.5, 2.0, 160) * 2.0 ** rng.integers(-8, 4, 160)).astype(np.float32):
        c = onf4.bf16_bits_to_f32(onf4.bf16_rn_bits(np.array([c])))[0]
        w = vals[np.abs(vals) <= c]
        w = w[rng.permutation(w.size)][: 63 * 200]
        w = np.pad(w, (0, (-w.size) % 63))
        b = np.concatenate([np.full((w.size // 63, 1), c, np.float32), w.reshape(-1, 63)], axis=1)
        blocks.append(b)
    data = torch.from_numpy(np.concatenate(blocks).ravel()).to(torch.bfloat16)
    _assert_codec_equal(data)


def test_quantize_llama_shapes_dq_full_codes_sampled():
    """Full-size LLaMA-7B gate (11008x4096): absmax-derived DQ exactly, codes on sampled blocks."""
    w = synth.normal_bf16((11008, 4096), 0.02, synth.seed_for(2, 4))
    codes, e, c2, mean, _ = _gpu_quant(w)
    wf = w.float().numpy().ravel()
    absmax = onf4.block_absmax(wf)
    dq = onf4.double_quantize(absmax)
    assert mean.view(np.uint32) == np.float32(dq["mean"]).view(np.uint32)
    assert np.array_equal(c2.view(np.uint32), dq["c2"].view(np.uint32))
    assert np.array_equal(e, dq["scale_codes"])
    rng = np.random.default_rng(3)
    blocks = np.sort(rng.choice(absmax.size, 4000, replace=False))
    sub = wf.reshape(-1, 64)[blocks].ravel()
    _, ref_codes = onf4.level1_codes(sub)
    assert np.array_equal(codes.reshape(-1, 32)[blocks].ravel(), ref_codes)


def test_dequant_bitexact_from_oracle_codes():
    cases = [synth.normal_bf16((1024, 1024), 0.02, synth.seed_for(1, 0)),
             synth.robust_weight_bf16(4000, 3000, synth.seed_for(5, 0)),
             synth.normal_bf16((64 * 1000 + 37,), 0.02, 11),
             torch.zeros(64 * 10, dtype=torch.bfloat16)]
    for w in cases:
        ref = onf4.quantize_nf4_dq(w.float().numpy().ravel())
        want = onf4.dequant_nf4_dq(ref["codes"], ref["scale_codes"], ref["c2"], ref["mean"], w.numel())
        Q = q.NF4Tensor(torch.from_numpy(ref["codes"]).cuda(), torch.from_numpy(ref["scale_codes"]).cuda(),
                        torch.from_numpy(ref["c2"]).cuda(),
                        torch.from_numpy(np.array([ref["mean"]], np.float32)).cuda(), w.shape)
        out = q.nf4_dequant(Q)
        torch.cuda.synchronize()
        got = out.cpu().contiguous().view(torch.int16).numpy().view(np.uint16).ravel()
        assert np.array_equal(got, want)


def test_quantize_then_dequant_round_trip_exact_zero():
    w = synth.robust_weight_bf16(4000, 3000, synth.seed_for(5, 0))
    Q = q.nf4_quantize_dq(w.cuda())
    out = q.nf4_dequant(Q).cpu()
    zero = (w == 0)
    assert zero.sum() > 0
    assert torch.all(out[zero] == 0)


def test_e4m3_encoders_match_oracle():
    rng = np.random.default_rng(9)
    pos = onf4.e4m3_decode(np.arange(127))
    mids = (pos[:-1] + pos[1:]) / 2
    near = []
    for m in mids:
        f = np.float32(m)
        near += [f, np.nextafter(f, np.float32(-1)), np.nextafter(f, np.float32(2))]
    v = np.concatenate([np.array(near, np.float32), -np.array(near, np.float32),
                        rng.uniform(-1, 1, 2_000_000).astype(np.float32),
                        (rng.uniform(-1, 1, 200_000) * 2.0 ** -7).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, -1.0, 448.0, 500.0, -1e-30], np.float32)])
    want = onf4.e4m3_encode_rn(v)
    vt = torch.from_numpy(v).cuda()
    for mode in (0, 1):
        got = q.e4m3_encode(vt, mode).cpu().numpy()
        assert np.array_equal(got, want), f"mode {mode}: {int((got != want).sum())} mismatches"


def test_zero_size_is_rejected():
    with pytest.raises(q.QNF4Error):
        q.nf4_quantize_dq(torch.zeros(0, dtype=torch.bfloat16, device="cuda"))
