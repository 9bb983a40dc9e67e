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


def _reachable_blocks(c_exponents=(0, -20, 30)):
    """Blocks [c or -c, w1..w63] covering, for every bf16 absmax significand c (128 of them, at
    each exponent in `c_exponents`), every bf16 weight w with |w| <= c whose exponent lies
    within 10 binades of c's (both signs), plus exact zeros.  The normalised value
    n = fp32(w / c) depends only on the two significands and the exponent gap, and any gap
    above 5 puts |n| below 1/32, far under the smallest midpoint (code 7), so these blocks
    reach every normalised value that can decide a code."""
    blocks = []
    mant = np.arange(128, dtype=np.float64)
    for ec in c_exponents:
        for mc in range(128):
            c = (1.0 + mc / 128.0) * 2.0 ** ec
            ws = []
            for k in range(11):
                w = (1.0 + mant / 128.0) * 2.0 ** (ec - k)
                w = w[w <= c]
                ws += [w, -w]
            ws.append(np.zeros(5))
            w = np.concatenate(ws).astype(np.float32)
            w = np.pad(w, (0, (-w.size) % 63))
            lead = np.full((w.size // 63, 1), c if mc % 2 == 0 else -c, np.float32)
            blocks.append(np.concatenate([lead, w.reshape(-1, 63)], axis=1))
    return np.concatenate(blocks).ravel()


def test_nearest_level_exhaustive_over_reachable_quotients():
    """Every normalised value a bf16 weight and a bf16 absmax can produce (and that can decide
    a code) goes through the GPU quantizer: codes, scale codes, c2 and mean bit-exact."""
    data = _reachable_blocks()
    assert data.size > 1_000_000
    ref, _ = _assert_codec_equal(torch.from_numpy(data).to(torch.bfloat16))
    codes = onf4.unpack_codes(ref["codes"], data.size)
    assert set(np.unique(codes).tolist()) == set(range(16))


def test_e4m3_hardware_and_software_encoders_agree_on_every_fp32_in_unit_interval():
    """All 2 x (0x3F800000 + 1) fp32 values in [-1, 1], in chunks, through both encoders on the
    GPU (the hardware conversion is the one the quantizer uses)."""
    step = 1 << 27
    for sign in (0, 0x80000000):
        lo, hi = 0, 0x3F800000 + 1
        for a in range(lo, hi, step):
            b = min(hi, a + step)
            bits = torch.arange(a, b, dtype=torch.int64, device="cuda") | sign
            v = bits.to(torch.int32).view(torch.float32) if sign == 0 else \
                (bits - (1 << 32)).to(torch.int32).view(torch.float32)
            hw = q.e4m3_encode(v, 0)
            sw = q.e4m3_encode(v, 1)
            bad = int((hw != sw).sum())
            assert bad == 0, f"{bad} mismatches in [{a:#x}, {b:#x}) sign {sign:#x}"
    torch.cuda.synchronize()


def test_e4m3_encoders_match_oracle_near_every_midpoint():
    """Every fp32 within 64 ulp of each midpoint between neighbouring E4M3 values in [0, 1]
    (and their negatives), plus every E4M3 value's own neighbourhood."""
    pos = onf4.e4m3_decode(np.arange(127))
    pos = pos[pos <= 1.0]
    pts = np.concatenate([(pos[:-1] + pos[1:]) / 2, pos]).astype(np.float32)
    bits = pts.view(np.uint32).astype(np.int64)
    offs = np.arange(-64, 65, dtype=np.int64)
    allb = (bits[:, None] + offs[None, :]).ravel()
    allb = allb[(allb >= 0) & (allb <= 0x3F800000)]
    v = allb.astype(np.uint32).view(np.float32)
    v = np.concatenate([v, -v])
    want = onf4.e4m3_encode_rn(v)
    vt = torch.from_numpy(v).cuda()
    for mode in (0, 1):
        got = q.e4m3_encode(vt, mode).cpu().numpy()
        assert np.array_equal(got, want), f"mode {mode}: {int((got != want).sum())} mismatches"
