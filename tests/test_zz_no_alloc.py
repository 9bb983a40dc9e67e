"""nf4_quantize_dq_noalloc, the quantizer that keeps its scratch in a static device array of
the library instead of a caller workspace, against nf4_quantize_dq on the same weights.

The codec is bit-exact, so the test tolerance is equality: codes, scale codes, group
constants c2 and the mean must match nf4_quantize_dq exactly, on two calls in a row and
across a sequence of sizes (a smaller call after a larger one must not see the larger call's
leftover scratch).  Every call goes through the C ABI.
"""

import ctypes

import pytest
import torch

import synth
from bit_nf4_quantized_dq_b200 import binding

pytestmark = pytest.mark.gpu

MAX_NUMEL = 268435456   # QNF4_NOALLOC_MAX_NUMEL in include/qlora_nf4.h


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _outputs(numel, dev, poison):
    nb = (numel + 63) // 64
    ng = (nb + 255) // 256
    codes = torch.full((32 * nb,), poison, dtype=torch.uint8, device=dev)
    sc = torch.full((nb,), poison, dtype=torch.uint8, device=dev)
    c2 = torch.full((ng,), float("nan"), dtype=torch.float32, device=dev)
    mean = torch.full((1,), float("nan"), dtype=torch.float32, device=dev)
    return codes, sc, c2, mean


def _reference(L, W):
    """Outputs of nf4_quantize_dq with a caller workspace."""
    numel = W.numel()
    out = _outputs(numel, W.device, 0x5A)
    ws = torch.empty(L.nf4_quantize_workspace_bytes(numel), dtype=torch.uint8, device=W.device)
    rc = L.nf4_quantize_dq(_ptr(W), numel, *map(_ptr, out), _ptr(ws), ws.numel(), _stream())
    assert rc == 0, L.qnf4_last_error()
    return out


def _noalloc(L, W, poison):
    out = _outputs(W.numel(), W.device, poison)
    rc = L.nf4_quantize_dq_noalloc(_ptr(W), W.numel(), *map(_ptr, out), _stream())
    assert rc == 0, L.qnf4_last_error()
    return out


def _assert_same(ref, got):
    torch.cuda.synchronize()
    for name, a, b in zip(("codes", "scale_codes", "c2", "mean"), ref, got):
        if a.dtype == torch.float32:
            a, b = a.view(torch.int32), b.view(torch.int32)
        assert torch.equal(a, b), name


def _weight(N, K, seed):
    return synth.robust_weight_bf16(N, K, seed).to("cuda")


@pytest.mark.parametrize("N,K", [(4000, 3000), (5120, 5120), (3, 100)])
def test_two_calls_in_a_row_match_workspace_entry_point(N, K):
    L = binding.lib()
    W = _weight(N, K, 7100 + N)
    ref = _reference(L, W)
    first = _noalloc(L, W, 0xA5)
    second = _noalloc(L, W, 0x3C)
    _assert_same(ref, first)
    _assert_same(ref, second)


def test_sequence_of_sizes_matches_workspace_entry_point():
    L = binding.lib()
    for i, (N, K) in enumerate([(5120, 5120), (1, 64), (777, 1000), (4096, 11008)]):
        W = _weight(N, K, 7200 + i)
        _assert_same(_reference(L, W), _noalloc(L, W, 0xC3))


def test_binding_wrapper_writes_into_given_buffers():
    W = _weight(640, 960, 7300)
    ref = binding.nf4_quantize_dq(W)
    out = binding.nf4_quantize_dq_noalloc(W, out=binding.nf4_quantize_dq(W))
    for _ in range(2):
        got = binding.nf4_quantize_dq_noalloc(W, out=out)
        assert got is out
        _assert_same((ref.codes, ref.scale_codes, ref.c2, ref.mean), (got.codes, got.scale_codes, got.c2, got.mean))


def test_above_the_static_limit_is_rejected_before_device_work():
    L = binding.lib()
    small = torch.zeros(64, dtype=torch.uint8, device="cuda")
    p = _ptr(small)
    assert L.nf4_quantize_dq_noalloc(p, MAX_NUMEL + 1, p, p, p, p, _stream()) == -2
    assert b"static scratch limit" in L.qnf4_last_error()
    assert binding.NOALLOC_MAX_NUMEL == MAX_NUMEL


def _oracle_sampled(W_cpu, blocks):
    """Oracle scale codes / c2 / mean of the whole weight, and the codes of `blocks` only
    (a block's codes depend on its own 64 weights and absmax alone)."""
    import numpy as np
    from oracle import nf4 as onf4
    w = W_cpu.float().numpy().ravel()
    absmax = onf4.block_absmax(w)
    dq = onf4.double_quantize(absmax)
    nb = absmax.size
    wp = np.zeros(nb * 64, np.float32)
    wp[:w.size] = w
    _, packed = onf4.level1_codes(wp.reshape(nb, 64)[blocks].ravel())
    return dq, packed.reshape(len(blocks), 32)


@pytest.mark.parametrize("numel", [MAX_NUMEL, MAX_NUMEL - 32])
def test_size_limit_fills_the_static_scratch(numel):
    """numel at the limit (every absmax slot and group sum of the static array in use) and
    just below it (a ragged last block): equal to the workspace entry point bit for bit, and
    to the oracle on the DQ parts and on sampled blocks' codes."""
    import numpy as np
    L = binding.lib()
    W_cpu = synth.normal_bf16((numel,), 0.02, 7400 + (numel & 63))
    W = W_cpu.to("cuda")
    ref = _reference(L, W)
    got = _noalloc(L, W, 0x99)
    _assert_same(ref, got)
    nb = (numel + 63) // 64
    rng = np.random.default_rng(numel)
    blocks = np.unique(np.concatenate([rng.choice(nb, 3000, replace=False), [0, nb - 2, nb - 1]]))
    dq, packed = _oracle_sampled(W_cpu, blocks)
    codes = got[0].view(-1, 32)[torch.as_tensor(blocks, device="cuda")].cpu().numpy()
    assert np.array_equal(codes, packed)
    assert np.array_equal(got[1].cpu().numpy(), dq["scale_codes"])
    assert np.array_equal(got[2].cpu().numpy(), dq["c2"])
    assert got[3].cpu().numpy()[0] == dq["mean"]
    del W, ref, got
    torch.cuda.empty_cache()


def test_binding_rejects_out_buffers_too_small_for_the_weight():
    small = binding.nf4_quantize_dq(_weight(64, 64, 7500))
    W = _weight(640, 960, 7501)
    with pytest.raises(binding.QNF4Error, match="codes"):
        binding.nf4_quantize_dq_noalloc(W, out=small)
    wrong = binding.nf4_quantize_dq(W)
    wrong.c2 = wrong.c2.to(torch.float64)
    with pytest.raises(binding.QNF4Error, match="c2"):
        binding.nf4_quantize_dq_noalloc(W, out=wrong)
    # a correctly sized buffer from a weight of another shape is accepted and takes W's shape
    other = binding.nf4_quantize_dq(_weight(960, 640, 7502))
    got = binding.nf4_quantize_dq_noalloc(W, out=other)
    assert got.shape == (640, 960)
