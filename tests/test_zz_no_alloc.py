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
