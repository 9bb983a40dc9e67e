"""The bounded waits on the GPU, without a fault: a kernel waits, through the same bounded-wait
code as every pipeline wait of the library, on a barrier that nothing completes.  The wait must
give up after its limit, report through the device error word, and leave the context usable."""

import ctypes

import pytest
import torch

import bit_nf4_quantized_dq_b200 as q
from bit_nf4_quantized_dq_b200 import binding

pytestmark = pytest.mark.gpu

SELFTEST_FLAG = 0x20


def test_bounded_wait_gives_up_reports_and_leaves_the_context_usable():
    L = binding.lib()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    word = ctypes.c_uint32(0)
    torch.cuda.synchronize()
    L.qnf4_device_error(st, ctypes.byref(word))          # start from a clear word
    assert L.qnf4_selftest_bounded_wait(50_000_000, st) == 0   # 50 ms
    rc = L.qnf4_device_error(st, ctypes.byref(word))
    assert rc == -5, L.qnf4_last_error()
    assert word.value & SELFTEST_FLAG
    # the word was cleared by the read, and the library still works on this context
    W = (torch.randn(256, 512, device="cuda") * 0.02).to(torch.bfloat16)
    Q = q.nf4_quantize_dq(W)
    Wd = q.nf4_dequant(Q)
    torch.cuda.synchronize()
    assert torch.isfinite(Wd.float()).all()
    assert L.qnf4_device_error(st, ctypes.byref(word)) == 0 and word.value == 0
