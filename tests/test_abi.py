"""The C-ABI library loads without a GPU, exports every function include/qlora_nf4.h declares,
and rejects bad arguments on the host before touching the device."""

import ctypes
import os
import re

import pytest

from bit_nf4_quantized_dq_b200 import binding

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "qlora_nf4.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"^\s*(?:int|size_t|const char\s*\*)\s+(\w+)\s*\(", text, flags=re.M))


def test_library_exports_every_declared_function():
    L = binding.lib()
    names = declared_functions()
    assert {"nf4_quantize_dq", "nf4_dequant", "qlora_linear_fwd", "qlora_linear_bwd"} <= names
    for n in names:
        assert hasattr(L, n), n
    assert set(binding.SIGNATURES) == names


def test_version_and_last_error():
    L = binding.lib()
    assert L.qnf4_version() >= 100
    assert isinstance(L.qnf4_last_error(), bytes)


def test_workspace_sizes():
    L = binding.lib()
    nb = 4096 * 4096 // 64
    ng = nb // 256
    assert L.nf4_quantize_workspace_bytes(4096 * 4096) == nb * 4 + ng * 8
    assert L.nf4_quantize_workspace_bytes(0) == 0
    # forward: t hi/lo in bf16, no split at 8192 tokens
    assert L.qlora_linear_fwd_workspace_bytes(8192, 5120, 5120, 64) >= 2 * 8192 * 64 * 2
    assert L.qlora_linear_bwd_workspace_bytes(8192, 5120, 5120, 64) > 0
    assert L.qlora_linear_fwd_workspace_bytes(-1, 5120, 5120, 64) == 0


FAKE = ctypes.c_void_p(1 << 20)        # 256-byte aligned, never dereferenced by these calls


def test_null_and_size_errors_before_any_device_work():
    L = binding.lib()
    assert L.nf4_quantize_dq(None, 64, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == -1
    assert L.nf4_quantize_dq(FAKE, 0, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == -1
    assert L.nf4_quantize_dq(FAKE, 1 << 40, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == -2
    assert L.nf4_quantize_dq(FAKE, 4096, FAKE, FAKE, FAKE, FAKE, FAKE, 16, None) == -6
    assert L.nf4_dequant(FAKE, FAKE, FAKE, FAKE, -5, FAKE, None) == -1
    assert L.nf4_dequant(ctypes.c_void_p((1 << 20) + 4), FAKE, FAKE, FAKE, 64, FAKE, None) == -2
    assert b"16 B" in L.qnf4_last_error()


def _fwd(L, M, K, N, r, ws_bytes=1 << 30, x=FAKE):
    return L.qlora_linear_fwd(x, M, K, N, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, r, 1.0, FAKE, FAKE, FAKE,
                              ws_bytes, None)


def test_selftest_rejects_limits_outside_range_before_any_device_work():
    L = binding.lib()
    assert L.qnf4_selftest_bounded_wait(999_999, None) == -1          # below 1 ms
    assert L.qnf4_selftest_bounded_wait(10_000_000_001, None) == -1   # above 10 s
    assert b"limit_ns" in L.qnf4_last_error()


def test_linear_shape_errors():
    L = binding.lib()
    assert _fwd(L, 128, 1024, 1024, 16, x=None) == -1
    assert _fwd(L, 0, 1024, 1024, 16) == -1
    assert _fwd(L, 128, 1020, 1024, 16) == -2          # K % 8
    assert _fwd(L, 128, 1024, 1020, 16) == -2          # N % 8
    assert _fwd(L, 128, 1024, 1024, 12) == -2          # r % 8
    assert _fwd(L, 128, 1024, 1024, 264) == -2         # r > 256
    assert _fwd(L, 128, 1024, 1024, 16, ws_bytes=10) == -6
    assert _fwd(L, 128, 1024, 1024, 16, x=ctypes.c_void_p((1 << 20) + 2)) == -2
    rc = L.qlora_linear_bwd(FAKE, FAKE, FAKE, 128, 1024, 1024, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, 1.0,
                            None, FAKE, None, FAKE, 1 << 30, None)
    assert rc == -1                                     # dB is required


def test_binding_refuses_cpu_tensors():
    torch = pytest.importorskip("torch")
    w = torch.zeros(64, dtype=torch.bfloat16)
    with pytest.raises(binding.QNF4Error):
        binding.nf4_quantize_dq(w)
