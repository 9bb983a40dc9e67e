"""Thin Python binding over the C ABI in include/qlora_nf4.h.

Argument marshalling only: PyTorch provides device memory and the current stream, every
step of the computation runs in the library's CUDA kernels.  There is no fallback: if the
shared library is missing or cannot be loaded, every call raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import build as _build

_LIB: Optional[ctypes.CDLL] = None

c_void_p = ctypes.c_void_p
c_int64 = ctypes.c_int64
c_int = ctypes.c_int
c_size_t = ctypes.c_size_t
c_float = ctypes.c_float

# name -> (restype, argtypes); mirrors include/qlora_nf4.h
SIGNATURES = {
    "qnf4_version": (c_int, []),
    "qnf4_last_error": (ctypes.c_char_p, []),
    "qnf4_device_error": (c_int, [c_void_p, ctypes.POINTER(ctypes.c_uint32)]),
    "nf4_quantize_workspace_bytes": (c_size_t, [c_int64]),
    "nf4_quantize_dq": (c_int, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                c_size_t, c_void_p]),
    "nf4_quantize_dq_noalloc": (c_int, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "nf4_dequant": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_void_p]),
    "qlora_linear_fwd_workspace_bytes": (c_size_t, [c_int64, c_int64, c_int64, c_int]),
    "qlora_linear_fwd": (c_int, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_int, c_float, c_void_p, c_void_p,
                                 c_void_p, c_size_t, c_void_p]),
    "qlora_linear_bwd_workspace_bytes": (c_size_t, [c_int64, c_int64, c_int64, c_int]),
    "qlora_linear_bwd": (c_int, [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_float,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "nf4_e4m3_encode": (c_int, [c_void_p, c_int64, c_void_p, c_int, c_void_p]),
    "qnf4_set_timing_events": (c_int, [c_void_p, c_int]),
    "qlora_linear_plan": (c_int, [c_int64, c_int64, c_int64, c_int, ctypes.POINTER(c_int),
                                  ctypes.POINTER(c_int), ctypes.POINTER(c_int), ctypes.POINTER(c_int)]),
}


class QNF4Error(RuntimeError):
    pass


def library_path() -> str:
    return _build.LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded library (building it first if it is missing or stale and nvcc exists)."""
    global _LIB
    if _LIB is None:
        path = _build.LIB_PATH
        if not os.path.exists(path) or _build.is_stale():
            try:
                _build.build()
            except Exception as e:  # no nvcc: only an existing library can be used
                if not os.path.exists(path):
                    raise QNF4Error(f"the CUDA library {path} is missing and cannot be built: {e}")
        handle = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = handle
    return _LIB


def _check(rc: int, what: str) -> None:
    if rc != 0:
        msg = lib().qnf4_last_error().decode(errors="replace")
        raise QNF4Error(f"{what} failed with status {rc}: {msg}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise QNF4Error("operands must be contiguous CUDA tensors")


def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _bf16_bits(t: torch.Tensor) -> torch.Tensor:
    if t.dtype != torch.bfloat16:
        raise QNF4Error("expected a bfloat16 tensor")
    return t


def check_device_error() -> int:
    """Synchronise the current stream; raise if a kernel gave up waiting."""
    word = ctypes.c_uint32(0)
    rc = lib().qnf4_device_error(_stream(), ctypes.byref(word))
    if rc != 0:
        raise QNF4Error(f"device error word 0x{word.value:x}: {lib().qnf4_last_error().decode()}")
    return word.value


class NF4Tensor:
    """A quantized weight: codes, E4M3 scale codes, fp32 group constants, fp32 mean."""

    def __init__(self, codes, scale_codes, c2, mean, shape):
        self.codes = codes
        self.scale_codes = scale_codes
        self.c2 = c2
        self.mean = mean
        self.shape = tuple(shape)

    @property
    def numel(self) -> int:
        n = 1
        for d in self.shape:
            n *= d
        return n

    def nbytes(self) -> int:
        return (self.codes.numel() + self.scale_codes.numel() + 4 * self.c2.numel() + 4 * self.mean.numel())


def nf4_quantize_dq(W: torch.Tensor, workspace: Optional[torch.Tensor] = None) -> NF4Tensor:
    """Quantize a bf16 weight (any shape, flattened row-major) to NF4 + DQ."""
    W = _bf16_bits(W)
    _require_cuda(W)
    numel = W.numel()
    nb = (numel + 63) // 64
    ng = (nb + 255) // 256
    dev = W.device
    codes = torch.empty(32 * nb, dtype=torch.uint8, device=dev)
    scale_codes = torch.empty(nb, dtype=torch.uint8, device=dev)
    c2 = torch.empty(ng, dtype=torch.float32, device=dev)
    mean = torch.empty(1, dtype=torch.float32, device=dev)
    L = lib()
    need = L.nf4_quantize_workspace_bytes(numel)
    if workspace is None or workspace.numel() < need:
        workspace = _ws(need, dev)
    _check(L.nf4_quantize_dq(_ptr(W), numel, _ptr(codes), _ptr(scale_codes), _ptr(c2), _ptr(mean),
                             _ptr(workspace), workspace.numel(), _stream()), "nf4_quantize_dq")
    return NF4Tensor(codes, scale_codes, c2, mean, W.shape)


def _check_out_buffer(t: torch.Tensor, dtype, count: int, device, name: str) -> None:
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or not t.is_contiguous() or t.device != device:
        raise QNF4Error(f"out.{name} must be a contiguous {dtype} tensor on {device}")
    if t.numel() < count:
        raise QNF4Error(f"out.{name} holds {t.numel()} elements, the weight needs {count}")


def nf4_quantize_dq_noalloc(W: torch.Tensor, out: Optional[NF4Tensor] = None) -> NF4Tensor:
    """nf4_quantize_dq without a workspace: the library's static scratch holds the absmax and
    group sums (numel <= NOALLOC_MAX_NUMEL; overlapping calls on one device race on it).  Pass
    `out` to write into existing buffers, so that the call itself allocates nothing; they are
    checked against W (device, dtype, contiguity, size) before the call."""
    W = _bf16_bits(W)
    _require_cuda(W)
    numel = W.numel()
    nb = (numel + 63) // 64
    ng = (nb + 255) // 256
    dev = W.device
    if out is None:
        out = NF4Tensor(torch.empty(32 * nb, dtype=torch.uint8, device=dev),
                        torch.empty(nb, dtype=torch.uint8, device=dev),
                        torch.empty(ng, dtype=torch.float32, device=dev),
                        torch.empty(1, dtype=torch.float32, device=dev), W.shape)
    else:
        _check_out_buffer(out.codes, torch.uint8, 32 * nb, dev, "codes")
        _check_out_buffer(out.scale_codes, torch.uint8, nb, dev, "scale_codes")
        _check_out_buffer(out.c2, torch.float32, ng, dev, "c2")
        _check_out_buffer(out.mean, torch.float32, 1, dev, "mean")
    with torch.cuda.device(dev):
        _check(lib().nf4_quantize_dq_noalloc(_ptr(W), numel, _ptr(out.codes), _ptr(out.scale_codes), _ptr(out.c2),
                                             _ptr(out.mean), _stream()), "nf4_quantize_dq_noalloc")
    out.shape = tuple(W.shape)
    return out


NOALLOC_MAX_NUMEL = 1 << 28   # QNF4_NOALLOC_MAX_NUMEL


def nf4_dequant(q: NF4Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """NF4 + DQ -> bf16 tensor of the original shape."""
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.codes.device)
    _require_cuda(out, q.codes)
    _check(lib().nf4_dequant(_ptr(q.codes), _ptr(q.scale_codes), _ptr(q.c2), _ptr(q.mean), q.numel,
                             _ptr(out), _stream()), "nf4_dequant")
    return out


def qlora_linear_fwd(x: torch.Tensor, q: NF4Tensor, A: torch.Tensor, B: torch.Tensor, s: float,
                     workspace: Optional[torch.Tensor] = None):
    """y = x W'^T + s (x A^T) B^T.  Returns (y, t_saved)."""
    _require_cuda(x, A, B)
    M, K = x.shape
    N = q.shape[0]
    r = A.shape[0]
    if q.shape != (N, K) or tuple(A.shape) != (r, K) or tuple(B.shape) != (N, r):
        raise QNF4Error("shape mismatch between x, W, A and B")
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    t = torch.empty((M, r), dtype=torch.float32, device=x.device)
    L = lib()
    need = L.qlora_linear_fwd_workspace_bytes(M, K, N, r)
    if workspace is None or workspace.numel() < need:
        workspace = _ws(need, x.device)
    _check(L.qlora_linear_fwd(_ptr(x), M, K, N, _ptr(q.codes), _ptr(q.scale_codes), _ptr(q.c2), _ptr(q.mean),
                              _ptr(A), _ptr(B), r, float(s), _ptr(y), _ptr(t), _ptr(workspace),
                              workspace.numel(), _stream()), "qlora_linear_fwd")
    return y, t


def qlora_linear_bwd(dY: torch.Tensor, x: torch.Tensor, t_saved: torch.Tensor, q: NF4Tensor,
                     A: torch.Tensor, B: torch.Tensor, s: float, need_dx: bool = True,
                     workspace: Optional[torch.Tensor] = None):
    """Returns (dX or None, dA, dB)."""
    _require_cuda(dY, x, t_saved, A, B)
    M, K = x.shape
    N = q.shape[0]
    r = A.shape[0]
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=x.device) if need_dx else None
    dA = torch.empty((r, K), dtype=torch.bfloat16, device=x.device)
    dB = torch.empty((N, r), dtype=torch.bfloat16, device=x.device)
    L = lib()
    need = L.qlora_linear_bwd_workspace_bytes(M, K, N, r)
    if workspace is None or workspace.numel() < need:
        workspace = _ws(need, x.device)
    _check(L.qlora_linear_bwd(_ptr(dY), _ptr(x), _ptr(t_saved), M, K, N, _ptr(q.codes), _ptr(q.scale_codes),
                              _ptr(q.c2), _ptr(q.mean), _ptr(A), _ptr(B), r, float(s), _ptr(dX), _ptr(dA),
                              _ptr(dB), _ptr(workspace), workspace.numel(), _stream()), "qlora_linear_bwd")
    return dX, dA, dB


def set_timing_events(events) -> None:
    """Record these torch.cuda.Event objects at the stage boundaries of later fwd / bwd calls
    made from this thread (see qnf4_set_timing_events); None stops recording."""
    global _EVENT_ARRAY
    if not events:
        _EVENT_ARRAY = None
        _check(lib().qnf4_set_timing_events(None, 0), "qnf4_set_timing_events")
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _EVENT_ARRAY = arr                       # keep the handle array alive while recording
    _check(lib().qnf4_set_timing_events(ctypes.cast(arr, ctypes.c_void_p), len(events)),
           "qnf4_set_timing_events")


_EVENT_ARRAY = None


def linear_plan(M: int, K: int, N: int, r: int) -> dict:
    """Kernel launches per forward / backward call and the fused GEMMs' K-split factors."""
    v = [c_int(0) for _ in range(4)]
    _check(lib().qlora_linear_plan(M, K, N, r, *[ctypes.byref(x) for x in v]), "qlora_linear_plan")
    return {"fwd_launches": v[0].value, "bwd_launches": v[1].value, "fwd_splits": v[2].value,
            "dx_splits": v[3].value}


def e4m3_encode(v: torch.Tensor, mode: int = 0) -> torch.Tensor:
    _require_cuda(v)
    out = torch.empty(v.numel(), dtype=torch.uint8, device=v.device)
    _check(lib().nf4_e4m3_encode(_ptr(v), v.numel(), _ptr(out), mode, _stream()), "nf4_e4m3_encode")
    return out
