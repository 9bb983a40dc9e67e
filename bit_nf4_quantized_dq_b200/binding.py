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
c_double = ctypes.c_double

# name -> (restype, argtypes); mirrors include/qlora_nf4.h
SIGNATURES = {
    "qnf4_version": (c_int, []),
    "qnf4_last_error": (ctypes.c_char_p, []),
    "qnf4_device_error": (c_int, [c_void_p, ctypes.POINTER(ctypes.c_uint32)]),
    "qnf4_selftest_bounded_wait": (c_int, [ctypes.c_uint64, c_void_p]),
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
    "qnf4_quantize_workspace_bytes_ex": (c_size_t, [c_int64, c_int]),
    "qnf4_quantize_ex": (c_int, [c_void_p, c_int64, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                 c_size_t, c_void_p]),
    "qnf4_dequant_ex": (c_int, [c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_void_p]),
    "qlora_linear_fwd_ex": (c_int, [c_void_p, c_int64, c_int64, c_int64, c_int, c_int, c_void_p, c_void_p,
                                    c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_float, c_void_p, c_void_p,
                                    c_void_p, c_size_t, c_void_p]),
    "qnf4_paged_alloc": (c_int, [c_size_t, ctypes.POINTER(c_void_p)]),
    "qnf4_paged_free": (c_int, [c_void_p]),
    "qnf4_paged_prefetch": (c_int, [c_void_p, c_size_t, c_int, c_void_p]),
    "qlora_adamw_step": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_double, c_double,
                                 c_double, c_double, c_double, c_int, c_void_p]),
    "qlora_merge_workspace_bytes": (c_size_t, [c_int64, c_int64, c_int, c_int]),
    "qlora_merge_requantize": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int, c_int,
                                       c_void_p, c_void_p, c_int, c_float, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_size_t, c_void_p]),
    "qlora_linear_bwd_ex": (c_int, [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64, c_int, c_int,
                                    c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_float,
                                    c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
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


CODEBOOKS = {"nf4": 0, "fp4_e2m1": 1, "int4": 2}   # QNF4_CODEBOOK_* in include/qlora_nf4.h


class NF4Tensor:
    """A quantized weight: 4-bit codes and their block scales.

    With double quantization (the default): E4M3 scale codes, fp32 group constants `c2` and
    the fp32 mean.  Without it: `c2` holds one fp32 absmax per block and `scale_codes` and
    `mean` are None.  `codebook` names the 16 levels ("nf4", "fp4_e2m1" or "int4")."""

    def __init__(self, codes, scale_codes, c2, mean, shape, codebook: str = "nf4", double_quant: bool = True):
        if codebook not in CODEBOOKS:
            raise QNF4Error(f"unknown code book {codebook!r}")
        self.codes = codes
        self.scale_codes = scale_codes
        self.c2 = c2
        self.mean = mean
        self.shape = tuple(shape)
        self.codebook = codebook
        self.double_quant = bool(double_quant)

    @property
    def scales(self):
        return self.c2

    def _format(self):
        return CODEBOOKS[self.codebook], 1 if self.double_quant else 0

    @property
    def numel(self) -> int:
        n = 1
        for d in self.shape:
            n *= d
        return n

    def nbytes(self) -> int:
        n = self.codes.numel() + 4 * self.c2.numel()
        if self.double_quant:
            n += self.scale_codes.numel() + 4 * self.mean.numel()
        return n


def quantize(W: torch.Tensor, codebook: str = "nf4", double_quant: bool = True,
             workspace: Optional[torch.Tensor] = None) -> NF4Tensor:
    """Blockwise 4-bit quantization of a bf16 weight with any of the code books, with or
    without double quantization of the block scales."""
    if codebook == "nf4" and double_quant:
        return nf4_quantize_dq(W, workspace)
    W = _bf16_bits(W)
    _require_cuda(W)
    numel = W.numel()
    nb = (numel + 63) // 64
    ng = (nb + 255) // 256
    dev = W.device
    codes = torch.empty(32 * nb, dtype=torch.uint8, device=dev)
    if double_quant:
        sc = torch.empty(nb, dtype=torch.uint8, device=dev)
        scales = torch.empty(ng, dtype=torch.float32, device=dev)
        mean = torch.empty(1, dtype=torch.float32, device=dev)
    else:
        sc, mean = None, None
        scales = torch.empty(nb, dtype=torch.float32, device=dev)
    out = NF4Tensor(codes, sc, scales, mean, W.shape, codebook, double_quant)
    cb, dq = out._format()
    L = lib()
    need = L.qnf4_quantize_workspace_bytes_ex(numel, dq)
    if workspace is None or workspace.numel() < need:
        workspace = _ws(need, dev)
    _check(L.qnf4_quantize_ex(_ptr(W), numel, cb, dq, _ptr(codes), _ptr(sc), _ptr(scales), _ptr(mean),
                              _ptr(workspace), workspace.numel(), _stream()), "qnf4_quantize_ex")
    return out


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
    cb, dq = q._format()
    _check(lib().qnf4_dequant_ex(_ptr(q.codes), cb, dq, _ptr(q.scale_codes), _ptr(q.c2), _ptr(q.mean), q.numel,
                                 _ptr(out), _stream()), "qnf4_dequant_ex")
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
    cb, dq = q._format()
    _check(L.qlora_linear_fwd_ex(_ptr(x), M, K, N, cb, dq, _ptr(q.codes), _ptr(q.scale_codes), _ptr(q.c2),
                                 _ptr(q.mean), _ptr(A), _ptr(B), r, float(s), _ptr(y), _ptr(t), _ptr(workspace),
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
    cb, dq = q._format()
    _check(L.qlora_linear_bwd_ex(_ptr(dY), _ptr(x), _ptr(t_saved), M, K, N, cb, dq, _ptr(q.codes),
                                 _ptr(q.scale_codes), _ptr(q.c2), _ptr(q.mean), _ptr(A), _ptr(B), r, float(s),
                                 _ptr(dX), _ptr(dA), _ptr(dB), _ptr(workspace), workspace.numel(), _stream()),
           "qlora_linear_bwd")
    return dX, dA, dB


def merge_requantize(q: NF4Tensor, A: torch.Tensor, B: torch.Tensor, s: float, return_merged: bool = False):
    """Fold the adapters into the base and quantize the result again in the same format:
    W'' = bf16(W' + s B A), then quantized.  Returns the new NF4Tensor (and W'' as a bf16
    tensor when `return_merged`)."""
    _require_cuda(A, B, q.codes)
    N, K = q.shape
    r = A.shape[0]
    if tuple(A.shape) != (r, K) or tuple(B.shape) != (N, r):
        raise QNF4Error("shape mismatch between W, A and B")
    dev = q.codes.device
    nb = (N * K + 63) // 64
    ng = (nb + 255) // 256
    codes = torch.empty(32 * nb, dtype=torch.uint8, device=dev)
    if q.double_quant:
        sc = torch.empty(nb, dtype=torch.uint8, device=dev)
        scales = torch.empty(ng, dtype=torch.float32, device=dev)
        mean = torch.empty(1, dtype=torch.float32, device=dev)
    else:
        sc, mean = None, None
        scales = torch.empty(nb, dtype=torch.float32, device=dev)
    out = NF4Tensor(codes, sc, scales, mean, (N, K), q.codebook, q.double_quant)
    merged = torch.empty((N, K), dtype=torch.bfloat16, device=dev) if return_merged else None
    cb, dq = q._format()
    L = lib()
    ws = _ws(L.qlora_merge_workspace_bytes(N, K, dq, 1 if merged is not None else 0), dev)
    _check(L.qlora_merge_requantize(_ptr(q.codes), _ptr(q.scale_codes), _ptr(q.c2), _ptr(q.mean), N, K, cb, dq,
                                    _ptr(A), _ptr(B), r, float(s), _ptr(codes), _ptr(sc), _ptr(scales), _ptr(mean),
                                    _ptr(merged), _ptr(ws), ws.numel(), _stream()), "qlora_merge_requantize")
    return (out, merged) if return_merged else out


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
