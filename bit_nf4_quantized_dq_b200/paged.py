"""Paged AdamW for the LoRA adapters.

"QLoRA Paper Breakdown: 4-Bit NormalFloat (NF4), Double Quantization, and Paged Optimizers"
(fullstackaihub), section 5: the AdamW states m_t and v_t of the adapters live in CUDA unified
memory; under a memory spike the driver (or the caller, with ``evict``) moves their pages to
host RAM, and they are paged back for the optimizer step.  "QLoRA, explained." step 6.

The step itself is the library's ``qlora_adamw_step`` kernel; this module only manages the
state buffers and the order of prefetches and launches.
"""

from __future__ import annotations

import ctypes
from typing import List, Optional, Sequence

import torch

from .binding import QNF4Error, _check, _stream, lib


class _Managed:
    """A managed-memory fp32 buffer of `n` elements, exposed to torch without a copy."""

    def __init__(self, L, n: int, device: torch.device):
        self.L = L
        self.n = n
        self.nbytes = 4 * n
        ptr = ctypes.c_void_p(0)
        _check(L.qnf4_paged_alloc(self.nbytes, ctypes.byref(ptr)), "qnf4_paged_alloc")
        self.ptr = ptr.value
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "<f4", "data": (self.ptr, False), "version": 3}
        with torch.cuda.device(device):
            # on the device before the first kernel touches it
            _check(L.qnf4_paged_prefetch(ctypes.c_void_p(self.ptr), self.nbytes, 1, _stream()), "qnf4_paged_prefetch")
            self.tensor = torch.as_tensor(self, device=device)

    def free(self):
        if self.ptr:
            self.tensor = None
            _check(self.L.qnf4_paged_free(ctypes.c_void_p(self.ptr)), "qnf4_paged_free")
            self.ptr = 0


class PagedAdamW:
    """AdamW (decoupled weight decay) over fp32 master copies of the adapters.

    params: fp32 CUDA tensors (updated in place); bf16_params: matching bf16 tensors that
    receive the updated values (the adapters the linear layer reads), or None.  With
    ``paged=True`` the states live in managed memory: ``step`` prefetches them to the device
    on the current stream before the update, ``evict`` sends them to host RAM."""

    def __init__(self, params: Sequence[torch.Tensor], bf16_params: Optional[Sequence[Optional[torch.Tensor]]] = None,
                 lr: float = 1e-4, betas=(0.9, 0.999), eps: float = 1e-8, weight_decay: float = 0.0,
                 paged: bool = True, library=None):
        self.L = library if library is not None else lib()
        self._managed = _Managed if library is None else getattr(library, "managed_buffer", _Managed)
        self.params = list(params)
        self.bf16 = list(bf16_params) if bf16_params is not None else [None] * len(self.params)
        if len(self.bf16) != len(self.params):
            raise QNF4Error("bf16_params must match params")
        for p, b in zip(self.params, self.bf16):
            if p.dtype != torch.float32 or not p.is_contiguous() or (library is None and not p.is_cuda):
                raise QNF4Error("parameters must be contiguous fp32 CUDA tensors")
            if b is not None and (b.dtype != torch.bfloat16 or b.numel() != p.numel() or not b.is_contiguous()):
                raise QNF4Error("bf16 copies must be contiguous bf16 tensors of the same size")
        self.lr, self.b1, self.b2, self.eps, self.wd = lr, betas[0], betas[1], eps, weight_decay
        self.paged = paged
        self.t = 0
        self.m: List = []
        self.v: List = []
        for p in self.params:
            if paged:
                m, v = self._managed(self.L, p.numel(), p.device), self._managed(self.L, p.numel(), p.device)
                m.tensor.zero_()
                v.tensor.zero_()
            else:
                m, v = torch.zeros_like(p), torch.zeros_like(p)
            self.m.append(m)
            self.v.append(v)

    def _state(self, s):
        return s.tensor if hasattr(s, "ptr") else s

    def state_bytes(self) -> int:
        return sum(8 * p.numel() for p in self.params)

    def prefetch(self, to_device: bool) -> None:
        """Move every state buffer to the device (True) or to host RAM (False), stream-ordered."""
        if not self.paged:
            return
        st = _stream()
        for s in self.m + self.v:
            _check(self.L.qnf4_paged_prefetch(ctypes.c_void_p(s.ptr), s.nbytes, 1 if to_device else 0, st),
                   "qnf4_paged_prefetch")

    def evict(self) -> None:
        self.prefetch(False)

    def step(self, grads: Sequence[torch.Tensor]) -> None:
        if len(grads) != len(self.params):
            raise QNF4Error("one gradient per parameter")
        self.t += 1
        self.prefetch(True)
        st = _stream()
        for p, g, m, v, b in zip(self.params, grads, self.m, self.v, self.bf16):
            if g.dtype != torch.bfloat16 or g.numel() != p.numel() or not g.is_contiguous():
                raise QNF4Error("gradients must be contiguous bf16 tensors of the parameters' sizes")
            mp = m.ptr if hasattr(m, "ptr") else m.data_ptr()
            vp = v.ptr if hasattr(v, "ptr") else v.data_ptr()
            _check(self.L.qlora_adamw_step(ctypes.c_void_p(p.data_ptr()), ctypes.c_void_p(g.data_ptr()),
                                           ctypes.c_void_p(mp), ctypes.c_void_p(vp),
                                           ctypes.c_void_p(b.data_ptr()) if b is not None else None, p.numel(),
                                           self.lr, self.b1, self.b2, self.eps, self.wd, self.t, st),
                   "qlora_adamw_step")

    def close(self) -> None:
        for s in self.m + self.v:
            if hasattr(s, "free"):
                s.free()
        self.m, self.v = [], []
