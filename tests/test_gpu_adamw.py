"""GPU parity of the AdamW step (qlora_adamw_step) against the float64 oracle, with the states
in plain device memory and in managed (paged) memory evicted to the host between steps.

Tolerance: the kernel computes in fp32 with IEEE division and square root.  m and v within
1e-6 relative; the parameters within two fp32 ulps of the reference plus 1e-5 of the update
(the update is small against the parameter, so the parameter's own rounding dominates)."""

import ctypes

import numpy as np
import pytest
import torch

import bit_nf4_quantized_dq_b200 as q
from bit_nf4_quantized_dq_b200 import binding
from oracle import adamw as oadamw

pytestmark = pytest.mark.gpu

HP = dict(lr=2e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.01)


def _run(paged: bool, sizes=(64 * 5120, 13824 * 64 + 3, 7)):
    torch.manual_seed(0)
    rng = np.random.default_rng(1)
    p_host = [rng.standard_normal(n).astype(np.float32) * 0.05 for n in sizes]
    params = [torch.from_numpy(x.copy()).cuda() for x in p_host]
    bf = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for n in sizes]
    opt = q.PagedAdamW(params, bf, paged=paged, **HP)
    ref = [(x.astype(np.float64), np.zeros(x.size), np.zeros(x.size)) for x in p_host]
    for step in range(1, 4):
        grads = [torch.from_numpy((rng.standard_normal(n) * 0.1).astype(np.float32)).to(torch.bfloat16).cuda()
                 for n in sizes]
        opt.step(grads)
        if paged:
            opt.evict()            # the states leave the device between steps and come back for the next
        new = []
        for (p0, m0, v0), g in zip(ref, grads):
            gg = g.float().cpu().numpy().astype(np.float64)
            new.append(oadamw.adamw_step(p0, gg, m0, v0, HP["lr"], HP["betas"][0], HP["betas"][1], HP["eps"],
                                         HP["weight_decay"], step))
        ref = new
    torch.cuda.synchronize()
    assert q.check_device_error() == 0
    for i, (p_ref, m_ref, v_ref) in enumerate(ref):
        p = params[i].cpu().numpy().astype(np.float64)
        m = opt._state(opt.m[i]).cpu().numpy().astype(np.float64)
        v = opt._state(opt.v[i]).cpu().numpy().astype(np.float64)
        upd = np.abs(p_ref - p_host[i].astype(np.float64))
        assert np.all(np.abs(p - p_ref) <= 2 * np.spacing(np.abs(p_ref).astype(np.float32)) + 1e-5 * upd)
        assert np.all(np.abs(m - m_ref) <= 1e-6 * np.abs(m_ref) + 1e-12)
        assert np.all(np.abs(v - v_ref) <= 1e-6 * np.abs(v_ref) + 1e-15)
        b = bf[i].float().cpu().numpy()
        assert np.array_equal(b, torch.from_numpy(params[i].cpu().numpy()).to(torch.bfloat16).float().numpy())
    opt.close()


def test_adamw_device_states():
    _run(paged=False)


def test_adamw_paged_states_evicted_between_steps():
    _run(paged=True)


def test_paged_alloc_and_prefetch_through_the_abi():
    L = binding.lib()
    ptr = ctypes.c_void_p(0)
    assert L.qnf4_paged_alloc(1 << 20, ctypes.byref(ptr)) == 0 and ptr.value
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.qnf4_paged_prefetch(ptr, 1 << 20, 1, st) == 0
    assert L.qnf4_paged_prefetch(ptr, 1 << 20, 0, st) == 0
    torch.cuda.synchronize()
    assert L.qnf4_paged_free(ptr) == 0
    assert L.qnf4_paged_alloc(0, ctypes.byref(ptr)) == -1
