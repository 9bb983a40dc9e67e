"""GPU parity of the AdamW step (qlora_adamw_step) against the float64 oracle, with the states
in plain device memory and in managed (paged) memory evicted to the host between steps.

Tolerance, from the arithmetic: the kernel keeps p, m and v in fp32 and rounds p once per step
(the final subtraction, at most half an ulp of the larger of the old and new |p|); the update
lr (m_hat / (sqrt(v_hat) + eps) + wd p) is formed from fp32 m and v through a handful of
correctly rounded operations on values of magnitude at most about 4 (the bias-corrected Adam
ratio is bounded near (1 - b1) / sqrt(1 - b2) = 3.2 for these betas), so it carries at most
16 units of 2^-24 times lr.  Errors of earlier steps pass on unchanged (the decay factor
1 - lr wd is below one).  The parameter bound is the sum of both terms over the steps, on the
oracle's own trajectory.  m and v see only their own roundings: per step at most 4 units of
2^-24 of b1 |m| + (1 - b1) |g| (the fp32 constants b1 and 1 - b1, the product and the fused
multiply-add), earlier errors shrinking by b1; v is a sum of positive terms, so the same
count gives 1e-6 relative over three steps."""

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
    bound = [np.zeros(n) for n in sizes]
    bound_m = [np.zeros(n) for n in sizes]
    for step in range(1, 4):
        grads = [torch.from_numpy((rng.standard_normal(n) * 0.1).astype(np.float32)).to(torch.bfloat16).cuda()
                 for n in sizes]
        opt.step(grads)
        if paged:
            opt.evict()            # the states leave the device between steps and come back for the next
        new = []
        for i, ((p0, m0, v0), g) in enumerate(zip(ref, grads)):
            gg = g.float().cpu().numpy().astype(np.float64)
            p1, m1, v1 = oadamw.adamw_step(p0, gg, m0, v0, HP["lr"], HP["betas"][0], HP["betas"][1], HP["eps"],
                                           HP["weight_decay"], step)
            big = np.maximum(np.abs(p0), np.abs(p1)).astype(np.float32)
            bound[i] += 0.5 * np.spacing(big).astype(np.float64) + 16 * 2.0 ** -24 * HP["lr"]
            b1 = HP["betas"][0]
            bound_m[i] = b1 * bound_m[i] + 4 * 2.0 ** -24 * (b1 * np.abs(m0) + (1 - b1) * np.abs(gg))
            new.append((p1, m1, v1))
        ref = new
    torch.cuda.synchronize()
    assert q.check_device_error() == 0
    for i, (p_ref, m_ref, v_ref) in enumerate(ref):
        p = params[i].cpu().numpy().astype(np.float64)
        m = opt._state(opt.m[i]).cpu().numpy().astype(np.float64)
        v = opt._state(opt.v[i]).cpu().numpy().astype(np.float64)
        err = np.abs(p - p_ref)
        assert np.all(err <= bound[i]), (i, float(np.max(err / bound[i])))
        assert np.all(np.abs(m - m_ref) <= bound_m[i])
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
