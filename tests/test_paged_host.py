"""Host-side logic of the paged AdamW (no GPU): the states are allocated as managed memory, each
step pages them to the device before the updates on the same stream, ``evict`` pages them to
host RAM, ``close`` frees them.  A fake library records the calls."""

import ctypes

import pytest
import torch

from bit_nf4_quantized_dq_b200 import binding, paged


class FakeLib:
    def __init__(self):
        self.calls = []
        self.next_ptr = 1 << 20

    class managed_buffer:            # stands in for managed memory: a host tensor and a fake address
        def __init__(self, L, n, device):
            self.L, self.n, self.nbytes = L, n, 4 * n
            self.ptr = L.next_ptr
            L.next_ptr += 1 << 16
            self.tensor = torch.zeros(n)
            L.calls.append(("alloc", self.ptr, self.nbytes))

        def free(self):
            self.L.calls.append(("free", self.ptr))
            self.ptr = 0

    def qnf4_paged_prefetch(self, ptr, nbytes, to_device, stream):
        self.calls.append(("prefetch", ptr.value, nbytes, to_device))
        return 0

    def qlora_adamw_step(self, p, g, m, v, b, n, lr, b1, b2, eps, wd, step, stream):
        self.calls.append(("step", m.value, v.value, n, step))
        return 0

    def qnf4_last_error(self):
        return b""


@pytest.fixture
def fake(monkeypatch):
    L = FakeLib()
    monkeypatch.setattr(paged, "_stream", lambda: ctypes.c_void_p(0))
    return L


def test_states_are_paged_in_before_every_step(fake):
    params = [torch.zeros(10), torch.zeros(6)]
    opt = paged.PagedAdamW(params, lr=1e-3, library=fake)
    allocs = [c for c in fake.calls if c[0] == "alloc"]
    assert len(allocs) == 4 and [c[2] for c in allocs] == [40, 40, 24, 24]
    fake.calls.clear()
    grads = [torch.zeros(10, dtype=torch.bfloat16), torch.zeros(6, dtype=torch.bfloat16)]
    opt.step(grads)
    opt.step(grads)
    kinds = [c[0] for c in fake.calls]
    assert kinds == ["prefetch"] * 4 + ["step"] * 2 + ["prefetch"] * 4 + ["step"] * 2
    assert all(c[3] == 1 for c in fake.calls if c[0] == "prefetch")
    steps = [c for c in fake.calls if c[0] == "step"]
    assert [c[4] for c in steps] == [1, 1, 2, 2]
    m_ptrs = {a[1] for a in allocs[0::2]}
    assert {c[1] for c in steps} == m_ptrs


def test_evict_pages_out_and_close_frees(fake):
    opt = paged.PagedAdamW([torch.zeros(8)], library=fake)
    fake.calls.clear()
    opt.evict()
    assert [c[0] for c in fake.calls] == ["prefetch", "prefetch"] and all(c[3] == 0 for c in fake.calls)
    fake.calls.clear()
    opt.close()
    assert [c[0] for c in fake.calls] == ["free", "free"]


def test_unpaged_states_need_no_paging(fake):
    opt = paged.PagedAdamW([torch.zeros(8)], paged=False, library=fake)
    fake.calls.clear()
    opt.step([torch.zeros(8, dtype=torch.bfloat16)])
    assert [c[0] for c in fake.calls] == ["step"]


def test_bad_arguments(fake):
    with pytest.raises(binding.QNF4Error):
        paged.PagedAdamW([torch.zeros(8, dtype=torch.float64)], library=fake)
    opt = paged.PagedAdamW([torch.zeros(8)], library=fake)
    with pytest.raises(binding.QNF4Error):
        opt.step([torch.zeros(8)])               # fp32 gradient: must be bf16
