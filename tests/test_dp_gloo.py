"""World-size-2 data parallelism on CPU (gloo): token sharding, and the all-reduce of the
adapter gradients reproduces the full-batch gradients of the oracle."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_nf4_quantized_dq_b200.dp import allreduce_adapter_grads, token_shard


def test_token_shard_covers_all_tokens():
    for total in (1, 7, 8192, 16385):
        for world in (1, 2, 3, 8):
            spans = [token_shard(total, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [e - s for s, e in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        token_shard(10, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import linear as olin
        rng = np.random.default_rng(0)
        M, N, K, r, s = 24, 12, 10, 4, 0.5
        x = rng.standard_normal((M, K)); dY = rng.standard_normal((M, N))
        A = rng.standard_normal((r, K)); B = rng.standard_normal((N, r))
        lo, hi = token_shard(M, rank, world)
        g = olin.adapter_grads(dY[lo:hi], x[lo:hi], A, B, s)
        dA = torch.from_numpy(g["dA"].copy())
        dB = torch.from_numpy(g["dB"].copy())
        allreduce_adapter_grads([dA, dB])
        full = olin.adapter_grads(dY, x, A, B, s)
        ok = np.allclose(dA.numpy(), full["dA"], atol=1e-12) and np.allclose(dB.numpy(), full["dB"], atol=1e-12)
        # bf16 tensors are reduced in fp32 and averaged on request
        h = torch.full((3,), float(rank + 1), dtype=torch.bfloat16)
        allreduce_adapter_grads([h], average=True)
        ok = ok and bool(torch.all(h.float() == 1.5))
        if rank == 0:
            with open(out_path, "w") as f:
                f.write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


def test_allreduce_reproduces_full_batch_gradients(tmp_path):
    out = str(tmp_path / "res.txt")
    mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
    assert open(out).read() == "ok"
