"""Host-side pieces of bench.py that need no GPU: the DRAM-traffic figures of the fused GEMMs
are reported only while the kernel sources they were captured on are unchanged; the bf16 peak
follows the clock record; `--gpus N` launches N ranks and checks the world size; the timed
region's rank orchestration (barriers, max over ranks, adapter-gradient all-reduce) runs on
two gloo ranks."""

import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _sources_hash(root):
    import hashlib
    h = hashlib.sha256()
    for f in bench.FUSED_SOURCES:
        with open(os.path.join(root, "bit_nf4_quantized_dq_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def test_traffic_reported_only_for_the_captured_sources():
    assert bench.FUSED_TRAFFIC["dx"] > 0 and bench.FUSED_TRAFFIC["fwd"] > 0
    same = _sources_hash(ROOT) == bench.FUSED_TRAFFIC["sources_sha256"]
    for k in ("dx", "fwd"):
        assert bench.fused_traffic(k) == (bench.FUSED_TRAFFIC[k] if same else None)


def test_traffic_withdrawn_when_a_kernel_source_changes(tmp_path, monkeypatch):
    # a copy of the package with one fused-GEMM source edited
    fake_root = tmp_path / "root"
    shutil.copytree(os.path.join(ROOT, "bit_nf4_quantized_dq_b200", "csrc"),
                    fake_root / "bit_nf4_quantized_dq_b200" / "csrc")
    with open(fake_root / "bit_nf4_quantized_dq_b200" / "csrc" / "gemm.cuh", "a") as f:
        f.write("\n// edited\n")
    monkeypatch.setattr(bench, "ROOT", str(fake_root))
    assert bench.fused_traffic("dx") is None
    assert bench.fused_traffic("fwd") is None


@pytest.mark.parametrize("name", ["gemm.cuh", "gemm.h", "common.cuh", "nf4_device.cuh", "qlora_nf4.cu"])
def test_every_fused_source_exists(name):
    assert name in bench.FUSED_SOURCES
    assert os.path.exists(os.path.join(ROOT, "bit_nf4_quantized_dq_b200", "csrc", name))


def test_peak_follows_the_clock_record():
    peaks = {"bf16_tflops": 1659.6, "bf16_tflops_sustained": 1382.4, "hbm_gbs": 6552.6}
    assert bench.pick_bf16_peak(peaks, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}) == (1659.6, "burst")
    assert bench.pick_bf16_peak(peaks, {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0}) == (1659.6, "burst")
    assert bench.pick_bf16_peak(peaks, {"sm_mhz": 1327.0, "sm_max_mhz": 1965.0}) == (1382.4, "sustained")
    assert bench.pick_bf16_peak(peaks, {"sm_mhz": None, "sm_max_mhz": None}) == (1659.6, "burst")


def test_world_size_must_match_gpus():
    import argparse
    args = argparse.Namespace(gpus=8)
    with pytest.raises(SystemExit):
        bench.check_world(args, {"WORLD_SIZE": "1"})
    assert bench.check_world(argparse.Namespace(gpus=2), {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"}) \
        == (1, 2, 1)
    assert bench.check_world(argparse.Namespace(gpus=1), {}) == (0, 1, 0)


def test_launcher_command_starts_n_ranks_on_loopback():
    import argparse
    cmd = bench.launcher_command(argparse.Namespace(gpus=4), ["--gpus", "4", "--steps", "2"])
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "2"] and cmd[-5].endswith("bench.py")


def _orchestration_worker(rank, world, port, out_path):
    import time
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sys.path.insert(0, ROOT)
        import bench as b
        from bit_nf4_quantized_dq_b200.dp import allreduce_adapter_grads
        dA = torch.zeros(4, 6, dtype=torch.bfloat16)
        dB = torch.zeros(5, 4, dtype=torch.bfloat16)
        calls = []

        def step(k):
            # stands in for the GPU step: this rank's partial gradients, then the exchange
            dA.fill_(rank + 1)
            dB.fill_(2 * (rank + 1))
            allreduce_adapter_grads([dA, dB])
            calls.append(k)
            if rank == 1:
                time.sleep(0.05)

        class WallTimer:
            def start(self):
                self.t = time.perf_counter()

            def stop(self):
                self.e = time.perf_counter()

            def elapsed_ms(self):
                return (self.e - self.t) * 1e3

        ms = b.timed_region(step, 3, 2, dist, lambda: None, WallTimer(), b.make_reduce_max(dist, "cpu"))
        ok = calls == [None, None, 0, 1, 2]
        ok = ok and bool(torch.all(dA.float() == 3)) and bool(torch.all(dB.float() == 6))
        ok = ok and ms >= 150.0          # the slow rank's time is the one reported, on every rank
        res = torch.tensor([ms], dtype=torch.float64)
        gathered = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, res)
        ok = ok and gathered[0].item() == gathered[1].item()
        with open(f"{out_path}.{rank}", "w") as f:
            f.write("ok" if ok else f"bad {calls} {ms}")
    finally:
        dist.destroy_process_group()


def test_timed_region_two_gloo_ranks(tmp_path):
    import socket
    import torch.multiprocessing as mp
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    out = str(tmp_path / "res")
    mp.start_processes(_orchestration_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
    assert open(out + ".0").read() == "ok" and open(out + ".1").read() == "ok"
