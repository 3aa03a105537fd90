"""Host logic of bench.py: the algorithmic FLOP/byte counts and the
multi-rank plumbing (max over ranks, adapter-gradient averaging), the latter
run as two gloo ranks on the CPU."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from bit_nf4_quantized_qlora_b200 import workloads as WL


def test_flop_counts_of_the_7b_mlp():
    f = bench.linear_flops(4096, 11008, 4096, 64)
    assert f["fwd"] == 2 * 4096 * 11008 * 4096 + 2 * 4096 * 64 * (11008 + 4096)
    assert abs(f["fwd"] / 1e9 - 377.3) < 0.1           # forward of one 11008x4096 projection
    assert f["fwd"] == f["bwd_dx"]
    assert f["fused_fwd_kernel"] == 2 * 4096 * 11008 * (4096 + 64)
    cases = [WL.mlp_7b(p) for p in bench.PROJECTIONS]
    assert bench.step_flops(cases) == sum(bench.linear_flops(c.m, c.n, c.k, c.r)["total"] for c in cases)


def test_weight_bytes_match_the_format():
    assert bench.weight_bytes(4096, 4096) == 8388608 + 262144 + 4 * 1024
    assert abs(bench.weight_bytes(28672, 8192) / 1e6 - 121.2) < 0.5


def test_peaks_file_or_fallback():
    peaks, kind = bench.load_peaks()
    assert kind in ("measured", "fallback")
    assert peaks["hbm_gbs"] > 1000 and peaks["bf16_tflops_sustained"] > 100


def test_profile_traffic_requires_matching_source(tmp_path, monkeypatch):
    p = tmp_path / "summary.txt"
    p.write_text("kernel_source_sha256: abc\ntraffic_bytes_per_launch: 123.0\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(p))
    assert bench.profile_traffic("abc") == 123.0
    assert bench.profile_traffic("other") is None


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.reduce_max(1.5 * (rank + 1), world)
        flat = torch.full((12,), float(rank + 1), dtype=torch.float32)
        bench.allreduce_grads(flat, world)
        cases = [WL.LinearCase("c", n=16, k=64, m=4, r=16, alpha=32.0)]
        buf, views = bench._grad_buffer(cases, "cpu")
        a, b = views[0]
        a.fill_(rank + 1)
        b.fill_(2 * (rank + 1))
        buf32 = buf.float()
        bench.allreduce_grads(buf32, world)
        out[rank] = (t, flat.tolist(), float(buf32[:a.numel()].mean()), float(buf32[a.numel():].mean()),
                     buf.numel())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_gradient_average():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    for rank in range(world):
        t, flat, ma, mb, numel = out[rank]
        assert t == 3.0                                   # max over ranks
        assert flat == [1.5] * 12                         # average of 1 and 2
        assert ma == pytest.approx(1.5) and mb == pytest.approx(3.0)
        assert numel == 16 * 64 + 16 * 16


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the CPU oracle, rank 0) prints one JSON
    line carrying the contract's keys, its own cpu_baseline and an e2e entry
    with zero host-device bytes."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=300, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1 and d["vs_baseline"] is None
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"]
