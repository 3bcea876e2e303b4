"""Host-side logic of bench.py without a GPU: the reference arm's JSON line,
and the multi-rank path (per-rank shards, max-over-ranks step time,
whole-job throughput) on two gloo ranks on the CPU."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from camera_bev_view_b200 import inputs as I  # noqa: E402


def test_reference_arm_prints_the_contract_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "1", "--workload", "tiny"], capture_output=True, text=True, env=env,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "elements/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 2 and line["warmup"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--workload", "tiny"], capture_output=True, text=True, env=env,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_whole_job_rate():
    assert bench.whole_job_rate(1000, 1, 1.0) == pytest.approx(1e6)
    assert bench.whole_job_rate(1000, 4, 2.0) == pytest.approx(2e6)
    assert bench.max_over_ranks(3.5, 1) == 3.5


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = I.WORKLOADS["tiny"]
        F = I.make_features(w, shard=rank)
        K, E = I.make_rigs(w, shard=rank)
        # a stand-in per-rank step time; the slowest rank sets the job's step time
        ms_local = 1.0 + rank
        ms = bench.max_over_ranks(ms_local, world)
        rate = bench.whole_job_rate(w.out_elems, world, ms)
        sums = torch.tensor([float(F.double().sum()), float(E.double().sum())], dtype=torch.float64)
        gathered = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, sums)
        if rank == 0:
            json.dump({"ms": ms, "rate": rate, "sums": [g.tolist() for g in gathered]},
                      open(os.path.join(outdir, "result.json"), "w"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_aggregate(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    res = json.load(open(tmp_path / "result.json"))
    w = I.WORKLOADS["tiny"]
    assert res["ms"] == 2.0                                  # max over ranks
    assert res["rate"] == pytest.approx(2 * w.out_elems / 2e-3)
    s0, s1 = res["sums"]
    assert not np.allclose(s0, s1)                           # each rank transforms its own batch


def test_recorded_traffic_names_known_kernels_and_sources():
    """Every kernel in the committed traffic table maps to source files that
    exist, so a stale entry is detected by its digest rather than by a crash;
    entries whose digest matches the sources are returned, others are not."""
    table = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for kernel, per_workload in table.items():
        assert kernel in bench.KERNEL_SOURCES, kernel
        for f in bench.KERNEL_SOURCES[kernel]:
            assert os.path.exists(os.path.join(ROOT, "camera_bev_view_b200", "csrc", f)), f
        for workload, entry in per_workload.items():
            got = bench.recorded_traffic(kernel, workload)
            if entry.get("source_digest") == bench.source_digest(kernel):
                assert got == float(entry["dram_bytes_per_launch"]) and got > 0
            else:
                assert got is None


@pytest.mark.parametrize("op,workload", [("ms", "ms_tiny"), ("deform", "deform_tiny"), ("lss", "lss_tiny")])
def test_reference_arm_of_the_further_operators(op, workload):
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--op", op, "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--workload", workload], capture_output=True, text=True,
                       env=env, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
