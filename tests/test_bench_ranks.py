"""Multi-process host logic of bench.py, on CPU with gloo (world size 2).

With N GPUs every rank runs an independent replica of the layer (weak scaling,
no data-path collective); the only communication is the max over ranks of the
timings, from which rank 0 reports bytes of all ranks / the slowest time.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        mine = [1.5 * rank + 1.0, 10.0 - rank, 3.0]
        got = bench.max_over_ranks(dist, mine, "cpu")
        value = bench.whole_job_gbs(4e9, world, got[1])
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"max": got, "value": value}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value(tmp_path):
    import socket

    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(2)]
    for r in res:
        assert r["max"] == [2.5, 10.0, 3.0]
        # 2 ranks x 4 GB each over the slowest rank's 10 ms
        assert r["value"] == pytest.approx(8e9 / 10e-3 / 1e9)


def test_single_process_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(None, [1.0, 2.0], "cpu") == [1.0, 2.0]
    assert bench.whole_job_gbs(6.5e9, 1, 1.0) == pytest.approx(6500.0)
    b = bench.algorithmic_bytes(8, 4096, 8, 7168)
    assert b["dispatch"] == 4228907008 and b["combine"] == 4229955584
    # captured DRAM traffic belongs to one workload: never reported for another
    assert bench.ncu_traffic("ep8_e32_k4_s256_h512", 0.2, 0) == {}
    assert bench.ncu_traffic("ep8_e256_k8_s4096_h7168", 20.0, 0) == {}
    assert bench.ncu_traffic("ep8_e256_k8_s4096_h7168", 0.2, 1) == {}


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_runs_on_rank_zero_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "ep8_e32_k4_s256_h512", "--steps", "3", "--warmup", "1",
                        "--reference-budget-s", "5"], capture_output=True, text=True, env=env,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    if rank == 0:
        assert len(lines) == 1
        d = json.loads(lines[0])
        assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
        assert d["cpu_baseline"]["kind"] == "oracle" and d["n_gpus"] == 2
        assert d["e2e"]["h2d_bytes_per_step"] == 0
    else:
        assert lines == []


def test_oracle_baseline_threads_cover_the_same_work():
    """The threaded CPU baseline splits each step over disjoint tokens or experts: every
    thread count must leave exactly the single-threaded results behind."""
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    from moonep_inputs import WORKLOADS
    w = WORKLOADS["ep8_e32_k4_s256_h512"]
    res = {}
    for n in (1, 3, 8):
        smp = bench.OracleSample(w, 5.0, 0, s=40, p=4096)
        assert smp.n_local > 0
        ks = smp.kernels()
        for name in ("dispatch", "reduce_grad", "prefetch"):
            ks[name](n)
        res[n] = (smp.recv.copy(), smp.home.copy(), smp.rep_w.copy())
    for n in (3, 8):
        for a, b in zip(res[1], res[n]):
            assert np.array_equal(a, b)
    smp = bench.OracleSample(w, 5.0, 0, s=40, p=4096)
    ks = smp.kernels()
    for name in ("combine", "combine_bwd", "dispatch_bwd"):
        ks[name](4)  # runs over every token without error


def test_reference_line_carries_the_gpu_arm_config():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "ep8_e32_k4_s256_h512", "--steps", "2", "--warmup", "1",
                        "--reference-budget-s", "5"], capture_output=True, text=True, env=env,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    sys.path.insert(0, ROOT)
    import bench
    from moonep_inputs import WORKLOADS, make_routing
    w = WORKLOADS["ep8_e32_k4_s256_h512"]
    _, alpha, mv = make_routing(w.R, w.E, w.K, w.S, w.maxvio[0], 0)
    assert d["config"] == bench.workload_config(w, mv, alpha, 1)
    assert d["cpu_baseline"]["cores"] == bench.host_cores()


def test_profiles_name_the_current_sources():
    """Every ncu summary under profiles/ states the sha256 (16 hex digits) of the sources
    it was captured on; each stated hash is that of the file as it is now."""
    import glob
    import hashlib
    import re
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    csrc = os.path.join(root, "token_dispatch_moonep_b200", "csrc")
    now = {f: hashlib.sha256(open(os.path.join(csrc, f), "rb").read()).hexdigest()[:16]
           for f in os.listdir(csrc) if f.endswith((".cu", ".cuh"))}
    files = sorted(glob.glob(os.path.join(root, "profiles", "*.md")))
    assert files
    for path in files:
        text = open(path).read()
        stated = re.findall(r"`csrc/([\w.]+)` ([0-9a-f]{16})", text)
        assert stated, f"{os.path.basename(path)} names no source hash"
        for name, h in stated:
            assert now.get(name) == h, f"{os.path.basename(path)}: {name} is {now.get(name)}, not {h}"
    for ln in open(os.path.join(root, "profiles", "ncu_traffic.txt")):
        if ln.startswith("#") or not ln.strip():
            continue
        parts = dict(kv.split("=", 1) for kv in ln.split())
        assert now[parts["source"]] == parts["sha"]
        assert now["moonep_internal.cuh"] == parts["header_sha"]
    # bench.py's own reader finds a current line for each of the step's seven kernels,
    # so the headline run's roofline carries the measured traffic
    import bench
    got = bench.ncu_traffic(bench.DEFAULT_WORKLOAD, 0.2, 0)
    assert set(got) == {"plan", "prefetch", "dispatch", "combine", "combine_bwd", "dispatch_bwd",
                        "reduce_grad"}, sorted(got)
    assert all(v > 0 for v in got.values())
