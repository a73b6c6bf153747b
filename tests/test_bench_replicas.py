"""Multi-process host logic of bench.py (replicas, no data-path collective), on CPU with gloo.

The decode path runs on one GPU; with N > 1 every rank is an independent replica and
the only collectives are the timing barrier and the max over ranks of the per-rank
time.  These tests cover that plumbing with world size 2 on the gloo backend.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        got = bench.max_over_ranks(10.0 * (rank + 1) + 0.25, world)
        out.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(world))
    assert res == {0: 20.25, 1: 20.25}


def test_reference_arm_under_torchrun():
    """--impl reference with 2 ranks: rank 0 alone runs the oracle and prints one line; the other exits 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny4k_fp32"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["n_gpus"] == 2
    assert line["higher_is_better"] is False
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


if __name__ == "__main__":
    pytest.main([__file__, "-q"])


def test_sweep_crossover():
    """The crossover is interpolated in log N between the bracketing sweep points."""
    import math
    sys.path.insert(0, ROOT)
    import bench
    pts = [(32768, 150.0, 34.0), (262144, 200.0, 105.0), (524288, 140.0, 190.0), (1048576, 220.0, 350.0)]
    x = bench.crossover(pts)
    g0, g1 = 105.0 - 200.0, 190.0 - 140.0
    want = math.exp(math.log(262144) + (math.log(524288) - math.log(262144)) * (-g0) / (g1 - g0))
    assert x == int(round(want)) and 262144 < x < 524288
    assert bench.crossover([(1024, 1.0, 2.0), (2048, 1.0, 3.0)]) == "<= 1024"
    assert bench.crossover([(1024, 3.0, 2.0), (2048, 4.0, 3.0)]) is None


def test_union_bytes_counts_each_group_once():
    """Algorithmic bytes: planes scored and keys attended are counted once per (sequence, KV group)."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    from synth.workloads import Workload
    w = Workload("t", d=64, n_q_heads=4, n_kv_heads=2, n_tokens=1000, block=4, levels=2, n_refs=2, p=0.9,
                 batch=1, dtype="bf16", gen="topics", seed=0)
    # heads 0,1 share KV head 0; 2,3 share KV head 1
    scored = np.array([[[5, 6, 7, 0], [6, 7, 8, 0], [1, 0, 0, 0], [2, 0, 0, 0]]], dtype=np.int32)
    nscored = np.array([[3, 3, 1, 1]])
    kept = np.array([[[0, 3, 0], [3, 4, 0], [9, 0, 0], [9, 0, 0]]], dtype=np.int32)
    kcnt = np.array([[2, 2, 1, 1]])
    route, attend, kph = bench.union_bytes(w, scored, nscored, kept, kcnt, 1002)
    plane = 2 * (64 * 2 + 4)
    assert route == (4 + 2) * plane                       # {5,6,7,8} and {1,2}
    kv = 2 * 64 * 2
    tail = 1002 - 250 * 4                                 # 2 tail tokens
    # group 0: leaves {0,3,4} (block 0 kept: no extra sink); group 1: {9} + sink
    assert attend == (3 * 4 + tail) * kv + (1 * 4 + tail + 1) * kv + 1 * 4 * 64 * (2 + 4)
    assert kph == [2 * 4 + tail, 2 * 4 + tail + 1, 4 + tail + 1, 4 + tail + 1]
    w4 = Workload("t4", d=64, n_q_heads=4, n_kv_heads=2, n_tokens=1000, block=4, levels=2, n_refs=2, p=0.9,
                  batch=1, dtype="bf16", gen="topics", seed=0, planes="fp4")
    route4, _, _ = bench.union_bytes(w4, scored, nscored, kept, kcnt, 1002)
    assert route4 == (4 + 2) * 2 * (32 + 4 + 4)


def test_traffic_figure_only_for_the_measured_kernels(tmp_path, monkeypatch):
    """roofline.traffic is read from the ncu summary only while its workload and source hash match."""
    sys.path.insert(0, ROOT)
    import bench
    f = tmp_path / "traffic.txt"
    f.write_text(f"# comment: x\nworkload: deep256k_bf16\nsource_hash: {bench.kernel_source_hash()}\n"
                 "dram_bytes_per_decode: 123456\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.measured_traffic("deep256k_bf16") == 123456
    assert bench.measured_traffic("wide256k_bf16") is None
    f.write_text("workload: deep256k_bf16\nsource_hash: 0000000000000000\ndram_bytes_per_decode: 123456\n")
    assert bench.measured_traffic("deep256k_bf16") is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.txt"))
    assert bench.measured_traffic("deep256k_bf16") is None
