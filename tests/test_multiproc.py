"""Host logic of the N > 1 path on CPU: gloo ranks, no GPU.

The attention path shards into independent problems (one per rank, weak
scaling) with no collective on the data path; the only collectives are the
bench's timing reductions (max / sum over ranks), checked here with gloo.
"""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench

    r, lr, w = bench.dist_env()
    dist = bench.init_dist(w, "gloo")
    res = {
        "env": [r, lr, w],
        "max": bench.max_over_ranks(1.0 + 2.0 * rank, dist),
        "sum": bench.sum_over_ranks(1.0 + rank, dist),
        "seed": bench.rank_seed(2, rank),
    }
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump(res, f)


def test_rank_reductions_with_gloo(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for r, x in enumerate(res):
        assert x["env"] == [r, r, world]
        assert x["max"] == 3.0  # every rank sees the slowest rank's time
        assert x["sum"] == 3.0
    assert res[0]["seed"] == 2 and res[1]["seed"] != res[0]["seed"]


def test_weak_scaling_value():
    sys.path.insert(0, ROOT)
    import bench

    # 2 ranks x 10 steps x 1e12 FLOP in 4 s -> 5 TFLOP/s for the whole job
    assert bench.weak_scaling_value(1e12, 2, 10, 4.0) == pytest.approx(5.0)


def test_reference_arm_under_torchrun_prints_once():
    """Two ranks on CPU: rank 0 times the oracle and prints one line, rank 1 exits 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "b1h1n256d64", "--ref-step-seconds", "0.3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["value"] > 0 and line["unit"] == "TFLOP/s"


def test_committed_traffic_reads_the_profile_summary(tmp_path, monkeypatch):
    """The bench reports DRAM traffic from the committed ncu summary only while its
    kernel source hash matches the current sources."""
    sys.path.insert(0, ROOT)
    import bench

    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", [])  # the hash of no sources
    (prof / "fa_fwd_wl_ncu.md").write_text(
        "- kernel_source_sha256: `%s` (note)\n- dram_bytes_per_launch: 1234\n" % bench.kernel_source_hash())
    (prof / "fa_fwd_old_ncu.md").write_text(
        "- kernel_source_sha256: `0000000000000000` (note)\n- dram_bytes_per_launch: 99\n")
    assert bench.committed_traffic("wl") == 1234.0
    assert bench.committed_traffic("old") is None
    assert bench.committed_traffic("missing") is None
