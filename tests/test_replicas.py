"""Multi-process replicas on CPU (gloo, two ranks): the benchmark's max-over-ranks
timing and whole-job throughput, and the reference arm printing on rank 0 only.
The path has no exchange step: ranks are independent replicas."""
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


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [1.5, 2.5][rank]  # rank 1 is the slow one
        dist.barrier()
        ms = bench.max_over_ranks_of(local_ms, dist, "cpu")
        value = bench.replica_throughput(100.0, ms, world)
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, value in got:
        assert ms == 2.5                      # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 100.0 / 2.5e-3)  # both ranks' units over that time


def test_single_process_has_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks_of(3.0) == 3.0
    assert bench.replica_throughput(10.0, 2.0, 1) == pytest.approx(5000.0)


def test_reference_arm_prints_on_rank0_only():
    """Under torchrun only rank 0 runs the oracle sample; other ranks exit 0 at once."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr
    assert res.stdout.strip() == ""


def test_profiled_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    """The roofline's `traffic` comes from a committed ncu summary only while the kernel source
    still has the sha256 recorded beside it; an edited source (or a summary without the fields)
    gives None rather than stale counters."""
    import hashlib
    sys.path.insert(0, ROOT)
    import bench
    (tmp_path / "profiles").mkdir()
    csrc = tmp_path / "latent_kv_attention_down_b200" / "csrc"
    csrc.mkdir(parents=True)
    src = csrc / "k.cu"
    src.write_text("kernel body\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles" / "k.md").write_text(f"source_sha256: {sha}\n| dram_bytes_per_launch: 42190592 | r+w |\n")
    (tmp_path / "profiles" / "bare.md").write_text("no fields here\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("k.cu", "k.md") == 42190592.0
    assert bench.profiled_traffic("k.cu", "bare.md") is None
    assert bench.profiled_traffic("missing.cu", "k.md") is None
    src.write_text("kernel body, edited\n")
    assert bench.profiled_traffic("k.cu", "k.md") is None
