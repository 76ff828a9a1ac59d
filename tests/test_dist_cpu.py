"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the barrier,
max-over-ranks timing and the weak-scaling throughput. No GPU."""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist = bench.dist_init("gloo", timeout_s=60)
    bench.barrier()
    mx = bench.max_over_ranks(10.0 * (rank + 1))
    sm = bench.sum_over_ranks(rank + 1)
    # rank r ran 1000 steps of 6 units in (r+1) * 100 ms: the job is as slow as rank 1
    value, ms = bench.throughput(6, 1000, 100.0 * (rank + 1))
    q.put((rank, mx, sm, value, ms))
    dist.destroy_process_group()


def test_two_rank_timing_and_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, mx, sm, value, ms in res:
        assert mx == 20.0
        assert sm == 3.0
        assert ms == 200.0
        assert value == pytest.approx(6 * 1000 * 2 / 0.2)


def test_single_process_helpers_without_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    value, ms = bench.throughput(10, 5, 50.0)
    assert ms == 50.0 and value == pytest.approx(1000.0)


def _run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True,
                          text=True, timeout=600, env=env, cwd=ROOT)


def test_reference_arm_runs_the_oracle_on_cpu():
    r = _run_bench(["--impl", "reference", "--workload", "small", "--steps", "3", "--warmup", "3",
                    "--reference-seconds", "1"])
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["unit"] == "channel-steps/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench(["--impl", "reference", "--workload", "small", "--steps", "3"],
                   {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_recorded_traffic_follows_the_sources(tmp_path, monkeypatch):
    """A profile's traffic line counts only while the kernels and their launch
    code hash to the digest it names; the XU figure is optional."""
    sys.path.insert(0, ROOT)
    import bench
    csrc = tmp_path / "wkv_recurrence_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cuh").write_text("kernel one")
    (csrc / "api.cu").write_text("launch one")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d = bench.source_digest()
    (tmp_path / "profiles" / "a.md").write_text(
        f"traffic: kernel=kx workload=layer source={d} bytes_per_launch=123 xu_pct=21.5\n"
        f"traffic: kernel=ky workload=layer source={d} bytes_per_launch=456\n"
        "traffic: kernel=kz workload=layer source=0000000000000000 bytes_per_launch=789\n")
    assert bench.recorded_traffic("kx", "layer") == (123, 21.5)
    assert bench.recorded_traffic("ky", "layer") == (456, None)
    assert bench.recorded_traffic("kz", "layer") == (None, None)  # another build's capture
    assert bench.recorded_traffic("kx", "long") == (None, None)
    (csrc / "api.cu").write_text("launch two")  # launch code changed: the capture no longer counts
    assert bench.source_digest() != d
    assert bench.recorded_traffic("kx", "layer") == (None, None)
