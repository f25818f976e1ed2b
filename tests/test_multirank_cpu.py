"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the
max-over-ranks reduction of device times, the whole-job rate, and the
reference arm under torch.distributed.run (rank 0 alone prints one line)."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _torchrun(nproc, args, timeout=240):
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", OMP_NUM_THREADS="1", CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(nproc),
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port())] + args
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=timeout)


def test_job_rate_single_rank():
    assert bench.max_over_ranks([3.0, 4.5], 1) == [3.0, 4.5]
    assert bench.job_rate(100, 1, 50.0) == pytest.approx(2000.0)
    # weak scaling: N ranks with the same per-rank time give N times the rate
    assert bench.job_rate(100, 4, 50.0) == pytest.approx(8000.0)


def test_max_over_ranks_gloo_world2(tmp_path):
    r = _torchrun(2, [os.path.join("tests", "mr_worker.py"), str(tmp_path)])
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    res = [json.load(open(tmp_path / ("rank%d.json" % i))) for i in range(2)]
    for x in res:
        assert x["world"] == 2
        # the slowest rank's time, on every rank
        assert x["ms"] == pytest.approx(125.0)
        assert x["e2e"] == pytest.approx(7.0)
        # 50 steps on each of 2 ranks over the slowest rank's 125 ms
        assert x["rate"] == pytest.approx(100 / 0.125)
    assert res[0]["mine"] != res[1]["mine"]


def test_reference_arm_world2_rank0_only():
    r = _torchrun(2, ["bench.py", "--impl", "reference", "--workload", "tiny", "--gpus", "2",
                      "--steps", "2", "--warmup", "1"])
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["n_gpus"] == 2
    assert line["unit"] == "steps/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_parallel_cpu_baseline_uses_several_cores():
    """bench.py's all-cores oracle baseline (spawn-started workers, one pair
    each, timed together) on a tiny workload."""
    wl = dict(bench.WORKLOADS["tiny"], batch=2, H=2)
    r = bench.cpu_baseline_parallel(wl, 0, queries=2, max_workers=2)
    assert r["kind"] == "oracle" and r["unit"] == "steps/s"
    assert r["cores"] == min(2, os.cpu_count() or 1)
    assert r["value"] > 0
