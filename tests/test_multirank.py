"""The N > 1 host logic of bench.py, on the CPU with two ranks (torchrun,
gloo): the job's time is the max over ranks and its work the sum, every rank
agrees on both; the reference arm prints one line from rank 0 only."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _torchrun(args, timeout):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port())] + args
    env = dict(os.environ, OMP_NUM_THREADS="2", CUDA_VISIBLE_DEVICES="")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=timeout)
    assert r.returncode == 0, r.stderr[-2000:]
    return [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]


def test_aggregate_ranks_two_gloo_ranks():
    lines = _torchrun([os.path.join("tests", "_rank_worker.py")], timeout=180)
    assert len(lines) == 1
    d = lines[0]
    assert d["world"] == 2
    # max of 10 and 15 ms; 1000 + 2000 bytes; the same answer on both ranks
    assert d["per_rank"] == [[15.0, 3000.0], [15.0, 3000.0]]


def test_aggregate_ranks_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate_ranks(12.5, 4096, 1, "cpu") == (12.5, 4096.0)


def test_reference_arm_prints_once_under_two_ranks():
    lines = _torchrun(["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"], timeout=600)
    assert len(lines) == 1, lines
    d = lines[0]
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
