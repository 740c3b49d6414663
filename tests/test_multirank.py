"""bench.py's multi-process path on two CPU ranks (gloo), launched the way the driver
launches the GPU bench: torchrun, one process per rank, rendezvous on 127.0.0.1."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_timing_and_replicas():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "tests", "multirank_worker.py")]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout                  # rank 0 alone prints (rank 1 also ran the reference arm)
    out = json.loads(lines[0])
    assert out["world"] == 2
    assert out["max_ms"] == 125.0                     # the slowest rank's time on every rank
    assert out["distinct"]                            # replicas draw different inputs
    assert abs(out["value"] - 8192 * 2 / 0.125) < 1e-6


def test_reference_arm_other_ranks_do_no_work(capsys):
    """bench.py --impl reference under torchrun: a rank other than 0 returns at once."""
    sys.path.insert(0, ROOT)
    import bench

    class A:
        steps, warmup, ref_tokens, gpus = 1, 0, 1, 2
    bench.run_reference(A, 2, 1)
    assert capsys.readouterr().out == ""
