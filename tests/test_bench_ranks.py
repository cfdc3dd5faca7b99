"""The benchmark's multi-rank path on two CPU ranks (gloo): each rank its own
seeded batch element, the job time is the slowest rank's, the value is all
ranks' work over that time; the reference arm prints on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def torchrun(args, timeout=240):
    env = dict(os.environ, PYTHONPATH=ROOT, OMP_NUM_THREADS="1", CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={free_port()}"] + args
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=timeout)
    assert p.returncode == 0, p.stdout[-2000:] + p.stderr[-4000:]
    return [json.loads(x) for x in p.stdout.splitlines() if x.startswith("{")]


def test_two_rank_seeding_max_and_aggregate():
    lines = sorted(torchrun([os.path.join(ROOT, "tests", "dist_bench_worker.py")]), key=lambda d: d["rank"])
    assert [d["rank"] for d in lines] == [0, 1]
    c0, c1 = lines[0]["checksums"], lines[1]["checksums"]
    assert c0 == c1 and c0[0] != c0[1]                 # same gather everywhere, different inputs per rank
    for d in lines:
        assert d["world"] == 2
        assert d["max_ms"] == 15.0                     # the slower rank's time on every rank
        assert abs(d["value"] - 2 * 2e12 * 4 / 0.015 / 1e12) < 1e-9


def test_reference_arm_prints_on_rank_zero_only():
    lines = torchrun([os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--L", "128",
                      "--ref-rows", "8", "--steps", "1", "--warmup", "0"])
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
