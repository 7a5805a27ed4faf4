"""bench.py's N > 1 path on CPU: two processes over gloo, launched the way the benchmark is
(torch.distributed.run, rendezvous on 127.0.0.1)."""
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


def _torchrun(args, timeout=300):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port())] + args
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=timeout)


def _json_lines(text):
    return [json.loads(line) for line in text.splitlines() if line.startswith("{")]


def test_max_over_ranks_and_token_batches_on_two_gloo_ranks(tmp_path):
    r = _torchrun([os.path.join("tests", "multirank_worker.py"), str(tmp_path)])
    assert r.returncode == 0, r.stderr[-3000:]
    lines = []
    for rank in range(2):
        with open(tmp_path / f"rank{rank}.json") as f:
            lines.append(json.load(f))
    assert [d["rank"] for d in lines] == [0, 1]
    for d in lines:
        assert d["backend"] == "gloo"
        assert d["step_max"] == 20.0          # the slower rank's time, on every rank
        assert d["e2e_max"] == 0.0
    assert lines[0]["seed"] != lines[1]["seed"]   # replicas time distinct token batches


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    r = _torchrun(["bench.py", "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "1",
                   "--warmup", "1"])
    assert r.returncode == 0, r.stderr[-3000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
