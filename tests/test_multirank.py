"""The benchmark's multi-rank host logic on CPU: two gloo ranks under torchrun.

The hot path shards into independent replicas (no data-path collective), so what
needs checking with more than one rank is the host side: rank setup, the
max-over-ranks step time, the whole-job (weak scaling) aggregate, per-rank seeds,
and that the reference arm runs on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _torchrun(args, timeout=240):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_port())] + args
    env = dict(os.environ, OMP_NUM_THREADS="2", CUDA_VISIBLE_DEVICES="")
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=timeout)


def _json_lines(out):
    return [json.loads(x) for x in out.splitlines() if x.startswith("{")]


def test_two_gloo_ranks_share_the_slowest_time_and_own_their_batches(tmp_path):
    r = _torchrun([os.path.join("tests", "multirank_worker.py"), str(tmp_path)])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.load(open(tmp_path / ("rank%d.json" % i))) for i in range(2)]
    assert [j["rank"] for j in lines] == [0, 1]
    for j in lines:
        assert j["ws"] == 2
        assert j["tmax"] == 2.5                      # max of 1.5 and 2.5, on every rank
        assert j["value"] == pytest.approx(2 * 1e9 / 2.5e-3 / 1e9)
        assert j["sums"][0] != j["sums"][1]          # the replicas' inputs differ
    assert lines[0]["sums"] == lines[1]["sums"]


def test_reference_arm_prints_once_from_rank_zero():
    r = _torchrun(["bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    j = lines[0]
    assert j["impl"] == "reference" and j["n_gpus"] == 2 and j["unit"] == "GB/s" and j["value"] > 0
    assert j["cpu_baseline"]["kind"] == "oracle"
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["d2h_bytes_per_step"] == 0
