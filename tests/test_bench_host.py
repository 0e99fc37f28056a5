"""Host-side logic of bench.py, including the multi-rank path on CPU (gloo, 2 ranks)."""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_aggregate_is_total_work_over_slowest_rank():
    assert bench.aggregate(2e12, 0.5, 1) == pytest.approx(4.0)
    assert bench.aggregate(2e12, 0.5, 8) == pytest.approx(32.0)


def test_parse_defaults():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.workload == "wan14b_720p" and a.impl == "mcs"
    # the default line carries e2e through the pipelined host call, the fast grouping and the grouping effect
    assert not a.no_e2e and a.e2e_chunks == 20 and a.fast_krylov == 8 and a.grouping_effect
    # ... and the other workloads' group/anchor/reuse/dense timings
    assert a.per_workload
    assert [n for n, _ in bench.PER_WORKLOAD_CASES] == ["tiny", "wan13b_480p", "h3_768p", "h3_768p", "asset3d"]
    b = bench.parse_args(["--fast-krylov", "0", "--no-grouping-effect", "--e2e-chunks", "4", "--no-per-workload"])
    assert b.fast_krylov == 0 and not b.grouping_effect and b.e2e_chunks == 4 and not b.per_workload


def test_profiled_traffic_stale_hash_reads_null(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "k.md").write_text(
        "kernel: attn_reuse\nworkload: x\nsource_sha: abc\ndram_bytes_per_launch: 123\n")
    assert bench.profiled_traffic("attn_reuse", "abc") == 123.0
    assert bench.profiled_traffic("attn_reuse", "def") is None
    assert bench.profiled_traffic("other", "abc") is None


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


WORKER = r"""
import os, sys, datetime
sys.path.insert(0, {root!r})
import torch.distributed as dist
import bench
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
r = dist.get_rank()
t = bench.reduce_max([1.0 + r, 10.0 - r], dist.get_world_size())
v = bench.aggregate(1e12, t[0] / 1e3, dist.get_world_size())
print("RESULT", r, t, v, flush=True)
dist.destroy_process_group()
"""


def test_reduce_max_over_two_gloo_ranks(tmp_path):
    script = tmp_path / "w.py"
    script.write_text(WORKER.format(root=ROOT))
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE="2", LOCAL_RANK=str(r), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT, text=True))
    outs = [p.communicate(timeout=120)[0] for p in procs]
    assert all(p.returncode == 0 for p in procs), outs
    for out in outs:
        line = [ln for ln in out.splitlines() if ln.startswith("RESULT")][0]
        # max over ranks of [1 + r, 10 - r] is [2, 10]; value = 2 ranks x 1 TFLOP / 2 ms
        assert "[2.0, 10.0]" in line and line.endswith(" 1000.0")


def test_reference_arm_nonzero_rank_exits_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference"]) == 0
    assert capsys.readouterr().out == ""
