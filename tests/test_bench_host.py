"""Host-side logic of bench.py without a GPU: whole-job throughput of
independent replicas, max-over-ranks timing over a 2-rank gloo group, and the
CPU oracle arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_replica_value():
    # 2 ranks, 1 GB each, slowest rank 0.5 s -> 4 GB/s for the job
    assert bench.replica_value(1.0, 2, 0.5) == pytest.approx(4.0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


WORKER = r"""
import os, sys, json
sys.path.insert(0, os.environ["ROOT"])
import bench
d = bench.Dist()
d.init("gloo")
t = 0.25 if d.rank == 0 else 0.75       # per-rank elapsed seconds
m = d.max(t)
d.barrier()
if d.rank == 0:
    print(json.dumps({"max": m, "value": bench.replica_value(2.0, d.world, m)}))
d.close()
"""


def test_max_over_ranks_gloo():
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, ROOT=ROOT, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=120) for p in procs]
    assert all(p.returncode == 0 for p in procs), outs
    res = json.loads(outs[0][0].strip().splitlines()[-1])
    assert res["max"] == pytest.approx(0.75)
    assert res["value"] == pytest.approx(2.0 * 2 / 0.75)


def test_reference_arm_json(monkeypatch, capsys):
    fake = {"value": 1.5, "unit": "GB/s", "cores": 8, "kind": "oracle", "sample": "s", "cpu": "x"}
    monkeypatch.setattr(bench, "cpu_sample", lambda seconds=10.0: fake)
    bench.main(["--impl", "reference", "--steps", "2", "--warmup", "3"])
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["value"] == 1.5
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 8
    assert line["e2e"] == {"value": 1.5, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["metric"] == bench.METRIC


def test_reference_arm_other_ranks_do_no_work(monkeypatch, capsys):
    # under torchrun only rank 0 times the oracle and prints; another rank
    # returns at once, without a process group or any oracle call
    def no_call(seconds=10.0):
        raise AssertionError("rank 1 ran the oracle")
    monkeypatch.setattr(bench, "cpu_sample", no_call)
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--steps", "2", "--warmup", "3"])
    assert capsys.readouterr().out == ""


def test_cpu_sample_is_bounded():
    r = bench.cpu_sample(seconds=0.0)       # one pass of the oracle on c1
    assert r["kind"] == "oracle" and r["value"] > 0 and r["cores"] >= 1


def test_traffic_keyed_by_kernel_device_sources(tmp_path, monkeypatch):
    # the roofline's DRAM traffic is reported only while the code of the
    # profiled kernel is the one the counters were taken on; a host-only
    # launch header and comments do not count, a code change in the kernel's
    # file does
    csrc = tmp_path / "gguf_quant_dequant_q4_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("kq_qmv_stream.cu", "kq_device.cuh", "kq_launch.h"):
        (csrc / f).write_text(f"// {f}\nint v_{f.split('.')[0]} = 1;\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    tag = "qmv_q6_K_m1_14336x4096"
    h = bench.kernel_source_hash(tag)
    (tmp_path / "profiles" / "p.txt").write_text(f"summary\ntraffic {tag} 48223488 {h}\n")
    assert bench.profiled_traffic(tag) == 48223488
    (csrc / "kq_launch.h").write_text("// a new host declaration\nint launch(int);\n")
    assert bench.profiled_traffic(tag) == 48223488
    (csrc / "kq_qmv_stream.cu").write_text("/* reworded */ // comments only\nint v_kq_qmv_stream  =  1;\n")
    assert bench.profiled_traffic(tag) == 48223488
    (csrc / "kq_qmv_stream.cu").write_text("// the kernel changed\nint v_kq_qmv_stream = 2;\n")
    assert bench.profiled_traffic(tag) is None
