"""Host-side logic of bench.py on the CPU: the max-over-ranks timing
reduction with two gloo ranks, and the reference (oracle) arm's JSON line."""

import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from exact_io_aware_56_b200 import DECODE_WORKLOADS, FP8_WORKLOADS, WORKLOADS, DecodeWorkload, Workload  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, w = bench.init_dist("gloo")
    bench.barrier()
    got = bench.max_over_ranks(10.0 * (r + 1))
    bench.barrier()
    import torch.distributed as dist

    dist.destroy_process_group()
    q.put((r, w, got))


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, 2, 20.0), (1, 2, 20.0)]


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5


def test_reference_arm_json(monkeypatch, capsys):
    tiny = Workload("tiny_ref", 1, 2, 1, 64, 64, True, True, seed=3)
    monkeypatch.setitem(WORKLOADS, "tiny_ref", tiny)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.main(["--impl", "reference", "--workload", "tiny_ref", "--steps", "2", "--warmup", "1"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["config"]["workload"] == "tiny_ref"


def test_decode_reference_arm_json(monkeypatch, capsys):
    tiny = DecodeWorkload("decode_tiny_ref", 2, 4, 2, 1, 300, 64, seed=5)
    monkeypatch.setitem(DECODE_WORKLOADS, "decode_tiny_ref", tiny)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.main(["--impl", "reference", "--workload", "decode_tiny_ref", "--steps", "2", "--warmup", "1"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["metric"] == bench.DECODE_METRIC and line["config"]["Nk"] == 300
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["d2h_bytes_per_step"] == 0


def test_fp8_reference_arm_json(monkeypatch, capsys):
    tiny = Workload("fwd_fp8_tiny", 1, 2, 1, 256, 128, True, False, seed=4)
    monkeypatch.setitem(FP8_WORKLOADS, "fwd_fp8_tiny", tiny)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.main(["--impl", "reference", "--workload", "fwd_fp8_tiny", "--steps", "1", "--warmup", "1"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.FP8_METRIC and line["value"] > 0


def test_decode_workload_bytes():
    w = DECODE_WORKLOADS["decode_b16_hq32_hkv8_nq1_nk8192_d128"]
    kv = 2 * 16 * 8 * 8192 * 128 * 2
    assert w.bytes_moved() == kv + 2 * 16 * 32 * 1 * 128 * 2 + 4 * 16 * 32
    assert w.flops() == 4.0 * 16 * 32 * 1 * 8192 * 128


def test_reference_arm_other_ranks_exit_quietly(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"]) == 0
    assert capsys.readouterr().out == ""


def test_workload_flops():
    w = WORKLOADS["fwdbwd_b2_h16_n8192_d128_causal_peaky"]
    assert w.fwd_flops() == pytest.approx(549.755813888e9)
    assert w.bwd_flops() == pytest.approx(2.5 * 549.755813888e9)
    assert WORKLOADS["fwd_b1_h1_n128_d64"].fwd_flops() == 4 * 128 * 128 * 64


def test_captured_traffic_requires_unchanged_sources(tmp_path, monkeypatch):
    import hashlib

    csrc = tmp_path / "exact_io_aware_56_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_bytes(b"kernel source v1")
    digest = hashlib.sha256(b"kernel source v1").hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"captures": [{"kernel": "kern", "workload": "wl", "sources": ["k.cu"], "sha256_16": digest,
                       "traffic_bytes": 12345}]}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.captured_traffic("kern", "wl") == 12345
    assert bench.captured_traffic("kern", "other") is None
    (csrc / "k.cu").write_bytes(b"kernel source v2")
    assert bench.captured_traffic("kern", "wl") is None


def test_clock_summary_keeps_only_the_timed_window():
    c = bench.ClockSampler(None)
    c.samples = [(0.0, 1200.0, 1965.0, set()), (1.0, 1965.0, 1965.0, {"sw_power_cap"}),
                 (1.5, 1900.0, 1965.0, set()), (3.0, 800.0, 1965.0, {"hw_slowdown"})]
    c.t_begin, c.t_end = 0.9, 2.0
    sm = c.summary()
    assert sm["samples"] == 2 and sm["sm_mhz"] == (1965.0 + 1900.0) / 2
    assert sm["reasons"] == ["sw_power_cap"] and sm["sm_max_mhz"] == 1965.0
    c.t_begin, c.t_end = 2.1, 2.2  # shorter than the polling period: nearest sample to its middle
    assert c.summary()["samples"] == 1 and c.summary()["sm_mhz"] == 1900.0


def test_peak_value_measured_fallback_and_malformed(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.peak_value("bf16_tflops") == (bench.FALLBACK_PEAKS["bf16_tflops"], "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6431.7, "bf16_tflops": 1656.9}))
    assert bench.peak_value("bf16_tflops") == (1656.9, "measured")
    assert bench.peak_value("hbm_gbs") == (6431.7, "measured")
    # A key the file lacks, or holds as something other than a positive
    # number, takes the fallback figure and says so.
    assert bench.peak_value("bf16_tflops_sustained") == (bench.FALLBACK_PEAKS["bf16_tflops_sustained"],
                                                         "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"bf16_tflops": {"burst": 1656.9}, "hbm_gbs": -1}))
    assert bench.peak_value("bf16_tflops")[1] == "fallback" and bench.peak_value("hbm_gbs")[1] == "fallback"
    (tmp_path / "MEASURED_PEAKS.json").write_text("[1, 2]")
    assert bench.peak_value("hbm_gbs") == (bench.FALLBACK_PEAKS["hbm_gbs"], "fallback")
