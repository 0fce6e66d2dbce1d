"""Host-side logic of bench.py: closed forms, the max-over-ranks timing
reduction on two gloo ranks, and the JSON contract of the reference arm."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden", "table_bytes.txt")


def test_materialised_table_bytes_match_the_printed_values():
    units = {"GB": 1e9, "MiB": 2 ** 20}
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    assert len(rows) == 5
    for H, P, b, val, unit in rows:
        got = bench.materialised_bytes(int(H), int(P), int(b)) / units[unit]
        # the page rounds to the printed digits
        assert abs(got - float(val)) <= 0.005 * float(val), (H, P, b, got, val)


def test_flop_and_byte_counts():
    assert bench.attn_flops(1, 16, 11616, 64, False) == 4 * 16 * 11616 ** 2 * 64
    assert bench.attn_flops(8, 12, 1024, 64, True) == 2 * 8 * 12 * 1024 ** 2 * 64
    assert abs(bench.attn_flops(1, 16, 11616, 64, False) / 1e9 - 552.7) < 0.1
    assert bench.algorithmic_bytes(1, 16, 11616, 64) == 16 * 11616 * (8 * 64 + 4)
    assert bench.output_bytes(1, 16, 11616, 64) == 24532992
    # the extra-memory cap of the target: 1.1 x (O + LSE) = 26.99 MB at 3 MP
    assert abs(1.1 * bench.output_bytes(1, 16, 11616, 64) / 1e6 - 26.99) < 0.01


def test_peaks_fall_back_when_absent(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback" and p["bf16_tflops"] == 1590.0


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.0][rank]
        out[rank] = bench.reduce_max(local_ms, dist, torch.device("cpu"))
    finally:
        dist.destroy_process_group()


def test_timing_is_max_over_two_gloo_ranks():
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True)
    assert out[0] == 5.0 and out[1] == 5.0


def test_reduce_max_single_process_is_identity():
    assert bench.reduce_max(2.5) == 2.5


def test_reference_arm_prints_the_contract_line():
    env = dict(os.environ, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--cpu-budget", "1"], capture_output=True, text=True, env=env,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    for key in ("value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "config",
                "cpu_baseline", "e2e"):
        assert key in line
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["value"] > 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, PYTHONPATH=ROOT, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env, timeout=120,
                       cwd=ROOT)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_warmup_below_three_rejected():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_backward_flops_and_configs():
    # five N x N x d products in the backward (S recomputed, dP, dV, dK, dQ)
    assert bench.bwd_flops(1, 16, 11616, 64, False) == 10 * 16 * 11616 ** 2 * 64
    assert bench.bwd_flops(1, 16, 16384, 128, True) == 5 * 16 * 16384 ** 2 * 128
    # every workload of the pages is reachable by name, the default is the headline
    assert bench.CONFIGS["headline"] is bench.WORKLOAD
    assert {c["N"] for c in bench.CONFIGS.values()} >= {128, 1944, 11616, 38400, 1024, 16384}
    args = type("A", (), {"config": "causal_d128"})()
    w = bench.workload(args)
    assert (w["B"], w["H"], w["N"], w["d"], w["causal"]) == (1, 16, 16384, 128, True)
    # the headline keeps the metric name it is quoted on; others name their shape
    assert bench.metric_name(bench.WORKLOAD) == bench.METRIC
    assert bench.metric_name(w) == "attn fwd TFLOP/s at B1 H16 N16384 d128 causal"
    assert bench.metric_name(bench.WORKLOAD, "bwd").startswith("attn bwd TFLOP/s at B1 H16 N11616 d64")


def test_reference_arm_other_config():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                          "--steps", "1", "--warmup", "3", "--cpu-budget", "1"],
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["config"]["N"] == 128 and line["metric"].endswith("N128 d64")
