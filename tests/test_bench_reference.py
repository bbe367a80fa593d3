"""The reference arm (the oracle timed on the host cores): any --steps K stays
within the wall-time budget with a fixed per-step sample, and its JSON line
carries the contract's keys."""
import json
import os
import subprocess
import sys
import time

import numpy as np

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_all_steps_when_they_fit():
    assert bench.reference_steps(10, 120.0, 0.15) == 10


def test_steps_capped_by_the_budget():
    run = bench.reference_steps(10000, 120.0, 0.15)
    assert run == 800 and run * 0.15 <= 120.0
    assert bench.reference_steps(10000, 120.0, 500.0) == 1  # at least one step


def test_reference_line_on_the_tiny_workload():
    t0 = time.time()
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                          "tiny-f32", "--steps", "5", "--warmup", "3", "--ref-budget", "20"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert time.time() - t0 < 300
    assert line["impl"] == "reference" and line["value"] > 0 and line["higher_is_better"] is True
    assert line["steps"] == 5 and line["steps_requested"] == 5
    for k in ("metric", "unit", "n_gpus", "warmup", "ms_per_step", "scaling", "dtype", "data", "config"):
        assert k in line, k
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_cpu_baseline_reports_all_threads_and_one():
    import argparse

    from ddtree_speculative_decode_b200 import synth
    shape = synth.tiny_f32()
    x, logits = bench.oracle_inputs(shape)
    cb = bench.cpu_baseline(argparse.Namespace(cpu_seconds=1.0), shape, x, logits)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1
    assert cb["value_1thread"] is None or cb["value_1thread"] > 0
    assert "nothing scaled" in cb["sample"]


def test_request_step_is_the_whole_step_of_one_request():
    """The oracle timings' unit: one request of the workload, rebased to pool
    row 0, whose whole step (every node attended) runs without scaling."""
    from ddtree_speculative_decode_b200 import synth
    shape = synth.custom(B=3, D=3, K=2, N=6, H=2, d_l=16, d_r=8, V=50, L=(4, 9, 2), seed=5)
    x, logits = bench.oracle_inputs(shape)
    r = bench.request_slice(x, logits, 1)
    assert r["kv"].shape[0] == x.cache_cap[1] and int(r["off"][0]) == 0
    assert np.array_equal(r["kv"], x.kv[x.cache_off[1]:x.cache_off[1] + x.cache_cap[1]])
    t, ta, m, n = bench.oracle_request_step(shape, r)
    assert m == n == 6 and 0 < ta <= t
    t, ta, m, n = bench.oracle_request_step(shape, r, attn_nodes=2)
    assert m == 2 and n == 6
    assert bench.synth_nodes(shape) == 6


def test_seed_flag_changes_the_draws():
    def run(*extra):
        out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                              "tiny-f32", "--steps", "2", "--warmup", "3", "--ref-budget", "10", *extra],
                             capture_output=True, text=True, timeout=600, cwd=ROOT)
        assert out.returncode == 0, out.stderr
        return json.loads(out.stdout.strip().splitlines()[-1])
    default, seeded = run(), run("--seed", "77")
    assert seeded["config"]["seed"] == 77 and default["config"]["seed"] != 77
    assert seeded["config"]["cache_len"] == default["config"]["cache_len"]


def test_two_ranks_under_torchrun_print_one_line():
    """--impl reference under torchrun: rank 0 alone runs and prints; the other
    rank exits 0 without work."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    out = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                          "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
                          "--impl", "reference", "--gpus", "2", "--config", "tiny-f32", "--steps", "2", "--warmup",
                          "3", "--ref-budget", "10"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2


def test_profiled_traffic_follows_the_captured_sources(tmp_path):
    """roofline.traffic is the captured DRAM count only while the captured
    kernel sources are unchanged (the table records their sha256), and only
    for the captured workload."""
    import hashlib

    from ddtree_speculative_decode_b200 import synth
    csrc = tmp_path / "ddtree_speculative_decode_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "verify_attn_tc.cu").write_text("kernel A\n")
    (csrc / "sm100_ptx.cuh").write_text("helpers B\n")

    def sha(name):
        return hashlib.sha256((csrc / name).read_bytes()).hexdigest()

    table = {"kimi-1req-L4096-N64": {"bytes": 9.5e6 + 512,
                                     "sources": {"verify_attn_tc.cu": sha("verify_attn_tc.cu"),
                                                 "sm100_ptx.cuh": sha("sm100_ptx.cuh")}}}
    shape = synth.kimi_1req()
    assert bench.profiled_traffic(shape, table, str(tmp_path)) == 9.5e6 + 512
    assert bench.profiled_traffic(synth.NAMED["kimi-16req"](), table, str(tmp_path)) is None  # not captured
    (csrc / "sm100_ptx.cuh").write_text("helpers B, changed\n")
    assert bench.profiled_traffic(shape, table, str(tmp_path)) is None
