"""The reference arm (the oracle timed on the host cores): any --steps K stays
within the wall-time budget with a fixed per-step sample, and its JSON line
carries the contract's keys."""
import json
import os
import subprocess
import sys
import time

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

    import oracle
    from ddtree_speculative_decode_b200 import synth
    shape = synth.tiny_f32()
    x = synth.make_step(shape)
    tree = oracle.build_tree(x.logp, x.tok, x.root_tok, x.cache_len, shape.N)
    logits = synth.target_logits(shape, tree["parent"], tree["node_tok"], tree["n_nodes"])
    cb = bench.cpu_baseline(argparse.Namespace(ref_nodes=8, cpu_seconds=1.0), shape, x, logits, None)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1
    assert cb["value_1thread"] is None or cb["value_1thread"] > 0
    assert int(cb["sample"].split()[0]) > 1  # many step estimates within the second


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


def test_profiled_traffic_follows_the_captured_sources(tmp_path, monkeypatch):
    """roofline.traffic comes from the ncu summary only while the captured
    kernel sources are unchanged (the summary records their sha256), and only
    for the captured workload."""
    import hashlib

    from ddtree_speculative_decode_b200 import synth
    csrc = tmp_path / "ddtree_speculative_decode_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "verify_attn_tc.cu").write_text("kernel A\n")
    (csrc / "sm100_ptx.cuh").write_text("helpers B\n")

    def sha(name):
        return hashlib.sha256((csrc / name).read_bytes()).hexdigest()

    (tmp_path / "profiles" / "attn_tc_kimi-1req.md").write_text(
        "Source captured (sha256):\n\n"
        f"    verify_attn_tc.cu {sha('verify_attn_tc.cu')}\n"
        f"    sm100_ptx.cuh     {sha('sm100_ptx.cuh')}\n\n"
        "| metric | value |\n|---|---|\n"
        "| dram__bytes_read.sum | 9.5 MB |\n| dram__bytes_write.sum | 512 B |\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    shape = synth.kimi_1req()
    assert bench.profiled_traffic(shape) == 9.5e6 + 512
    assert bench.profiled_traffic(synth.NAMED["kimi-16req"]()) is None  # no capture of that workload
    (csrc / "sm100_ptx.cuh").write_text("helpers B, changed\n")
    assert bench.profiled_traffic(shape) is None
