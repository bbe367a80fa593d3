#!/usr/bin/env python
"""Benchmark of one DDTree tree-verify step on B200s.

A step = ddt_build_tree -> ddt_verify_attn -> ddt_accept_compact (all three
calls of the C ABI, one stream) over one batch of synthetic Kimi-K2.6-shaped
inputs. Metric: verified tree nodes per second (whole job), with the verify
attention's TFLOP/s against the measured bf16 dense peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

N > 1 runs under torch.distributed.run, one process per GPU. Requests are
independent, so every rank runs its own replica of the workload (weak scaling)
with no collective on the data path; NCCL only carries the timing barrier and
the max-over-ranks of the elapsed time.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from ddtree_speculative_decode_b200 import synth  # noqa: E402

METRIC = "verified tree-nodes/s per B200; verify-attn TFLOP/s as % of BF16 peak"
UNIT = "nodes/s"
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------


# (B, N, L) points of the Kimi-shaped sweep: every batch x tree budget x
# context length of the workload definition (36 points)
SWEEP_POINTS = [(b, n, l) for b in (1, 4, 16, 64) for n in (16, 64, 256) for l in (512, 4096, 65536)]


def max_over_ranks(x: float, device) -> float:
    """The largest value of x over the ranks of the default process group (x
    itself without one): a multi-GPU time is the slowest replica's."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(nodes_per_step: int, steps: int, world: int, elapsed_ms: float) -> float:
    """Whole-job tree nodes/s of `world` replicas that each ran `steps` steps of
    `nodes_per_step` nodes, timed by the slowest replica."""
    return nodes_per_step * world * steps / (elapsed_ms / 1e3)


# DRAM bytes (read + write) of one verify-attention launch, from one ncu
# capture per workload (the capture command and figures are summarised under
# profiles/), valid only while the kernel sources still have the sha256 they
# had when captured.
PROFILED_ATTN_DRAM = {
    # ncu --set full, one launch of the long-context workload's attention
    # (bench.py --steps 3 --warmup 3 --no-cpu-baseline --e2e-steps 3 --layers 1
    # --extra=, -k regex:attn_tc -s 2 -c 1): dram__bytes_read.sum 317.055488 MB
    # + dram__bytes_write.sum 81.800960 MB
    "kimi-4req-L32768-N128": {
        "bytes": 398856448.0,
        "sources": {"verify_attn_tc.cu": "d7cd1b6e74e4b64c5a98ba4b00855840b7f11254464a9dc0bb6f3fbd65277c7a",
                    "sm100_ptx.cuh": "742a701fc79bc45f49ed1e6b9494f89da884dc911c9353fdb120e72dbac572a6"}},
}


def profiled_traffic(shape: synth.Shape, table=None, root=None):
    """roofline.traffic: the captured DRAM bytes of one verify-attention launch
    of this workload, or None when there is no capture of it or the kernel
    sources changed since (a stale count says nothing about the kernel as it
    is)."""
    import hashlib
    entry = (PROFILED_ATTN_DRAM if table is None else table).get(shape.name)
    if entry is None:
        return None
    csrc = os.path.join(root or ROOT, "ddtree_speculative_decode_b200", "csrc")
    for fname, digest in entry["sources"].items():
        path = os.path.join(csrc, fname)
        if not os.path.exists(path) or hashlib.sha256(open(path, "rb").read()).hexdigest() != digest:
            return None
    return float(entry["bytes"])


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def attn_flops(shape: synth.Shape, cache_len, depth, n_nodes) -> float:
    """Algorithmic FLOPs of one verify-attention launch: for every real row
    (b, i, h), 2 * (visible keys) * (d_qk + d_l); visible keys = L_b + depth_i + 1."""
    f = 0.0
    for b in range(len(n_nodes)):
        n = int(n_nodes[b])
        vis = int(cache_len[b]) * n + int(np.sum(depth[b, :n] + 1))
        f += 2.0 * shape.H * vis * (shape.d_qk + shape.d_l)
    return f


class ClockSampler:
    """nvidia-smi sampler (200 ms) for SM clock and throttle reasons."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.proc = None
        self.path = None
        if uuid is None:
            return
        try:
            fd, self.path = tempfile.mkstemp(prefix="ddt_clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", uuid, f"--query-gpu={self.Q}", "--format=csv,noheader",
                                          "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append({"sm": float(f[1].split()[0]), "max": float(f[2].split()[0]),
                             "hw_slowdown": f[5] == "Active", "hw_thermal_slowdown": f[6] == "Active",
                             "sw_thermal_slowdown": f[7] == "Active", "sw_power_cap": f[8] == "Active"})
            except Exception:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = sorted({k for r in rows for k in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                                    "sw_power_cap") if r[k]})
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": reasons, "samples": len(rows)}


class RegionClocks:
    """SM clock and clock-event reasons polled through NVML (about once a
    millisecond) while the timed region runs. nvidia-smi's 200 ms period is
    longer than a short timed region, so its samples over the whole run are
    mostly taken outside it, with the GPU idle or lightly loaded."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, uuid: str | None):
        self.nv = None
        self.h = None
        self.th = None
        self.rows = []
        self.done = threading.Event()
        if uuid is None:
            return
        try:
            import pynvml
            pynvml.nvmlInit()
        except Exception:
            return
        self.nv = pynvml
        try:
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        except Exception:
            self.h = None
            try:
                pynvml.nvmlShutdown()
            except Exception:
                pass

    def start(self):
        if self.h is None:
            return
        nv, h = self.nv, self.h

        def poll():
            while not self.done.is_set():
                try:
                    self.rows.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                      int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))))
                except Exception:
                    return
                time.sleep(0.001)

        self.th = threading.Thread(target=poll, daemon=True)
        self.th.start()

    def stop(self):
        if self.th is None:
            return None
        self.done.set()
        self.th.join(timeout=5)
        try:
            self.nv.nvmlShutdown()  # balances the nvmlInit of this sampler
        except Exception:
            pass
        if not self.rows:
            return None
        reasons = sorted({k for _, bits in self.rows for k, name in self.REASONS
                          if bits & int(getattr(self.nv, name, 0))})
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": self.max_mhz,
                "sm_min_mhz": min(r[0] for r in self.rows), "reasons": reasons, "samples": len(self.rows),
                "source": "NVML, polled about every millisecond during the timed region"}


def clock_record(region: dict | None, whole: dict | None) -> dict | None:
    """The clocks key: the timed region's NVML samples when there are any,
    else nvidia-smi's samples over the whole run; the nvidia-smi summary is
    kept beside the first."""
    if region is None:
        return None if whole is None else dict(whole, source="nvidia-smi every 200 ms over the whole run")
    return dict(region, nvidia_smi_whole_run=whole)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline; never the product path)
# ---------------------------------------------------------------------------


def request_slice(x, logits, b):
    """Request b of a step as a one-request step (its pool rows rebased to
    row 0): the unit of work of the oracle timings."""
    off, cap = int(x.cache_off[b]), int(x.cache_cap[b])
    return {"logp": x.logp[b:b + 1], "tok": x.tok[b:b + 1], "root": x.root_tok[b:b + 1],
            "L": x.cache_len[b:b + 1], "off": np.zeros(1, np.int64), "cap": x.cache_cap[b:b + 1],
            "kv": x.kv[off:off + cap], "q": x.q[b:b + 1], "logits": logits[b:b + 1]}


def oracle_request_step(shape: synth.Shape, r: dict, attn_nodes=None):
    """Wall seconds of the oracle's whole step on one request: tree build,
    attention (for the first `attn_nodes` nodes if given, else all of them,
    every head), accept and compaction. Returns (seconds, attention seconds,
    nodes attended, nodes of the request). The pool slice it compacts is a
    copy made before the clock starts."""
    import oracle

    kv = r["kv"].copy()
    t0 = time.perf_counter()
    tree = oracle.build_tree(r["logp"], r["tok"], r["root"], r["L"], shape.N)
    n = int(tree["n_nodes"][0])
    m = n if attn_nodes is None else max(1, min(n, int(attn_nodes)))
    rows = None if m == n else [(0, i) for i in range(m)]
    t1 = time.perf_counter()
    oracle.verify_attn(r["q"], kv, r["off"], r["L"], tree["mask"], tree["n_nodes"], shape.H, shape.d_l, shape.d_r,
                       shape.scale, shape.dtype, rows=rows)
    t2 = time.perf_counter()
    oracle.accept_compact(r["logits"], shape.dtype, tree["node_tok"], tree["parent"], tree["n_nodes"], kv, r["off"],
                          r["L"], r["cap"])
    t3 = time.perf_counter()
    return t3 - t0, t2 - t1, m, n


def reference_steps(steps: int, budget_s: float, step_wall_s: float) -> int:
    """How many of the requested steps the reference arm times: all of them if
    they fit the wall-time budget, else as many as it holds (at least one)."""
    if step_wall_s <= 0:
        return steps
    return int(max(1, min(steps, budget_s // step_wall_s)))


def oracle_inputs(shape: synth.Shape):
    """The workload's step drawn on the host and the oracle's tree and target
    logits for it (inputs of the oracle timings; not timed)."""
    import oracle

    x = synth.make_step(shape)
    tree = oracle.build_tree(x.logp, x.tok, x.root_tok, x.cache_len, shape.N)
    logits = synth.target_logits(shape, tree["parent"], tree["node_tok"], tree["n_nodes"])
    return x, logits


def run_reference(args, shape: synth.Shape, rank: int):
    """--impl reference: the oracle as it stands, timed on the host cores.
    A step is the oracle's whole step on one request of the workload
    (requests in turn), nothing sampled or scaled: ms_per_step is what a step
    took."""
    if rank != 0:
        return
    x, logits = oracle_inputs(shape)
    reqs = [request_slice(x, logits, b) for b in range(shape.B)]
    # one untimed step (whatever W is) also measures a step's wall time
    t, _, _, _ = oracle_request_step(shape, reqs[0])
    run = reference_steps(args.steps, args.ref_budget, t)
    secs, nodes = [], 0
    for k in range(run):
        t, _, _, n = oracle_request_step(shape, reqs[k % shape.B])
        secs.append(t)
        nodes += n
    sec = float(sum(secs))
    value = nodes / sec
    desc = (f"each step the oracle's whole step on one of the workload's {shape.B} requests in turn (tree build, "
            f"attention on all its nodes and heads, accept + compaction), nothing sampled or scaled; {run} of "
            f"{args.steps} requested steps timed (wall-time budget {args.ref_budget:.0f} s)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": run, "steps_requested": args.steps, "warmup": args.warmup, "ms_per_step": sec / run * 1e3,
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(shape),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(shape: synth.Shape, extra=None):
    d = {"workload": shape.name, "seed": shape.seed, "B": shape.B, "N": shape.N, "D": shape.D, "K": shape.K,
         "H": shape.H,
         "d_latent": shape.d_l, "d_rope": shape.d_r, "V": shape.V, "cache_len": list(shape.L)[:4] +
         (["..."] if len(shape.L) > 4 else []), "in_dtype": shape.dtype}
    if extra:
        d.update(extra)
    return d


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------


def measure_step(args, shape: synth.Shape, dev, world: int, full: bool, clock_uuid: str | None = None):
    """One workload on this GPU: the timed loop of K whole steps, the per-stage
    kernel times and (when `full`) the drafter, compaction and end-to-end
    legs. Returns a dict of results (and the host-side step for the CPU
    baseline)."""
    import torch
    import torch.distributed as dist

    from ddtree_speculative_decode_b200 import lib

    bf = shape.dtype == "bf16"
    tdt = torch.bfloat16 if bf else torch.float32

    def dev_t(a, as_bf16=False):
        a = np.ascontiguousarray(a)
        if as_bf16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    # ---- inputs (host draw, then resident in HBM; sweep points: the latent
    # rows, queries and logits drawn on the device, same distributions) ------
    on_device = bool(args.sweep)
    x = synth.make_step(shape, rows=not on_device)
    logp, tok = dev_t(x.logp), dev_t(x.tok)
    root, cl0 = dev_t(x.root_tok), dev_t(x.cache_len)
    off, cap = dev_t(x.cache_off), dev_t(x.cache_cap)
    tree = lib.build_tree(logp, tok, root, cl0, shape.N)
    torch.cuda.synchronize()
    t_host = {k: v.cpu().numpy() for k, v in tree.items()}
    if on_device:
        logits_h = None
        set_bytes = device_set_bytes(shape, x)
        n_sets = max(1, min(16, math.ceil(2 * L2_BYTES / set_bytes)))
        sets = [device_set(shape, x, t_host, dev, k) for k in range(n_sets)]
    else:
        logits_h = synth.target_logits(shape, t_host["parent"], t_host["node_tok"], t_host["n_nodes"])
        set_bytes = x.kv.nbytes + x.q.nbytes + logits_h.nbytes
        n_sets = max(1, min(16, math.ceil(2 * L2_BYTES / set_bytes)))
        sets = []
        for _ in range(n_sets):
            sets.append({"kv": dev_t(x.kv, bf), "q": dev_t(x.q, bf), "logits": dev_t(logits_h, bf)})
    maxL = int(max(shape.L))
    B, N, H = shape.B, shape.N, shape.H
    ws_attn = torch.zeros(max(256, lib.verify_attn_workspace_size(B, N, H, shape.d_l, shape.d_r, maxL, tdt)),
                          dtype=torch.uint8, device=dev)
    ws_acc = torch.zeros(max(256, lib.accept_compact_workspace_size(B, N, shape.V)), dtype=torch.uint8, device=dev)
    out = torch.empty(B, N, H, shape.d_l, dtype=tdt, device=dev)
    lse = torch.empty(B, N, H, dtype=torch.float32, device=dev)
    acc = lib.alloc_accept(B, N, dev)
    cl = cl0.clone()
    stream = torch.cuda.current_stream(dev)
    n_nodes_total = int(t_host["n_nodes"].sum())

    def step(s, ev=None):
        st = torch.cuda.current_stream(dev)  # the capture stream while a graph is recorded
        # restore cache_len (the accept advances it) with a small kernel rather
        # than a memcpy, which would break the chain of programmatic launches
        torch.add(cl0, 0, out=cl)
        if ev is not None:
            ev[0].record(st)
        lib.build_tree(logp, tok, root, cl, N, out=tree, stream=st)
        if ev is not None:
            ev[1].record(st)
        lib.verify_attn(s["q"], s["kv"], off, cl, tree["mask"], tree["n_nodes"], shape.d_l, shape.d_r, shape.scale,
                        maxL, out=out, lse=lse, workspace=ws_attn, stream=st)
        if ev is not None:
            ev[2].record(st)
        lib.accept_compact(s["logits"], tree["node_tok"], tree["parent"], tree["n_nodes"], s["kv"], off, cl, cap,
                           out=acc, workspace=ws_acc, stream=st)
        if ev is not None:
            ev[3].record(st)

    # ---- warm-up ---------------------------------------------------------------
    for w in range(args.warmup):
        step(sets[w % n_sets])
    torch.cuda.synchronize()
    # one CUDA graph per input set holds one whole step (the library's launches
    # keep their programmatic-launch edges), so the timed loop is not bound by
    # Python's per-call cost; --no-graph times plain calls instead
    graphs = None
    if args.graph:
        try:
            graphs = []
            for k in range(n_sets):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    step(sets[k])
                graphs.append(g)
            for k in range(max(3, n_sets)):
                graphs[k % n_sets].replay()
            torch.cuda.synchronize()
        except Exception as e:  # capture unsupported here: fall back to plain calls
            print(f"graph capture failed ({e}); timing plain calls", file=sys.stderr)
            graphs = None
            torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    # ---- timed region: exactly K steps ------------------------------------------
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    region = RegionClocks(clock_uuid)
    region.start()
    t_start.record(stream)
    for k in range(args.steps):
        if graphs is not None:
            graphs[k % n_sets].replay()
        else:
            step(sets[k % n_sets])
    t_end.record(stream)
    torch.cuda.synchronize()
    region_clocks = region.stop()
    if world > 1:
        dist.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    # ---- per-stage kernel times: a separate pass (events between the kernels
    # cut their programmatic overlap, so they stay out of the timed region),
    # captured as one graph with event nodes between the stages so that the
    # host's per-call cost never shows up as GPU time ------------------------------
    n_stage = max(3, min(args.steps, 300))
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(n_stage)]
    stage_pass = "one CUDA graph of the steps with timing-event nodes between the stages"
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for k in range(n_stage):
                step(sets[k % n_sets], evs[k])
        g.replay()
        torch.cuda.synchronize()
        del g
    except Exception as e:  # no event nodes in graphs here: plain calls (host gaps included)
        print(f"stage graph failed ({e}); timing stages with plain calls", file=sys.stderr)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_stage)]
        for k in range(n_stage):
            step(sets[k % n_sets], evs[k])
        torch.cuda.synchronize()
        stage_pass = "plain library calls with events between the stages"
    build_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    accept_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    acc_len = acc["acc_len"].cpu().numpy().astype(np.int64)
    res = {"shape": shape, "x": x, "logits_h": logits_h, "t_host": t_host, "n_sets": n_sets, "set_bytes": set_bytes,
           "region_clocks": region_clocks,
           "elapsed_ms": max_over_ranks(elapsed_ms, dev), "nodes": n_nodes_total,
           "flops": attn_flops(shape, x.cache_len, t_host["depth"], t_host["n_nodes"]),
           "acc_bytes": float(n_nodes_total) * shape.V * (2 if bf else 4),
           "stages_ms": {"build_tree": build_ms, "verify_attn": attn_ms, "accept_compact": accept_ms},
           "stage_pass": f"{stage_pass}, {n_stage} steps",
           "acc_len": acc_len, "graphs": graphs is not None,
           "split_keys": lib.verify_attn_workspace_size(B, N, H, shape.d_l, shape.d_r, maxL, tdt) > 256}
    if full:
        if args.dump:
            dump_step(args.dump, shape, x, logits_h, tree, out, lse, acc, cl)
        res["drafter"] = measure_drafter(args, shape, lib, dev, tdt)
        res["compaction"] = None if args.layers < 2 else measure_compaction(
            args, shape, lib, dev, tdt, sets[0], tree, cl0, off, cap, acc, ws_acc)
        # ---- end to end through the public API with host buffers --------------------
        res["e2e"] = run_e2e(args, shape, x, logits_h, dev, stream, lib, tree, acc, ws_attn, ws_acc, out, lse, off,
                             cap, maxL, world)
        # ---- the same step with the target's LM head folded into the accept -------
        if args.lmhead and shape.dtype == "bf16":
            lm = measure_lmhead(args, shape, lib, dev, x, t_host,
                                {"cl0": cl0, "cl": cl, "tree": tree, "off": off, "cap": cap, "ws_acc": ws_acc,
                                 "acc": acc, "kv": sets[0]["kv"]})
            w_head, hid = lm.pop("w"), lm.pop("hidden")

            def step_lm(s):
                st = torch.cuda.current_stream(dev)
                torch.add(cl0, 0, out=cl)
                lib.build_tree(logp, tok, root, cl, N, out=tree, stream=st)
                lib.verify_attn(s["q"], s["kv"], off, cl, tree["mask"], tree["n_nodes"], shape.d_l, shape.d_r,
                                shape.scale, maxL, out=out, lse=lse, workspace=ws_attn, stream=st)
                lib.accept_compact_lmhead(hid, w_head, tree["node_tok"], tree["parent"], tree["n_nodes"], s["kv"],
                                          off, cl, cap, out=acc, workspace=ws_acc, stream=st)

            for k in range(3):
                step_lm(sets[k % n_sets])
            torch.cuda.synchronize()
            n_lm = max(3, min(args.steps, 50))
            gl = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gl):
                for k in range(n_lm):
                    step_lm(sets[k % n_sets])
            gl.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            gl.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            ms = max_over_ranks(e0.elapsed_time(e1), dev)
            del gl
            lm["step"] = {"value": replica_throughput(n_nodes_total, n_lm, world, ms), "unit": UNIT,
                          "ms_per_step": ms / n_lm, "steps": n_lm,
                          "what": "build -> verify attention -> accept with the LM head folded in (one graph)"}
            lm["step"]["e2e"] = run_e2e(args, shape, x, logits_h, dev, stream, lib, tree, acc, ws_attn, ws_acc, out,
                                        lse, off, cap, maxL, world,
                                        head={"w": w_head, "hidden_h": hid.cpu()})
            res["lmhead"] = lm
            del w_head, hid
    del sets, graphs
    return res


def lmhead_width(shape: synth.Shape) -> int:
    """Hidden size of the target whose head the fused accept folds in: Kimi
    K2.6's 7168 for the Kimi-shaped workloads, the pages' tiny model's 64
    otherwise."""
    return 7168 if shape.V == 163840 else 64


def measure_lmhead(args, shape, lib, dev, x, t_host, step_parts):
    """The accept with the target's LM head folded in (ddt_accept_compact_lmhead)
    on this workload's verify rows: a random-init bf16 head [V, d] and hidden
    states drawn on the device (planted rows pushed toward a child's token as
    the logits recipe biases them). Times the call alone (graph of calls after
    a restore of cache_len), then the whole step with it in place of the
    materialised-logits accept, then that step end to end with the hidden
    states copied in each step."""
    import torch
    B, N, V = shape.B, shape.N, shape.V
    d = lmhead_width(shape)
    g = torch.Generator(device=dev)
    g.manual_seed(shape.seed + 77)
    w = (torch.randn(V, d, generator=g, device=dev) / math.sqrt(d)).to(torch.bfloat16)
    hidden = torch.randn(B, N, d, generator=g, device=dev)
    rng = np.random.default_rng(shape.seed + 78)
    for b in range(B):
        n = int(t_host["n_nodes"][b])
        for i in range(n):
            kids = np.flatnonzero(t_host["parent"][b, :n] == i)
            if len(kids) and rng.random() < shape.accept_p:
                t = int(t_host["node_tok"][b, int(kids[rng.integers(len(kids))])])
                wt = w[t].float()
                hidden[b, i] += shape.accept_bias * wt / (wt @ wt)
    hidden = hidden.to(torch.bfloat16)
    cl0, cl, tree, off, cap, ws_acc, acc, kv = (step_parts[k] for k in
                                                 ("cl0", "cl", "tree", "off", "cap", "ws_acc", "acc", "kv"))
    stream = torch.cuda.current_stream(dev)

    def call(st):
        torch.add(cl0, 0, out=cl)
        lib.accept_compact_lmhead(hidden, w, tree["node_tok"], tree["parent"], tree["n_nodes"], kv, off, cl, cap,
                                  out=acc, workspace=ws_acc, stream=st)

    for _ in range(3):
        call(stream)
    torch.cuda.synchronize()
    reps = max(3, min(50, int(0.2 / (2.0 * B * N * d * V / 1.0e15 + 1e-5))))
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for _ in range(reps):
            call(torch.cuda.current_stream(dev))
    gr.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    gr.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) / reps * 1e3
    del gr
    acc_len = acc["acc_len"].cpu().numpy().astype(np.int64)
    return {"rows": B * N, "d_model": d, "V": V, "us": us, "flops": 2.0 * B * N * d * V,
            "head_bytes": float(V * d * 2), "tokens_per_call": int((acc_len + 1).sum()),
            "w": w, "hidden": hidden, "timing": f"graph of {reps} calls, each after a cache_len restore"}


def device_set_bytes(shape: synth.Shape, x) -> int:
    elt = 2 if shape.dtype == "bf16" else 4
    rows = int(x.cache_cap.astype(np.int64).sum())
    return elt * (rows * shape.d_qk + shape.B * shape.N * shape.H * shape.d_qk + shape.B * shape.N * shape.V)


def device_set(shape: synth.Shape, x, t_host: dict, dev, k: int) -> dict:
    """One input set drawn on the device with seeded generators, the host
    recipe's distributions (latent rows N(0, 1) x kv_scale, queries N(0, 1),
    logits N(0, 1) with +bias on a uniformly chosen child's token at the
    workload's fraction of nodes), for points too large to draw on the host
    in reasonable time."""
    import torch
    tdt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
    g = torch.Generator(device=dev)
    g.manual_seed(shape.seed * 1000 + k)
    rows = int(x.cache_cap.astype(np.int64).sum())
    kv = (torch.randn(rows, shape.d_qk, generator=g, device=dev) * shape.kv_scale).to(tdt)
    q = torch.randn(shape.B, shape.N, shape.H, shape.d_qk, generator=g, device=dev).to(tdt)
    logits = torch.empty(shape.B, shape.N, shape.V, dtype=tdt, device=dev)
    rng = np.random.default_rng([shape.seed, 11, k])
    for b in range(shape.B):
        z = torch.randn(shape.N, shape.V, generator=g, device=dev)
        n = int(t_host["n_nodes"][b])
        rows_i, toks = [], []
        for i in range(n):
            u, pick = rng.random(), rng.random()
            kids = np.flatnonzero(t_host["parent"][b, :n] == i)
            if len(kids) and u < shape.accept_p:
                rows_i.append(i)
                toks.append(int(t_host["node_tok"][b, int(kids[min(len(kids) - 1, int(pick * len(kids)))])]))
        if rows_i:
            z[torch.tensor(rows_i, device=dev), torch.tensor(toks, device=dev)] += shape.accept_bias
        logits[b] = z.to(tdt)
        del z
    return {"kv": kv, "q": q, "logits": logits}


def stage_rooflines(res: dict, pk: dict) -> dict:
    """Attention TFLOP/s and accept GB/s from the per-stage kernel times, as
    fractions of the burst peaks (the stage pass is a short burst of work)."""
    attn_ms = res["stages_ms"]["verify_attn"]
    accept_ms = res["stages_ms"]["accept_compact"]
    achieved = res["flops"] / (attn_ms / 1e3) / 1e12
    gbs = res["acc_bytes"] / (accept_ms / 1e3) / 1e9
    return {"attn_tflops": achieved, "attn_frac": achieved / pk["bf16_tflops"], "accept_gbs": gbs,
            "accept_frac": gbs / pk["hbm_gbs"]}


def run_ours(args, shape: synth.Shape, rank: int, world: int, local_rank: int):
    import torch

    from ddtree_speculative_decode_b200 import lib

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    lib.load()
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        if not uuid.startswith("GPU-"):
            uuid = "GPU-" + uuid
    except Exception:
        uuid = None
    sampler = ClockSampler(uuid) if rank == 0 else ClockSampler(None)
    res = measure_step(args, shape, dev, world, full=not args.sweep, clock_uuid=uuid if rank == 0 else None)
    clocks = sampler.stop()
    extra = {}
    if not args.sweep:
        for name in [n for n in (args.extra or "").split(",") if n]:
            sh = synth.NAMED[name]() if args.seed is None else dataclasses.replace(synth.NAMED[name](), seed=args.seed)
            if sh.name == shape.name:
                continue
            r = measure_step(args, sh, dev, world, full=False)
            extra[sh.name] = r
            torch.cuda.empty_cache()
    if rank != 0:
        return
    pk = peaks()
    rf = stage_rooflines(res, pk)
    value = replica_throughput(res["nodes"], args.steps, world, res["elapsed_ms"])
    launches_per_step = 1 + attn_launches(shape) + 2  # build, attention, accept argmax + walk (cache_len restore excluded)
    acc_len = res["acc_len"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["elapsed_ms"] / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": shape.dtype, "data": "synthetic",
        "config": config_dict(shape, {"parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                                      "l2": f"{res['n_sets']} rotating input set(s) of {res['set_bytes'] / 2**20:.1f} "
                                            f"MiB (each larger than the 126 MiB L2, or together > 2x L2)"}),
        "roofline": {"bound": "tensor", "achieved": rf["attn_tflops"], "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": rf["attn_frac"], "traffic": profiled_traffic(shape),
                     "kernel": "ddt_verify_attn",
                     "achieved_from": f"algorithmic FLOPs {res['flops'] / 1e9:.1f} G per launch / mean launch time "
                                      f"{res['stages_ms']['verify_attn'] * 1e3:.1f} us ({res['stage_pass']})",
                     "peak_kind": f"bf16 dense, burst (kernel timed in a short pass), {pk['source']}"},
        "stages_ms": res["stages_ms"],
        "accept_hbm": {"achieved_gbs": rf["accept_gbs"], "peak_gbs": pk["hbm_gbs"], "frac": rf["accept_frac"],
                       "bytes": res["acc_bytes"]},
        "nodes_per_step": res["nodes"],
        "accept_len_hist": np.bincount(acc_len, minlength=min(shape.D, shape.N - 1) + 1).tolist(),
        "tokens_per_step": int((acc_len + 1).sum()),
        "attn_gflop_per_step": res["flops"] / 1e9,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clock_record(res["region_clocks"], clocks),
        "timed_loop": "cuda-graph replays of the step" if res["graphs"] else "plain library calls",
    }
    if args.sweep:
        line["sweep_point"] = True
        line["attn_split_keys"] = res["split_keys"]
    else:
        dr, comp = res["drafter"], res["compaction"]
        line["drafter_topk"] = dict(dr, frac=dr["gbs"] / pk["hbm_gbs"], peak_gbs=pk["hbm_gbs"])
        line["compaction_layers"] = None if comp is None else dict(
            comp, frac=comp["marginal_gbs"] / pk["hbm_gbs"], peak_gbs=pk["hbm_gbs"])
        line["e2e"] = res["e2e"]
        lm = res.get("lmhead")
        if lm is not None:
            t_tc = lm["flops"] / (pk["bf16_tflops"] * 1e12)
            t_hbm = lm["head_bytes"] / (pk["hbm_gbs"] * 1e9)
            lm.update({"tflops": lm["flops"] / (lm["us"] * 1e-6) / 1e12,
                       "head_gbs": lm["head_bytes"] / (lm["us"] * 1e-6) / 1e9,
                       "bound": "tensor" if t_tc >= t_hbm else "hbm",
                       "roofline_frac": max(t_tc, t_hbm) / (lm["us"] * 1e-6),
                       "peaks": f"bf16 {pk['bf16_tflops']} TFLOP/s burst, HBM {pk['hbm_gbs']} GB/s ({pk['source']})"})
            line["lmhead"] = lm
        line["workloads"] = {}
        for name, r in extra.items():
            rr = stage_rooflines(r, pk)
            line["workloads"][name] = {
                "value": replica_throughput(r["nodes"], args.steps, world, r["elapsed_ms"]), "unit": UNIT,
                "ms_per_step": r["elapsed_ms"] / args.steps, "stages_ms": r["stages_ms"],
                "attn_tflops": rr["attn_tflops"], "attn_frac": rr["attn_frac"], "accept_gbs": rr["accept_gbs"],
                "accept_frac": rr["accept_frac"], "nodes_per_step": r["nodes"],
                "tokens_per_step": int((r["acc_len"] + 1).sum())}
        if args.cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(args, shape, res["x"], res["logits_h"], res["t_host"])
    print(json.dumps(line), flush=True)


def attn_launches(shape: synth.Shape) -> int:
    """The verify attention is one launch (split partials merge in-kernel)."""
    return 1


def _tdtype(shape):
    import torch
    return torch.bfloat16 if shape.dtype == "bf16" else torch.float32


def dump_step(path, shape, x, logits_h, tree, out, lse, acc, cl):
    """Writes the step's host inputs and the library's outputs of the last
    stage-pass step (stepio format) for replay elsewhere."""
    from ddtree_speculative_decode_b200 import stepio
    inputs = {"logp": x.logp, "tok": x.tok, "root_tok": x.root_tok, "cache_len": x.cache_len,
              "cache_off": x.cache_off, "cache_cap": x.cache_cap, "q": x.q, "kv": x.kv, "logits": logits_h}
    outputs = {k: v.cpu().numpy() for k, v in tree.items()}
    outputs.update({f"acc_{k}": v.cpu().numpy() for k, v in acc.items()})
    outputs["attn_out"] = out.float().cpu().numpy()
    outputs["lse"] = lse.cpu().numpy()
    outputs["cache_len_after"] = cl.cpu().numpy()
    meta = {"workload": shape.name, "B": shape.B, "N": shape.N, "D": shape.D, "K": shape.K, "H": shape.H,
            "d_latent": shape.d_l, "d_rope": shape.d_r, "V": shape.V, "dtype": shape.dtype, "scale": shape.scale}
    stepio.save_step(path, inputs, outputs, meta)


def measure_compaction(args, shape, lib, dev, tdt, s, tree, cl0, off, cap, acc, ws_acc):
    """ddt_accept_compact on a pool of args.layers copies of the workload's
    latent cache at a layer stride (every layer compacted along the same
    accepted path), against the same call on one layer. The target logits are
    the step's with one change: along each tree's deepest path (to its
    deepest node, the lowest index on ties) the next node's token is made the
    argmax, so every request accepts that whole path (several tokens per step,
    as the pages' runs do). Each call is timed
    alone with events after writing a buffer larger than L2, so the moved rows
    come from HBM. The marginal bandwidth counts the extra layers' bytes (each
    accepted row read once and written once) over the extra time."""
    import torch
    layers = args.layers
    par, tokn = tree["parent"].cpu().numpy(), tree["node_tok"].cpu().numpy()
    dep, nn = tree["depth"].cpu().numpy(), tree["n_nodes"].cpu().numpy()
    logits = s["logits"].clone()
    for b in range(len(nn)):
        node = int(np.argmax(dep[b, :int(nn[b])]))
        while node > 0:
            logits[b, int(par[b, node]), int(tokn[b, node])] = 30.0  # above every drawn logit
            node = int(par[b, node])
    kv1 = s["kv"]
    stride = kv1.shape[0]
    pool = kv1.unsqueeze(0).expand(layers, stride, kv1.shape[1]).contiguous().view(layers * stride, kv1.shape[1])
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    cl = cl0.clone()
    stream = torch.cuda.current_stream(dev)

    def timed(n_layers, kv, reps):
        ts = []
        for _ in range(reps):
            torch.add(cl0, 0, out=cl)
            flush.zero_()  # also keeps the GPU busy while the host enqueues the call
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            lib.accept_compact(logits, tree["node_tok"], tree["parent"], tree["n_nodes"], kv, off, cl, cap,
                               n_layers=n_layers, layer_stride_rows=stride, out=acc, workspace=ws_acc,
                               stream=stream)
            e1.record(stream)
            ts.append((e0, e1))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ts) * 1e3

    timed(1, kv1, 3)
    timed(layers, pool, 3)
    us1 = timed(1, kv1, 30)
    usL = timed(layers, pool, 30)
    a = acc["acc_len"].cpu().numpy().astype(np.int64)
    row_bytes = kv1.shape[1] * kv1.element_size()
    per_layer = float(2 * (a + 1).sum() * row_bytes)
    del pool, flush, logits
    return {"layers": layers, "accepted_rows": int((a + 1).sum()), "us_1_layer": us1, "us": usL,
            "bytes_per_layer": per_layer,
            "marginal_gbs": per_layer * (layers - 1) / max(usL - us1, 1e-3) * 1e-3,
            "gbs": per_layer * layers / usL * 1e-3,
            "timing": "one call per pair of events after a 252 MiB L2 flush; median of 30"}


def measure_drafter(args, shape, lib, dev, tdt):
    """ddt_drafter_topk on the workload's B x D rows of V drafter logits (the
    build's inputs), timed alone over rotating sets larger than 2 x L2 (random
    device-side logits; its parity is covered by the tests)."""
    import torch
    R, V, K = shape.B * shape.D, shape.V, shape.K
    row_bytes = R * V * (2 if tdt == torch.bfloat16 else 4)
    n = max(2, math.ceil(2 * L2_BYTES / row_bytes))
    g = torch.Generator(device=dev)
    g.manual_seed(shape.seed)
    z = (torch.randn(n, R, V, device=dev, generator=g) * shape.drafter_sigma).to(tdt)
    views = [z[i] for i in range(n)]
    out = lib.drafter_topk(views[0], K)
    for i in range(3):
        lib.drafter_topk(views[i % n], K, out=out)
    torch.cuda.synchronize()
    # one graph launches the kernel once per set, so Python's per-call cost
    # stays out of the kernel time
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            lib.drafter_topk(views[i], K, out=out, stream=torch.cuda.current_stream(dev))
    g.replay()
    torch.cuda.synchronize()
    reps = max(2, min(50, math.ceil(400 / n)))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) / (reps * n) * 1e3
    del g, views, z
    return {"us": us, "gbs": row_bytes / (us / 1e6) / 1e9, "rows": R, "V": V, "K": K}


def run_e2e(args, shape, x, logits_h, dev, stream, lib, tree, acc, ws_attn, ws_acc, out, lse, off, cap, maxL, world,
            head=None):
    """Same step through the public API, inputs from pinned host memory each
    step (drafter output, queries, the tree rows' latent KV, target logits,
    cache lengths) and the committed tokens read back. With `head` (device
    head weights and host hidden states) the accept runs the fused LM head:
    the verify rows' hidden states are copied in instead of logits."""
    import torch
    import torch.distributed as dist

    bf = shape.dtype == "bf16"

    def pin(a, as_bf16=False):
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if as_bf16 else np.ascontiguousarray(a))
        t = t.pin_memory()
        return t.view(torch.bfloat16) if as_bf16 else t

    B, N = shape.B, shape.N
    h = {"logp": pin(x.logp), "tok": pin(x.tok), "root": pin(x.root_tok), "cl": pin(x.cache_len),
         "q": pin(x.q, bf)}
    if head is None:
        h["logits"] = pin(logits_h, bf)
    else:
        h["hidden"] = head["hidden_h"].pin_memory()
    tree_rows = [pin(x.kv[int(x.cache_off[b]) + int(x.cache_len[b]):int(x.cache_off[b]) + int(x.cache_len[b]) + N],
                     bf) for b in range(B)]
    # two device copies of the per-step inputs: the next step's host-to-device
    # copies run on a copy stream while this step computes
    dd = [{k: torch.empty(v.shape, dtype=v.dtype, device=dev) for k, v in h.items()} for _ in range(2)]
    kv = torch.from_numpy(x.kv.view(np.int16) if bf else x.kv).to(dev)
    kv = kv.view(torch.bfloat16) if bf else kv
    res_h = {"out_tok": torch.empty(B, N, dtype=torch.int32).pin_memory(),
             "acc_len": torch.empty(B, dtype=torch.int32).pin_memory(),
             "bonus": torch.empty(B, dtype=torch.int32).pin_memory()}
    h2d = sum(v.numel() * v.element_size() for v in h.values()) + sum(t.numel() * t.element_size() for t in tree_rows)
    d2h = sum(v.numel() * v.element_size() for v in res_h.values())
    copy_stream = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    freed = [torch.cuda.Event() for _ in range(2)]
    for e in freed:
        e.record(stream)
    counter = [0]

    def step():
        i = counter[0] & 1
        counter[0] += 1
        d = dd[i]
        if args.e2e_serial:
            for k in h:
                d[k].copy_(h[k], non_blocking=True)
        else:
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(freed[i])
                for k in h:
                    d[k].copy_(h[k], non_blocking=True)
                copied[i].record(copy_stream)
            stream.wait_event(copied[i])
        for b in range(B):
            o = int(x.cache_off[b]) + int(x.cache_len[b])
            kv[o:o + N].copy_(tree_rows[b], non_blocking=True)
        lib.build_tree(d["logp"], d["tok"], d["root"], d["cl"], N, out=tree, stream=stream)
        lib.verify_attn(d["q"], kv, off, d["cl"], tree["mask"], tree["n_nodes"], shape.d_l, shape.d_r, shape.scale,
                        maxL, out=out, lse=lse, workspace=ws_attn, stream=stream)
        if head is None:
            lib.accept_compact(d["logits"], tree["node_tok"], tree["parent"], tree["n_nodes"], kv, off, d["cl"], cap,
                               out=acc, workspace=ws_acc, stream=stream)
        else:
            lib.accept_compact_lmhead(d["hidden"], head["w"], tree["node_tok"], tree["parent"], tree["n_nodes"], kv,
                                      off, d["cl"], cap, out=acc, workspace=ws_acc, stream=stream)
        freed[i].record(stream)
        res_h["out_tok"].copy_(acc["out_tok"], non_blocking=True)
        res_h["acc_len"].copy_(acc["acc_len"], non_blocking=True)
        res_h["bonus"].copy_(acc["bonus"], non_blocking=True)

    steps = max(3, min(args.steps, args.e2e_steps))
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_stream.wait_event(e0)  # the first step's copies start inside the timed region
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), dev)
    nodes = int(tree["n_nodes"].sum().item())
    return {"value": replica_throughput(nodes, steps, world, ms), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps,
            "copies": "on the compute stream" if args.e2e_serial else "next step's copies overlap this step's kernels",
            "h2d_gbs": h2d * steps / (ms / 1e3) / 1e9}


def cpu_baseline(args, shape, x, logits_h, t_host=None):
    """The oracle's throughput on this workload on the host cores: its whole
    step on three of the workload's requests (requests in turn; each step
    complete, nothing scaled), numpy's BLAS on all its threads; then one
    request on one thread, with attention on as many of its nodes as fit
    about args.cpu_seconds and scaled to all of them (labelled)."""
    reqs = [request_slice(x, logits_h, b) for b in range(shape.B)]
    secs, nodes, per_node = [], 0, []
    for k in range(3):
        t, ta, m, n = oracle_request_step(shape, reqs[k % shape.B])
        secs.append(t)
        nodes += n
        per_node.append(ta / max(1, m))
    value = nodes / float(sum(secs))
    one, one_desc = None, None
    try:
        from threadpoolctl import threadpool_limits
        r0 = reqs[0]
        n0 = int(synth_nodes(shape))
        # one thread runs the BLAS part several times slower: size the node
        # sample from the all-threads rate, at least one node
        m = max(1, min(n0, int(args.cpu_seconds / (4.0 * max(min(per_node), 1e-6)))))
        with threadpool_limits(limits=1, user_api="blas"):
            t, ta, m, n = oracle_request_step(shape, r0, attn_nodes=m)
        full = (t - ta) + ta * n / m
        one = n / full
        one_desc = (f"one request, whole step on one BLAS thread" if m == n else
                    f"one request on one BLAS thread: build, accept + compaction whole, attention on {m} of its "
                    f"{n} nodes scaled by {n}/{m} (extrapolated)")
    except Exception:  # no BLAS thread control here: report the all-threads figure only
        one = None
    return {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "median_step_s": float(statistics.median(secs)),
            "value_1thread": one, "sample_1thread": one_desc,
            "sample": f"3 steps, each the oracle's whole step on one of the workload's {shape.B} requests in turn "
                      f"(tree build, attention on all its nodes and heads, accept + compaction); "
                      f"{nodes} nodes in {sum(secs):.1f} s, nothing scaled"}


def synth_nodes(shape: synth.Shape) -> int:
    """Tree nodes of one request (the budget, when the drafter's tree can fill
    it, as every workload's can)."""
    total, width = 1, 1
    for _ in range(shape.D):
        width *= shape.K
        total += width
        if total >= shape.N:
            return shape.N
    return total


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="kimi-4req-32k", choices=sorted(synth.NAMED),
                    help="the workload of the headline line (default: the long-context step, the largest that "
                         "one GPU runs)")
    ap.add_argument("--extra", default="kimi-1req,kimi-16req",
                    help="comma list of further workloads measured after the headline one and reported under "
                         "'workloads' ('' for none)")
    ap.add_argument("--seed", type=int, default=None,
                    help="seed of the step's draws (drafter output, cache, queries, logits) instead of the "
                         "workload's own; the workload's cache lengths stay as defined")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--layers", type=int, default=61,
                    help="layers of the multi-layer compaction measurement (< 2: skip it)")
    ap.add_argument("--ref-budget", type=float, default=120.0,
                    help="wall seconds the reference arm's timed steps may take")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="about how long the one-thread oracle run of cpu_baseline may take")
    ap.add_argument("--dump", default=None,
                    help="write one step's inputs and the library's outputs to this .npz (replayable)")
    ap.add_argument("--e2e-serial", action="store_true",
                    help="end-to-end leg: copy each step's inputs on the compute stream (no overlap)")
    ap.add_argument("--sweep", default=None,
                    help="context/budget sweep on Kimi shapes: 'default' or a comma list of B:N:L points; one "
                         "JSON line per point (no end-to-end leg, no CPU baseline)")
    ap.add_argument("--no-lmhead", dest="lmhead", action="store_false",
                    help="skip the fused LM-head accept leg (head kernel, step and end to end)")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="time plain library calls instead of CUDA-graph replays of the step")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    def seeded(sh):
        return sh if args.seed is None else dataclasses.replace(sh, seed=args.seed)

    shape = seeded(synth.NAMED[args.config]())
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, shape, rank)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    try:
        if args.sweep:
            pts = SWEEP_POINTS if args.sweep == "default" else [tuple(int(v) for v in p.split(":"))
                                                                 for p in args.sweep.split(",")]
            for (b, n, l) in pts:
                sh = seeded(synth.kimi_sweep(b, n, l))
                # about half a second of timed steps per point (at least 5, at most --steps)
                est_s = 2.0 * b * n * sh.H * (l + 8) * (sh.d_qk + sh.d_l) / 1.0e15 + 60e-6
                pa = dataclasses.replace(args) if dataclasses.is_dataclass(args) else argparse.Namespace(**vars(args))
                pa.steps = int(max(5, min(args.steps, 0.5 / est_s)))
                run_ours(pa, sh, rank, world, local_rank)
                torch.cuda.empty_cache()
        else:
            run_ours(args, shape, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
