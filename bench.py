#!/usr/bin/env python
"""Benchmark of the Medusa decode-verify step on B200.

One step = heads + top-k, tree build, tree attention, verify/accept and KV
compaction for one batch (three C-ABI calls: heads with the tree build,
attention, verification with the compaction).  Default workload: the
Llama-3-8B-shaped configuration (batch 8, hidden 4096, vocab 128256, 4 heads,
64-node sparse tree, GQA 32/8 heads of 128, ragged prefixes 4096..8192, bf16,
greedy acceptance).  Inputs are seeded synthetic data of those shapes; every
step touches ~4.7 GB (larger than the 126 MB L2), so no flush is needed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own batch (sequences are independent; no
collective on the data path): weak scaling, value = all ranks' steps / the
slowest rank's time.  `--impl reference` times the CPU oracle (the only
reference implementation) on a bounded sample, rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "Medusa decode-verify steps/s (heads+tree attn+accept); % of HBM roofline"
UNIT = "steps/s"
KERNELS_PER_STEP = 9  # stream-K flags, W1 GEMM, W2 GEMM, top-k merge with the tree
#                       build, attention counters, attention, attention exact pass (empty
#                       list: reads a count), verify rows, verify path with the KV compaction


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j.get("bf16_tflops", 1590.0)), "measured"
    return 6650.0, 1590.0, "fallback"


def workload_of(args, W):
    """The named workload with the --nodes and --batch overrides applied."""
    w = W.WORKLOADS[args.workload]
    over = {}
    if args.nodes:
        over["N"] = args.nodes
    if args.batch:
        over["B"] = args.batch
    return W.scaled(w, **over) if over else w


def heads_traffic(algorithmic):
    """DRAM bytes of one heads call, scaled from the profiled ratio; None when
    the kernel sources changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "heads_topk_traffic.json")
    try:
        with open(path) as f:
            j = json.load(f)
        h = hashlib.sha256()
        for name in j["source_files"]:
            with open(os.path.join(ROOT, name), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != j["source_sha256"]:
            return None, "kernel changed since the ncu capture"
        return algorithmic * float(j["traffic_ratio"]), j["measured_on"]
    except (OSError, KeyError, ValueError):
        return None, "no ncu record"


def algorithmic_bytes(w, prefix_lens, N):
    """Bytes the step must move at minimum (bf16 = 2 B)."""
    e = 2 if w.dtype == "bf16" else 4
    heads = w.K * (w.d * w.d + w.d + w.V * w.d) * e + w.B * w.d * e
    kv_prefix = sum(int(p) for p in prefix_lens) * w.Hkv * w.dh * 2 * e
    tree_qkv = w.B * N * (w.Hq + 2 * w.Hkv) * w.dh * e
    tree_out = w.B * N * w.Hq * w.dh * e
    tree_kv_write = w.B * N * w.Hkv * w.dh * 2 * e
    logits = w.B * N * w.V * e
    return {"heads": heads, "attention": kv_prefix + tree_qkv + tree_out + tree_kv_write,
            "verify": logits, "total": heads + kv_prefix + tree_qkv + tree_out + tree_kv_write + logits}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.lines = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", gpu_index], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def _gpu_index(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample
# ---------------------------------------------------------------------------
def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return int(max([i.get("num_threads", 1) for i in threadpool_info()] + [1]))
    except Exception:
        return os.cpu_count() or 1


class OracleSample:
    """A bounded sample of one decode-verify step, run by the CPU oracle and
    extrapolated to the whole step.

    Sample (``frac`` = 1): head 0 on a 16384-token slice of its vocabulary for
    every sequence (scaled by K * V / 16384); tree attention of 4 (sequence,
    node) query rows with all heads (scaled by B*N/4 and the mean prefix);
    verification statistics of 8 rows (scaled by B*N/8); tree build and KV
    compaction in full.  ``frac`` < 1 shrinks the vocabulary slice (to at
    least 256 tokens) so that long runs stay within a few minutes.  Inputs
    are drawn once, outside the timed calls."""

    def __init__(self, w, n_nodes=None, seed=0, frac=1.0):
        from speculative_decoding_medusa_b200 import workloads as W

        self.w = w
        self.N = N = n_nodes or w.N
        self.spec = spec = W.tree_for(w, n_nodes=N)
        f64 = lambda t: t.to(torch.float64).numpy()
        self.rows_v = min(w.V, max(256, int(16384 * frac)))
        self.h = f64(W.randn((w.B, w.d), seed, 1, 1.0, w.dtype))
        self.W1 = f64(W.randn((1, w.d, w.d), seed, 2, 0.02, w.dtype))
        self.b1 = f64(W.randn((1, w.d), seed, 3, 0.02, w.dtype))
        self.W2 = f64(W.randn((1, self.rows_v, w.d), seed, 4, 0.02, w.dtype))
        self.P = W.prefix_lengths(w, seed).numpy().astype(np.int64)
        cap = w.ctx_hi + N
        self.b0 = int(np.argmax(self.P))
        self.q = f64(W.randn((1, N, w.Hq, w.dh), seed, 11, 1.0, w.dtype))
        self.kn = f64(W.randn((1, N, w.Hkv, w.dh), seed, 12, 1.0, w.dtype))
        self.vn = f64(W.randn((1, N, w.Hkv, w.dh), seed, 13, 1.0, w.dtype))
        self.Kc = f64(W.randn((1, w.Hkv, cap, w.dh), seed, 14, 1.0, w.dtype))
        self.Vc = f64(W.randn((1, w.Hkv, cap, w.dh), seed, 15, 1.0, w.dtype))
        self.logits = f64(W.randn((1, 9, w.V), seed, 21, 1.0, w.dtype))
        # 4 query nodes (all heads) of the longest sequence: a 4-node chain
        chain = [0]
        while len(chain) < 4 and any(spec.parent[c] == chain[-1] for c in range(1, N)):
            chain.append(next(c for c in range(1, N) if spec.parent[c] == chain[-1]))
        self.chain = chain
        self.mm = np.zeros((len(chain), 1), dtype=np.uint32)
        for r in range(len(chain)):
            self.mm[r, 0] = (1 << (r + 1)) - 1
        B, K, V = w.B, w.K, w.V
        self.scale = {
            "heads": K * V / self.rows_v, "tree_build": 1.0,
            "attention": B * N / len(chain) * (float(np.mean(self.P)) + N / 2)
            / (float(self.P[self.b0]) + len(chain) / 2),
            "verify": B * N / 8, "kv_compact": float(B)}

    def run(self):
        """Time the oracle on the sample once: (measured seconds, extrapolated
        seconds of one whole step, extrapolated seconds per stage)."""
        from oracle import medusa_oracle as O

        w, spec, N = self.w, self.spec, self.N
        t = {}
        t0 = time.perf_counter()
        z = O.head_logits(self.h, self.W1, self.b1, self.W2)
        O.topk(z, w.kmax)
        t["heads"] = time.perf_counter() - t0
        t0 = time.perf_counter()
        ids = np.zeros((w.B, w.K, w.kmax), dtype=np.int64)
        O.tree_build(spec.parent, spec.depth, spec.rank, np.zeros(w.B, np.int64), ids, self.P)
        t["tree_build"] = time.perf_counter() - t0
        t0 = time.perf_counter()
        b0, ch = self.b0, self.chain
        O.tree_attention(self.q[:, ch], self.kn[:, ch], self.vn[:, ch], self.Kc, self.Vc,
                         self.P[b0:b0 + 1], self.mm, 1.0 / math.sqrt(w.dh))
        t["attention"] = time.perf_counter() - t0
        t0 = time.perf_counter()
        O.row_argmax(self.logits[:, :8])
        if w.accept == "typical":  # a 9-node chain: statistics of its first 8 rows
            O.typical_log_margin(self.logits, np.zeros((1, 9), np.int64), np.arange(-1, 8),
                                 w.temperature, w.eps, w.delta)
        t["verify"] = time.perf_counter() - t0
        t0 = time.perf_counter()
        nodes = np.full((1, spec.max_depth + 1), -1, dtype=np.int64)
        nodes[0, 0] = 0
        O.kv_compact(self.Kc, self.Vc, self.P[b0:b0 + 1], nodes, np.array([0]))
        t["kv_compact"] = time.perf_counter() - t0
        measured = sum(t.values())
        stages = {k: v * self.scale[k] for k, v in t.items()}
        return measured, sum(stages.values()), stages

    def describe(self) -> str:
        w = self.w
        return (f"head 0 on {self.rows_v} of {w.V} vocab rows x {w.B} sequences "
                f"(x{self.scale['heads']:.1f}); {len(self.chain)} query nodes x {w.Hq} heads of "
                f"one sequence (x{w.B * self.N / len(self.chain):.0f}, scaled by mean prefix); "
                f"verify stats of 8 rows (x{self.scale['verify']:.0f}); tree build and "
                f"compaction in full; fp64 numpy")


def oracle_sample(w, n_nodes=None, seed=0, frac=1.0):
    """One timed oracle sample of a step: extrapolated seconds per step, the
    measured seconds, stages, threads used and the sample's description."""
    s = OracleSample(w, n_nodes, seed, frac)
    measured, sec, stages = s.run()
    return {"seconds_per_step": sec, "sample_s": measured, "stages": stages,
            "cores": _oracle_threads(), "sample": s.describe(),
            "scale": sec / measured if measured > 0 else None}


def single_core_figures():
    """Steps/s of the oracle on one host thread (Tiny and Vicuna-7B shapes,
    bounded samples as above)."""
    from threadpoolctl import threadpool_limits

    from speculative_decoding_medusa_b200 import workloads as W
    out = {}
    with threadpool_limits(limits=1):
        for name in ("tiny", "vicuna7b"):
            r = oracle_sample(W.WORKLOADS[name])
            out[name] = {"value": 1.0 / r["seconds_per_step"], "unit": UNIT, "cores": 1,
                         "sample_s": r["sample_s"]}
    return out


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------
def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama3_8b")
    ap.add_argument("--nodes", type=int, default=None, help="tree size override (long: 16/64/128)")
    ap.add_argument("--batch", type=int, default=None, help="batch override (llama3_8b: 1..8)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--loop-steps", type=int, default=16,
                    help="decode steps per CUDA graph (--stage loop)")
    ap.add_argument("--stage", choices=["all", "attention", "verify", "lmhead", "loop"],
                    default="all",
                    help="time one stage alone (profiling aid; prints a stage line, not the metric)")
    return ap.parse_args()


def run_loop(args):
    """Decode steps chained on the device and replayed from one CUDA graph:
    heads -> tree -> (synthetic base model: node hidden states) -> tree
    attention -> lm_head verify -> KV compaction -> next step.  Reports
    tokens per second (kept candidates + the bonus token, all sequences)
    with the mean accept_len the synthetic base model produced."""
    import math
    import speculative_decoding_medusa_b200 as M
    from speculative_decoding_medusa_b200 import workloads as W
    from speculative_decoding_medusa_b200.step import DecodeLoop

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workload_of(args, W)
    R = args.loop_steps
    spec = W.tree_for(w)
    N = spec.n_nodes
    tree = M.Tree.from_spec(spec, dev)
    heads = W.heads_inputs(w, seed=0, device=dev)
    max_prefix = w.ctx_hi + R * (spec.max_depth + 1)
    cap = max_prefix + N
    att = W.attention_inputs(W.scaled(w, ctx_hi=cap - N), seed=0, device=dev, n_nodes=N)
    p0 = W.prefix_lengths(w, seed=0, device=dev)
    lm = W.randn((w.V, w.d), 0, 77, 1.0 / math.sqrt(w.d), "bf16", dev)
    bm = W.SyntheticBaseModel(w, spec, lm, R, seed=0, device=dev)
    loop = DecodeLoop(B=w.B, d=w.d, V=w.V, K=w.K, kmax=w.kmax, tree=tree, Hq=w.Hq, Hkv=w.Hkv,
                      dh=w.dh, cap=cap, max_prefix=max_prefix, steps=R, accept=w.accept,
                      temperature=w.temperature, eps=w.eps, delta=w.delta, device=dev)
    h0 = heads["h"].clone()
    r0 = W.random_root_tokens(w, 0, device=dev)
    h, root, pl = h0.clone(), r0.clone(), p0.clone()

    def reset():
        h.copy_(h0)
        root.copy_(r0)
        pl.copy_(p0)

    def steps():
        for r in range(R):
            loop.step(r, h, root, heads["W1"], heads["b1"], heads["W2"], lm, bm, att["q"],
                      att["k_new"], att["v_new"], att["Kc"], att["Vc"], pl)

    reset()
    steps()  # eager warm-up (first-call setup outside the capture)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            steps()
    torch.cuda.current_stream().wait_stream(side)
    times, toks = [], []
    for i in range(max(args.warmup, 3) + args.steps):
        reset()
        loop.status.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        assert int(loop.status.item()) == 0, int(loop.status.item())
        if i >= max(args.warmup, 3):
            times.append(e0.elapsed_time(e1) / 1e3)
            toks.append(int(loop.history.sum()) + R * w.B)
    del graph
    sec = sum(times)
    line = {"stage": "loop", "workload": args.workload, "n_nodes": N, "steps_per_graph": R,
            "graphs": len(times), "us_per_step": sec / (len(times) * R) * 1e6,
            "tokens_per_s": sum(toks) / sec,
            "mean_accept_len": (sum(toks) - len(times) * R * w.B) / (len(times) * R * w.B),
            "tokens_per_step_per_seq": sum(toks) / (len(times) * R * w.B),
            "base_model": "synthetic node hidden states (p_match %.2f planted matches)" % w.p_match}
    print(json.dumps(line))
    return 0


def run_stage(args):
    """One stage in a loop on the workload's inputs (for per-kernel timing
    and profiling): tree attention or verify/accept."""
    import speculative_decoding_medusa_b200 as M
    from speculative_decoding_medusa_b200 import workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workload_of(args, W)
    N = w.N
    spec = W.tree_for(w, n_nodes=N)
    tree = M.Tree.from_spec(spec, dev)
    att = W.attention_inputs(w, seed=0, device=dev, n_nodes=N)
    root = W.random_root_tokens(w, 0, device=dev)
    topk = W.random_topk_ids(w, 0, device=dev)
    i32 = dict(dtype=torch.int32, device=dev)
    cand = torch.empty(w.B, N, **i32)
    pos = torch.empty(w.B, N, **i32)
    mask = torch.empty(N, (N + 31) // 32, **i32)
    retrieve = torch.empty(spec.n_leaves, spec.max_depth + 1, **i32)
    status = M.new_status(dev)
    M.medusa_tree_build(tree, root, topk, att["prefix_len"], cand, pos, mask, retrieve, status)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    if args.stage == "attention":
        out = torch.empty(w.B, N, w.Hq, w.dh, dtype=dt, device=dev)
        ws = M.workspace(M.medusa_tree_attention_workspace_size(
            w.B, N, w.Hq, w.Hkv, w.dh, w.ctx_hi, M.MEDUSA_BF16 if dt == torch.bfloat16 else M.MEDUSA_F32), dev)
        fn = lambda: M.medusa_tree_attention(att["q"], att["k_new"], att["v_new"], att["Kc"], att["Vc"],
                                             att["prefix_len"], mask, w.ctx_hi, out, None, ws, status)
        e = 2 if dt == torch.bfloat16 else 4
        P = att["prefix_len"].tolist()
        nbytes = (sum(P) * w.Hkv * w.dh * 2 + w.B * N * (2 * w.Hq + 4 * w.Hkv) * w.dh) * e
        flops = 4.0 * w.Hq * w.dh * N * sum(p + N for p in P)
    elif args.stage == "lmhead":
        # verification from the nodes' hidden states: lm_head GEMM + reduction
        hidden, lm = W.lmhead_inputs(w, spec, cand.cpu(), seed=0, device=dev)
        Wd = spec.max_depth + 1
        outs = [torch.empty(w.B, **i32), torch.empty(w.B, Wd, **i32), torch.empty(w.B, Wd, **i32),
                torch.empty(w.B, **i32)]
        ws = M.workspace(M.medusa_lmhead_verify_workspace_size(w.B, N, w.d, w.V), dev)
        mode = M.MEDUSA_ACCEPT_TYPICAL if w.accept == "typical" else M.MEDUSA_ACCEPT_GREEDY
        fn = lambda: M.medusa_lmhead_verify(hidden, lm, cand, tree, *outs, mode, w.temperature,
                                            w.eps, w.delta, ws=ws, dev_status=status)
        nbytes = (w.V * w.d + w.B * N * w.d) * 2
        flops = 2.0 * w.B * N * w.V * w.d
    else:
        torch.cuda.synchronize()
        logits = W.verify_logits(w, spec, cand, seed=0, device=dev)
        Wd = spec.max_depth + 1
        outs = [torch.empty(w.B, **i32), torch.empty(w.B, Wd, **i32), torch.empty(w.B, Wd, **i32),
                torch.empty(w.B, **i32)]
        ws = M.workspace(M.medusa_verify_accept_workspace_size(w.B, N, w.V), dev)
        mode = M.MEDUSA_ACCEPT_TYPICAL if w.accept == "typical" else M.MEDUSA_ACCEPT_GREEDY
        fn = lambda: M.medusa_verify_accept(logits, cand, tree, *outs, mode, w.temperature, w.eps,
                                            w.delta, ws, status)
        nbytes = logits.numel() * logits.element_size()
        flops = 0.0
    for _ in range(max(args.warmup, 3)):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, int(status.item())
    us = e0.elapsed_time(e1) * 1e3 / args.steps
    hbm, tflops, kind = _peaks()
    line = {"stage": args.stage, "workload": args.workload, "n_nodes": N, "us_per_call": us,
            "algorithmic_bytes": nbytes, "achieved_gbs": nbytes / us / 1e3,
            "hbm_frac": nbytes / us / 1e3 / hbm, "tflops": flops / us / 1e6,
            "tensor_frac": flops / us / 1e6 / tflops if flops else None, "peaks": kind}
    print(json.dumps(line))
    return 0


def run_reference(args):
    """The CPU oracle as the reference arm: warmup + steps timed samples of
    the workload's step, each extrapolated to the whole step.  ms_per_step is
    what was measured (oracle seconds of one sample); value is the
    extrapolated whole-step rate; the sample is sized so the whole run takes
    a few minutes at most."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from speculative_decoding_medusa_b200 import workloads as W
    w = workload_of(args, W)
    N = w.N
    n_total = args.warmup + args.steps
    # size the sample: one full sample first (untimed), then shrink the
    # vocabulary slice so that all steps take about 120 s of oracle time
    probe = OracleSample(w, N, seed=0)
    t_full, _, _ = probe.run()
    frac = min(1.0, 120.0 / max(n_total * t_full, 1e-9))
    sample = OracleSample(w, N, seed=0, frac=frac) if frac < 1.0 else probe
    measured, extrap = [], []
    for i in range(n_total):
        m, sec, _ = sample.run()
        if i >= args.warmup:
            measured.append(m)
            extrap.append(sec)
    sec = statistics.mean(extrap)
    value = 1.0 / sec
    sample_s = statistics.mean(measured)
    cores = _oracle_threads()
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference",
            "n_gpus": args.gpus, "steps": len(measured), "warmup": args.warmup,
            "ms_per_step": sample_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "value_basis": "extrapolated: each timed step is a bounded sample of the step "
                           "(ms_per_step = its measured oracle time), scaled to the whole step",
            "sample_s": sample_s, "scale": sec / sample_s if sample_s > 0 else None,
            "ms_per_step_extrapolated": sec * 1e3,
            "config": {"workload": args.workload, "global_batch": w.B, "n_nodes": N,
                       "prefix": [w.ctx_lo, w.ctx_hi], "parallelism": "none (CPU oracle)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample.describe(), "cpu_model": _cpu_model(),
                             "sample_s": sample_s},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.stage == "loop":
        return run_loop(args)
    if args.stage != "all":
        return run_stage(args)

    import speculative_decoding_medusa_b200 as M
    from speculative_decoding_medusa_b200 import workloads as W
    from speculative_decoding_medusa_b200.step import DecodeVerifyStep

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    M.lib()  # fails loudly when the library is missing

    w = workload_of(args, W)
    N = w.N
    spec = W.tree_for(w, n_nodes=N)
    seed = rank
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    # weights and caches drawn on the device (seeded); parity is tested elsewhere
    hin = W.heads_inputs(w, seed=seed, device=dev)
    att = W.attention_inputs(w, seed=seed, device=dev, n_nodes=N)
    root = W.random_root_tokens(w, seed, device=dev)
    tree = M.Tree.from_spec(spec, dev)
    step = DecodeVerifyStep(B=w.B, d=w.d, V=w.V, K=w.K, kmax=w.kmax, tree=tree, Hq=w.Hq, Hkv=w.Hkv,
                            dh=w.dh, cap=w.cap, max_prefix=w.ctx_hi, dtype=dt, accept=w.accept,
                            temperature=w.temperature, eps=w.eps, delta=w.delta, device=dev)
    # candidates of this batch -> verify logits that agree with some of them
    M.medusa_heads_topk(hin["h"], hin["W1"], hin["b1"], hin["W2"], w.kmax, step.topk_ids,
                        step.topk_vals, None, step.ws_heads, step.status)
    M.medusa_tree_build(tree, root, step.topk_ids, att["prefix_len"], step.cand_ids, step.pos_ids,
                        step.anc_mask, step.retrieve, step.status)
    torch.cuda.synchronize()
    logits = W.verify_logits(w, spec, step.cand_ids, seed=seed, device=dev)
    prefix0 = att["prefix_len"].clone()
    prefix_list = prefix0.tolist()
    stream = torch.cuda.current_stream()

    def one_step(evs=None):
        att["prefix_len"].copy_(prefix0)  # same prefixes every step
        if evs is None:
            step.run(hin["h"], hin["W1"], hin["b1"], hin["W2"], root, att["q"], att["k_new"],
                     att["v_new"], att["Kc"], att["Vc"], att["prefix_len"], logits)
            return
        evs[0].record(stream)
        M.medusa_heads_topk_tree(hin["h"], hin["W1"], hin["b1"], hin["W2"], w.kmax, step.topk_ids,
                                 step.topk_vals, tree, root, att["prefix_len"], step.cand_ids,
                                 step.pos_ids, step.anc_mask, step.retrieve, None, step.ws_heads,
                                 step.status)
        evs[1].record(stream)
        M.medusa_tree_attention(att["q"], att["k_new"], att["v_new"], att["Kc"], att["Vc"],
                                att["prefix_len"], step.anc_mask, w.ctx_hi, step.attn_out, None,
                                step.ws_attn, step.status)
        evs[2].record(stream)
        M.medusa_verify_accept_compact(logits, step.cand_ids, tree, step.accept_len,
                                       step.accepted_nodes, step.accepted_tokens, step.bonus,
                                       att["Kc"], att["Vc"], att["prefix_len"], step.compact_src,
                                       step.mode, w.temperature, w.eps, w.delta, step.ws_verify,
                                       step.status)
        evs[3].record(stream)

    for _ in range(max(args.warmup, 3)):
        one_step()
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0, f"device status {int(step.status.item())}"

    sampler = ClockSampler(_gpu_index(local_rank))
    time.sleep(0.2)
    # ---- timed region: K steps through the product path (no events between
    # the calls: an event record between two kernels stops the second from
    # being launched while the first drains) ----
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(args.steps):
        one_step()
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    ms_total = t_start.elapsed_time(t_end)
    if world > 1:
        tt = torch.tensor([ms_total], device=dev, dtype=torch.float64)
        torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
        ms_total = float(tt.item())
    ms_step = ms_total / args.steps
    # stage breakdown from a separate, untimed pass with events between the calls
    n_stage = min(args.steps, 50)
    stage_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_stage)]
    for k in range(n_stage):
        one_step(stage_evs[k])
    torch.cuda.synchronize()
    names = ["heads_topk_tree", "tree_attention", "verify_accept_compact"]
    stages = {n: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in stage_evs) * 1e3
              for i, n in enumerate(names)}  # us
    assert int(step.status.item()) == 0

    # ---- the step captured in one CUDA graph and replayed: per-step
    # percentiles (an event between replays) ----
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            one_step()
    stream.wait_stream(side)
    n_rep = min(max(args.steps, 20), 200)
    rep_evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_rep + 1)]
    for _ in range(3):
        graph.replay()
    rep_evs[0].record(stream)
    for k in range(n_rep):
        graph.replay()
        rep_evs[k + 1].record(stream)
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    per_step = sorted(rep_evs[k].elapsed_time(rep_evs[k + 1]) * 1e3 for k in range(n_rep))
    step_us = {"graph": True, "replays": n_rep, "p10": per_step[n_rep // 10],
               "p50": per_step[n_rep // 2], "p90": per_step[(9 * n_rep) // 10]}
    del graph

    # ---- end to end through the public API with host buffers ----
    host_in = {k: v.cpu().pin_memory() for k, v in
               {"h": hin["h"], "root": root, "q": att["q"], "k_new": att["k_new"],
                "v_new": att["v_new"], "logits": logits, "prefix_len": prefix0}.items()}
    dev_in = {"h": hin["h"], "root": root, "q": att["q"], "k_new": att["k_new"],
              "v_new": att["v_new"], "logits": logits, "prefix_len": att["prefix_len"]}
    host_out = {k: torch.empty_like(getattr(step, k), device="cpu").pin_memory()
                for k in ("accept_len", "accepted_tokens", "bonus", "compact_src")}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())

    # Two device copies of the step inputs: the inputs of step i + 1 are
    # uploaded on a copy stream while step i runs (as a server stages its next
    # batch), and a slot is overwritten only once the step that read it is
    # done.  Every step's upload, kernels and result read-back are inside the
    # timed region; the first upload is not overlapped.
    copy_stream = torch.cuda.Stream()
    dev_sets = [dev_in, {k: torch.empty_like(v) for k, v in dev_in.items()}]
    uploaded = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]

    def upload(slot):
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(consumed[slot])
            for k, t in host_in.items():
                dev_sets[slot][k].copy_(t, non_blocking=True)
            uploaded[slot].record(copy_stream)

    def e2e_run(n):
        copy_stream.wait_stream(stream)
        upload(0)
        for i in range(n):
            slot = i % 2
            if i + 1 < n:
                upload(1 - slot)
            stream.wait_event(uploaded[slot])
            d = dev_sets[slot]
            step.run(d["h"], hin["W1"], hin["b1"], hin["W2"], d["root"], d["q"], d["k_new"],
                     d["v_new"], att["Kc"], att["Vc"], d["prefix_len"], d["logits"])
            consumed[slot].record(stream)
            for k, t in host_out.items():
                t.copy_(getattr(step, k), non_blocking=True)

    e2e_run(3)
    torch.cuda.synchronize()
    n_e2e = max(1, args.e2e_steps)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(n_e2e)
    e1.record(stream)
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    ms_e2e = e0.elapsed_time(e1)
    if world > 1:
        tt = torch.tensor([ms_e2e], device=dev, dtype=torch.float64)
        torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
        ms_e2e = float(tt.item())
    e2e_value = world * n_e2e / (ms_e2e / 1e3)

    # ---- roofline of the dominant call (heads + top-k with the tree build: W1 + W2 weight stream) ----
    hbm_peak, _, peak_kind = _peaks()
    ab = algorithmic_bytes(w, prefix_list, N)
    heads_gbs = ab["heads"] / (stages["heads_topk_tree"] * 1e-6) / 1e9
    traffic, traffic_src = heads_traffic(ab["heads"])
    step_gbs = ab["total"] / (ms_step * 1e-3) / 1e9
    value = world * args.steps / (ms_total / 1e3)
    # tree attention (attention kernel + combine): HBM and tensor rooflines
    _, tc_peak, _ = _peaks()
    attn_s = stages["tree_attention"] * 1e-6
    attn_flops = 4.0 * w.Hq * w.dh * N * sum(P + N for P in prefix_list)
    attention = {"us": stages["tree_attention"], "bytes": ab["attention"], "flops": attn_flops,
                 "achieved_gbs": ab["attention"] / attn_s / 1e9,
                 "frac_hbm": ab["attention"] / attn_s / 1e9 / hbm_peak,
                 "achieved_tflops": attn_flops / attn_s / 1e12,
                 "frac_tensor": attn_flops / attn_s / 1e12 / tc_peak,
                 "peaks": f"{peak_kind} hbm_gbs {hbm_peak:.0f}, bf16_tflops {tc_peak:.0f} (burst)",
                 "flops_def": "4 Hq dh N sum_b (P_b + N): QK and PV over prefix and tree tiles"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = oracle_sample(w, N)
        cpu = {"value": 1.0 / r["seconds_per_step"], "unit": UNIT, "cores": r["cores"],
               "kind": "oracle", "sample": r["sample"], "sample_s": r["sample_s"],
               "scale": r["scale"], "basis": "extrapolated from the timed sample",
               "cpu_model": _cpu_model(), "single_core": single_core_figures()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if dt == torch.bfloat16 else "f32",
            "data": "synthetic (seeded, on-device draws of the workload's shapes; random weights)",
            "config": {"workload": args.workload, "global_batch": w.B * world, "batch_per_gpu": w.B,
                       "hidden": w.d, "vocab": w.V, "heads": w.K, "kmax": w.kmax, "n_nodes": N,
                       "attn_heads": [w.Hq, w.Hkv, w.dh], "prefix": [w.ctx_lo, w.ctx_hi],
                       "accept": w.accept, "parallelism": f"dp{world} (independent batches)",
                       "l2": "no flush: each step streams ~%.2f GB (> 126 MB L2)" % (ab["total"] / 1e9)},
            "hbm_roofline_frac_step": step_gbs / hbm_peak,
            "step_bytes": ab["total"],
            "stages_us": stages,
            "step_us": step_us,
            "roofline": {"bound": "hbm", "kernel": "medusa_heads_topk_tree (W1 GEMM + W2 GEMM + top-k merge with the tree build)",
                         "achieved": heads_gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": heads_gbs / hbm_peak, "traffic": traffic,
                         "traffic_source": "ncu dram bytes ratio, " + traffic_src,
                         "peak_source": f"{peak_kind} hbm_gbs", "algorithmic_bytes": ab["heads"]},
            "attention": attention,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": n_e2e,
                    "overlap": "step i+1 inputs uploaded during step i"},
            "gpu_launches": KERNELS_PER_STEP * args.steps,
            "clocks": clocks,
            "mean_accept_len": float(step.accept_len.float().mean().item()),
        }
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
