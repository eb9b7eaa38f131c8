#!/usr/bin/env python
"""Benchmark of the DSA hot path (Lightning Indexer -> Top-K -> sparse MLA).

Default workload: decode, batch 32 x 8192 context, one new token each
(H_I=64, d_I=128, K=2048, 128 MLA heads, 512+64 latent dims, BF16), timed as
one ``dsa_fused_decode`` call per step through the C ABI. Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config c2|c3|c4|c5]
  python bench.py --impl reference ...     # the CPU oracle, timed on host cores

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a
device synchronize, timed with CUDA events on the launch stream; max over
ranks. Each step reads one of 4 rotating input copies (all caches and
queries), 1.5 GB in total for the default workload, so no step finds its
inputs in the 126 MB L2. Per-kernel times come from events the fused call
records on its stream between its stages.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DSA query tokens/sec (indexer+TopK+sparse MLA) at 32×8K decode; % HBM roofline"
UNIT = "query_tokens/s"
FALLBACK_HBM_GBS = 6650.0

WORKLOAD_TEXT = {
    "c2": "decode: batch 32 x 8192 context, 1 query each; H_I=64 d_I=128 BF16 index keys; K=2048; "
          "128 MLA heads, d_c=512 + d_rope=64 BF16",
    "c3": "ragged decode: batch 64, context U[1024,65536]; FP8 E4M3 index keys (per-key fp32 scale); K=2048; "
          "128 MLA heads, 576-dim BF16 latent rows",
    "c4": "causal prefill: 1 x 32768 tokens; H_I=64 d_I=128 BF16; K=2048; 128 MLA heads, 576/512 dims",
    "c5": "chunked prefill: 4 x (131072 prefix + 8192 chunk); FP8 index keys; K=2048; 128 MLA heads",
}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(wl, n_selected: int):
    """Bytes each stage must move at least once (inputs read + outputs written).

    indexer: index-key rows of every causal candidate, q_I, w, the fp32 score row
    written and read back by the Top-K; attention: the selected latent rows
    (D bf16 each), q, idx and the bf16 output."""
    nv = wl.n_valid().astype(np.int64)
    key_row = wl.dI * (1 if wl.key_dtype == "fp8" else 2) + (4 if wl.key_dtype == "fp8" else 0)
    # distinct key rows read: every sequence's rows up to its longest causal history
    b = wl.seq_of_token()
    rows_per_seq = np.zeros(wl.B, np.int64)
    np.maximum.at(rows_per_seq, b, nv)
    idx_bytes = int(rows_per_seq.sum()) * key_row + wl.T * wl.HI * wl.dI * 2 + wl.T * wl.HI * 4
    scores = int(nv.sum()) * 4
    attn = n_selected * wl.D * 2 + wl.T * wl.H * wl.D * 2 + wl.T * wl.K * 4 + wl.T * wl.H * wl.dc * 2
    return {"indexer": idx_bytes + scores, "topk": scores + wl.T * wl.K * 4, "sparse_mla": attn,
            "step": idx_bytes + attn}


class ClockSampler:
    """SM clock, power and clock-event reasons sampled during the timed region.

    Reads (never sets) NVML in a background thread every 2 ms, so even a
    few-millisecond timed region gets samples; falls back to polling
    nvidia-smi when NVML is unavailable."""

    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device):
        self.dev = torch_device
        self.samples = []
        self.stop = False
        self.thread = None
        self.handle = None
        self.error = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            pr = torch.cuda.get_device_properties(self.dev)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons

            def loop():
                while not self.stop:
                    try:
                        self.samples.append((pynvml.nvmlDeviceGetClockInfo(self.handle, pynvml.NVML_CLOCK_SM),
                                             pynvml.nvmlDeviceGetPowerUsage(self.handle) / 1000.0,
                                             int(get_reasons(self.handle))))
                    except Exception as e:  # keep sampling; record the first problem
                        self.error = self.error or repr(e)
                    time.sleep(0.002)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
        except Exception as e:
            self.error = repr(e)
        return self

    def __exit__(self, *a):
        self.stop = True
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": self.error}
        seen = sorted({name for _, _, r in self.samples for bit, name in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(c for c, _, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": seen, "samples": len(self.samples),
                "power_w_max": max(p for _, p, _ in self.samples)}


def run_cpu_oracle(wl, n_tokens: int, seed: int = 0, min_seconds: float = 0.0):
    """Time the fp64 oracle (indexer + Top-K + attention) on n_tokens sampled
    query tokens of the workload, repeated until at least min_seconds of CPU
    work have been timed. Returns (tokens processed, seconds, threads)."""
    import oracle
    from indexed_sparse_attention_relu_b200 import workloads as W
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(wl.T, size=min(n_tokens, wl.T), replace=False))
    sub, rows = W.restrict(wl, rows)
    kw = {}
    if wl.key_dtype == "fp8":
        codes, scales = oracle.quantize_keys(sub.k_idx, sub.scale_group)
        kw = dict(k_codes=codes, k_scales=scales)
    done, dt = 0, 0.0
    while done == 0 or dt < min_seconds:
        t0 = time.perf_counter()
        oracle.dsa(sub, **kw)
        dt += time.perf_counter() - t0
        done += len(rows)
    return done, dt, oracle.num_threads()


def reference_arm(args, rank: int):
    """The base contract's reference arm, here the CPU oracle timed on host cores."""
    if rank != 0:
        return
    from indexed_sparse_attention_relu_b200 import workloads as W
    wl = W.make(args.config, with_caches=False)
    per_step = max(1, args.ref_tokens)
    for _ in range(args.warmup if args.warmup < 2 else 1):
        run_cpu_oracle(wl, 1, seed=999)
    tok, sec = 0, 0.0
    threads = 1
    for s in range(args.steps):
        n, dt, threads = run_cpu_oracle(wl, per_step, seed=s)
        tok += n
        sec += dt
    value = tok / sec
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sec / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.config], "name": args.config},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{per_step} query token(s) per step, full causal history, fp64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="c2", choices=sorted(WORKLOAD_TEXT))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--copies", type=int, default=4, help="rotating input copies (L2 defeat)")
    ap.add_argument("--cpu-tokens", type=int, default=8, help="query tokens in the oracle baseline sample")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="minimum CPU time of the oracle baseline")
    ap.add_argument("--ref-tokens", type=int, default=1, help="query tokens per reference-arm step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager launches instead of one CUDA graph")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        reference_arm(args, rank)
        return

    import torch
    import torch.distributed as dist
    from indexed_sparse_attention_relu_b200 import binding as B
    from indexed_sparse_attention_relu_b200 import build as build_mod
    from indexed_sparse_attention_relu_b200 import device as DV
    from indexed_sparse_attention_relu_b200 import multi
    from indexed_sparse_attention_relu_b200 import workloads as W

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    build_mod.build()
    B.load()

    # ---- inputs: one workload, cloned into rotating copies on the device
    wl = W.make(args.config, with_caches=False)
    base = DV.to_device(wl, dev)
    copies = [base]
    for _ in range(args.copies - 1):
        c = DV.DeviceWorkload(wl, base.batch, base.q_idx.clone(), base.w.clone(), base.k_cache.clone(),
                              None if base.k_scale is None else base.k_scale.clone(), None, base.q.clone(),
                              base.kv.clone())
        copies.append(c)
    T, K = wl.T, wl.K
    stream = torch.cuda.current_stream(dev)
    outs = [torch.empty((T, wl.H, wl.dc), dtype=torch.bfloat16, device=dev) for _ in copies]
    lses = [torch.empty((T, wl.H), dtype=torch.float32, device=dev) for _ in copies]
    ws_bytes = B.dsa_workspace_size(B.DSA_OP_FUSED_DECODE, base.batch, K)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    idx_in = [c.indexer_in() for c in copies]
    mla_in = [c.mla_in() for c in copies]

    def step(i, events=None, st=None):
        j = i % len(copies)
        B.dsa_fused_decode(copies[j].batch, idx_in[j], mla_in[j], K, outs[j], lses[j], None, ws, ws_bytes,
                           stage_events=events, stream=stream if st is None else st)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    status = B.dsa_read_device_status(stream)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    for e in [x for row in ev for x in row] + [t_start, t_end]:
        e.record(stream)            # creates the CUDA events outside the timed region
    torch.cuda.synchronize(dev)
    # The K timed steps are captured once as one CUDA graph and replayed once,
    # so host launch overhead cannot hide in the device time (every call of
    # the library is capture-safe: no allocation, no synchronisation).
    graph = None
    timing_mode = "eager"
    if not args.eager:
        try:
            graph = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream(dev)
            with torch.cuda.graph(graph, stream=cap):
                for i in range(args.steps):
                    step(i, None, st=cap)
            timing_mode = "cuda_graph"
        except Exception as e:  # report and fall back to eager launches
            graph = None
            timing_mode = f"eager (graph capture failed: {type(e).__name__})"
            torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    # timed region: K steps exactly as a caller runs them (programmatic launch
    # between the kernels, no events in between)
    with ClockSampler(dev) as clocks:
        t_start.record(stream)
        if graph is not None:
            graph.replay()
        else:
            for i in range(args.steps):
                step(i)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    # per-kernel durations: a second pass of K steps, launched eagerly with an
    # event recorded on the launch stream right before and after each stage
    # (events inside a graph cannot be timed; an event between two kernels also
    # turns the programmatic launch off on that edge)
    for i in range(args.steps):
        step(i, ev[i])
    torch.cuda.synchronize(dev)
    stage_ms = {
        "indexer": statistics.mean(e[0].elapsed_time(e[1]) for e in ev),
        "topk": statistics.mean(e[1].elapsed_time(e[2]) for e in ev),
        "sparse_mla": statistics.mean(e[2].elapsed_time(e[3]) for e in ev),
    }
    # the job's time is its slowest rank's; every rank ran its own T queries
    total_ms = multi.max_over_ranks(total_ms, dist if world > 1 else None, dev)
    ms_per_step = total_ms / args.steps
    value = multi.job_throughput([T] * world, ms_per_step)

    # ---- end to end through the C ABI with host buffers (pinned), copies timed
    h_qidx = base.q_idx.cpu().pin_memory()
    h_w = base.w.cpu().pin_memory()
    h_q = base.q.cpu().pin_memory()
    h_out = torch.empty(outs[0].shape, dtype=torch.bfloat16).pin_memory()
    h2d = h_qidx.numel() * 2 + h_w.numel() * 4 + h_q.numel() * 2
    d2h = h_out.numel() * 2

    def e2e_step(i):
        j = i % len(copies)
        c = copies[j]
        c.q_idx.copy_(h_qidx, non_blocking=True)
        c.w.copy_(h_w, non_blocking=True)
        c.q.copy_(h_q, non_blocking=True)
        B.dsa_fused_decode(c.batch, idx_in[j], mla_in[j], K, outs[j], lses[j], None, ws, ws_bytes, stream=stream)
        h_out.copy_(outs[j], non_blocking=True)

    for i in range(max(3, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / args.steps
    e2e_ms = multi.max_over_ranks(e2e_ms, dist if world > 1 else None, dev)
    status2 = B.dsa_read_device_status(stream)

    # ---- roofline of the dominant stage
    n_sel = int(np.minimum(wl.n_valid(), K).sum())
    algo = algorithmic_bytes(wl, n_sel)
    dom = max(stage_ms, key=stage_ms.get)
    peak, peak_kind = _peaks()
    achieved = algo[dom] / (stage_ms[dom] * 1e-3) / 1e9
    step_gbs = algo["step"] / (ms_per_step * 1e-3) / 1e9
    # DRAM bytes per launch of the dominant kernel from the committed ncu
    # capture, used only while the kernel's sources are the ones it measured
    traffic = None
    prof = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if os.path.exists(prof):
        try:
            rec = json.load(open(prof)).get(dom)
            if rec and rec.get("workload") == args.config:
                h = hashlib.sha256()
                for src in rec["sources"]:
                    h.update(open(os.path.join(ROOT, src), "rb").read())
                if h.hexdigest() == rec["sources_sha256"]:
                    traffic = rec["dram_bytes_read"] + rec["dram_bytes_write"]
        except (OSError, KeyError, ValueError):
            traffic = None

    # kernels launched per step: indexer, Top-K, attention (split partials merge
    # inside a cluster, so there is no separate combine launch)
    launches_per_step = 3

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.config], "name": args.config, "B": wl.B, "L_max": wl.Lmax,
                   "T": T, "K": K, "H_I": wl.HI, "d_I": wl.dI, "H": wl.H, "d_c": wl.dc, "d_rope": wl.dr,
                   "index_keys": wl.key_dtype, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"{len(copies)} rotating input copies "
                         f"({len(copies) * (base.kv.numel() * 2 + base.k_cache.numel() * base.k_cache.element_size()) / 1e9:.2f} GB) > 126 MB L2"},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind, "traffic": traffic,
                     "algorithmic_bytes": algo[dom], "avg_launch_ms": stage_ms[dom]},
        "step_roofline": {"bound": "hbm", "achieved": step_gbs, "peak": peak, "unit": "GB/s",
                          "frac": step_gbs / peak, "frac_of_8TBps": step_gbs / 8000.0,
                          "algorithmic_bytes": algo["step"]},
        "stage_ms": stage_ms,
        "stage_ms_note": "second K-step pass, eager launches with CUDA events between the stages",
        "clocks": clocks.summary(),
        "e2e": {"value": world * T / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches_per_step * args.steps,
        "timing": timing_mode,
        "device_status": [status, status2],
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n, dt, thr = run_cpu_oracle(wl, args.cpu_tokens, min_seconds=args.cpu_seconds)
        line["cpu_baseline"] = {"value": n / dt, "unit": UNIT, "cores": thr, "kind": "oracle",
                                "sample": f"{min(args.cpu_tokens, wl.T)} query tokens of the same workload (full "
                                          f"causal history), fp64, repeated to {n} tokens in {dt:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
