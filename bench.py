#!/usr/bin/env python
"""Benchmark of the DSA hot path (Lightning Indexer -> Top-K -> sparse MLA).

Default workload: decode, batch 32 x 8192 context, one new token each
(H_I=64, d_I=128, K=2048, 128 MLA heads, 512+64 latent dims, BF16), timed as
one ``dsa_fused_decode`` call per step through the C ABI. Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config c2|c3|c4|c5] [--extra c3,c3mx,c2kv8,c2pg,c4,c5]
  python bench.py --impl reference ...     # the CPU oracle, timed on host cores

The JSON line's headline is the decode workload; ``configs`` adds one block
per extra workload (the ragged decode with FP8 or MXFP8 index inputs, the
decode over an FP8 latent KV cache or over paged caches against the HBM
roofline, the prefills against the dense tensor-core peak), each graph-timed
the same way.

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
    "c3mx": "ragged decode: batch 64, context U[1024,65536]; MXFP8 index queries and keys (E4M3, one E8M0 "
            "scale per 32 elements); K=2048; 128 MLA heads, 576-dim BF16 latent rows",
    "c2pg": "decode: batch 32 x 8192 context, 1 query each; H_I=64 d_I=128 BF16; K=2048; 128 MLA heads; "
            "paged caches (64-row pages in a shuffled pool, one block table)",
    "c2kv8": "decode: batch 32 x 8192 context, 1 query each; H_I=64 d_I=128 BF16 index keys; K=2048; "
             "128 MLA heads; FP8 latent KV cache (4 x 128-element tiles per token, fp32 scales, rope BF16: "
             "656-byte rows)",
}

# Workloads that are another one's inputs with the latent KV cache in FP8, or
# with MXFP8 index queries and keys.
FP8_KV = {"c2kv8": "c2"}
MX_INDEX = {"c3mx": "c3"}
PAGED = {"c2pg": "c2"}  # every cache in a pool of 64-row pages under a block table
# Ragged batches whose sequences are split across ranks (longest first, no
# exchange: sequences are independent); the others run one copy per rank.
SHARDED = ("c3",)


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _peak_tflops():
    """(burst, sustained) dense bf16 TFLOP/s measured on this machine, or the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 1590.0, 1400.0, "fallback"


def algorithmic_flops(wl, n_selected: int):
    """Tensor-core FLOPs each stage must do (2 per multiply-add): the indexer's
    q_I . k_I products over every causal candidate and head, and the attention's
    QK^T (D dims) and PV (d_c dims) over every selected row and head."""
    nv = wl.n_valid().astype(np.int64)
    idx = int(nv.sum()) * wl.HI * wl.dI * 2
    attn = int(n_selected) * wl.H * (wl.D + wl.dc) * 2
    return {"indexer": idx, "sparse_mla": attn, "step": idx + attn}


def algorithmic_bytes(wl, n_selected: int, kv_row_bytes: int | None = None, key_row_bytes: int | None = None):
    """Bytes each stage must move at least once (inputs read + outputs written).

    indexer: index-key rows of every causal candidate, q_I, w, the fp32 score row
    written and read back by the Top-K; attention: the selected latent rows
    (D bf16 each, or kv_row_bytes for an FP8 cache), q, idx and the bf16 output."""
    nv = wl.n_valid().astype(np.int64)
    key_row = wl.dI * (1 if wl.key_dtype == "fp8" else 2) + (4 if wl.key_dtype == "fp8" else 0)
    if key_row_bytes is not None:  # MXFP8: codes + one scale byte per 32
        key_row = key_row_bytes
    # distinct key rows read: every sequence's rows up to its longest causal history
    b = wl.seq_of_token()
    rows_per_seq = np.zeros(wl.B, np.int64)
    np.maximum.at(rows_per_seq, b, nv)
    idx_bytes = int(rows_per_seq.sum()) * key_row + wl.T * wl.HI * wl.dI * 2 + wl.T * wl.HI * 4
    scores = int(nv.sum()) * 4
    row = wl.D * 2 if kv_row_bytes is None else kv_row_bytes
    attn = n_selected * row + wl.T * wl.H * wl.D * 2 + wl.T * wl.K * 4 + wl.T * wl.H * wl.dc * 2
    return {"indexer": idx_bytes + scores, "topk": scores + wl.T * wl.K * 4, "sparse_mla": attn,
            "step": idx_bytes + attn}


class ClockSampler:
    """SM clock, power and clock-event reasons sampled during the timed region.

    Reads (never sets) NVML in a background thread every 0.2 ms from before the
    timed region until after it; mark() brackets the region with host
    timestamps and summary() keeps only the samples taken inside it."""

    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device, period_s: float = 0.0002):
        self.dev = torch_device
        self.samples = []
        self.stop = False
        self.thread = None
        self.handle = None
        self.error = None
        self.period = period_s
        self.t0 = self.t1 = None
        self.max_mhz = None

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
            started = threading.Event()

            def loop():
                while not self.stop:
                    try:
                        self.samples.append((time.perf_counter(),
                                             pynvml.nvmlDeviceGetClockInfo(self.handle, pynvml.NVML_CLOCK_SM),
                                             pynvml.nvmlDeviceGetPowerUsage(self.handle) / 1000.0,
                                             int(get_reasons(self.handle))))
                    except Exception as e:  # keep sampling; record the first problem
                        self.error = self.error or repr(e)
                    started.set()
                    time.sleep(self.period)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            started.wait(timeout=2.0)   # the sampler is running before the region starts
        except Exception as e:
            self.error = repr(e)
        return self

    def mark(self, which: str):
        if which == "start":
            self.t0 = time.perf_counter()
        else:
            self.t1 = time.perf_counter()

    def __exit__(self, *a):
        time.sleep(2 * self.period)
        self.stop = True
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        inside = [s for s in self.samples
                  if self.t0 is None or self.t1 is None or self.t0 <= s[0] <= self.t1]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "note": self.error}
        seen = sorted({name for _, _, _, r in inside for bit, name in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(c for _, c, _, _ in inside), "sm_max_mhz": self.max_mhz,
                "reasons": seen, "samples": len(inside), "power_w_max": max(p for _, _, p, _ in inside)}


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


def _stage_events(B, steps):
    import torch
    return [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]


class Runner:
    """One workload resident on the device in rotating copies, run through
    dsa_fused_decode (the whole chain as one C-ABI call per step)."""

    def __init__(self, name, dev, copies, rank=0, world=1):
        import torch
        from indexed_sparse_attention_relu_b200 import binding as B
        from indexed_sparse_attention_relu_b200 import device as DV
        from indexed_sparse_attention_relu_b200 import workloads as W
        self.B = B
        wl = W.make(FP8_KV.get(name, MX_INDEX.get(name, PAGED.get(name, name))), with_caches=False)
        # tokens each rank processes per step (one full copy per rank unless sharded)
        self.units = [wl.T] * world
        if world > 1 and name in SHARDED:
            from indexed_sparse_attention_relu_b200 import multi
            shards = multi.shard_sequences(wl.seq_lens, world)
            self.units = [int(sum(wl.cu_q[b + 1] - wl.cu_q[b] for b in sh)) for sh in shards]
            wl = W.select_sequences(wl, shards[rank])
        self.wl = wl
        self.dev = dev
        base = DV.to_device(wl, dev, keep_bf16_keys=name in MX_INDEX)
        self.kv_row_bytes = None
        self.key_row_bytes = None
        if name in MX_INDEX:  # the library's MXFP8 quantisation of q_I and k_I, outside the timed region
            base = DV.with_mxfp8_index(base)
            self.key_row_bytes = wl.dI + wl.dI // 32
        if name in PAGED:
            base = DV.to_paged(base, 64, seed=wl.seed)
        if name in FP8_KV:  # the library's FP8 KV cache write, outside the timed region
            base = DV.with_fp8_kv(base)
            self.kv_row_bytes = B.dsa_kv_fp8_row_bytes(wl.dc, wl.dr)
        self.copies = [base]
        for _ in range(copies - 1):
            self.copies.append(DV.DeviceWorkload(wl, base.batch, base.q_idx.clone(), base.w.clone(),
                                                 base.k_cache.clone(),
                                                 None if base.k_scale is None else base.k_scale.clone(), None,
                                                 base.q.clone(), base.kv.clone(),
                                                 None if base.q_mx is None else base.q_mx.clone(),
                                                 None if base.k_mx is None else base.k_mx.clone()))
        T, K = wl.T, wl.K
        self.outs = [torch.empty((T, wl.H, wl.dc), dtype=torch.bfloat16, device=dev) for _ in self.copies]
        self.lses = [torch.empty((T, wl.H), dtype=torch.float32, device=dev) for _ in self.copies]
        self.ws_bytes = B.dsa_workspace_size(B.DSA_OP_FUSED_DECODE, base.batch, K, wl.HI, wl.dI)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.idx_in = [c.indexer_in() for c in self.copies]
        self.mla_in = [c.mla_in() for c in self.copies]
        self.resident_bytes = sum(c.kv.numel() * c.kv.element_size() + c.k_cache.numel() * c.k_cache.element_size()
                                  + c.q.numel() * 2 for c in self.copies)

    def step(self, i, stream, events=None):
        j = i % len(self.copies)
        self.B.dsa_fused_decode(self.copies[j].batch, self.idx_in[j], self.mla_in[j], self.wl.K, self.outs[j],
                                self.lses[j], None, self.ws, self.ws_bytes, stage_events=events, stream=stream)


def time_steps(run, steps, warmup, stream, dev, dist=None, eager=False):
    """W warm-up steps, then K steps captured once as a CUDA graph and replayed
    (host launch overhead cannot hide in the device time), bracketed by a
    barrier and a device synchronize, timed with CUDA events on the launch
    stream. Returns (total_ms, clock summary, timing mode, device status)."""
    import torch
    for i in range(warmup):
        run.step(i, stream)
    torch.cuda.synchronize(dev)
    status = run.B.dsa_read_device_status(stream)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    for e in (t_start, t_end):
        e.record(stream)
    torch.cuda.synchronize(dev)
    graph, mode = None, "eager"
    if not eager:
        try:
            graph = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream(dev)
            with torch.cuda.graph(graph, stream=cap):
                for i in range(steps):
                    run.step(i, cap)
            mode = "cuda_graph"
        except Exception as e:
            graph, mode = None, f"eager (graph capture failed: {type(e).__name__})"
            torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clocks:
        clocks.mark("start")
        t_start.record(stream)
        if graph is not None:
            graph.replay()
        else:
            for i in range(steps):
                run.step(i, stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        clocks.mark("end")
    if dist is not None:
        dist.barrier()
    del graph
    return t_start.elapsed_time(t_end), clocks.summary(), mode, status


def stage_times(run, steps, stream, dev):
    """Per-kernel durations: eager launches with an event recorded on the launch
    stream right before and after each stage (an event between two kernels
    turns the programmatic launch off on that edge, and the gaps include host
    launch latency, so these slightly overstate the in-graph stage times)."""
    import torch
    ev = _stage_events(run.B, steps)
    for row in ev:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize(dev)
    for i in range(steps):
        run.step(i, stream, ev[i])
    torch.cuda.synchronize(dev)
    return {
        "indexer": statistics.mean(e[0].elapsed_time(e[1]) for e in ev),
        "topk": statistics.mean(e[1].elapsed_time(e[2]) for e in ev),
        "sparse_mla": statistics.mean(e[2].elapsed_time(e[3]) for e in ev),
    }


def e2e_pipelined(run, steps, warmup, dev):
    """End to end through the public call with host buffers: every step copies
    its inputs (q_I, w, q) from pinned host memory to the device and its output
    back to pinned host memory. Copies run on their own streams, double
    buffered, so step i+1's upload and step i-1's download overlap step i's
    kernels; the timed region runs from the first upload to the last download."""
    import torch
    wl = run.wl
    base = run.copies[0]
    h_in = [(base.q_idx.cpu().pin_memory(), base.w.cpu().pin_memory(), base.q.cpu().pin_memory()) for _ in range(2)]
    h_out = [torch.empty(run.outs[0].shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    s_in, s_run, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    nb = min(2, len(run.copies))
    in_done = [torch.cuda.Event() for _ in range(nb)]
    run_done = [torch.cuda.Event() for _ in range(nb)]
    out_done = [torch.cuda.Event() for _ in range(nb)]
    h2d = sum(t.numel() * t.element_size() for t in h_in[0])
    d2h = h_out[0].numel() * 2

    def one(i):
        j = i % nb
        c = run.copies[j]
        with torch.cuda.stream(s_in):
            if i >= nb:
                s_in.wait_event(run_done[j])          # the kernels of step i - nb no longer read buffer j
            for dst, src in zip((c.q_idx, c.w, c.q), h_in[j]):
                dst.copy_(src, non_blocking=True)
            in_done[j].record(s_in)
        s_run.wait_event(in_done[j])
        if i >= nb:
            s_run.wait_event(out_done[j])             # the download of step i - nb has read out[j]
        run.B.dsa_fused_decode(c.batch, run.idx_in[j], run.mla_in[j], wl.K, run.outs[j], run.lses[j], None, run.ws,
                               run.ws_bytes, stream=s_run)
        run_done[j].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(run_done[j])
            h_out[j].copy_(run.outs[j], non_blocking=True)
            out_done[j].record(s_out)

    # untimed warm-up: at least `warmup` steps and 0.2 s, so the host link has
    # left any idle power state before the timed steps
    t_end = time.perf_counter() + 0.2
    i = 0
    while i < max(3, warmup) or time.perf_counter() < t_end:
        one(i)
        i += 1
        if i % 64 == 0:
            torch.cuda.synchronize(dev)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        one(i)
    s_out.wait_event(out_done[(steps - 1) % nb])
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1) / steps, h2d, d2h


def extra_block(name, args, dev, stream):
    """One graph-timed measurement of another workload, with its roofline."""
    import torch
    t0 = time.time()
    decode = name in ("c3", "c3mx", "c2kv8", "c2pg")
    steps = args.extra_steps_decode if decode else args.extra_steps_prefill
    run = Runner(name, dev, copies=2)
    wl = run.wl
    total_ms, clocks, mode, status = time_steps(run, steps, 2, stream, dev)
    stages = stage_times(run, min(steps, 3), stream, dev)
    ms = total_ms / steps
    n_sel = int(np.minimum(wl.n_valid(), wl.K).sum())
    block = {"name": name, "workload": WORKLOAD_TEXT[name], "steps": steps, "warmup": 2, "ms_per_step": ms,
             "query_tokens_per_s": wl.T / (ms * 1e-3), "stage_ms": stages, "clocks": clocks, "timing": mode,
             "device_status": [status, run.B.dsa_read_device_status(stream)],
             "l2": f"2 rotating input copies ({run.resident_bytes / 1e9:.2f} GB) > 126 MB L2"}
    if decode:
        peak, kind = _peaks()
        ab = algorithmic_bytes(wl, n_sel, run.kv_row_bytes, run.key_row_bytes)
        b = ab["step"]
        block["roofline"] = {"bound": "hbm", "achieved": b / (ms * 1e-3) / 1e9, "peak": peak, "unit": "GB/s",
                             "frac": b / (ms * 1e-3) / 1e9 / peak, "peak_kind": kind, "algorithmic_bytes": b,
                             "frac_of_8TBps": b / (ms * 1e-3) / 1e9 / 8000.0,
                             "stage_frac": {k: ab[k] / (stages[k] * 1e-3) / 1e9 / peak
                                            for k in ("indexer", "topk", "sparse_mla")}}
    else:
        burst, sustained, kind = _peak_tflops()
        f = algorithmic_flops(wl, n_sel)
        ach = f["step"] / (ms * 1e-3) / 1e12
        block["roofline"] = {"bound": "tensor", "achieved": ach, "unit": "TFLOP/s", "peak": sustained,
                             "frac": ach / sustained, "peak_kind": f"{kind} sustained bf16",
                             "frac_of_burst": ach / burst, "burst_peak": burst, "frac_of_nominal_2250": ach / 2250.0,
                             "algorithmic_flops": f["step"],
                             "stage_tflops": {k: f[k] / (stages[k] * 1e-3) / 1e12 for k in ("indexer", "sparse_mla")}}
    block["setup_s"] = round(time.time() - t0 - total_ms / 1e3, 1)
    del run
    torch.cuda.empty_cache()
    return block


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
    ap.add_argument("--extra", default="c3,c3mx,c2kv8,c2pg,c4,c5",
                    help="comma-separated extra workloads measured after the headline (single GPU only; '' for none)")
    ap.add_argument("--extra-steps-decode", type=int, default=20)
    ap.add_argument("--extra-steps-prefill", type=int, default=3)
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
    from indexed_sparse_attention_relu_b200 import multi

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    build_mod.build()
    B.load()

    run = Runner(args.config, dev, args.copies, rank=rank, world=world)
    sharded = world > 1 and args.config in SHARDED
    wl = run.wl
    T, K = wl.T, wl.K
    stream = torch.cuda.current_stream(dev)
    total_ms, clocks, timing_mode, status = time_steps(run, args.steps, args.warmup, stream, dev,
                                                      dist if world > 1 else None, eager=args.eager)
    stage_ms = stage_times(run, args.steps, stream, dev)
    # the job's time is its slowest rank's; every rank ran its own T queries
    total_ms = multi.max_over_ranks(total_ms, dist if world > 1 else None, dev)
    ms_per_step = total_ms / args.steps
    value = multi.job_throughput(run.units, ms_per_step)

    e2e_ms, h2d, d2h = e2e_pipelined(run, args.steps, args.warmup, dev)
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
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong" if sharded else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.config], "name": args.config, "B": wl.B, "L_max": wl.Lmax,
                   "T": T, "K": K, "H_I": wl.HI, "d_I": wl.dI, "H": wl.H, "d_c": wl.dc, "d_rope": wl.dr,
                   "index_keys": wl.key_dtype,
                   "parallelism": (f"sequences sharded x{world} (longest first)" if sharded else f"replicas x{world}")
                   if world > 1 else "single GPU",
                   "l2": f"{len(run.copies)} rotating input copies ({run.resident_bytes / 1e9:.2f} GB) > 126 MB L2"},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind, "traffic": traffic,
                     "algorithmic_bytes": algo[dom], "avg_launch_ms": stage_ms[dom]},
        "step_roofline": {"bound": "hbm", "achieved": step_gbs, "peak": peak, "unit": "GB/s",
                          "frac": step_gbs / peak, "frac_of_8TBps": step_gbs / 8000.0,
                          "algorithmic_bytes": algo["step"]},
        "stage_ms": stage_ms,
        "stage_ms_note": "second K-step pass, eager launches with CUDA events between the stages",
        "clocks": clocks,
        "e2e": {"value": sum(run.units) / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "note": "pinned host buffers; uploads and downloads on their own streams, double buffered"},
        "gpu_launches": launches_per_step * args.steps,
        "timing": timing_mode,
        "device_status": [status, status2],
    }
    del run
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n, dt, thr = run_cpu_oracle(wl, args.cpu_tokens, min_seconds=args.cpu_seconds)
        line["cpu_baseline"] = {"value": n / dt, "unit": UNIT, "cores": thr, "kind": "oracle",
                                "sample": f"{min(args.cpu_tokens, wl.T)} query tokens of the same workload (full "
                                          f"causal history), fp64, repeated to {n} tokens in {dt:.1f} s"}
        # the same oracle on one core (OpenMP threads = 1), a shorter sample
        import oracle
        oracle.set_num_threads(1)
        n1, dt1, _ = run_cpu_oracle(wl, 1, min_seconds=min(args.cpu_seconds, 3.0))
        oracle.set_num_threads(thr)
        line["cpu_baseline"]["single_core"] = {"value": n1 / dt1, "unit": UNIT, "cores": 1,
                                               "sample": f"1 query token, repeated to {n1} in {dt1:.1f} s"}
    if world == 1 and args.extra:
        line["configs"] = []
        for name in [x for x in args.extra.split(",") if x and x != args.config]:
            try:
                line["configs"].append(extra_block(name, args, dev, stream))
            except Exception as e:  # report, keep the headline
                line["configs"].append({"name": name, "error": f"{type(e).__name__}: {e}"})
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
