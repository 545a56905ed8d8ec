#!/usr/bin/env python
"""Benchmark of the CSA2 decode hot path on B200.

Default workload: the full 20-layer decoder attention stack (five groups:
Full + 3 Reuse, then four Reindex + 3 Reuse), batch 4, context 1,048,576,
one decode step = append the new token's FP4 KV row, then every layer's
indexing (scan / pool / top-512 or Reindex rescoring) and sparse attention.

Metric: decode layer-steps/s (layers of the stack / time of one decode step of
the whole batch), plus the dominant kernel (the Full layer's indexer scan)
against the HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl csa2|reference]

N > 1 runs one process per GPU (torchrun); each rank decodes its own batch
(weak scaling, no data-path collective: sequences are independent).
`--impl reference` times the CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA2 decode layer-steps/s at 128K–1M ctx; achieved HBM GB/s vs roofline"
UNIT = "layer-steps/s"
DEFAULT_WORKLOAD = "decoder_stack20_b4_ctx1m"
FALLBACK_HBM_GBS = 6650.0


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def _scan_traffic(workload: str):
    """DRAM bytes per scan launch from the committed ncu summary, or None if the
    scan source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "index_full_scan.traffic.txt")
    src = os.path.join(ROOT, "sparse_attention_fp4_kv_b200", "csrc", "indexer.cu")
    if not os.path.exists(p):
        return None
    kv = {}
    for line in open(p):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    if kv.get("indexer_cu_sha256") != sha or kv.get("workload") != workload:
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock/throttle sampling every 200 ms during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        text = self.file.read()
        os.unlink(self.file.name)
        return summarize_clocks(text)


def summarize_clocks(text: str) -> dict:
    """Median SM clock, the largest max clock and the throttle reasons seen in
    nvidia-smi CSV lines of ClockSampler.FIELDS (noheader, nounits)."""
    sm, smax, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in text.splitlines():
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            smax.append(float(parts[2]))
        except ValueError:
            continue
        for n, v in zip(names, parts[5:9]):
            if v.lower().startswith("active"):
                reasons.add(n)
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(smax) if smax else None,
            "reasons": sorted(reasons), "samples": len(sm)}


def _config(w, name):
    return {"workload": name, "batch_per_gpu": w.B, "ctx": w.ctx, "layers": w.n_layers,
            "schedule": "".join("FRU"[m] for m in w.modes), "main_kv": f"fp4 e2m1+e4m3/16, {w.C} ch",
            "q_heads": w.Hq, "indexer": f"int8 {w.H_idx}x{w.D_idx}", "pool_blocks": 2048,
            "topk": 512, "n_win": w.n_win,
            "l2": "inputs larger than L2: every step streams "
                  f"{w.B * w.ctx * w.H_idx * w.D_idx / 1e9:.2f} GB of indexer keys",
            "parallelism": "replicas (weak scaling, no collective)"}


# ----------------------------------------------------------------------------- oracle timing
def _host_cores() -> dict:
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:
        usable = os.cpu_count()
    return {"cpu_count": os.cpu_count(), "usable": usable}


def _oracle_sequence_step(inp):
    """The oracle's decode step for one sequence of the stack (all layers)."""
    import oracle
    modes = inp["modes"]
    ctx = inp["ctx"]
    kn, sn, kv = inp["k_idx"], inp["k_scale"], inp["kv_bf16"]
    pool = inp.get("pool0")
    top = None
    outs = []
    for l, m in enumerate(modes):
        if m == 0:
            r = oracle.full_layer(inp["q_idx"][l], kn, sn, ctx)
            pool, top = r["pool"], r["top"]
        elif m == 1:
            top, _, _ = oracle.reindex_layer(inp["q_idx"][l], kn, sn, pool, ctx)
        outs.append(oracle.sparse_attention(inp["q"][l], lambda P: kv[P], top, inp["swa"][l],
                                            ctx - 1, ctx - inp["swa_rows"], inp["scale"]))
    return outs


def _bits(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _oracle_inputs_from_device(wl, b):
    """Host copies of sequence b's inputs: the buffers the GPU arm uses, with
    the bf16 main-KV rows (before quantization) re-drawn on the device."""
    from sparse_attention_fp4_kv_b200 import synth
    import oracle
    w = wl.w
    inp = dict(modes=list(wl.modes), ctx=w.ctx, k_idx=wl.k_idx[b].cpu().numpy(),
               k_scale=wl.k_scale[b].cpu().numpy(),
               kv_bf16=_bits(synth.main_kv_bf16(w, b, 0, w.ctx, wl.device)),
               q_idx={l: q[b, 0].cpu().numpy() for l, q in enumerate(wl.q_idx) if q is not None},
               q=[_bits(q[b, 0]) for q in wl.q], swa=[_bits(s[b]) for s in wl.swa],
               swa_rows=wl.swa_rows, scale=wl.scale)
    if wl.pool_ready:
        inp["pool0"] = oracle.full_layer(wl.pool_q_idx[b, 0].cpu().numpy(), inp["k_idx"],
                                         inp["k_scale"], w.ctx)["pool"]
    return inp


def _oracle_inputs_on_host(w, b):
    """Sequence b's inputs drawn on the host by the seeded generators alone (no
    GPU, no libcsa2): the same shapes and distributions as the GPU arm's
    (values drawn on the CPU differ from values drawn on a GPU)."""
    from sparse_attention_fp4_kv_b200 import synth
    import oracle
    rows = min(w.n_win, w.ctx)
    k_idx = synth.indexer_keys(w, b, w.ctx, "cpu")
    q_idx = {l: synth.indexer_q(w, l, 1, "cpu") for l, m in enumerate(w.modes) if m != synth.REUSE}
    inp = dict(modes=list(w.modes), ctx=w.ctx, k_scale=synth.indexer_key_scale(w, b, w.ctx, "cpu").numpy(),
               kv_bf16=_bits(synth.main_kv_bf16(w, b, 0, w.ctx, "cpu")),
               q=[_bits(synth.main_q(w, l, 1, "cpu")[b, 0]) for l in range(w.n_layers)],
               swa=[_bits(synth.swa_kv(w, l, rows, "cpu")[b]) for l in range(w.n_layers)],
               swa_rows=rows, scale=1.0 / np.sqrt(w.C))
    if w.modes[0] == synth.REINDEX:
        # set-up: plant the correlated blocks, then the pool of a preceding Full layer
        q_r = q_idx[0]
        if w.planted_blocks:
            synth.plant(w, b, k_idx, q_r[b, 0])
        inp["pool0"] = oracle.full_layer(synth.pool_builder_q(w, q_r)[b, 0].numpy(), k_idx.numpy(),
                                         inp["k_scale"], w.ctx)["pool"]
    inp["k_idx"] = k_idx.numpy()
    inp["q_idx"] = {l: q[b, 0].numpy() for l, q in q_idx.items()}
    return inp


def _time_oracle(inp, reps=3):
    """Seconds per oracle step of one sequence: one untimed warm-up, then the
    median of `reps` timed runs on the same pre-drawn inputs."""
    _oracle_sequence_step(inp)
    ts = []
    for _ in range(reps):
        t0 = time.perf_counter()
        _oracle_sequence_step(inp)
        ts.append(time.perf_counter() - t0)
    return statistics.median(ts)


# ----------------------------------------------------------------------------- arms
REFERENCE_BUDGET_S = 150.0


def run_reference(args, name):
    """CPU oracle arm (the OpenMP build, every usable host core). A step is the
    oracle's decode step (every layer) of S sequences of the batch: the whole
    batch (S = B) when K + W such steps fit in REFERENCE_BUDGET_S, else as many
    sequences as fit (at least one). ms_per_step is the measured time of those
    S sequences; value is the batch rate at that time per sequence."""
    from sparse_attention_fp4_kv_b200 import synth
    import oracle
    threads = oracle.use_openmp(True)
    w = synth.WORKLOADS[name]
    t_setup = time.perf_counter()
    inputs = [_oracle_inputs_on_host(w, 0)]
    t_seq = _time_oracle(inputs[0], reps=1)
    n_steps = args.steps + args.warmup
    S = int(max(1, min(w.B, REFERENCE_BUDGET_S // max(n_steps * t_seq, 1e-9))))
    for b in range(1, S):
        inputs.append(_oracle_inputs_on_host(w, b))
    t_setup = time.perf_counter() - t_setup

    def step():
        for inp in inputs:
            _oracle_sequence_step(inp)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    ms = (time.perf_counter() - t0) / args.steps * 1e3
    value = w.n_layers * S / w.B / (ms / 1e3)
    sample = (f"{S} of {w.B} sequences per step (all {w.n_layers} layers each: Full-layer scan over "
              f"all {w.ctx} tokens, pool, every layer's top-512 and attention); value = rate of the "
              f"{w.B}-sequence batch at the measured time per sequence; inputs drawn on the host by "
              f"the seeded generators ({t_setup:.0f} s set-up, untimed); OpenMP oracle build, "
              f"{threads} threads")
    cfg = _config(w, name)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int64/fp64", "data": "synthetic", "config": cfg, "host_cores": _host_cores(),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def synth_n_new(name: str) -> int:
    """New tokens (queries) per sequence of a workload: more than one means the
    multi-query Full-layer path (chunked prefill, multi-token decode)."""
    from sparse_attention_fp4_kv_b200 import synth
    return int(getattr(synth.WORKLOADS[name], "n_new", 1) or 1)


def run_prefill(args, name, rank, world, local_rank):
    """Chunked-prefill workload (one Full layer, n_new causal queries): tokens
    (queries) per second, and the tensor-core indexer against the int8 roofline."""
    from sparse_attention_fp4_kv_b200 import synth
    from sparse_attention_fp4_kv_b200.workload import PrefillWorkload
    import torch.distributed as dist
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    from sparse_attention_fp4_kv_b200 import replicas
    w = replicas.rank_workload(synth.WORKLOADS[name], rank, world)
    pw = PrefillWorkload(w, dev)
    stream = torch.cuda.current_stream()
    K, W = args.steps, args.warmup
    for _ in range(W):
        pw.step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    clocks = ClockSampler(dev)
    time.sleep(0.4)
    if world > 1:
        dist.barrier(device_ids=[local_rank])
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(K):
        pw.step(scan_events=ev[k])
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1) / K
    scan_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    from sparse_attention_fp4_kv_b200 import replicas
    ms, scan_ms = replicas.slowest([ms, scan_ms], dev)
    peaks = {}
    pth = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pth):
        peaks = json.load(open(pth))
    bf16 = float(peaks.get("bf16_tflops", 1590.0))
    # int8 dense is twice the bf16 dense rate (nominal 4.5 vs 2.25 PFLOP/s)
    int8_peak = 2.0 * bf16
    ops = pw.index_ops()
    tops = ops / (scan_ms / 1e3) / 1e12
    tokens = world * w.B * w.n_new
    # A few queries per sequence (multi-token decode): the scan streams every
    # key once and is bound by HBM, not by the tensor cores.
    key_bytes = w.B * w.ctx * (w.H_idx * w.D_idx + 4)
    hbm_bound = ops / key_bytes < 2.0 * bf16 * 1e12 / (float(peaks.get("hbm_gbs", 6650.0)) * 1e9)
    if hbm_bound:
        hbm_peak = float(peaks.get("hbm_gbs", 6650.0))
        gbs = key_bytes / (scan_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": "index_mma_kernel (tcgen05 kind::i8, few queries)",
                "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                "peak_kind": "measured" if "hbm_gbs" in peaks else "fallback",
                "traffic": None, "algorithmic_bytes": key_bytes, "launch_ms": scan_ms}
    else:
        roof = {"bound": "tensor", "kernel": "index_mma_kernel (tcgen05 kind::i8)",
                "achieved": tops, "peak": int8_peak, "unit": "TOPS", "frac": tops / int8_peak,
                "peak_kind": "measured bf16 burst x 2 (nominal int8/bf16 ratio)"
                if peaks else "fallback bf16 x 2",
                "traffic": None, "algorithmic_ops": ops, "launch_ms": scan_ms}
    line = {"metric": "CSA2 chunked-prefill tokens/s (Full layer: append, causal indexer, "
                      "pool, top-512, attention)", "value": tokens / (ms / 1e3),
            "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int8/fp32", "data": "synthetic",
            "config": {"workload": name, "batch_per_gpu": w.B, "ctx": w.ctx, "new_tokens": w.n_new,
                       "indexer": f"int8 {w.H_idx}x{w.D_idx}", "q_heads": w.Hq, "C": w.C},
            "roofline": roof, "clocks": clk, "gpu_launches": pw.launches_per_step() * K}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_csa2(args, name, rank, world, local_rank):
    from sparse_attention_fp4_kv_b200 import synth
    from sparse_attention_fp4_kv_b200.workload import DecodeWorkload
    import torch.distributed as dist
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    from sparse_attention_fp4_kv_b200 import replicas
    w = replicas.rank_workload(synth.WORKLOADS[name], rank, world)
    wl = DecodeWorkload(w, dev)
    stream = torch.cuda.current_stream()
    K, W = args.steps, args.warmup

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    scan_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
    for a, b in scan_ev:  # materialise the event handles
        a.record(stream)
        b.record(stream)
    for _ in range(W):
        wl.step()
    torch.cuda.synchronize()

    clocks = ClockSampler(dev)
    time.sleep(0.4)
    barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(K):
        wl.stack(stream, scan_events=scan_ev[k])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms_total = t_start.elapsed_time(t_end)
    scan_ms = statistics.mean(a.elapsed_time(b) for a, b in scan_ev)

    # ---- the same step captured once as a CUDA graph and replayed K times (the
    # kernels keep their programmatic dependencies as graph edges)
    graph_ms, graph_note = None, None
    graph = None
    try:
        graph = wl.capture_step_graph()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(K):
            graph.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        graph_ms = g0.elapsed_time(g1)
    except Exception as e:  # capture unsupported here: report the direct launches
        graph_note = f"graph capture failed: {type(e).__name__}: {str(e)[:120]}"
    barrier()
    ms_direct, scan_ms = replicas.slowest([ms_total, scan_ms], dev)
    if graph_ms is not None:
        ms_total = replicas.slowest([graph_ms], dev)[0]
    else:
        ms_total = ms_direct
    ms_step = ms_total / K
    value = replicas.aggregate_rate(w.n_layers, world, ms_step)

    # ---- end to end through the public API with host buffers
    e2e = _e2e(wl, args, stream, world, local_rank)
    from sparse_attention_fp4_kv_b200 import binding
    # every bounded wait of the timed steps completed (0); otherwise the outputs are invalid
    status = binding.device_status()

    nbytes = wl.step_bytes()
    peak, peak_kind = _peaks()
    # the dominant kernel is timed inside the step: the first Full layer's
    # scan, or the first Reindex rescoring in a stack without a Full layer
    n_full, n_ri = wl.modes.count(synth.FULL), wl.modes.count(synth.REINDEX)
    if n_full:
        kernel = "index_full_kernel (Full-layer indexer scan)"
        kbytes = nbytes["scan"] / n_full
        traffic = _scan_traffic(name)
    else:
        kernel = "index_reindex_kernel (Reindex rescoring of the pool)"
        kbytes = nbytes["reindex"] / max(n_ri, 1)
        traffic = None
    scan_gbs = kbytes / (scan_ms / 1e3) / 1e9
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8/fp32", "data": "synthetic",
            "config": _config(w, name),
            "roofline": {"bound": "hbm", "kernel": kernel,
                         "achieved": scan_gbs, "peak": peak, "unit": "GB/s",
                         "frac": scan_gbs / peak, "peak_kind": peak_kind,
                         "traffic": traffic, "algorithmic_bytes": kbytes,
                         "launch_ms": scan_ms},
            "step_hbm": {"algorithmic_bytes": nbytes["total"],
                         "achieved_gbs": nbytes["total"] / (ms_step / 1e3) / 1e9,
                         "frac": nbytes["total"] / (ms_step / 1e3) / 1e9 / peak},
            "clocks": clk, "e2e": e2e, "gpu_launches": wl.launches_per_step() * K,
            "timing": {"value_from": "CUDA graph replays" if graph_ms is not None else "direct launches",
                       "graph_ms_per_step": graph_ms / K if graph_ms is not None else None,
                       "direct_ms_per_step": ms_direct / K, "note": graph_note}}
    line["device_status"] = status
    line["host_cores"] = _host_cores()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        threads = oracle.use_openmp(True)
        inp = _oracle_inputs_from_device(wl, 0)
        t_seq = _time_oracle(inp, reps=3)
        line["cpu_baseline"] = {"value": w.n_layers / (w.B * t_seq), "unit": UNIT, "cores": threads,
                                "kind": "oracle",
                                "sample": f"sequence 0 of {w.B}, all {w.n_layers} layers, the GPU arm's "
                                          f"inputs copied to the host; median of 3 runs after one "
                                          f"warm-up ({t_seq:.2f} s per sequence); rate of the "
                                          f"{w.B}-sequence batch at that time per sequence; OpenMP "
                                          f"oracle build, {threads} threads"}
    if world == 1 and not args.no_extra_configs and name == DEFAULT_WORKLOAD:
        del graph, wl
        torch.cuda.empty_cache()
        line["configs"] = _extra_configs(dev)
        status = status or binding.device_status()
        line["device_status"] = status
    if rank == 0:
        print(json.dumps(line), flush=True)
    if status != 0:
        raise SystemExit(f"a kernel gave up a bounded wait (csa2_device_status = {status}): "
                         "the step's outputs are invalid")


# The metric is quoted for 128K-1M contexts: the other decode workloads of that
# range and the chunked prefill are measured in the same run (one GPU), each
# after the previous one's buffers are freed.
EXTRA_CONFIGS = ("decoder_group1_b8_ctx128k", "reindex_group_b32_ctx256k", "prefill_4096_at_64k")
EXTRA_STEPS, EXTRA_WARMUP = 30, 3


def _extra_configs(dev):
    from sparse_attention_fp4_kv_b200 import synth
    from sparse_attention_fp4_kv_b200.workload import DecodeWorkload, PrefillWorkload
    peak, peak_kind = _peaks()
    out = {}
    for name in EXTRA_CONFIGS:
        w = synth.WORKLOADS[name]
        stream = torch.cuda.current_stream()
        if synth_n_new(name) > 1:
            pw = PrefillWorkload(w, dev)
            for _ in range(EXTRA_WARMUP):
                pw.step()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(EXTRA_STEPS // 6):
                pw.step()
            b.record(stream)
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / (EXTRA_STEPS // 6)
            out[name] = {"metric": "chunked-prefill tokens/s", "value": w.B * w.n_new / (ms / 1e3),
                         "unit": "tokens/s", "ms_per_step": ms, "steps": EXTRA_STEPS // 6,
                         "gpu_launches_per_step": pw.launches_per_step()}
            del pw
        else:
            wl = DecodeWorkload(w, dev)
            for _ in range(EXTRA_WARMUP):
                wl.step()
            torch.cuda.synchronize()
            g = wl.capture_step_graph()
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(EXTRA_STEPS):
                g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / EXTRA_STEPS
            nbytes = wl.step_bytes()["total"]
            out[name] = {"metric": METRIC, "value": w.n_layers / (ms / 1e3), "unit": UNIT,
                         "ms_per_step": ms, "steps": EXTRA_STEPS, "timing": "CUDA graph replays",
                         "step_hbm": {"algorithmic_bytes": nbytes,
                                      "achieved_gbs": nbytes / (ms / 1e3) / 1e9,
                                      "frac": nbytes / (ms / 1e3) / 1e9 / peak, "peak_kind": peak_kind},
                         "gpu_launches_per_step": wl.launches_per_step()}
            del g, wl
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


def _e2e(wl, args, stream, world, local_rank):
    """Same metric through the public API with pinned host buffers: every step
    copies that step's inputs host->device (the new KV row, every layer's main Q
    and indexer Q), runs the decode stack, and reads every layer's output and
    top-k indices back to the host. As in a serving loop, the copies overlap the
    neighbouring steps' compute: inputs go up on one stream and results come
    back on another, two sets of per-step device buffers alternate, events
    order each step's copy-in, compute and copy-out, and compute stays strictly
    in step order on one stream. The timed region spans the first copy-in to
    the last copy-out."""
    import torch.distributed as dist
    dev = wl.device
    sets = []
    for k in range(2):
        if k == 0:
            stack = wl.stack
            d_in, d_out = wl.io_tensors()
        else:
            stack, d_in, d_out = wl.io_set()
        h_in = [torch.empty_like(t, device="cpu").pin_memory() for t in d_in]
        h_out = [torch.empty_like(t, device="cpu").pin_memory() for t in d_out]
        for d, h in zip(d_in, h_in):
            h.copy_(d)
        sets.append((stack, list(zip(d_in, h_in)), list(zip(d_out, h_out))))
    h2d = sum(h.numel() * h.element_size() for _, h in sets[0][1])
    d2h = sum(h.numel() * h.element_size() for _, h in sets[0][2])
    E = max(1, min(args.steps, 200))
    up = torch.cuda.Stream(device=dev)
    down = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    started = [False, False]

    def enqueue(k):
        i = k % 2
        stack, ins, outs = sets[i]
        with torch.cuda.stream(up):
            if started[i]:
                up.wait_event(ev_done[i])  # the set's previous step has read its inputs
            for d, h in ins:
                d.copy_(h, non_blocking=True)
            ev_in[i].record(up)
        stream.wait_event(ev_in[i])
        if started[i]:
            stream.wait_event(ev_out[i])  # ... and its outputs have been read back
        stack(stream)
        ev_done[i].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(ev_done[i])
            for d, h in outs:
                h.copy_(d, non_blocking=True)
            ev_out[i].record(down)
        started[i] = True

    for k in range(4):
        enqueue(k)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier(device_ids=[local_rank])
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    up.wait_event(a)
    for k in range(E):
        enqueue(k)
    stream.wait_event(ev_out[(E - 1) % 2])
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / E
    from sparse_attention_fp4_kv_b200 import replicas
    ms = replicas.slowest([ms], dev)[0]
    return {"value": replicas.aggregate_rate(wl.w.n_layers, world, ms), "unit": UNIT, "ms_per_step": ms,
            "steps": E, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "overlap": "inputs and results copied on two more streams, two alternating buffer sets"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="csa2", choices=["csa2", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-configs", action="store_true",
                    help="skip the other decode workloads and the prefill in the line's 'configs'")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, args.workload)
        return
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        if synth_n_new(args.workload) > 1:
            run_prefill(args, args.workload, rank, world, local_rank)
        else:
            run_csa2(args, args.workload, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
