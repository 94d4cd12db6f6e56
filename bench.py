"""Throughput of query-aware top-k selective attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the hot path over one batch of synthetic input:
  headline  ESA chunked prefill of a Llama-3-8B attention layer, 32768 tokens in
            chunks of 512 (compress keys and queries, score, correct, chunk-sum,
            neighbour max-pool, top-k, attention over initial + selected + local);
  also      ESA decode at 128K context, batch 16, and MoBA causal prefill at 64K
            (32 heads, 64 blocks of 1024, top-3 + current), each timed the same way.
Every rank runs its own replica (weak scaling, no collective on the data path);
time is the max over ranks of the CUDA-event time. L2 is flushed (256 MB write)
between timed steps, outside the events. Rank 0 prints one JSON line.

--impl reference times the CPU oracle (oracle/, float64 numpy on the host cores)
on a bounded sample of the same workload per step; it needs no GPU.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ESA decode tok/s @128K & chunked-prefill tok/s; % of HBM/tensor roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true", help="time the headline workload only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--prefill-ctx", type=int, default=0,
                    help="shorter prefill context (profiling a small case); the line then names that workload")
    ap.add_argument("--only", choices=["decode", "decode_per_head", "decode_varlen", "decode_1m", "moba",
                                       "moba_decode", "cca", "tiny_decode", "fit"],
                    default=None,
                    help="profiling: run one of the other workloads alone and print its figures")
    ap.add_argument("--decode-batch", type=int, default=0, help="profiling: decode batch (default: the workload's)")
    ap.add_argument("--moba-seq", type=int, default=0, help="profiling: MoBA sequence length (default: the workload's)")
    return ap.parse_args()


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "query_aware_selective_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, sources):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    kernel as it is now (same source hash); else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        t = json.load(f)
    e = t.get(kernel)
    if not e or e.get("source_hash") != source_hash(*sources):
        return None
    return e.get("dram_bytes_per_launch")


def choose_tensor_peak(clocks, peaks, peak_src):
    """The dense bf16 peak a tensor-core kernel of this run is held against, chosen from
    the run's own clock record: the burst figure (measured at the full clock) when the
    median SM clock under load stayed at its maximum, whatever reasons were sampled (a
    power-cap flag with the clock at its maximum did not slow the kernel), else the
    sustained one (measured under the power cap at a lower clock). Returns (peak,
    regime, source text)."""
    burst, sustained = peaks["bf16_tflops"], peaks["bf16_tflops_sustained"]
    if clocks and clocks.get("sm_mhz") and clocks.get("sm_max_mhz"):
        reasons = clocks.get("reasons") or []
        if clocks["sm_mhz"] >= 0.97 * clocks["sm_max_mhz"]:
            return burst, "burst", (f"{peak_src} bf16 burst: median SM clock under load {clocks['sm_mhz']:.0f} of "
                                    f"{clocks['sm_max_mhz']:.0f} MHz (reasons sampled: {reasons})")
        return sustained, "sustained", (f"{peak_src} bf16 sustained: median SM clock under load "
                                        f"{clocks['sm_mhz']:.0f} of {clocks['sm_max_mhz']:.0f} MHz, reasons {reasons}")
    return burst, "burst", f"{peak_src} bf16 burst (no clock record: the higher peak, so the lower fraction)"


def finish_tensor_roofline(r, clocks, peaks, peak_src):
    """Fill peak and fraction of a tensor-bound roofline entry whose 'achieved' is set."""
    peak, regime, src = choose_tensor_peak(clocks, peaks, peak_src)
    r["peak"] = peak
    r["frac"] = round(r["achieved"] / peak, 4)
    r["frac_of_burst"] = round(r["achieved"] / peaks["bf16_tflops"], 4)
    r["frac_of_sustained"] = round(r["achieved"] / peaks["bf16_tflops_sustained"], 4)
    r["peak_regime"] = regime
    r["peak_source"] = src


def finish_rooflines(line, clocks, peaks, peak_src):
    entries = [line.get("roofline")] + [e.get("roofline") for e in (line.get("also") or {}).values()]
    for r in entries:
        if r and r.get("bound") == "tensor":
            finish_tensor_roofline(r, clocks, peaks, peak_src)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples every 100 ms while running (clocks, power, throttle reasons)."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "utilization.gpu", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id: str):
        self.gpu_id, self.proc, self.lines = gpu_id, None, []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + ",".join(self.FIELDS),
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [[x.strip() for x in ln.split(",")] for ln in out.strip().splitlines() if ln.strip()]
        rows = [r for r in rows if len(r) == len(self.FIELDS)]
        if not rows:
            return None

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        busy = [r for r in rows if (num(r[3]) or 0) >= 50] or rows
        sm = [num(r[0]) for r in busy if num(r[0]) is not None]
        reasons = set()
        for r in busy:
            for name, val in zip(["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"],
                                 r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(rows[0][1]),
                "power_w_max": max((num(r[2]) or 0) for r in rows), "samples": len(rows),
                "samples_under_load": len(busy), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- timing

def time_steps(fn, steps, warmup, flush, dist_max, after_step=None):
    """Warm up, then time each of `steps` calls with CUDA events (L2 flushed between
    steps, outside the events). after_step, if given, runs after each step once the
    device is idle (outside the events; it reads timing events of the step). Returns
    per-step ms and their sum (the sum after max over ranks)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    dist_barrier()
    torch.cuda.synchronize()
    evs = []
    for _ in range(steps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        evs.append((a, b))
        if after_step is not None:
            torch.cuda.synchronize()
            after_step()
    torch.cuda.synchronize()
    dist_barrier()
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in evs]
    total = dist_max(sum(ms))
    return ms, total


L2_NOTE = ("flushed between timed steps: 256 MB written, then another 256 MB read (no input line left in the "
           "126 MB L2, and no dirty line left to be written back inside the step)")


def make_flush(dev):
    """L2 flush between timed steps, outside the events: write a 256 MB buffer (twice the
    L2), then read another 256 MB one, so that the lines the write left dirty are evicted
    (and written back) before the next step starts rather than during it."""
    import torch
    wbuf = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    rbuf = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    sink = torch.empty(1, dtype=torch.float32, device=dev)

    def flush():
        wbuf.zero_()
        torch.sum(rbuf, dim=0, keepdim=True, out=sink)
    return flush


_dist = None


def dist_barrier():
    if _dist is not None:
        _dist.barrier()


def make_dist_max(device="cuda"):
    """x -> the max of x over the ranks (identity without a process group). The
    reduction tensor lives on `device`: the rank's GPU under NCCL, the CPU under gloo."""
    import torch
    if _dist is None:
        return lambda x: x

    def f(x):
        t = torch.tensor([x], dtype=torch.float64, device=device)
        _dist.all_reduce(t, op=_dist.ReduceOp.MAX)
        return float(t.item())
    return f


# ----------------------------------------------------------------------------- our arm

def run_only(args):
    """Profiling helper: one of the secondary workloads alone (optionally smaller), on
    one GPU, printing its figures as one JSON line."""
    import torch
    import query_aware_selective_b200 as qas
    torch.cuda.set_device(0)
    qas.load()
    dev = torch.device("cuda", 0)
    peaks, peak_src = load_peaks()
    flush = make_flush(dev)
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid)).start()
    if args.only == "moba":
        out = bench_moba(args, dev, flush, make_dist_max(), peaks, peak_src, 1)
    elif args.only == "moba_decode":
        out = bench_moba_decode(args, dev, flush, make_dist_max(), peaks, peak_src, 1)
    elif args.only == "cca":
        out = bench_cca(args, dev, flush, make_dist_max(), peaks, peak_src, 1)
    elif args.only == "decode_varlen":
        out = bench_decode_varlen(args, dev, flush, make_dist_max(), peaks, peak_src, 1)
    elif args.only == "decode_1m":
        from query_aware_selective_b200 import synthetic
        out = bench_decode(args, dev, flush, make_dist_max(), peaks, peak_src, 1, workload=synthetic.DECODE_1M)
    elif args.only == "tiny_decode":
        out = bench_tiny_decode(args, dev, flush, make_dist_max(), world=1)
    elif args.only == "fit":
        out = bench_fit(args, dev, flush, make_dist_max(), peaks, peak_src, 1)
    else:
        out = bench_decode(args, dev, flush, make_dist_max(), peaks, peak_src, 1, per_head=args.only == "decode_per_head")
    out["clocks"] = sampler.stop()
    if out.get("roofline", {}).get("bound") == "tensor":
        finish_tensor_roofline(out["roofline"], out["clocks"], peaks, peak_src)
    print(json.dumps({"only": args.only, **out}), flush=True)


def run_ours(args):
    import torch
    import query_aware_selective_b200 as qas
    from query_aware_selective_b200 import cost, pipeline, synthetic

    global _dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        _dist = dist
    dist_max = make_dist_max()
    qas.load()
    dev = torch.device("cuda", local)
    props = torch.cuda.get_device_properties(dev)
    peaks, peak_src = load_peaks()
    flush = make_flush(dev)
    sampler = ClockSampler("GPU-" + str(props.uuid)).start()

    # ---------------------------------------------------------------- headline: prefill
    w = synthetic.PREFILL_32K
    if args.prefill_ctx:
        import dataclasses
        w = dataclasses.replace(w, n_ctx=args.prefill_ctx, name=f"esa_prefill_llama3_8b_ctx{args.prefill_ctx}_chunk512")
    p = qas.params(w.n_init, w.window, w.topk, w.eps, w.clamp_c)
    inp = synthetic.make_esa_inputs(w, device=dev)
    pf = pipeline.EsaPrefill(w.batch, w.n_ctx, w.chunk, w.hq, w.hkv, w.head_dim, w.d_c, p, device=dev)
    # The whole step (weight packing + every chunk) is one CUDA graph; the attention
    # launches carry external timing events, read after each replay.
    attn_events = []

    def prefill_run(ev=None):
        pf.run(inp["q"], inp["k"], inp["v"], inp["wq"], inp["wk"], attn_events=ev, external_events=True)

    launches0 = qas._abi.launch_count()
    prefill_run()
    torch.cuda.synchronize()
    launches_per_step = qas._abi.launch_count() - launches0

    def capture_body():
        attn_events.clear()
        prefill_run(attn_events)

    graph = pipeline.graph_of(capture_body)
    attn_ms = []
    ms, total_ms = time_steps(graph.replay, args.steps, args.warmup, flush, dist_max,
                              after_step=lambda: attn_ms.extend(a.elapsed_time(b) for a, b in attn_events))
    launches = launches_per_step * args.steps
    tokens = w.batch * w.n_ctx
    value = world * tokens * args.steps / (total_ms / 1e3)
    fl = cost.prefill_flops(w.n_ctx, w.chunk, w.hq, w.head_dim, w.d_c, w.n_init, w.window, w.topk)
    n_attn = len(attn_ms)
    attn_time_s = sum(attn_ms) / 1e3
    achieved = fl["attention"] * args.steps / attn_time_s / 1e12
    # peak and frac are filled in from this run's clock record (finish_rooflines)
    roofline = {"bound": "tensor", "kernel": "attn_tc_kernel<EsaTcProblem>", "achieved": round(achieved, 1),
                "peak": None, "unit": "TFLOP/s", "frac": None,
                "traffic": traffic_for("attn_tc_kernel<EsaTcProblem>", ["attn_tc.cuh", "common.cuh", "keylist.cuh"]),
                "flops_per_launch": fl["attention"] // (n_attn // args.steps),
                "launches": n_attn, "avg_launch_us": round(1e3 * sum(attn_ms) / n_attn, 2),
                "share_of_step": round(sum(attn_ms) / sum(ms), 3)}

    # ---------------------------------------------------------------- e2e through host buffers
    host = {n: inp[n].cpu().pin_memory() for n in ("q", "k", "v")}
    out_host = torch.empty(pf.out.shape, dtype=pf.out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size()

    # the library's own host-buffer entry: chunk by chunk, inputs up on one copy stream
    # and outputs back on another, overlapping the compute; one CUDA graph per step
    e2e_graph = pipeline.graph_of(lambda: pf.run_from_host(host["q"], host["k"], host["v"], inp["q"], inp["k"],
                                                           inp["v"], inp["wq"], inp["wk"], out_host))
    e_ms, e_total = time_steps(e2e_graph.replay, args.e2e_steps, 1, flush, dist_max)
    e2e = {"value": round(world * tokens * args.e2e_steps / (e_total / 1e3), 1), "unit": "tok/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": round(e_total / args.e2e_steps, 3),
           "path": "EsaPrefill.run_from_host: per-chunk host-to-device copies on one stream, "
                   "device-to-host copies on another, overlapping the compute"}
    del host, out_host, e2e_graph

    line = {"metric": METRIC, "value": round(value, 1), "unit": "tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "model": "llama-3-8b attention layer (random weights)",
                       "global_batch": w.batch * world, "seq_len": w.n_ctx, "chunk": w.chunk, "hq": w.hq,
                       "hkv": w.hkv, "head_dim": w.head_dim, "d_c": w.d_c, "n_init": w.n_init,
                       "window": w.window, "topk": w.topk, "eps": w.eps, "clamp_c": w.clamp_c,
                       "parallelism": f"replicas x{world}", "l2": L2_NOTE,
                       "execution": "one CUDA graph per step (weight packing and all 64 chunks)",
                       "precision": "bf16 attention (fp32 accumulate), fp32 selection"},
            "roofline": roofline, "e2e": e2e, "gpu_launches": launches}

    # ---------------------------------------------------------------- also: decode, MoBA
    if not args.no_extras:
        del inp, pf, graph
        torch.cuda.empty_cache()
        line["also"] = {"esa_decode_128k": bench_decode(args, dev, flush, dist_max, peaks, peak_src, world)}
        torch.cuda.empty_cache()
        line["also"]["esa_tiny_decode"] = bench_tiny_decode(args, dev, flush, dist_max, world,
                                                            oracle=rank == 0 and world == 1)
        torch.cuda.empty_cache()
        line["also"]["esa_decode_128k_per_head"] = bench_decode(args, dev, flush, dist_max, peaks, peak_src, world,
                                                                per_head=True)
        torch.cuda.empty_cache()
        line["also"]["esa_decode_128k_varlen"] = bench_decode_varlen(args, dev, flush, dist_max, peaks, peak_src,
                                                                     world)
        torch.cuda.empty_cache()
        line["also"]["esa_decode_1m"] = bench_decode(args, dev, flush, dist_max, peaks, peak_src, world,
                                                     workload=synthetic.DECODE_1M)
        torch.cuda.empty_cache()
        line["also"]["moba_prefill_64k"] = bench_moba(args, dev, flush, dist_max, peaks, peak_src, world)
        torch.cuda.empty_cache()
        line["also"]["moba_decode_64k"] = bench_moba_decode(args, dev, flush, dist_max, peaks, peak_src, world)
        torch.cuda.empty_cache()
        line["also"]["cca_prefill_64k"] = bench_cca(args, dev, flush, dist_max, peaks, peak_src, world)
        torch.cuda.empty_cache()
        line["also"]["esa_fit_64k"] = bench_fit(args, dev, flush, dist_max, peaks, peak_src, world)
    line["clocks"] = sampler.stop()
    finish_rooflines(line, line["clocks"], peaks, peak_src)
    line["gpu"] = props.name
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_prefill()
    if _dist is not None:
        _dist.barrier()
        _dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def bench_decode(args, dev, flush, dist_max, peaks, peak_src, world, per_head=False, workload=None):
    """ESA decode at 128K, batch 16 (or `workload`, e.g. the 1M-token stress case).
    per_head: the per-head selection variant (one index set per KV head,
    block-diagonal compression maps) on the same inputs."""
    import torch
    import query_aware_selective_b200 as qas
    from query_aware_selective_b200 import cost, pipeline, synthetic
    w = workload or synthetic.DECODE_128K
    if args.decode_batch:
        import dataclasses
        w = dataclasses.replace(w, batch=args.decode_batch, name=f"esa_decode_llama3_8b_b{args.decode_batch}_ctx{w.n_ctx}")
    p = qas.params(w.n_init, w.window, w.topk, w.eps, w.clamp_c)
    inp = synthetic.make_esa_inputs(w, device=dev)
    if per_head:
        wq_g, wk_g = synthetic.make_group_maps(w, device=dev)
        inp["wq"], inp["wk"] = pipeline.block_diagonal(wq_g), pipeline.block_diagonal(wk_g)
    dec = pipeline.EsaDecode(w.batch, w.n_ctx, w.hq, w.hkv, w.head_dim, w.d_c, p, device=dev, per_head=per_head)
    dec.fill_cache(inp["k"], inp["wk"])
    torch.cuda.synchronize()
    # the headline replays the bare step; the phase split comes from a second graph of the
    # same step with timing events between the phases, replayed separately
    graph = pipeline.graph_of(lambda: dec.step(inp["q"], inp["k"], inp["v"], inp["wq"], inp["wk"]))
    steps = max(args.steps, 20)
    ms, total = time_steps(graph.replay, steps, args.warmup, flush, dist_max)
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
    graph_ev = pipeline.graph_of(lambda: dec.step(inp["q"], inp["k"], inp["v"], inp["wq"], inp["wk"], phase_events=ev))
    phases = []
    time_steps(graph_ev.replay, 10, args.warmup, flush, dist_max,
               after_step=lambda: phases.append((ev[1].elapsed_time(ev[2]), ev[2].elapsed_time(ev[3]))))
    by = cost.decode_bytes(w.batch, w.n_ctx, w.hq, w.hkv, w.head_dim, w.d_c, w.n_init, w.window, w.topk)
    sel_ms = statistics.mean(e[0] for e in phases)
    att_ms = statistics.mean(e[1] for e in phases)
    hbm = peaks["hbm_gbs"]
    step_gbs = by["total"] / (total / steps / 1e3) / 1e9
    sel_gbs = (by["compressed_keys"]) / (sel_ms / 1e3) / 1e9
    att_gbs = (by["kv_rows"]) / (att_ms / 1e3) / 1e9
    return {"workload": w.name + ("_per_head" if per_head else ""),
            "value": round(world * w.batch * steps / (total / 1e3), 1), "unit": "tok/s",
            "ms_per_step": round(total / steps, 4), "steps": steps, "execution": "one CUDA graph per step",
            "roofline": {"bound": "hbm", "achieved": round(step_gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(step_gbs / hbm, 4), "bytes_per_step": by["total"],
                         "peak_source": f"{peak_src} HBM copy"},
            "phases": {"score_select_ms": round(sel_ms, 4), "score_select_gbs": round(sel_gbs, 1),
                       "sparse_attn_ms": round(att_ms, 4), "sparse_attn_gbs": round(att_gbs, 1)}}


def bench_tiny_decode(args, dev, flush, dist_max, world, oracle=True):
    """The tiny fp32 ESA decode step (one sequence of 2048 cached tokens, 4 heads of 64,
    map 256 -> 16, top-128): a latency case, reported in microseconds per step, with the
    oracle's time for the same whole step beside it (host cores, float64)."""
    import torch
    import query_aware_selective_b200 as qas
    from query_aware_selective_b200 import pipeline, synthetic
    w = synthetic.TINY_DECODE
    p = qas.params(w.n_init, w.window, w.topk, w.eps, w.clamp_c)
    inp = synthetic.make_esa_inputs(w)
    dinp = {n: t.to(dev) for n, t in inp.items() if torch.is_tensor(t)}
    dec = pipeline.EsaDecode(w.batch, w.n_ctx, w.hq, w.hkv, w.head_dim, w.d_c, p, dtype=torch.float32, device=dev)
    dec.fill_cache(dinp["k"], dinp["wk"])
    torch.cuda.synchronize()
    graph = pipeline.graph_of(lambda: dec.step(dinp["q"], dinp["k"], dinp["v"], dinp["wq"], dinp["wk"]))
    steps = max(args.steps, 50)
    launches0 = qas._abi.launch_count()
    dec.step(dinp["q"], dinp["k"], dinp["v"], dinp["wq"], dinp["wk"])
    torch.cuda.synchronize()
    launches = qas._abi.launch_count() - launches0
    ms, total = time_steps(graph.replay, steps, args.warmup, flush, dist_max)
    us = 1e3 * total / steps
    out = {"workload": w.name, "value": round(world * w.batch * steps / (total / 1e3), 1), "unit": "tok/s",
           "us_per_step": round(us, 2), "steps": steps, "dtype": "f32", "kernels_per_step": launches,
           "execution": "one CUDA graph per step (query and key compression, selection, attention)",
           "bound": "latency (0.9 MB per step: launch and dependency latency, not bandwidth)"}
    if oracle:
        from oracle import esa as oesa
        args_np = [inp[n].numpy() for n in ("q", "k", "v", "wq", "wk")]
        reps, t0 = 0, time.perf_counter()
        while reps < 3 or time.perf_counter() - t0 < 2.0:
            oesa.decode_step(*args_np, w.n_init, w.window, w.topk, w.eps, w.clamp_c)
            reps += 1
        o_us = 1e6 * (time.perf_counter() - t0) / reps
        out["oracle"] = {"us_per_step": round(o_us, 1), "cores": blas_threads(), "kind": "oracle",
                         "sample": f"the whole step (compress the 2048 keys and the query, select, attend), "
                                   f"{reps} runs"}
    return out


def bench_fit(args, dev, flush, dist_max, peaks, peak_src, world):
    """Offline fit of the compression maps (4096 -> 128) from 65536 calibration tokens of
    the Llama-3-8B layer shape: Gram matrices on the tensor cores, fp64 factorisations and
    the subspace iteration, timed as one CUDA graph; the query Gram product (the tensor
    work) is also timed alone for its roofline."""
    import torch
    import query_aware_selective_b200 as qas
    from query_aware_selective_b200 import pipeline, synthetic
    w = synthetic.FIT_64K
    inp = synthetic.make_fit_inputs(w, device=dev)
    ws = torch.empty(qas._abi.fit_workspace_size(w.n_tokens, w.n_tokens, w.hq, w.hkv, w.head_dim, w.d_c,
                                                 w.oversample) + 256, dtype=torch.uint8, device=dev)
    graph = pipeline.graph_of(lambda: qas.fit_maps(inp["q"], inp["k"], w.d_c, inp["omega"], ridge=w.ridge,
                                                   power_iters=w.power_iters, workspace=ws))
    steps = max(3, args.steps // 3)
    ms, total = time_steps(graph.replay, steps, args.warmup, flush, dist_max)
    # the query Gram product alone: n * dq * (dq + 1) flops of symmetric X^T X
    dq = w.hq * w.head_dim
    x = inp["q"].view(w.n_tokens, dq)
    gws = torch.empty(qas._abi.load().esa_gram_workspace_size(w.n_tokens, dq) + 256, dtype=torch.uint8, device=dev)
    g = torch.empty((dq, dq), dtype=torch.float64, device=dev)
    gram_graph = pipeline.graph_of(lambda: qas.gram(x, workspace=gws, out=g))
    gms, gtotal = time_steps(gram_graph.replay, steps, args.warmup, flush, dist_max)
    flops = w.n_tokens * dq * (dq + 1)
    ach = flops / (gtotal / steps / 1e3) / 1e12
    return {"workload": w.name, "value": round(world * w.n_tokens * steps / (total / 1e3), 1),
            "unit": "calibration tok/s", "ms_per_step": round(total / steps, 3), "steps": steps,
            "execution": "one CUDA graph per fit (Grams, Cholesky, C, subspace iteration, Rayleigh-Ritz, maps)",
            "gram_ms": round(gtotal / steps, 4),
            "roofline": {"bound": "tensor", "kernel": "esa_gram: gram_kernel + fixed-order fp64 sum (query Gram X^T X, 65536 x 4096 bf16)",
                         "achieved": round(ach, 1), "peak": None, "unit": "TFLOP/s", "frac": None,
                         "flops_per_launch": flops}}


def bench_decode_varlen(args, dev, flush, dist_max, peaks, peak_src, world):
    """ESA decode, batch 16, caches of 128K rows holding a seeded mix of lengths
    (sequence 0 at 131072, the rest uniform in [8192, 131072]), lengths on the device."""
    import torch
    import query_aware_selective_b200 as qas
    from query_aware_selective_b200 import cost, pipeline, synthetic
    w = synthetic.DECODE_128K
    p = qas.params(w.n_init, w.window, w.topk, w.eps, w.clamp_c)
    lens = synthetic.varlen_lengths(w.batch, w.n_ctx, 8192, seed=w.seed + 2000)
    inp = synthetic.make_esa_inputs(w, device=dev)
    dec = pipeline.EsaDecodeVarlen(w.batch, w.n_ctx, w.hq, w.hkv, w.head_dim, w.d_c, p, device=dev)
    dec.fill_cache(inp["k"], inp["wk"], lens.tolist())
    seq_len = lens.to(dev)
    k_new = inp["k"][torch.arange(w.batch, device=dev), seq_len - 1].contiguous()
    torch.cuda.synchronize()
    graph = pipeline.graph_of(lambda: dec.step(inp["q"], k_new, inp["k"], inp["v"], inp["wq"], inp["wk"], seq_len))
    steps = max(args.steps, 20)
    ms, total = time_steps(graph.replay, steps, args.warmup, flush, dist_max)
    by = cost.decode_varlen_bytes(lens.tolist(), w.hq, w.hkv, w.head_dim, w.d_c, w.n_init, w.window, w.topk)
    gbs = by["total"] / (total / steps / 1e3) / 1e9
    hbm = peaks["hbm_gbs"]
    return {"workload": f"esa_decode_llama3_8b_b{w.batch}_varlen8192to131072",
            "lengths": lens.tolist(), "value": round(world * w.batch * steps / (total / 1e3), 1), "unit": "tok/s",
            "ms_per_step": round(total / steps, 4), "steps": steps, "execution": "one CUDA graph per step",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "bytes_per_step": by["total"],
                         "peak_source": f"{peak_src} HBM copy"}}


def bench_cca(args, dev, flush, dist_max, peaks, peak_src, world):
    """CCA-style causal prefill: 65536 tokens, 32 / 8 heads, groups of 128, window 1024."""
    import torch
    import query_aware_selective_b200 as qas
    from query_aware_selective_b200 import cost, pipeline, synthetic
    w = synthetic.CCA_64K
    inp = synthetic.make_cca_inputs(w, device=dev)
    out = torch.empty_like(inp["q"])
    ws = torch.empty(qas._abi.cca_workspace_size(w.batch, w.seq, w.hq, w.head_dim, w.group) + 256,
                     dtype=torch.uint8, device=dev)
    graph = pipeline.graph_of(lambda: qas.cca_attn(inp["q"], inp["k"], inp["v"], w.group, w.window, out=out,
                                                   workspace=ws))
    steps = max(3, args.steps // 2)
    ms, total = time_steps(graph.replay, steps, args.warmup, flush, dist_max)
    fl = cost.cca_flops(w.seq, w.hq, w.head_dim, w.group, w.window)
    ach = fl["total"] * w.batch / (total / steps / 1e3) / 1e12
    return {"workload": w.name, "value": round(world * w.batch * w.seq * steps / (total / 1e3), 1),
            "unit": "tok/s", "ms_per_step": round(total / steps, 3), "steps": steps,
            "execution": "one CUDA graph per step",
            "roofline": {"bound": "tensor", "achieved": round(ach, 1), "peak": None, "unit": "TFLOP/s",
                         "frac": None, "flops_per_step": fl["total"] * w.batch}}


def bench_moba_decode(args, dev, flush, dist_max, peaks, peak_src, world):
    """MoBA decode: batch 16, 32 heads, one query at position 65535, top-3 past blocks."""
    import torch
    from query_aware_selective_b200 import cost, pipeline, synthetic
    w = synthetic.MOBA_DECODE_64K
    if args.decode_batch:
        import dataclasses
        w = dataclasses.replace(w, batch=args.decode_batch,
                                name=f"moba_decode_h{w.heads}_b{args.decode_batch}_ctx{w.seq}_block{w.block}_top{w.topk}")
    inp = synthetic.make_moba_decode_inputs(w, device=dev)
    dec = pipeline.MobaDecode(w.batch, w.seq, w.heads, w.head_dim, w.block, w.topk, device=dev)
    dec.fill(inp["k"])
    torch.cuda.synchronize()
    graph = pipeline.graph_of(lambda: dec.step(inp["q"], inp["k"], inp["v"]))
    steps = max(args.steps, 20)
    ms, total = time_steps(graph.replay, steps, args.warmup, flush, dist_max)
    by = cost.moba_decode_bytes(w.batch, w.seq, w.heads, w.head_dim, w.block, w.topk)
    gbs = by["total"] / (total / steps / 1e3) / 1e9
    hbm = peaks["hbm_gbs"]
    return {"workload": w.name, "value": round(world * w.batch * steps / (total / 1e3), 1), "unit": "tok/s",
            "ms_per_step": round(total / steps, 4), "steps": steps, "execution": "one CUDA graph per step",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "bytes_per_step": by["total"],
                         "peak_source": f"{peak_src} HBM copy"}}


def bench_moba(args, dev, flush, dist_max, peaks, peak_src, world):
    import torch
    from query_aware_selective_b200 import cost, pipeline, synthetic
    w = synthetic.MOBA_64K
    if args.moba_seq:
        import dataclasses
        w = dataclasses.replace(w, seq=args.moba_seq, name=f"moba_prefill_h{w.heads}_seq{args.moba_seq}_block{w.block}_top{w.topk}")
    inp = synthetic.make_moba_inputs(w, device=dev)
    mb = pipeline.MobaPrefill(w.batch, w.seq, w.heads, w.head_dim, w.block, w.topk, device=dev)
    graph = pipeline.graph_of(lambda: mb.run(inp["q"], inp["k"], inp["v"]))
    steps = max(3, args.steps // 2)
    ms, total = time_steps(graph.replay, steps, args.warmup, flush, dist_max)
    fl = cost.moba_flops(w.seq, w.heads, w.head_dim, w.block, w.topk)
    ach = fl["total"] / (total / steps / 1e3) / 1e12
    return {"workload": w.name, "value": round(world * w.batch * w.seq * steps / (total / 1e3), 1),
            "unit": "tok/s", "ms_per_step": round(total / steps, 3), "steps": steps,
            "execution": "one CUDA graph per step",
            "roofline": {"bound": "tensor", "achieved": round(ach, 1), "peak": None, "unit": "TFLOP/s",
                         "frac": None, "flops_per_step": fl["total"]}}


# ----------------------------------------------------------------------------- oracle arm

def oracle_prefill_sample(w, inp_np, c0, rows):
    """One chunk of the oracle's chunked prefill: compress the chunk's keys and
    queries, select over the middle, attend `rows` of the chunk's queries.
    Returns (seconds, tokens-equivalent)."""
    import numpy as np
    from oracle import esa as oesa
    lq = w.chunk
    t0 = time.perf_counter()
    kc_new = oesa.compress(inp_np["k"][0, c0:c0 + lq], inp_np["wk"], w.hq)
    inp_np["k_c"][0, c0:c0 + lq] = kc_new
    q_c = oesa.compress(inp_np["q"][0, c0:c0 + lq], inp_np["wq"], w.hq)[None]
    idx, cnt, _ = oesa.score_select(q_c, inp_np["k_c"], c0, w.n_init, w.window, w.topk, w.eps, w.clamp_c)
    t_sel = time.perf_counter() - t0
    t1 = time.perf_counter()
    oesa.sparse_attn(inp_np["q"][:, c0:c0 + lq], inp_np["k"], inp_np["v"], c0, idx, cnt, w.n_init, w.window,
                     rows=[(0, i) for i in range(rows)])
    t_att = time.perf_counter() - t1
    per_token = t_sel / lq + t_att / rows
    return t_sel + t_att, 1.0 / per_token


def oracle_setup(device="cpu", n_chunks=1):
    """The prefill workload's inputs on the host for the oracle, with the compressed
    cache filled up to c0 = 16384 (untimed) and the queries of n_chunks chunks from c0."""
    import numpy as np
    from oracle import esa as oesa
    from query_aware_selective_b200 import synthetic
    w = synthetic.PREFILL_32K
    inp = synthetic.make_esa_inputs(w, device=device)
    c0 = (w.n_ctx // 2 // w.chunk) * w.chunk                     # the middle chunk (c0 = 16384)
    c1 = c0 + n_chunks * w.chunk
    inp_np = {"q": inp["q"][:, c0:c1].float().cpu().numpy(), "k": inp["k"].float().cpu().numpy(),
              "v": inp["v"].float().cpu().numpy(), "wq": inp["wq"].cpu().numpy(), "wk": inp["wk"].cpu().numpy()}
    # queries outside the sampled chunks are not needed: re-index so they sit at c0
    q_full = np.zeros((1, c1) + inp_np["q"].shape[2:], dtype=np.float32)
    q_full[:, c0:] = inp_np["q"]
    inp_np["q"] = q_full
    inp_np["k_c"] = np.zeros((1, w.n_ctx, w.d_c))
    inp_np["k_c"][0, :c0] = oesa.compress(inp_np["k"][0, :c0], inp_np["wk"], w.hq)   # cache state (untimed)
    return w, inp_np, c0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline_prefill(seconds_hint=12.0, max_chunks=16):
    """The oracle on consecutive chunks of the prefill from c0 = 16384 until about
    seconds_hint of CPU work (at most max_chunks chunks)."""
    w, inp_np, c0 = oracle_setup(n_chunks=max_chunks)
    rows = 16
    secs, per_tok, n = 0.0, [], 0
    while n < max_chunks and secs < seconds_hint:
        s, tps = oracle_prefill_sample(w, inp_np, c0 + n * w.chunk, rows)
        secs += s
        per_tok.append(1.0 / tps)
        n += 1
    value = 1.0 / (sum(per_tok) / len(per_tok))
    return {"value": round(value, 3), "unit": "tok/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} consecutive 512-token chunks of the 32768-token prefill from c0={c0}: per chunk, "
                      f"compress its keys and queries, select over its middle "
                      f"({c0 - w.window - w.n_init} tokens and up), attend {rows} of its query rows; "
                      f"tok/s = 1 / mean over chunks of (select time / 512 + attention time / {rows}); "
                      f"{secs:.1f} s of CPU work"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w, inp_np, c0 = oracle_setup()
    rows = 8
    for _ in range(args.warmup):
        oracle_prefill_sample(w, inp_np, c0, rows)
    vals, secs = [], 0.0
    for _ in range(args.steps):
        s, tps = oracle_prefill_sample(w, inp_np, c0, rows)
        vals.append(tps)
        secs += s
    per_tok = sum(1.0 / v for v in vals) / len(vals)
    value = 1.0 / per_tok
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tok/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * secs / args.steps, 1), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "seq_len": w.n_ctx, "chunk": w.chunk, "global_batch": w.batch},
            "cpu_baseline": {"kind": "oracle", "cores": blas_threads(), "value": round(value, 3), "unit": "tok/s",
                             "sample": f"per step: one 512-token chunk at c0={c0} (compress, select) plus "
                                       f"attention for {rows} of its query rows"},
            "e2e": {"value": round(value, 3), "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def spawn_command(argv, n, port):
    """The torch.distributed.run command that runs this script as n ranks on one node
    (one process per GPU), with the same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]


def self_spawn(n, argv):
    """`bench.py --gpus N` started as a single process: start the N ranks here and pass
    their exit status on (rank 0 prints the line)."""
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    return subprocess.call(spawn_command(argv, n, port))


def main():
    args = parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and not args.only:
        sys.exit(self_spawn(args.gpus, sys.argv[1:]))
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.only:
        run_only(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
