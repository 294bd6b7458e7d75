"""Benchmark of the verified sparse decode step (vattn_decode) on B200.

    python bench.py [--gpus N --steps K --warmup W] [--workload gqa_32k] [--eps E]
                    [--guarantee denominator|output]
    python bench.py --impl reference ...      # the CPU oracle, timed on host cores

One step = one vattn_decode call over the whole batch of the workload (every
row of the hot path: query prep, ranking-score pass, top-k select, pilot,
budget, gather, combine). Inputs are resident in HBM before the timed region
and larger than L2 (so no flush is needed). Prints one JSON line (rank 0).
The headline is --workload (default gqa_32k); at one GPU the line also carries
`per_config`, the same measurements for the other long-context workloads
(sparq_128k, loki_64k, paged_sweep at eps 0.05). The score pass's roofline is
timed by events on SCORE_SAMPLES further calls after the timed region. `host_kv`
times the HOST_KV workloads with their K and V caches in page-locked host memory,
against dense decode over the same host-resident caches.
Under torchrun each rank runs its own batch on its own GPU (weak scaling; no
collective on the data path, one max-reduction of the elapsed time); with
--shard heads|batch the ranks split one batch instead and all-gather its
outputs over NCCL in every step (strong scaling).
"""
import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from verified_sparse_attention_b200 import _abi, ranks, synth  # noqa: E402
from verified_sparse_attention_b200.decoder import decoder_for, params_for  # noqa: E402

METRIC = "sparse decode-attn calls/s & achieved HBM GB/s (% of ~8 TB/s) at 32k–128k ctx"
NOMINAL_HBM_GBS = 8000.0
SCORE_SAMPLES = 64   # score passes timed by events after the timed region
# the other long-context workloads measured in the same run (name, eps override)
PER_CONFIG = [("sparq_128k", None), ("loki_64k", None), ("paged_sweep", 0.05)]
# workloads also timed with their K and V caches in page-locked host memory
HOST_KV = ["loki_64k"]
KERNEL_SOURCE = "verified_sparse_attention_b200/csrc/vattn_kernels.cuh"
# the sections of KERNEL_SOURCE that hold the ranking-score pass (its kernels
# and their own helpers): the DRAM counters in profiles/ are keyed to them
SCORE_SECTIONS = ["score pass helpers", "k_score_rows", "k_score_sparq", "k_score_tma"]


def kernel_hash():
    """sha256 (16 hex digits) of the score-pass sections' source text."""
    with open(os.path.join(ROOT, KERNEL_SOURCE)) as f:
        text = f.read()
    marks = [(m.start(), m.group(1).strip()) for m in re.finditer(r"^// =+ (.*)$", text, re.M)]
    parts = {}
    for i, (pos, name) in enumerate(marks):
        parts[name] = text[pos:marks[i + 1][0] if i + 1 < len(marks) else len(text)]
    h = hashlib.sha256()
    for name in SCORE_SECTIONS:
        # a missing section changes the hash, so stale counters are not reported
        h.update(parts.get(name, f"<no section {name}>").encode())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def profiled_traffic(workload):
    """DRAM bytes per score-pass launch from the committed ncu summary, if still current."""
    path = os.path.join(ROOT, "profiles", f"score_pass_{workload}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_hash") != kernel_hash():
        return None
    return d.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock and throttle reasons sampled through NVML while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index, period=0.005):
        """index None: sample nothing."""
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self.ok = period, False
        self._stop = threading.Event()
        if index is None:
            return
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            get = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
            r = get(self.h)
            for bit, name in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)
        except Exception:
            pass

    def __enter__(self):
        if self.ok:
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ byte accounting
def algorithmic_bytes(w, x, res):
    """Bytes one call must move, from the call's own outputs: the score pass's K (or
    proxy) rows of the middle, the 4-byte ranking keys it writes (workspace, reported
    apart), and the gathers' K and V rows of every selected entry."""
    e = synth.bytes_per_elem(w)
    d = w.head_dim
    n = x["seq_lens"].to(torch.int64).cpu()
    s1 = torch.clamp(n, max=w.sinks)
    wst = torch.maximum(n - w.window, s1)
    mid = (wst - s1).clamp(min=0)                          # middle rows per sequence
    per_row = {"exact": d * e, "sparq": w.proxy_rank * e, "loki": w.proxy_rank * e}[w.proxy]
    rows = int(mid.sum()) * w.num_kv_heads
    cnt = res["sel_count"].to(torch.int64).cpu()            # [B, Hkv] rows gathered (K and V)
    gather = int(cnt.sum()) * 2 * d * e
    if w.guarantee == "output":
        # the numerator statistics read the V rows of I_f and the pilot once more
        # for every unit that drew a pilot (N_tail > p)
        kb = (n * w.topk_num) // w.topk_den if w.topk_den else torch.full_like(n, w.topk_abs)
        k = torch.minimum(kb, mid)
        p = (torch.clamp((n * w.pilot_num + w.pilot_den - 1) // w.pilot_den, min=w.pilot_min)
             if w.pilot_den else torch.full_like(n, w.pilot_min))
        n_if = s1 + k + (n - wst)
        piloted = (mid - k) > p
        gather += int(((n_if + p) * piloted).sum()) * w.num_kv_heads * d * e
    return {"score_read": rows * per_row, "key_write": rows * 4, "gather": gather,
            "call": rows * per_row + gather}


# ------------------------------------------------------------------ one workload
def run_config(w, args, dev, world, steps, *, headline):
    """Time `steps` decode calls of workload w (inputs resident in HBM, larger than L2),
    then 64 more with the score pass timed by events, then the dense decode on the same
    inputs. Returns (decoder, inputs, result dict)."""
    x = synth.make_inputs(w, device=dev)
    dec = decoder_for(w, device=dev)
    prm = params_for(w, x)
    outs = dec.alloc_outputs(w.batch)
    stream = torch.cuda.current_stream()

    def step():
        dec.decode(x["q"], x["k_cache"], x["v_cache"], x["page_table"], x["seq_lens"], prm,
                   outputs=outs, stream=stream)

    # untimed clock ramp-up (the GPU idles at a low clock before this)
    torch.cuda.synchronize()
    t_ramp = time.perf_counter()
    while time.perf_counter() - t_ramp < args.ramp_s:
        for _ in range(20):
            step()
        torch.cuda.synchronize()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dec.last_error():
        raise RuntimeError(f"{w.name}: device error word set during warm-up")
    launches_per_call = _abi.vattn_last_launch_count(dec.ctx)

    ranks.barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with (ClockSampler(torch.cuda.current_device()) if headline else ClockSampler(None)) as clk:
        t0.record(stream)
        for _ in range(steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
    ranks.barrier(world)
    ms = t0.elapsed_time(t1)
    ms_max = ranks.max_over_ranks(ms, world, dev)

    # the score pass alone: an event pair on the launching stream around it in each of
    # SCORE_SAMPLES further calls (the pair stops it overlapping its neighbours, so
    # these calls are kept out of the timed region above)
    _abi.vattn_score_pass_ms(dec.ctx, reset=True)
    _abi.vattn_set_timing(dec.ctx, 1)
    for _ in range(SCORE_SAMPLES):
        step()
    torch.cuda.synchronize()
    _abi.vattn_set_timing(dec.ctx, 0)
    score_ms, score_n = _abi.vattn_score_pass_ms(dec.ctx, reset=True)
    if dec.last_error():
        raise RuntimeError(f"{w.name}: device error word set")

    nbytes = algorithmic_bytes(w, x, outs)
    budgets = outs["budgets"].cpu()

    # dense decode attention on the same inputs (comparison baseline)
    dsteps = max(10, min(steps, 200))
    for _ in range(args.warmup):
        dec.dense(x["q"], x["k_cache"], x["v_cache"], x["page_table"], x["seq_lens"],
                  x["num_pages"], stream=stream)
    torch.cuda.synchronize()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for _ in range(dsteps):
        dec.dense(x["q"], x["k_cache"], x["v_cache"], x["page_table"], x["seq_lens"],
                  x["num_pages"], stream=stream)
    d1.record(stream)
    torch.cuda.synchronize()
    dense_ms = d0.elapsed_time(d1) / dsteps

    return dec, x, prm, dict(w=w, ms=ms_max, steps=steps, score_ms=score_ms, score_n=score_n,
                             bytes=nbytes, budgets=budgets, launches_per_call=launches_per_call,
                             clocks=clk.summary() if headline else None, dense_ms=dense_ms)


def summarize(r, world, peak):
    """Rates of one run_config result: calls/s, the score pass's roofline, whole-call GB/s."""
    calls_s = ranks.job_rate(world, r["steps"], r["ms"])
    call_s = r["ms"] / 1e3 / r["steps"]
    avg_score_s = (r["score_ms"] / max(1, r["score_n"])) / 1e3
    b = r["bytes"]
    achieved = b["score_read"] / avg_score_s / 1e9
    return {"calls_per_s": calls_s, "us_per_call": call_s * 1e6,
            "score_pass": {"achieved_gbs": achieved, "frac": achieved / peak,
                           "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                           "avg_launch_us": avg_score_s * 1e6, "samples": r["score_n"],
                           "read_bytes_per_launch": b["score_read"],
                           "key_write_bytes_per_launch": b["key_write"]},
            "call_kv_bytes": b["call"], "call_achieved_gbs": b["call"] / call_s / 1e9,
            "call_frac_of_peak": b["call"] / call_s / 1e9 / peak,
            "dense_calls_per_s": world / (r["dense_ms"] / 1e3),
            "speedup_vs_dense": r["dense_ms"] / (r["ms"] / r["steps"]),
            "budget_mean": float(r["budgets"].float().mean())}


def run_e2e(args, w, x, dec, prm, stream, dev, world):
    """Same metric through the C ABI with host buffers: pinned host -> device copies of
    every input and a device -> host read of every result (out, sel_idx, sel_count,
    budgets, head_need) inside the timed region."""
    keys = ["q", "k_cache", "v_cache", "page_table", "seq_lens"]
    extra = [k for k in ("k_t_cache", "k_proj_cache", "proj_basis") if k in x]
    host = {k: x[k].cpu().pin_memory() for k in keys + extra}
    devb = {k: torch.empty_like(x[k]) for k in keys + extra}
    outs = dec.alloc_outputs(w.batch)
    out_h = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in outs.items()}
    p = params_for(w, {**devb, "num_pages": x["num_pages"]}, eps=args.eps)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(v.numel() * v.element_size() for v in out_h.values())
    steps = max(1, min(args.steps, args.e2e_steps))

    def step():
        for k in host:
            devb[k].copy_(host[k], non_blocking=True)
        dec.decode(devb["q"], devb["k_cache"], devb["v_cache"], devb["page_table"],
                   devb["seq_lens"], p, outputs=outs, stream=stream)
        for k in out_h:
            out_h[k].copy_(outs[k], non_blocking=True)

    step()
    torch.cuda.synchronize()
    ranks.barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = ranks.max_over_ranks(a.elapsed_time(b), world, dev)
    del devb, host
    return {"value": ranks.job_rate(world, steps, ms), "unit": "calls/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps}


def run_host_kv(name, args, dev):
    """Workload `name` with its K and V caches in page-locked host memory (the proxy
    caches, q, page table and lengths on the GPU): sparse calls/s against dense decode
    over the same host-resident caches, both by CUDA events on the launching stream."""
    w = synth.WORKLOADS[name]
    xd = synth.make_inputs(w, device=dev)
    x = dict(xd, k_cache=xd["k_cache"].cpu().pin_memory(), v_cache=xd["v_cache"].cpu().pin_memory())
    del xd
    torch.cuda.empty_cache()
    dec = decoder_for(w, device=dev, kv_location="host")
    prm = params_for(w, x)
    outs = dec.alloc_outputs(w.batch)
    stream = torch.cuda.current_stream()

    def timed(fn, n):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    sparse_ms = timed(lambda: dec.decode(x["q"], x["k_cache"], x["v_cache"], x["page_table"],
                                         x["seq_lens"], prm, outputs=outs, stream=stream),
                      args.host_kv_steps)
    if dec.last_error():
        raise RuntimeError(f"{name} (host-resident caches): device error word set")
    dense_ms = timed(lambda: dec.dense(x["q"], x["k_cache"], x["v_cache"], x["page_table"],
                                       x["seq_lens"], x["num_pages"], stream=stream),
                     max(1, args.host_kv_steps // 4))
    b = algorithmic_bytes(w, x, outs)
    e = synth.bytes_per_elem(w)
    host_sparse = b["gather"] + (b["score_read"] if w.proxy == "exact" else 0)
    host_dense = int(x["seq_lens"].to(torch.int64).sum()) * w.num_kv_heads * 2 * w.head_dim * e
    dec.close()
    del x
    torch.cuda.empty_cache()
    return {"workload": synth.describe(w), "calls_per_s": 1e3 / sparse_ms,
            "dense_calls_per_s": 1e3 / dense_ms, "speedup_vs_dense": dense_ms / sparse_ms,
            "host_bytes_per_call": host_sparse, "dense_host_bytes_per_call": host_dense,
            "host_link_gbs": host_sparse / (sparse_ms / 1e3) / 1e9,
            "dense_host_link_gbs": host_dense / (dense_ms / 1e3) / 1e9,
            "steps": args.host_kv_steps}


def run_sharded(args, w, rank, world, dev):
    """One batch split over the ranks (--shard heads|batch): each rank decodes its slice
    and the outputs are all-gathered over NCCL inside every timed step, so a step is
    one whole-batch call (strong scaling)."""
    x = synth.make_inputs(w, device=dev)  # the whole batch (same seed on every rank)
    ws, boff, hoff = ranks.shard_workload(w, args.shard, world, rank)
    xs = ranks.shard_inputs(x, w, args.shard, world, rank)
    del x
    torch.cuda.empty_cache()
    dec = decoder_for(ws, device=dev)
    prm = params_for(ws, xs, batch_offset=boff, head_offset=hoff)
    outs = dec.alloc_outputs(ws.batch)
    stream = torch.cuda.current_stream()

    def step():
        dec.decode(xs["q"], xs["k_cache"], xs["v_cache"], xs["page_table"], xs["seq_lens"], prm,
                   outputs=outs, stream=stream)
        return ranks.gather_outputs(outs, args.shard, world)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dec.last_error():
        raise RuntimeError("device error word set during warm-up")
    ranks.barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        a.record(stream)
        for _ in range(args.steps):
            step()
        b.record(stream)
        torch.cuda.synchronize()
    ranks.barrier(world)
    ms = ranks.max_over_ranks(a.elapsed_time(b), world, dev)
    launches = _abi.vattn_last_launch_count(dec.ctx) * args.steps
    dec.close()
    return {"value": args.steps / (ms / 1e3), "ms": ms, "clocks": clk.summary(), "gpu_launches": launches,
            "shard": {"mode": args.shard, "units_per_rank": ws.units, "units": w.units,
                      "collective": "all_gather of out, sel_idx, sel_count, budgets, head_need"}}


def time_oracle_all_cores(w, cpu_inputs, budget_s):
    """The same oracle on every host core: one thread per core, each running whole
    (sequence, KV head) units (the C library releases the GIL) until budget_s.
    Returns (calls/s equivalent, units done, seconds, threads)."""
    import concurrent.futures
    import oracle
    pr = oracle.make_problem(w)
    U = w.units
    T = os.cpu_count() or 1
    t0 = time.perf_counter()

    def worker(tid):
        done, u = 0, tid
        while time.perf_counter() - t0 < budget_s and done < 5 * U:
            oracle.decode(pr, cpu_inputs, units=[u % U])
            done += 1
            u += T
        return done

    with concurrent.futures.ThreadPoolExecutor(T) as ex:
        done = sum(ex.map(worker, range(T)))
    el = time.perf_counter() - t0
    return (done / U) / el, done, el, T


def time_oracle(w, cpu_inputs, budget_s, units_per_step=None):
    """Run the oracle unit by unit on the host until budget_s elapses (or all units).
    Returns (calls/s equivalent, units done, seconds)."""
    import oracle
    pr = oracle.make_problem(w)
    U = w.units
    chunk = 4 if units_per_step is None else units_per_step
    done, t0 = 0, time.perf_counter()
    u = 0
    while True:
        oracle.decode(pr, cpu_inputs, units=[(u + i) % U for i in range(chunk)])
        done += chunk
        u += chunk
        el = time.perf_counter() - t0
        if units_per_step is not None or el >= budget_s or done >= 5 * U:
            break
    el = time.perf_counter() - t0
    return (done / U) / el, done, el


def emit(line):
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--ramp-s", type=float, default=0.3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="gqa_32k", choices=list(synth.WORKLOADS))
    ap.add_argument("--eps", type=float, default=None)
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences per call (default: the workload's own)")
    ap.add_argument("--guarantee", default="denominator", choices=["denominator", "output"],
                    help="what the sample size bounds: the softmax denominator, or the output too")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", dest="per_config", action="store_false",
                    help="skip the other long-context workloads")
    ap.add_argument("--per-config-steps", type=int, default=200)
    ap.add_argument("--shard", default=None, choices=list(ranks.SHARD_MODES),
                    help="split one batch over the ranks (by KV head or by sequence) and "
                         "all-gather the outputs, instead of one batch per rank")
    ap.add_argument("--host-kv-steps", type=int, default=8,
                    help="decode calls timed with the KV cache in host memory (0: skip)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world, rank, local_rank = ranks.rank_env()
    w = synth.WORKLOADS[args.workload].replace(guarantee=args.guarantee)
    if args.eps is not None:
        w = w.replace(eps=args.eps)
    if args.batch is not None:
        w = w.replace(batch=args.batch)
    cfg = {"workload": synth.describe(w), "name": w.name, "batch": w.batch,
           "ctx": w.max_ctx if w.min_ctx == w.max_ctx else [w.min_ctx, w.max_ctx],
           "l2": "inputs larger than L2 (no flush)", "parallelism": f"replicas{world}"}

    if args.impl == "reference":
        if not ranks.reports(rank):
            return
        t_gen = time.perf_counter()
        cpu = synth.make_inputs(w)
        gen_s = time.perf_counter() - t_gen
        ups = max(1, w.units // 16)
        for _ in range(args.warmup):
            time_oracle(w, cpu, 0, units_per_step=1)
        t0 = time.perf_counter()
        done = 0
        for _ in range(args.steps):
            _, d, _ = time_oracle(w, cpu, 0, units_per_step=ups)
            done += d
        el = time.perf_counter() - t0
        val = (done / w.units) / el
        emit({"impl": "reference", "metric": METRIC, "value": val, "unit": "calls/s",
              "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
              "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
              "vs_baseline": None, "dtype": w.dtype, "data": "synthetic", "config": cfg,
              "cpu_baseline": {"value": val, "unit": "calls/s", "cores": 1, "kind": "oracle",
                               "sample": f"{ups} of {w.units} (sequence, KV head) units per step, "
                                         f"single-threaded C oracle; input generation {gen_s:.1f}s untimed"},
              "e2e": {"value": val, "unit": "calls/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}})
        return

    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peak, peak_kind = load_peaks()
    if args.shard:
        r = run_sharded(args, w, rank, world, dev)
        cfg["parallelism"] = f"shard-{args.shard}{world}"
        if ranks.reports(rank):
            emit({"metric": METRIC, "value": r["value"], "unit": "calls/s", "n_gpus": world,
                  "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms"] / args.steps,
                  "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
                  "dtype": w.dtype, "data": "synthetic", "config": cfg, "shard": r["shard"],
                  "gpu_launches": r["gpu_launches"], "clocks": r["clocks"]})
        if world > 1:
            ranks.barrier(world)
            torch.distributed.destroy_process_group()
        return
    wr = ranks.rank_workload(w, rank)
    dec, x, prm, r = run_config(wr, args, dev, world, args.steps, headline=True)
    sm = summarize(r, world, peak)
    sp = sm["score_pass"]
    e2e = run_e2e(args, wr, x, dec, prm, torch.cuda.current_stream(), dev, world)
    line = {"metric": METRIC, "value": sm["calls_per_s"], "unit": "calls/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms"] / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic", "config": cfg,
            "roofline": {"bound": "hbm",
                         "kernel": "score pass (k_score_tma / k_score_rows / k_score_sparq)",
                         "achieved": sp["achieved_gbs"], "peak": peak, "peak_kind": peak_kind,
                         "unit": "GB/s", "frac": sp["frac"],
                         "frac_of_nominal_8tbs": sp["frac_of_nominal_8tbs"],
                         "traffic": profiled_traffic(w.name),
                         "algorithmic_bytes_per_launch": sp["read_bytes_per_launch"],
                         "key_write_bytes_per_launch": sp["key_write_bytes_per_launch"],
                         "avg_launch_us": sp["avg_launch_us"], "samples": sp["samples"]},
            "call_kv_bytes": sm["call_kv_bytes"], "call_achieved_gbs": sm["call_achieved_gbs"],
            "call_frac_of_peak": sm["call_frac_of_peak"],
            "dense_calls_per_s": sm["dense_calls_per_s"],
            "speedup_vs_dense": sm["speedup_vs_dense"], "budget_mean": sm["budget_mean"],
            "gpu_launches": r["launches_per_call"] * args.steps, "clocks": r["clocks"],
            "e2e": e2e}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = {k: (v.cpu() if hasattr(v, "cpu") else v) for k, v in x.items()}
        val, done, el = time_oracle(wr, cpu, args.cpu_budget_s)
        line["cpu_baseline"] = {"value": val, "unit": "calls/s", "cores": 1, "kind": "oracle",
                                "sample": f"{done} (sequence, KV head) units of a {w.units}-unit call "
                                          f"in {el:.1f}s, single-threaded C oracle"}
        val, done, el, T = time_oracle_all_cores(wr, cpu, args.cpu_budget_s)
        line["cpu_baseline_all_cores"] = {
            "value": val, "unit": "calls/s", "cores": T, "kind": "oracle",
            "sample": f"{done} units in {el:.1f}s, one unit per call on {T} threads of the same C oracle"}
        del cpu
    dec.close()
    del x, dec
    torch.cuda.empty_cache()

    # the other long-context workloads, same rules, at one GPU only (their inputs are
    # made after the headline's are freed)
    if world == 1 and args.per_config and args.guarantee == "denominator":
        per = {}
        for name, eps in PER_CONFIG:
            if name == w.name:
                continue
            wc = synth.WORKLOADS[name]
            if eps is not None:
                wc = wc.replace(eps=eps)
            dec_c, x_c, _, rc = run_config(wc, args, dev, world, max(args.steps, args.per_config_steps),
                                           headline=False)
            smc = summarize(rc, world, peak)
            smc["score_pass"]["traffic"] = profiled_traffic(name)
            smc["workload"] = synth.describe(wc)
            per[name] = smc
            dec_c.close()
            del x_c, dec_c
            torch.cuda.empty_cache()
        line["per_config"] = per
    if world == 1 and args.host_kv_steps > 0 and args.guarantee == "denominator":
        line["host_kv"] = {name: run_host_kv(name, args, dev) for name in HOST_KV}
    if ranks.reports(rank):
        emit(line)
    if world > 1:
        ranks.barrier(world)
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
