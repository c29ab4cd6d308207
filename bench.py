"""Benchmark: sparse-FFN decode tokens/s through the whole layer stack on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--batch B]
                    [--sparsity S] [--impl ours|reference] [--no-cpu-baseline]

A step is one decode step of one token block through every layer of the
workload: predictor, compaction, hot block, sparse up/gate + activation,
sparse down, split-K reduction and the residual+RMSNorm glue, all in libpi's
kernels.  Inputs (weights for every layer, the token blocks) are synthetic and
seeded (pi_workload) and resident in HBM before timing starts.  A resident
stack far larger than L2 needs no flush: each step streams every layer's
predictor and active rows.  A stack below 1 GiB (the tiny fp32 workload) is
timed step by step with L2 flushed before every step, outside the timed spans.

Prints ONE JSON line (rank 0).  With N > 1 (torchrun) every rank runs an
independent replica (the path has no exchange step): weak scaling, time = max
over ranks of the device-timed region.

--impl reference times the CPU oracle (the only other implementation of this
path) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
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

import pi_workload as W  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
POOL = 64         # distinct token blocks (one captured graph each), cycled over the timed steps
E2E_STEPS = 200   # steps of the end-to-end (host buffers) measurement
REF_SECONDS = 150.0  # cap on the timed oracle work of the reference arm
# DRAM bytes (read + write) per layer of the decode-step kernel, from an ncu
# capture of a few layers of the workload (the committed ncu summaries);
# per-layer traffic does not depend on the layer count, so a launch over L
# layers moves L times this.  Only for captures of the current kernel.
TRAFFIC_PER_LAYER = {("7b-reglu-fp16", 1): (271105792 + 3212032) / 4,
                     ("13b-reglu-q4_0", 1): (208271616 + 3159808) / 4,
                     ("70b-reglu-fp16", 1): (1318978816 + 4201984) / 4}
FALLBACK_HBM_GBS = 6650.0


def max_over_ranks(value: float, world: int, device) -> float:
    """The job's time is the slowest rank's device time (all ranks take this
    collective in the same order)."""
    if world <= 1:
        return value
    t_ = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t_, op=torch.distributed.ReduceOp.MAX)
    return float(t_.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the max-over-ranks time."""
    return world * tokens_per_rank / (ms / 1e3)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="70b-reglu-fp16", choices=sorted(W.WORKLOADS))
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--sparsity", type=float, default=None)
    ap.add_argument("--ptype", default=None, choices=["f16", "q4_0"],
                    help="predictor dtype instead of the workload's (q4_0: a quantised predictor, fp16 tokens)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None, help="run fewer layers (smoke only; not a bench number)")
    ap.add_argument("--token-ffn", default=None, choices=["warp_mma", "tcgen05"],
                    help="FFN kernels for token blocks of 3-16 (default: the library's, warp_mma)")
    return ap.parse_args()


def peak_hbm():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------------------
# clocks during the timed region


class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, sampled through NVML
    every few milliseconds while the timed region runs (a background thread),
    so that even a region of a few tens of milliseconds gets samples.  One
    extra sample is always taken when the region ends.  Without NVML it falls
    back to nvidia-smi's loop."""

    PERIOD_S = 0.005
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, device):
        self.device = device
        self.rows = []
        self._stop = None
        self._thread = None
        self._nv = None
        self._h = None
        self._smi = None

    def _handle(self):
        import pynvml as nv
        nv.nvmlInit()
        props = torch.cuda.get_device_properties(self.device)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            try:
                return nv, nv.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
            except Exception:
                pass
        return nv, nv.nvmlDeviceGetHandleByIndex(torch.cuda.current_device() if self.device is None else
                                                 torch.device(self.device).index or 0)

    def sample(self):
        nv, h = self._nv, self._h
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        try:
            power = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
        except Exception:
            power = None
        self.rows.append((float(sm), float(smax), int(reasons), power))

    def _loop(self):
        while not self._stop.is_set():
            try:
                self.sample()
            except Exception:
                return
            self._stop.wait(self.PERIOD_S)

    def __enter__(self):
        import threading
        try:
            self._nv, self._h = self._handle()
            self._stop = threading.Event()
            self._thread = threading.Thread(target=self._loop, daemon=True)
            self._thread.start()
        except Exception:
            self._nv = None
            try:
                fd, path = tempfile.mkstemp(suffix=".csv")
                os.close(fd)
                q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                     "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                     "clocks_event_reasons.sw_power_cap")
                self._smi = (subprocess.Popen(["nvidia-smi", "--query-gpu=" + q, "--format=csv,noheader,nounits",
                                               "-lms", "200"], stdout=open(path, "w"), stderr=subprocess.DEVNULL),
                             path)
            except Exception:
                self._smi = None
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
            try:
                self.sample()   # the end of the region is always sampled
            except Exception:
                pass
        if self._smi is not None:
            proc, path = self._smi
            proc.terminate()
            try:
                proc.wait(timeout=5)
            except Exception:
                proc.kill()
            for line in open(path):
                p = [x.strip() for x in line.split(",")]
                try:
                    bits = sum(m for (_, m), v in zip(self.REASONS[:4], p[3:7]) if v.lower() == "active")
                    self.rows.append((float(p[0]), float(p[1]), bits, float(p[2])))
                except (ValueError, IndexError):
                    continue
            os.unlink(path)
        return False

    def summary(self):
        if not self.rows:
            return None
        reasons = sorted({name for _, _, bits, _ in self.rows for name, m in self.REASONS if bits & m})
        powers = [p for *_, p in self.rows if p is not None]
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": max(r[1] for r in self.rows),
                "reasons": reasons, "samples": len(self.rows),
                "source": "nvml" if self._nv is not None else "nvidia-smi",
                "power_w_max": round(max(powers), 1) if powers else None}


# ----------------------------------------------------------------------------
# our arm


def run_ours(args, rank, world, local_rank):
    import activation_sparse_decode_predict_b200 as pi
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = W.WORKLOADS[args.workload]
    if args.sparsity is not None:
        wl = wl.with_(sparsity=args.sparsity)
    if args.ptype is not None:
        wl = wl.with_(ptype=args.ptype)
    B = args.batch or wl.batches[0]
    n_layers = args.layers or wl.layers
    desc = pi.desc_for(wl)
    if args.token_ffn is not None:
        pi.set_token_block_ffn(args.token_ffn)

    layers = [W.make_layer(wl, l, device=dev) for l in range(n_layers)]
    torch.cuda.synchronize()
    arr = pi.layer_array([pi.layer_weights(L) for L in layers])
    n_steps = args.warmup + args.steps
    P = min(POOL, n_steps)                    # distinct token blocks, cycled
    h_pool = torch.stack([W.make_tokens(wl, B, rank * 100003 + t, device=dev) for t in range(P)])
    ws = pi.workspace(desc, B, device=dev)
    C = wl.n_cold
    idx = torch.empty(n_layers, max(C, 1), dtype=torch.int32, device=dev)
    counts = torch.zeros(P, n_layers, dtype=torch.int32, device=dev)
    h_out = torch.empty(B, wl.d, dtype=h_pool.dtype, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(p, s):
        pi.decode_stack(desc, arr, h_pool[p], h_out, idx, counts[p], None, W.RMS_EPS, ws, stream=s)

    # one CUDA graph per token block; captured before timing
    graphs = []
    with torch.cuda.stream(stream):
        step(0, stream)                       # warm the code path once outside capture
        stream.synchronize()
        for p in range(P):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step(p, stream)
            graphs.append(g)
    torch.cuda.synchronize()

    for t in range(args.warmup):
        graphs[t % P].replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # a stack that L2 could hold is timed step by step, with L2 flushed (a
    # buffer larger than L2 written) before every step, outside the timed spans
    flush = _resident_bytes(layers) < FLUSH_BELOW
    fbuf = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev) if flush else None
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)] if flush else []
    with ClockSampler(dev) as clk:
        with torch.cuda.stream(stream):
            torch.cuda.synchronize()
            # profiler range = the timed region (ncu --profile-from-start off)
            torch.cuda.cudart().cudaProfilerStart()
            ev0.record(stream)
            for i, t in enumerate(range(args.warmup, n_steps)):
                if flush:
                    fbuf.fill_(float(i))
                    step_ev[i][0].record(stream)
                graphs[t % P].replay()
                if flush:
                    step_ev[i][1].record(stream)
            ev1.record(stream)
            torch.cuda.synchronize()
            torch.cuda.cudart().cudaProfilerStop()
    ms = sum(a.elapsed_time(b) for a, b in step_ev) if flush else ev0.elapsed_time(ev1)
    clocks = clk.summary()
    ms = max_over_ranks(ms, world, dev)
    if world > 1:
        torch.distributed.barrier()
    status = pi.device_status(ws)

    # measured active counts of the timed steps -> algorithmic bytes
    cnt_p = counts.double().cpu().numpy()
    cnt = np.stack([cnt_p[t % P] for t in range(args.warmup, n_steps)])
    per_block = [sum(W.layer_bytes(wl, B, float(a), wl.layer_rank(l)) for l, a in enumerate(cnt_p[p]))
                 for p in range(P)]
    total_bytes = sum(per_block[t % P] for t in range(args.warmup, n_steps))
    sec = ms / 1e3
    gbs = total_bytes / sec / 1e9
    peak, peak_kind = peak_hbm()
    tok_s = job_tokens_per_s(B * args.steps, world, ms)

    # end to end through the public API with host buffers: H2D of the step's
    # token block from pinned memory, the stack call, D2H of the result.
    h_host = h_pool.cpu().pin_memory()  # token block in its own dtype (fp16 unless fp32 predictors)
    out_host = torch.empty(B, wl.d, dtype=h_pool.dtype).pin_memory()
    h_dev_in = torch.empty(B, wl.d, dtype=h_pool.dtype, device=dev)
    e_steps = min(args.steps, E2E_STEPS)
    e_cnt = torch.zeros(n_layers, dtype=torch.int32, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for t in range(args.warmup):
            h_dev_in.copy_(h_host[t % P], non_blocking=True)
            pi.decode_stack(desc, arr, h_dev_in, h_out, idx, e_cnt, None, W.RMS_EPS, ws, stream=stream)
            out_host.copy_(h_out, non_blocking=True)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0.record(stream)
        for t in range(e_steps):
            h_dev_in.copy_(h_host[t % P], non_blocking=True)
            pi.decode_stack(desc, arr, h_dev_in, h_out, idx, e_cnt, None, W.RMS_EPS, ws, stream=stream)
            out_host.copy_(h_out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
    e_ms = e0.elapsed_time(e1)
    e_ms = max_over_ranks(e_ms, world, dev)
    e2e_tok_s = job_tokens_per_s(B * e_steps, world, e_ms)
    hb = B * wl.d * h_pool.element_size()

    launches_per_step = pi.stack_launches(desc, B, n_layers)
    out = {
        "metric": "sparse-FFN decode tokens/s",
        "value": round(tok_s, 3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16" if wl.wtype == "f16" else wl.wtype,
        "data": "synthetic (seeded Zipf-activity weights, low-rank predictor, RMS-normalised tokens)",
        "config": {"workload": wl.name, "d": wl.d, "ffn": wl.ffn, "layers": n_layers, "batch": B,
                   "sparsity": wl.sparsity, "hot": wl.n_hot, "rank": wl.rank, "act": wl.act, "weights": wl.wtype,
                   "predictor": wl.ptype,
                   "token_ffn": pi.token_block_ffn() if B >= 3 else None,
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": (("flushed: a %d MB buffer written before every step, outside the timed spans; "
                           "time = sum of per-step CUDA events (resident stack %.1f MB, L2 126 MB)") % (
                               FLUSH_BYTES >> 20, _resident_bytes(layers) / 1e6) if flush else
                          "no flush: resident stack %.1f GB, %.2f GB streamed per step (L2 126 MB)" % (
                              _resident_bytes(layers) / 1e9, total_bytes / args.steps / 1e9)),
                   "mean_active_cold": round(float(cnt.mean()), 1)},
        "gb_per_s": round(gbs, 1),
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4),
                     "traffic": (round(TRAFFIC_PER_LAYER[(wl.name, B)] * n_layers)
                                 if (wl.name, B) in TRAFFIC_PER_LAYER and args.sparsity is None
                                 and args.ptype is None else None),
                     "kernel": "whole decode step (%d launches)" % launches_per_step,
                     "peak_source": peak_kind},
        "e2e": {"value": round(e2e_tok_s, 3), "unit": "tokens/s", "h2d_bytes_per_step": hb, "d2h_bytes_per_step": hb,
                "steps": e_steps, "how": "pinned H2D of the token block, pi_decode_stack via the binding, D2H of h_out"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "device_status": status,
    }
    return out, (wl, B, layers, n_layers)


FLUSH_BELOW = 1 << 30   # resident stacks below 1 GiB are timed with an L2 flush before every step
FLUSH_BYTES = 512 << 20  # the flush buffer: four times L2


def _resident_bytes(layers):
    n = 0
    for L in layers:
        for k in ("Wg", "Wu", "WdT", "P1", "P2", "bp", "b1"):
            v = L.get(k)
            if v is None:
                continue
            for t in (v if isinstance(v, tuple) else (v,)):
                n += t.numel() * t.element_size()
    return n


# ----------------------------------------------------------------------------
# the CPU oracle on the host cores


def _host_layers(layers):
    host = []
    for L in layers:
        Ln = {}
        for k in ("Wg", "Wu", "WdT", "P1", "P2", "bp", "b1", "b2"):
            v = L.get(k)
            if isinstance(v, tuple):
                Ln[k] = tuple(np.ascontiguousarray(t.cpu().numpy()) for t in v)
            elif v is not None:
                Ln[k] = np.ascontiguousarray(v.cpu().numpy())
            else:
                Ln[k] = None
        Ln["thr"] = L["thr"]
        host.append(Ln)
    return host


def _oracle_layer_step(wl, B, Ln, step):
    import oracle
    h = W.make_tokens(wl, B, 7_000_000 + step).numpy()
    r = oracle.predict(h, Ln["P1"], Ln["P2"], Ln["bp"], Ln["thr"], wl.n_hot, wl.ffn)
    y = oracle.masked_ffn(h, r["idx"], Ln["Wg"], Ln["Wu"], Ln["WdT"], Ln["b1"], Ln["b2"], wl.act, wl.n_hot, wl.ffn)
    return oracle.residual_rmsnorm(h, y, W.RMS_EPS)


def oracle_sample(wl, B, layers, n_sample_layers, min_seconds=10.0, max_steps=200, threads=None, host=None):
    """Time the oracle (predictor + masked FFN + glue) on the first layers of
    the stack for token blocks until about `min_seconds` of CPU work are done;
    returns (tokens/s scaled to the full stack, seconds spent, threads used,
    description)."""
    import oracle
    if threads:
        oracle.set_threads(threads)
    if host is None:
        host = _host_layers(layers[:n_sample_layers])
    t0 = time.perf_counter()
    n_steps = 0
    while n_steps < max_steps and (n_steps == 0 or time.perf_counter() - t0 < min_seconds):
        s = n_steps
        n_steps += 1
        h = W.make_tokens(wl, B, 7_000_000 + s).numpy()
        for Ln in host:
            r = oracle.predict(h, Ln["P1"], Ln["P2"], Ln["bp"], Ln["thr"], wl.n_hot, wl.ffn)
            y = oracle.masked_ffn(h, r["idx"], Ln["Wg"], Ln["Wu"], Ln["WdT"], Ln["b1"], Ln["b2"], wl.act, wl.n_hot,
                                  wl.ffn)
            hn = oracle.residual_rmsnorm(h, y, W.RMS_EPS)
            h = hn.astype(h.dtype)
    dt = time.perf_counter() - t0
    n_layers = wl.layers
    tok_s = n_steps * B / (dt * n_layers / n_sample_layers)
    desc = "%d decode steps x %d of %d layers (B=%d), scaled by %d/%d (extrapolated)" % (
        n_steps, n_sample_layers, n_layers, B, n_layers, n_sample_layers)
    return tok_s, dt, oracle.get_threads(), desc


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def run_reference(args):
    """The reference arm: the CPU oracle, as it stands, on the host cores."""
    wl = W.WORKLOADS[args.workload]
    if args.sparsity is not None:
        wl = wl.with_(sparsity=args.sparsity)
    if args.ptype is not None:
        wl = wl.with_(ptype=args.ptype)
    B = args.batch or wl.batches[0]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    n_sample = 2
    layers = [W.make_layer(wl, l, device=dev) for l in range(n_sample)]
    import oracle
    oracle.set_threads(os.cpu_count() or 1)
    # Each reference step is one token block through ONE layer of the stack (the
    # sampled layers taken in turn); tokens/s is scaled to the full stack.
    host = _host_layers(layers)
    for t in range(args.warmup):
        _oracle_layer_step(wl, B, host[t % n_sample], t)
    # at most REF_SECONDS of timed oracle work: the CPU arm stays within minutes
    # for any workload; the line reports the steps actually timed
    t0 = time.perf_counter()
    done = 0
    for t in range(args.steps):
        _oracle_layer_step(wl, B, host[t % n_sample], 1000 + t)
        done += 1
        if time.perf_counter() - t0 > REF_SECONDS:
            break
    dt = time.perf_counter() - t0
    tok_s = done * B / (dt * wl.layers)
    cores = oracle.get_threads()
    desc = "%d steps of one token block (B=%d) through one of %d sampled layers, scaled by %d layers (extrapolated)" % (
        done, B, n_sample, wl.layers)
    ms = dt * 1e3 / done * wl.layers
    return {
        "impl": "reference",
        "metric": "sparse-FFN decode tokens/s",
        "value": round(tok_s, 4),
        "unit": "tokens/s",
        "n_gpus": 1,
        "steps": args.steps,
        "steps_timed": done,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded Zipf-activity weights, low-rank predictor, RMS-normalised tokens)",
        "config": {"workload": wl.name, "d": wl.d, "ffn": wl.ffn, "layers": wl.layers, "batch": B,
                   "sparsity": wl.sparsity},
        "cpu_baseline": {"value": round(tok_s, 4), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc, "cpu": cpu_model()},
        "e2e": {"value": round(tok_s, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    out, ctx = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        wl, B, layers, _ = ctx
        n_s = 2 if wl.d * wl.ffn <= 64e6 else 1
        host = _host_layers(layers[:n_s])
        tok_s, dt, cores, desc = oracle_sample(wl, B, layers, n_s, threads=os.cpu_count(), host=host)
        tok_1, dt_1, _, desc_1 = oracle_sample(wl, B, layers, n_s, min_seconds=5.0, threads=1, host=host)
        out["cpu_baseline"] = {"value": round(tok_s, 4), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                               "sample": desc, "cpu": cpu_model(), "seconds": round(dt, 2),
                               "single_thread": {"value": round(tok_1, 4), "unit": "tokens/s", "cores": 1,
                                                 "sample": desc_1, "seconds": round(dt_1, 2)}}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
