"""Phase trace of the persistent decode-step kernel.

    python -m activation_sparse_decode_predict_b200.phase_trace WORKLOAD B LAYERS [--sparsity S] [--ptype q4_0]

Builds the kernel with PI_TRACE (every CTA stamps `%globaltimer` at its phase
boundaries into a device buffer; libpi_trace.so beside libpi.so, not used by
anything else), runs 5 warm-up and 30 timed decode steps of the synthetic
workload through pi_decode_stack, and prints the median (p10, p90) time of
each phase of a layer over CTAs and layers, plus the barrier and stream-end
spreads.  A diagnostic: the stamps cost a little time themselves, so the
step time printed here is not a bench number.
"""
from __future__ import annotations

import argparse
import ctypes
import os
import sys

import numpy as np
import torch

from . import _binding as _b
from . import build as _build

TRACE_LIB = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpi_trace.so")
EVENTS = 16  # stamps per (layer, CTA); must match the kernel's kTraceEvents

# (name, first stamp, second stamp) of the layer phases
PHASES = [("P1", 0, 1), ("hotA", 1, 2), ("waitU", 2, 3), ("P2", 3, 4), ("list", 4, 5), ("stream", 5, 6),
          ("atomics", 6, 7), ("barY", 7, 8), ("glue", 8, 9)]


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("workload")
    ap.add_argument("batch", type=int)
    ap.add_argument("layers", type=int)
    ap.add_argument("--sparsity", type=float, default=None)
    ap.add_argument("--ptype", default=None, choices=["f16", "q4_0"])
    a = ap.parse_args(argv)
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import pi_workload as W
    import activation_sparse_decode_predict_b200 as pi

    pi._lib = _b.load(_build.build(defines=["PI_TRACE=1"], out=TRACE_LIB))
    pi._lib.pi_trace_buffer.argtypes = [ctypes.c_void_p]
    wl = W.WORKLOADS[a.workload]
    if a.sparsity is not None:
        wl = wl.with_(sparsity=a.sparsity)
    if a.ptype is not None:
        wl = wl.with_(ptype=a.ptype)
    B, NL = a.batch, a.layers
    desc = pi.desc_for(wl)
    dev = torch.device("cuda")
    layers = [W.make_layer(wl, l, device=dev) for l in range(NL)]
    arr = pi.layer_array([pi.layer_weights(L) for L in layers])
    ws = pi.workspace(desc, B)
    G = torch.cuda.get_device_properties(0).multi_processor_count
    idx = torch.empty(NL, max(wl.n_cold, 1), dtype=torch.int32, device=dev)
    counts = torch.zeros(NL, dtype=torch.int32, device=dev)
    h_out = torch.empty(B, wl.d, dtype=torch.float16 if wl.htype == "f16" else torch.float32, device=dev)
    hs = [W.make_tokens(wl, B, t, device=dev) for t in range(8)]
    tr = torch.zeros(NL * G * EVENTS, dtype=torch.int64, device=dev)
    pi._lib.pi_trace_buffer(tr.data_ptr())
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for i in range(5):
            pi.decode_stack(desc, arr, hs[i % 8], h_out, idx, counts, None, W.RMS_EPS, ws, stream=s)
        s.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = 30
        e0.record(s)
        for i in range(n):
            pi.decode_stack(desc, arr, hs[i % 8], h_out, idx, counts, None, W.RMS_EPS, ws, stream=s)
        e1.record(s)
        s.synchronize()
    ms = e0.elapsed_time(e1) / n
    print("%s B=%d L=%d: %.3f ms/step  %.1f us/layer  status %d  mean active cold %.0f (traced build)" % (
        wl.name, B, NL, ms, ms * 1e3 / NL, pi.device_status(ws), counts.float().mean().item()))
    t = tr.view(NL, G, EVENTS).cpu().numpy().astype(np.float64)
    lo = 1 if NL > 2 else 0

    def med(x):
        return float(np.median(x))

    print("phase      median_us   p10      p90   (over CTAs, layers %d..%d)" % (lo, NL - 1))
    for nm, i, j in PHASES:
        d = (t[lo:, :, j] - t[lo:, :, i]) / 1e3
        print("%-9s %8.2f %8.2f %8.2f" % (nm, med(d), np.percentile(d, 10), np.percentile(d, 90)))
    if NL > lo + 1:
        print("layer     %8.2f" % med((t[lo + 1:, :, 0] - t[lo:-1, :, 0]) / 1e3))
    spread = lambda k: med((t[lo:, :, k].max(1) - t[lo:, :, k].min(1)) / 1e3)
    print("barrier U: arrive -> pass (barrier warp) %.2f   arrive spread %.2f" % (
        med((t[lo:, :, 11] - t[lo:, :, 10]) / 1e3), spread(10)))
    print("barrier Y: arrive spread %.2f   pass spread %.2f   last arrive -> first pass %.2f" % (
        spread(7), spread(8), med((t[lo:, :, 8].min(1) - t[lo:, :, 7].max(1)) / 1e3)))
    se = (t[lo:, :, 6] - t[lo:, :, 6].min(1, keepdims=True)) / 1e3
    print("stream end after the first CTA's: median %.2f  p90 %.2f  max %.2f" % (
        med(se), np.percentile(se, 90), med(se.max(1))))
    last = np.argmax(t[lo:, :, 6], axis=1)
    ids, cnt = np.unique(last, return_counts=True)
    top = sorted(zip(cnt, ids), reverse=True)[:5]
    print("CTAs ending the stream last (layers %d..%d): %s" % (lo, NL - 1, ", ".join("%d x%d" % (i, c) for c, i in top)))
    # stream end vs the CTA's own predicted cold rows and its SM's position
    se_ctas = np.median(se, axis=0)
    nl = np.median(t[lo:, :, 15], axis=0)
    if np.std(nl) > 0:
        print("stream end vs local predicted rows: correlation %.2f" % float(np.corrcoef(se_ctas, nl)[0, 1]))
    half = G // 2
    print("median stream end after the first, CTAs 0..%d: %.2f  CTAs %d..%d: %.2f" % (
        half - 1, med(se[:, :half]), half, G - 1, med(se[:, half:])))
    nloc = t[lo:, :, 15]
    print("local predicted cold rows per CTA: mean %.1f  max %.1f (median over layers)" % (
        nloc.mean(), med(nloc.max(1))))
    return 0


if __name__ == "__main__":
    sys.exit(main())
