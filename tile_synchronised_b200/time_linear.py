"""Time mk_linear_tc at the projection shapes of the batched decode configurations.

    python -m tile_synchronised_b200.time_linear [--reps 30] [--shape B K M ...]
        [--streamk] [--swiglu-batch B]

Prints one JSON list: per (B, K, M) the K split, the mean microseconds per call
(CUDA events over back-to-back calls) and the achieved GB/s of the weights plus
x and y.  Weight copies are rotated so that the timed set exceeds the 126 MB L2.
--shape (repeatable) replaces the default shapes; --streamk also times the
stream-K launch (mk_linear_tc_streamk) of each shape; --swiglu-batch also times
the tensor-core fused SwiGLU first stage (MK_SWIGLU_TC) at the 70B-shard shape.
Also the command that ncu profiles the tensor-core kernels under.
"""
import argparse
import json
import os
import sys

import torch

SHAPES = [(1, 4096, 4096), (16, 4096, 4096), (32, 4096, 4096), (32, 4096, 6144), (32, 14336, 4096),
          (32, 4096, 14336), (16, 4096, 128256), (64, 4096, 14336)]


def main(argv=None):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import synth
    import tile_synchronised_b200 as mk

    ap = argparse.ArgumentParser()
    ap.add_argument("--reps", type=int, default=30)
    ap.add_argument("--peak-gbs", type=float, default=6550.4, help="the measured HBM copy bandwidth")
    ap.add_argument("--shape", type=int, nargs=3, action="append", metavar=("B", "K", "M"),
                    help="time this (batch, K, M) instead of the default shapes (repeatable)")
    ap.add_argument("--swiglu-batch", type=int, default=0, help="also time MK_SWIGLU_TC at this batch")
    ap.add_argument("--streamk", action="store_true", help="also time mk_linear_tc_streamk on each shape")
    a = ap.parse_args(argv)
    res = []
    for (B, K, M) in (a.shape or SHAPES):
        x, w = synth.make_linear_inputs(B, K, M, device="cuda")
        wb = M * K * 2
        ncopy = max(1, -(-300_000_000 // wb))
        ws = [w] + [w.clone() for _ in range(ncopy - 1)]
        y = torch.empty((B, M), dtype=torch.float32, device="cuda")
        calls = [("plain", lambda wi: mk.linear_tc(x, wi, out=y))]
        if a.streamk:
            calls.append(("streamk", lambda wi: mk.linear_tc_streamk(x, wi, out=y)))
        for kind, call in calls:
            for i in range(3):
                call(ws[i % ncopy])
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for i in range(a.reps):
                call(ws[i % ncopy])
            e1.record()
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / a.reps
            gbs = (wb + B * K * 2 + B * M * 4) / us / 1e3
            r = {"B": B, "K": K, "M": M, "split": mk.linear_tc_split(B, K, M), "us": round(us, 2),
                 "GBps": round(gbs, 1), "frac": round(gbs / a.peak_gbs, 3)}
            if a.streamk:
                r["kind"] = kind
                r["streamk_ctas"] = mk.linear_tc_streamk_grid(B, K, M)
            res.append(r)
        del ws
    if a.swiglu_batch:
        B = a.swiglu_batch
        x, wg, wu = synth.make_swiglu_inputs(B, device="cuda")
        out = torch.empty((B, wg.shape[1]), dtype=torch.float16, device="cuda")
        for i in range(3):
            mk.swiglu_stage1(x, wg, wu, out=out, variant=mk.MK_SWIGLU_TC)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(a.reps):
            mk.swiglu_stage1(x, wg, wu, out=out, variant=mk.MK_SWIGLU_TC)
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / a.reps
        K, N = wg.shape
        gbs = (2 * K * N * 2 + B * K * 2 + B * N * 2) / us / 1e3
        res.append({"swiglu_tc_B": B, "K": K, "N": N, "us": round(us, 2), "GBps": round(gbs, 1),
                    "frac": round(gbs / a.peak_gbs, 3)})
    print(json.dumps(res))


if __name__ == "__main__":
    main()
