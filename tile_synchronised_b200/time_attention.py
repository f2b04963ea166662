"""Time the split-KV decode attention (mk_attention_decode) on its own.

    python -m tile_synchronised_b200.time_attention [--reps 20]
        [--shape B NQ NKV D N_POS ...] [--chunks C]

Prints one JSON list: per shape the chunk count, the mean microseconds per
call (CUDA events around each call, with a 256 MB buffer written between
calls so that the cache is read from HBM) and the achieved GB/s of the K and
V rows read.  The default shapes are one layer of the decode configurations:
Llama-3.2-1B batch 1 at 1k, Qwen3-8B batch 16 at 1k and 16k, Llama-3.1-8B
batch 32 at 1k.  Also the command that ncu profiles the attention kernels
under.
"""
import argparse
import json
import os
import sys

import torch

SHAPES = [(1, 32, 8, 64, 1025), (16, 32, 8, 128, 1024), (16, 32, 8, 128, 16384), (32, 32, 8, 128, 1024)]


def main(argv=None):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import synth
    import tile_synchronised_b200 as mk

    ap = argparse.ArgumentParser()
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--peak-gbs", type=float, default=6550.4, help="the measured HBM copy bandwidth")
    ap.add_argument("--shape", type=int, nargs=5, action="append", metavar=("B", "NQ", "NKV", "D", "N_POS"),
                    help="time this shape instead of the defaults (repeatable)")
    ap.add_argument("--chunks", type=int, default=0, help="split-KV chunks (0: mk_attention_chunks)")
    a = ap.parse_args(argv)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    res = []
    for (B, nq, nkv, d, n_pos) in (a.shape or SHAPES):
        q, k, v = (t.cuda() for t in synth.make_attention_inputs(B, nq, nkv, d, n_pos + 16, n_pos))
        chunks = a.chunks or mk.attention_chunks(B, nkv, n_pos)
        need = int(mk._lib.load().mk_attention_scratch_bytes(B, nq, d, chunks))
        scratch = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
        out = torch.empty((B, nq, d), dtype=torch.float32, device="cuda")
        for _ in range(3):
            mk.attention_decode(q, k, v, n_pos, chunks=chunks, out=out, scratch=scratch)
        torch.cuda.synchronize()
        total = 0.0
        for _ in range(a.reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            mk.attention_decode(q, k, v, n_pos, chunks=chunks, out=out, scratch=scratch)
            e1.record()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
        us = total * 1e3 / a.reps
        gbs = B * nkv * n_pos * d * 2 * 2 / us / 1e3
        res.append({"B": B, "nq": nq, "nkv": nkv, "d": d, "n_pos": n_pos, "chunks": chunks, "us": round(us, 2),
                    "GBps": round(gbs, 1), "frac": round(gbs / a.peak_gbs, 3)})
        del q, k, v
    print(json.dumps(res))


if __name__ == "__main__":
    main()
