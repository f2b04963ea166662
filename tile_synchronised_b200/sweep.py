"""Row- versus column-tiled fused gate/up stage inside the decode step, swept
over batch size and KV length ("Deep Kernel Fusion for Transformers", Key
points: row-major tiling reuses the activations, column-major tiling the
weights, and the long-generation runs span outputs of 1024 to 16384 tokens at
batch 1, 4 and 16).

    python -m tile_synchronised_b200.sweep [--workload qwen3_8b] [--batches 1 4 16]
        [--kv 1024 4096 16384] [--steps 10] [--out table.md]

For every batch size one context is built with room for the longest KV
length; for every KV length C its cache positions below C are filled with
seeded N(0, 1) bf16 values (a step's cost depends on C, not on the values)
and decoding starts at C.  Both tilings are timed (CUDA events over `steps`
steps, the position rewound before each), then the one-time profiling pass
(mk_tune) runs at the same point and its pick is recorded.  Prints one JSON
object per (batch, C) and, with --out, writes a markdown table.
"""
from __future__ import annotations

import argparse
import json
import os
import sys


def rows_to_markdown(rows) -> str:
    """The sweep as a markdown table (one row per batch and KV length)."""
    out = ["| batch | KV length | row-tiled µs/step | column-tiled µs/step | faster | mk_tune picks |",
           "|---:|---:|---:|---:|---|---|"]
    for r in rows:
        faster = "row" if r["row_us"] < r["col_us"] else "column"
        out.append(f"| {r['batch']} | {r['kv']} | {r['row_us']:.1f} | {r['col_us']:.1f} | {faster} | {r['tuned']} |")
    return "\n".join(out) + "\n"


def main(argv=None):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch

    import synth
    import tile_synchronised_b200 as mk

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="qwen3_8b", choices=sorted(synth.MODELS))
    ap.add_argument("--batches", type=int, nargs="+", default=[1, 4, 16])
    ap.add_argument("--kv", type=int, nargs="+", default=[1024, 4096, 16384])
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--out", default=None)
    a = ap.parse_args(argv)
    shape = synth.MODELS[a.workload]
    tw = synth.make_weights(shape, device="cuda")
    names = {mk.MK_SWIGLU_ROW: "row", mk.MK_SWIGLU_COL: "column"}
    rows = []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for B in a.batches:
        max_seq = max(a.kv) + a.steps + 16
        model = mk.Model(shape, tw, batch=B, max_seq=max_seq)
        tok = synth.make_tokens(shape, 1, batch=B)[:, 0].contiguous().cuda()
        g = torch.Generator(device="cuda")
        g.manual_seed(11)
        filled = 0
        for C in sorted(a.kv):
            for t in model.kv_views():
                t[:, :, :, filled:C].normal_(generator=g)
            filled = C
            res = {"workload": a.workload, "batch": B, "kv": C}
            for variant in (mk.MK_SWIGLU_ROW, mk.MK_SWIGLU_COL):
                model.set_swiglu_tiling(variant)
                model.set_position(C)
                model.decode(tok)  # warm-up
                torch.cuda.synchronize()
                e0.record()
                for _ in range(a.steps):
                    model.set_position(C)
                    model.decode(tok)
                e1.record()
                torch.cuda.synchronize()
                res["row_us" if variant == mk.MK_SWIGLU_ROW else "col_us"] = 1e3 * e0.elapsed_time(e1) / a.steps
            model.set_position(C)
            res["tuned"] = names[model.tune()]
            if model.status() != 0:
                raise SystemExit(f"device status {model.status()}: {model.last_error()}")
            rows.append(res)
            print(json.dumps(res), flush=True)
        model.close()
        del model
        torch.cuda.empty_cache()
    if a.out:
        with open(a.out, "w") as f:
            f.write(rows_to_markdown(rows))
    print("sweep ok")


if __name__ == "__main__":
    main()
