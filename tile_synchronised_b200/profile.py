"""Profiling driver: run a few decode steps of a workload, optionally with the
per-instruction device trace, and summarise where the step's time goes.

    python -m tile_synchronised_b200.profile [--workload llama1b] [--batch 1]
        [--prefill 1024] [--steps 3] [--variant megakernel] [--trace out.json]

Used as the command under ncu (small --prefill keeps the capture short) and
for trace summaries: per phase (op, layer) the span from the first dependency
satisfied to the last instruction done, per op the mean instruction time, the
time spent waiting on counters, and how far the producer ran ahead, and per
edge of a layer's chain the gap from the producer phase's end to the
consumers' staged inputs.
"""
from __future__ import annotations

import argparse
import json
import sys

import numpy as np
import torch

OPS = {1: "qkv", 2: "attn", 3: "oproj", 4: "gateup", 5: "down", 6: "lmhead", 7: "acomb"}


# Edges of a layer's chain: (producer op, layer offset, consumer op).  The
# consumer stamps "inputs staged" (trace slot 7) once the words it reads carry
# the producer's tag; the gap from the producer phase's last instruction end
# to that stamp is the cost of the edge (an L2 round trip, the staging
# itself, and any wait for the slowest producer CTA).
EDGES = ((5, -1, 1, "down->qkv"), (1, 0, 2, "qkv->attn"), (7, 0, 3, "acomb->oproj"), (3, 0, 4, "oproj->gateup"),
         (4, 0, 5, "gateup->down"))


def edge_gaps(sched, tr):
    """Mean over the inner layers (1 .. L-2) of, per edge, the gap in µs from
    the producer phase's last end to the first and to the last consumer
    instruction's staged stamp."""
    t0 = tr[:, 0].astype(np.float64)
    origin = t0[t0 > 0].min()
    t2 = (tr[:, 2].astype(np.float64) - origin) / 1e3
    t7 = (tr[:, 7].astype(np.float64) - origin) / 1e3
    ops, layers = sched["op"].astype(np.int64), sched["layer"].astype(np.int64)
    n_layers = int(layers[ops != 6].max()) + 1
    out = {}
    for pop, dl, cop, name in EDGES:
        first, last = [], []
        for L in range(1, n_layers - 1):
            pm = (ops == pop) & (layers == L + dl)
            cm = (ops == cop) & (layers == L)
            if not pm.any() or not cm.any():
                continue
            end = t2[pm].max()
            first.append(t7[cm].min() - end)
            last.append(t7[cm].max() - end)
        if first:
            out[name] = {"to_first_staged_us": float(np.mean(first)), "to_last_staged_us": float(np.mean(last))}
    return out


def summarise(sched, base, tr):
    """sched: structured instruction array; tr: int64 [n, 8] stamps and waits (ns)."""
    t0, t1, t2, tp = (tr[:, k].astype(np.float64) for k in range(4))
    cwait, pwait = tr[:, 4].astype(np.float64), tr[:, 5].astype(np.float64)
    origin = t0[t0 > 0].min()
    t0, t1, t2 = t0 - origin, t1 - origin, t2 - origin
    tp = np.where(tp > 0, tp - origin, np.nan)
    out = {"step_us": float((t2.max()) / 1e3)}
    per_op = {}
    for code, name in OPS.items():
        m = sched["op"] == code
        if not m.any():
            continue
        dur = (t2[m] - t1[m]) / 1e3
        wait = (t1[m] - t0[m]) / 1e3
        lead = (t1[m] - tp[m]) / 1e3
        per_op[name] = {"n": int(m.sum()), "mean_us": float(dur.mean()), "p90_us": float(np.percentile(dur, 90)),
                        "sum_us_per_cta": float(dur.sum() / (len(base) - 1)),
                        "wait_sum_us_per_cta": float(wait.sum() / (len(base) - 1)),
                        "producer_lead_us": float(np.nanmean(lead)) if np.isfinite(lead).any() else None,
                        "consumer_data_wait_us": float(cwait[m].mean() / 1965.0),  # SM cycles at 1965 MHz
                        "producer_slot_wait_us": float(pwait[m].mean() / 1e3)}
    out["per_op"] = per_op
    phases = []
    keys = sched["op"].astype(np.int64) * 100000 + sched["layer"].astype(np.int64)
    for k in np.unique(keys):
        m = keys == k
        phases.append((float(t1[m].min() / 1e3), float(t2[m].max() / 1e3), OPS[int(k // 100000)], int(k % 100000)))
    phases.sort()
    out["phases"] = [{"op": o, "layer": l, "start_us": round(a, 2), "end_us": round(b, 2)} for a, b, o, l in phases]
    # per-CTA: total busy (sum of instruction durations) vs span
    busy = []
    for c in range(len(base) - 1):
        s, e = base[c], base[c + 1]
        if e > s:
            busy.append(float((t2[s:e] - t1[s:e]).sum() / max(1.0, t2[s:e].max())))
    out["cta_busy_frac_mean"] = float(np.mean(busy))
    out["edges"] = edge_gaps(sched, tr)
    return out


def main(argv=None):
    import os
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import synth
    import tile_synchronised_b200 as mk

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="llama1b", choices=sorted(synth.MODELS))
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--prefill", type=int, default=None)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--variant", default="megakernel", choices=sorted(mk.VARIANTS))
    ap.add_argument("--trace", default=None, help="write a trace summary (JSON) of the last step here")
    ap.add_argument("--max-seq", type=int, default=None)
    ap.add_argument("--prefetch", type=int, default=None, help="L2 prefetch distance (ring blocks)")
    ap.add_argument("--time", type=int, default=0, help="also time this many steps (CUDA events)")
    ap.add_argument("--sync", default="tags", choices=sorted(mk.SYNCS))
    ap.add_argument("--stages", type=int, default=0, help="ring slots in use (0: all that fit)")
    ap.add_argument("--synthetic-kv", type=int, default=0, metavar="C",
                    help="timing only: instead of a prefill, fill cache positions < C with seeded N(0,1) bf16 "
                         "values and start decoding at position C (the step's cost depends on C, not on the values)")
    ap.add_argument("--prefill-mode", default="auto", choices=["auto", "steps", "tc"],
                    help="how the prompt fills the cache: the tensor cores where the plan allows (auto), decode "
                         "steps, or the tensor cores (tc); the prefill is timed")
    ap.add_argument("--tcdec", action="store_true",
                    help="also time the tensor-core decode step (mk_tcdec_*) on the same cache, at the last position")
    a = ap.parse_args(argv)
    shape = synth.MODELS[a.workload]
    B = a.batch or shape.batch
    prefill = a.synthetic_kv or (shape.prefill if a.prefill is None else a.prefill)
    max_seq = a.max_seq or max(prefill + a.steps + 1, 16)
    tw = synth.make_weights(shape, device="cuda")
    model = mk.Model(shape, tw, batch=B, max_seq=max_seq, variant=a.variant)
    tokens = synth.make_tokens(shape, prefill + a.steps, batch=B)
    if a.prefetch is not None:
        model.set_prefetch(a.prefetch)
    model.set_sync(a.sync)
    model.set_ring_stages(a.stages)
    if a.synthetic_kv:
        g = torch.Generator(device="cuda")
        g.manual_seed(11)
        for t in model.kv_views():
            t[:, :, :, :prefill].normal_(generator=g)
        model.set_position(prefill)
    elif prefill:
        model.set_prefill(a.prefill_mode)
        dev_prompt = tokens[:, :prefill].cuda()
        torch.cuda.synchronize()
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record()
        model.prefill(dev_prompt)
        p1.record()
        torch.cuda.synchronize()
        print(json.dumps({"prefill_tokens": prefill, "batch": B, "prefill_mode": a.prefill_mode,
                          "prefill_ms": round(p0.elapsed_time(p1), 3)}))
    d_tok = tokens[:, prefill:].t().contiguous().cuda()  # [steps, B]
    for s in range(a.steps - 1):
        model.decode(d_tok[s])
    if a.time:
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for r in range(a.time):
            model.set_position(prefill + a.steps - 1)
            model.decode(d_tok[a.steps - 2 if a.steps > 1 else 0])
        e1.record()
        torch.cuda.synchronize()
        print(json.dumps({"timed_steps": a.time, "us_per_step": round(1e3 * e0.elapsed_time(e1) / a.time, 2),
                          "prefetch": a.prefetch, "sync": a.sync, "stages": a.stages}))
        model.set_position(prefill + a.steps - 1)
        if a.tcdec:
            dec = mk.TcDecoder(shape, tw, B, max_seq, kv_cache=model.kv)
            p_tc = prefill + a.steps - 1
            tok = d_tok[a.steps - 2 if a.steps > 1 else 0]
            for r in range(3):
                dec.step(tok, p_tc)
            torch.cuda.synchronize()
            e0.record()
            for r in range(a.time):
                dec.step(tok, p_tc)
            e1.record()
            torch.cuda.synchronize()
            if dec.status() != 0:
                raise SystemExit("tensor-core decode step: a token out of range")
            print(json.dumps({"tcdec_timed_steps": a.time,
                              "tcdec_us_per_step": round(1e3 * e0.elapsed_time(e1) / a.time, 2)}))
            dec.close()
    tr = None
    if a.trace:
        n = model.info()["n_instructions"]
        tr = torch.zeros((n, 8), dtype=torch.int64, device="cuda")
        model.set_trace(tr)
    model.decode(d_tok[a.steps - 1])
    torch.cuda.synchronize()
    st = model.status()
    if st != 0:
        raise SystemExit(f"device status {st}: {model.last_error()}")
    if a.trace:
        sched, base = model.schedule()
        stem = a.trace.replace(".json", "")
        np.save(stem + "_raw.npy", tr.cpu().numpy())
        np.save(stem + "_sched.npy", sched)
        np.save(stem + "_base.npy", base)
        summ = summarise(sched, base, tr.cpu().numpy())
        summ.update({"workload": a.workload, "batch": B, "prefill": prefill, "variant": a.variant,
                     "sync": a.sync, "schedule": model.info()})
        with open(a.trace, "w") as f:
            json.dump(summ, f, indent=1)
        print(json.dumps({k: v for k, v in summ.items() if k != "phases"}, indent=1))
        print("first phases:", summ["phases"][:12])
        print("last phases:", summ["phases"][-6:])
    print("profile run ok")


if __name__ == "__main__":
    main()
