#!/usr/bin/env python
"""Benchmark of one batch-1 decode step of the Llama-3.2-1B architecture.

Workload: 16 layers, hidden 2048, 32/8 heads, head_dim 64, SwiGLU 8192, vocab
128256, tied head, random-init bf16 weights; KV cache prefilled from 1024
seeded tokens, then teacher-forced decode steps at positions 1024..1279 (the
window is re-entered by rewinding the position, so every timed step attends
to 1025..1280 positions).  A step streams ~2.51 GB (weights + KV), far more
than the 126 MB L2, so no L2 flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mk|reference]

Prints one JSON line (rank 0).  For N > 1 launch it with torchrun: every rank
runs an independent replica (the step does not shard), timed on the device,
max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "bs=1 Llama-1B-arch decode tokens/s; achieved HBM GB/s vs B200 peak"
UNIT = "tokens/s"
PREFILL = 1024
WINDOW = 256
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
WORKLOAD_NAME = "Llama-3.2-1B-arch decode step, batch 1, KV 1024->1280, tied head, bf16 random-init"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="mk", choices=["mk", "reference"])
    ap.add_argument("--variant", default="megakernel",
                    choices=["megakernel", "graph", "graph_pdl", "tilesync", "tensor_cores"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-variants", action="store_true", help="skip timing the separate-kernel variants")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="budget of the CPU-baseline sample")
    return ap.parse_args()


# ---------------------------------------------------------------- helpers
def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(shape, batch, pos):
    """HBM bytes one step must move: every weight once (tied head = embedding
    table), the batch's embedding rows, the KV rows read (positions 0..pos-1)
    and the K/V rows written at `pos`."""
    kv_row = shape.n_layers * 2 * shape.n_kv_heads * shape.head_dim * 2
    return shape.weight_bytes() + batch * shape.hidden * 2 + batch * kv_row * pos + batch * kv_row


# The sources that decide what the decode step launches and what it reads:
# the megakernel, its plan and launch code, and the headers they share (not
# the isolated SwiGLU, attention and tensor-core kernels, nor mk_kernel.h,
# which only declares their entry points).
STEP_SOURCES = ("mk_api.cu", "mk_device.cuh", "mk_internal.h", "mk_kernel.cu", "mk_sched.cpp", "mk_sched.h")


def source_hash():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "tile_synchronised_b200", "csrc")
    for n in STEP_SOURCES:
        with open(os.path.join(d, n), "rb") as f:
            h.update(n.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "megakernel_llama1b_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        t = json.load(f)
    if t.get("source_hash") != source_hash():
        return None
    return t.get("dram_bytes_per_launch")


class ClockSampler:
    """NVML samples of SM clock and throttle reasons while running."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self.nv = None

    def _run(self):
        get_r = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = get_r(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv:
            self._t.join()

    def report(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def oracle_steps(shape, host_w, kc, vc, tokens_np, seconds, max_steps=None):
    """Time plain oracle decode steps from position PREFILL on (bounded)."""
    import numpy as np
    import oracle
    orc = oracle.OracleModel(shape, host_w, batch=1, max_seq=PREFILL + WINDOW)
    orc.kc[:, 0, :, :PREFILL] = kc
    orc.vc[:, 0, :, :PREFILL] = vc
    orc.pos[0] = PREFILL
    n, t0 = 0, time.perf_counter()
    while True:
        orc.step([int(tokens_np[0, PREFILL + (n % WINDOW)])], want_logits=False)
        n += 1
        if orc.pos[0] >= PREFILL + WINDOW:
            orc.pos[0] = PREFILL
        el = time.perf_counter() - t0
        if (n >= 2 and el >= seconds) or (max_steps and n >= max_steps):
            break
    del orc
    np.zeros(1)
    return n, el, oracle.num_threads()


def host_weights(tw):
    import synth
    hw = {k: (None if tw[k] is None else synth.to_u16(tw[k])) for k in ("embed", "final_norm", "lm_head")}
    hw["layers"] = [{a: (None if t is None else synth.to_u16(t)) for a, t in lw.items()} for lw in tw["layers"]]
    return hw


# ---------------------------------------------------------------- distributed plumbing
def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, v):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, batch, steps, ms_local):
    """Every rank decodes `batch` sequences for `steps` steps in `ms_local`
    device milliseconds; returns (the max over ranks of those ms, ms per step,
    whole-job tokens/s)."""
    ms = max_over_ranks(world, ms_local)
    return ms, ms / steps, world * batch * steps / (ms / 1e3)


# ---------------------------------------------------------------- the product arm
def run_mk(args, world, rank, local):
    import torch

    import synth
    import tile_synchronised_b200 as mk

    shape = synth.LLAMA1B
    B = 1
    tw = synth.make_weights(shape, device="cuda")
    model = mk.Model(shape, tw, batch=B, max_seq=PREFILL + WINDOW, variant=args.variant)
    tokens = synth.make_tokens(shape, PREFILL + WINDOW, batch=B)
    model.prefill(tokens[:, :PREFILL].cuda())
    win = tokens[0, PREFILL:].contiguous().cuda()  # teacher-forced inputs, resident in HBM
    stream = torch.cuda.current_stream()
    if args.variant == "megakernel":
        launches_per_step = 1
    elif args.variant == "tensor_cores":
        # per pass of up to 32 sequences: embed, rows, 13 per layer (norm, QKV GEMM, q/k/v post, 2 attention,
        # cast, O GEMM, residual, norm, gate/up GEMM, SiLU*mul, down GEMM, residual), final norm, LM GEMM,
        # argmax; then the position advance
        launches_per_step = ((B + 31) // 32) * (2 + 13 * shape.n_layers + 3) + 1
    else:
        launches_per_step = model.info()["n_phases"]

    def run_steps(n, start, e2e=None):
        rewinds = 0
        for s in range(start, start + n):
            j = s % WINDOW
            if j == 0 and model.position != PREFILL:
                model.set_position(PREFILL)
                rewinds += 1
            if e2e is None:
                model.decode(win[j:j + 1])
            else:
                h_tok, d_tok, h_out, k = e2e
                d_tok[k % 2].copy_(h_tok[s - start], non_blocking=True)
                nxt = model.decode(d_tok[k % 2], out=d_out[k % 2])
                h_out[s - start].copy_(nxt, non_blocking=True)
                e2e = (h_tok, d_tok, h_out, k + 1)
        return rewinds

    # warm-up, then the device-timed region
    run_steps(args.warmup, 0)
    model.set_position(PREFILL)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device() if world == 1 else local) as clk:
        e0.record(stream)
        rewinds = run_steps(args.steps, 0)
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ms_local = e0.elapsed_time(e1)
    ms, ms_per_step, value = job_throughput(world, B, args.steps, ms_local)
    st = model.status()
    if st != 0:
        raise RuntimeError(f"device status {st}: {model.last_error()}")
    total_tokens = world * B * args.steps

    # roofline of the (only) kernel: algorithmic bytes per launch / launch time
    pos_list = [PREFILL + (s % WINDOW) for s in range(args.steps)]
    mean_bytes = statistics.fmean(algorithmic_bytes(shape, B, p) for p in pos_list)
    peak, peak_kind = measured_peak()
    achieved = mean_bytes / (ms_local / args.steps / 1e3) / 1e9
    traffic = profiled_traffic()

    # e2e through the public API: pinned host tokens in, next token back to pinned host memory
    model.set_position(PREFILL)
    h_tok = tokens[0, PREFILL:].repeat((args.steps + WINDOW - 1) // WINDOW)[:args.steps].contiguous().pin_memory()
    h_tok = h_tok.view(args.steps, 1)
    h_out = torch.empty((args.steps, B), dtype=torch.int32).pin_memory()
    d_tok = [torch.empty(B, dtype=torch.int32, device="cuda") for _ in range(2)]
    d_out = [torch.empty(B, dtype=torch.int32, device="cuda") for _ in range(2)]
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    run_steps(args.steps, 0, e2e=(h_tok, d_tok, h_out, 0))
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(world, e0.elapsed_time(e1))
    e2e_value = total_tokens / (e2e_ms / 1e3)

    # the same ops as separate kernels in a CUDA graph (with and without PDL)
    variants = {}
    if not args.no_variants:
        for v in ("megakernel", "graph", "graph_pdl", "tilesync", "tensor_cores"):
            if v == args.variant:
                variants[v] = {"tokens_per_s": round(value / world, 2), "ms_per_step": round(ms_per_step, 5)}
                continue
            model.set_variant(v)
            n = min(args.steps, 2 * WINDOW)
            model.set_position(PREFILL)
            run_steps(8, 0)
            model.set_position(PREFILL)
            torch.cuda.synchronize()
            e0.record(stream)
            run_steps(n, 0)
            e1.record(stream)
            torch.cuda.synchronize()
            vms = e0.elapsed_time(e1) / n
            variants[v] = {"tokens_per_s": round(B / (vms / 1e3), 2), "ms_per_step": round(vms, 5)}
        model.set_variant(args.variant)
        if model.status() != 0:
            raise RuntimeError(model.last_error())

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        k, v = model.kv_views()
        kc = k[:, 0, :, :PREFILL].float().cpu().numpy()
        vc = v[:, 0, :, :PREFILL].float().cpu().numpy()
        hw = host_weights(tw)
        n, el, cores = oracle_steps(shape, hw, kc, vc, tokens.numpy(), args.cpu_seconds)
        cpu = {"value": round(B * n / el, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{n} oracle decode steps (batch 1, positions 1024+, KV handed over from the GPU "
                         f"prefill), {el:.1f} s on {cores} OpenMP threads"}
        import oracle
        oracle.set_num_threads(1)
        try:
            n1, el1, _ = oracle_steps(shape, hw, kc, vc, tokens.numpy(), args.cpu_seconds / 3)
        finally:
            oracle.set_num_threads(0)
        cpu["one_core"] = {"value": round(B * n1 / el1, 4), "unit": UNIT, "cores": 1,
                           "sample": f"{n1} oracle decode steps, {el1:.1f} s on 1 OpenMP thread"}

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_NAME, "batch": B, "kv_positions": [PREFILL + 1, PREFILL + WINDOW],
                   "variant": args.variant, "parallelism": f"replicas{world}",
                   "l2": "no flush: each step streams ~2.51 GB, > 126 MB L2"},
        "hbm_gbs": round(achieved, 1), "hbm_frac_of_spec_8tbs": round(achieved / SPEC_HBM_GBS, 4),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_source": peak_kind, "kernel": "mk::step_kernel<1> (the whole step)",
                     "algorithmic_bytes_per_launch": int(mean_bytes)},
        "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": 4 * B, "d2h_bytes_per_step": 4 * B},
        "gpu_launches": world * (args.steps * launches_per_step + rewinds),
        "clocks": clk.report(),
        "variants": variants,
        "cpu_baseline": cpu,
    }
    return line


# ---------------------------------------------------------------- the reference arm: the oracle on host cores
def run_reference(args, world, rank):
    if rank != 0:
        return None
    import numpy as np
    import torch

    import oracle
    import synth
    shape = synth.LLAMA1B
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    tw = synth.make_weights(shape, device=dev)
    hw = host_weights(tw)
    del tw
    tokens = synth.make_tokens(shape, PREFILL + WINDOW).numpy()
    # stand-in KV for positions < 1024: seeded N(0, 1) values (the oracle's
    # step cost does not depend on them; the GPU arm hands over real ones)
    rng = np.random.default_rng(123)
    kv_shape = (shape.n_layers, shape.n_kv_heads, PREFILL, shape.head_dim)
    kc = rng.standard_normal(kv_shape, dtype=np.float32)
    vc = rng.standard_normal(kv_shape, dtype=np.float32)
    oracle_steps(shape, hw, kc, vc, tokens, 0.0, max_steps=max(1, min(args.warmup, 2)))
    budget = 60.0
    n, el, cores = oracle_steps(shape, hw, kc, vc, tokens, budget, max_steps=args.steps)
    value = n / el
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": n, "steps_requested": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * el / n, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD_NAME, "batch": 1, "kv_positions": [PREFILL + 1, PREFILL + WINDOW],
                   "parallelism": "host cores of rank 0"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{n} of {args.steps} requested oracle decode steps (time-bounded to "
                                   f"{budget:.0f} s), KV positions < 1024 filled with seeded stand-ins"},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        line = run_reference(args, world, rank) if args.impl == "reference" else run_mk(args, world, rank, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
