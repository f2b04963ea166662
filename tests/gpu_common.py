"""Shared helpers of the GPU parity tests (comparison rules, model set-up)."""
import os

import numpy as np
import torch

import oracle
import synth

# Per-step logits tolerance: max|GPU - oracle| <= 2e-2 * max|oracle logit|
# (bf16 weights, fp32 accumulation; the method statement's bar).
LOGIT_TOL = 2e-2


def logits_close(gpu: np.ndarray, ref: np.ndarray) -> float:
    """Returns max|delta| after asserting it is within LOGIT_TOL * max|ref| per row.
    With MK_PARITY_LOG set, each row's max|delta| / max|ref| is appended to that
    file with the running test's name (to record the margin)."""
    worst = 0.0
    log = os.environ.get("MK_PARITY_LOG")
    for b in range(ref.shape[0]):
        d = float(np.max(np.abs(gpu[b].astype(np.float64) - ref[b])))
        scale = float(np.max(np.abs(ref[b])))
        bound = LOGIT_TOL * scale
        if log:
            with open(log, "a") as f:
                f.write(f"{os.environ.get('PYTEST_CURRENT_TEST', '?').split(' ')[0]}\t{d / scale:.3e}\n")
        assert d <= bound, f"row {b}: max|delta| {d:.4g} > {bound:.4g}"
        worst = max(worst, d)
    return worst


def check_argmax(nxt_gpu: np.ndarray, logits_gpu: np.ndarray, logits_ref: np.ndarray, max_delta: float):
    """(i) the GPU token is the exact argmax of the GPU's own logits (lowest
    index on ties); (ii) it equals the oracle's argmax wherever the oracle's
    top-1 / top-2 margin exceeds twice the observed logit error.  Returns the
    number of rows where (ii) was not decidable (appended to MK_PARITY_LOG,
    when set, as an "undecided" line)."""
    undecided = 0
    for b in range(logits_ref.shape[0]):
        g = logits_gpu[b]
        assert int(nxt_gpu[b]) == int(np.flatnonzero(g == g.max())[0])
        top2 = np.sort(logits_ref[b])[-2:]
        if top2[1] - top2[0] > 2 * max_delta:
            assert int(nxt_gpu[b]) == int(np.argmax(logits_ref[b]))
        else:
            undecided += 1
    log = os.environ.get("MK_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(f"{os.environ.get('PYTEST_CURRENT_TEST', '?').split(' ')[0]}\tundecided\t{undecided}"
                    f"/{logits_ref.shape[0]}\n")
    return undecided


def host_weights(tw):
    """The same weights as host uint16 bit patterns, for the oracle."""
    host = {kk: (None if tw[kk] is None else synth.to_u16(tw[kk])) for kk in ("embed", "final_norm", "lm_head")}
    host["layers"] = [{a: (None if t is None else synth.to_u16(t)) for a, t in lw.items()} for lw in tw["layers"]]
    return host


def widen_bf16(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def build_pair(shape, batch=None, max_seq=None, variant="megakernel", device="cuda", seed_tokens=synth.TOKEN_SEED,
               sync="tags"):
    """Weights on the GPU, the same bytes on the host for the oracle."""
    import tile_synchronised_b200 as mk
    b = shape.batch if batch is None else batch
    ms = shape.max_seq if max_seq is None else max_seq
    tw = synth.make_weights(shape, device=device)
    model = mk.Model(shape, tw, batch=b, max_seq=ms, variant=variant)
    model.set_sync(sync)
    orc = oracle.OracleModel.from_torch(shape, tw, batch=b, max_seq=ms)
    return tw, model, orc
