"""The trace summary of tile_synchronised_b200.profile on a synthetic trace
(no GPU): phases, per-op times and the edge gaps come out as constructed."""
import numpy as np

from tile_synchronised_b200 import profile


def synthetic(n_layers=4):
    """One CTA running every phase of every layer in order; each instruction
    starts 1 µs after the previous one ends, is staged 0.5 µs later and ends
    2 µs after its start."""
    order = [1, 2, 7, 3, 4, 5]
    rows = [(op, L) for L in range(n_layers) for op in order] + [(6, n_layers - 1)]
    sched = np.zeros(len(rows), dtype=[("op", "u1"), ("layer", "u2")])
    tr = np.zeros((len(rows), 8), dtype=np.int64)
    t = 1_000_000
    for i, (op, L) in enumerate(rows):
        sched[i] = (op, L)
        start = t + 1000
        tr[i, 0] = t
        tr[i, 1] = start
        tr[i, 7] = start + 500
        tr[i, 2] = start + 2000
        t = start + 2000
    base = np.array([0, len(rows)], dtype=np.int32)
    return sched, base, tr


def test_edge_gaps_of_a_synthetic_chain():
    sched, base, tr = synthetic()
    e = profile.edge_gaps(sched, tr)
    # the consumer follows its producer directly: 1 µs gap, 0.5 µs staging
    for name in ("down->qkv", "qkv->attn", "oproj->gateup", "gateup->down"):
        assert abs(e[name]["to_first_staged_us"] - 1.5) < 1e-9
        assert abs(e[name]["to_last_staged_us"] - 1.5) < 1e-9
    # acomb and oproj are adjacent too (attn -> acomb -> oproj)
    assert abs(e["acomb->oproj"]["to_first_staged_us"] - 1.5) < 1e-9


def test_summary_phases_and_per_op_times():
    sched, base, tr = synthetic()
    s = profile.summarise(sched, base, tr)
    assert s["per_op"]["qkv"]["n"] == 4
    assert abs(s["per_op"]["down"]["mean_us"] - 2.0) < 1e-9
    assert abs(s["per_op"]["gateup"]["wait_sum_us_per_cta"] - 4 * 1.0) < 1e-9
    assert s["phases"][0]["op"] == "qkv" and s["phases"][-1]["op"] == "lmhead"
    assert set(s["edges"]) == {"down->qkv", "qkv->attn", "acomb->oproj", "oproj->gateup", "gateup->down"}


def test_sweep_table_marks_the_faster_tiling():
    from tile_synchronised_b200 import sweep
    md = sweep.rows_to_markdown([{"batch": 4, "kv": 1024, "row_us": 10.0, "col_us": 12.5, "tuned": "row"},
                                 {"batch": 16, "kv": 16384, "row_us": 30.0, "col_us": 20.0, "tuned": "column"}])
    lines = md.strip().splitlines()
    assert len(lines) == 4
    assert lines[2].split("|")[5].strip() == "row" and lines[3].split("|")[5].strip() == "column"
