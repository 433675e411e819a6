"""Summaries of the megakernel's per-job timestamps (``Megakernel.trace()``).

Each job record (see ``mk_read_trace`` in mk.h) holds, in globaltimer
nanoseconds: the activation warp starting to wait for a free input slot, the
slot being free, the activation warp starting its part of the job, its part
being ready, compute warp 0 starting (its input polled from the producers'
tagged words inside the compute time), the first weight stage being ready, and
the job's last compute warp finishing. From these the summary separates, per
op, slot waits, the activation warp's staging, and compute (with the input
wait), and gives per layer the moment each op finished on its last SM -- the
step's critical path.
"""
from __future__ import annotations

import numpy as np

OPS = {1: "qkv", 2: "attn", 3: "oproj", 4: "gateup", 5: "down", 6: "lmhead"}
SLOT_WAIT, CTR_WAIT, CTR_DONE, READY, START, DONE, META, FILL = range(8)


def records(trace: np.ndarray):
    """Flatten to an array of valid job rows: [sm, job, stamps..., op, layer, chunk]."""
    n_sm, jobs, _ = trace.shape
    rows = []
    for s in range(n_sm):
        for j in range(jobs):
            r = trace[s, j].astype(np.int64)
            meta = int(r[META])
            op = meta & 0xFF
            if op == 0 or r[DONE] == 0:
                continue
            rows.append([s, j] + [int(x) for x in r[:6]] + [op, (meta >> 8) & 0xFFFF, meta >> 24,
                                                           int(r[FILL])])
    return np.array(rows, dtype=np.int64)


def summarize(trace: np.ndarray) -> dict:
    R = records(trace)
    if R.size == 0:
        return {}
    t = R[:, 2:8]
    t0 = t[t > 0].min()
    step_end = R[:, 2 + DONE].max()
    out = {"step_us": (step_end - t0) / 1e3, "jobs": int(len(R)), "ops": {}, "layers": []}
    op_col, layer_col = R[:, 8], R[:, 9]
    for op, name in OPS.items():
        m = op_col == op
        if not m.any():
            continue
        r = R[m]
        ctr = (r[:, 2 + CTR_DONE] - r[:, 2 + CTR_WAIT]) / 1e3
        prep = (r[:, 2 + READY] - r[:, 2 + CTR_DONE]) / 1e3
        comp = (r[:, 2 + DONE] - r[:, 2 + START]) / 1e3
        slot = (r[:, 2 + CTR_WAIT] - r[:, 2 + SLOT_WAIT]) / 1e3
        has_fill = r[:, 11] > 0
        fillw = ((r[has_fill, 11] - r[has_fill, 2 + START]) / 1e3) if has_fill.any() else np.zeros(1)
        out["ops"][name] = {
            "first_fill_wait_us": {"mean": float(fillw.mean()), "max": float(fillw.max())},
            "jobs": int(m.sum()),
            "counter_wait_us": {"mean": float(ctr.mean()), "max": float(ctr.max())},
            "prep_us": {"mean": float(prep.mean()), "max": float(prep.max())},
            "compute_us": {"mean": float(comp.mean()), "max": float(comp.max())},
            "slot_wait_us": {"mean": float(slot.mean()), "max": float(slot.max())},
        }
    for l in sorted(set(layer_col.tolist())):
        row = {"layer": int(l)}
        for op, name in OPS.items():
            m = (op_col == op) & (layer_col == l)
            if m.any():
                row[name + "_ready_first_us"] = float((R[m][:, 2 + CTR_DONE].min() - t0) / 1e3)
                row[name + "_done_last_us"] = float((R[m][:, 2 + DONE].max() - t0) / 1e3)
        out["layers"].append(row)
    return out


def format_summary(s: dict) -> str:
    lines = [f"step {s['step_us']:.1f} us, {s['jobs']} jobs"]
    lines.append(f"{'op':8s} {'jobs':>6s} {'ctr wait':>17s} {'prep':>17s} {'compute':>17s} "
                 f"{'slot wait':>17s} {'1st fill wait':>17s}")
    for name, o in s["ops"].items():
        f = lambda d: f"{d['mean']:7.2f}/{d['max']:8.2f}"
        lines.append(f"{name:8s} {o['jobs']:6d} {f(o['counter_wait_us']):>17s} {f(o['prep_us']):>17s} "
                     f"{f(o['compute_us']):>17s} {f(o['slot_wait_us']):>17s} "
                     f"{f(o['first_fill_wait_us']):>17s}")
    lines.append("per layer: time (us from step start) at which the op's last job finished")
    for row in s["layers"]:
        parts = [f"L{row['layer']:2d}"]
        for name in OPS.values():
            if name + "_done_last_us" in row:
                parts.append(f"{name}={row[name + '_done_last_us']:.1f}")
        lines.append("  " + " ".join(parts))
    return "\n".join(lines)
