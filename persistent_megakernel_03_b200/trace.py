"""Summaries of a megakernel per-task timeline (see mk_set_trace).

For every task the kernel records (%globaltimer, ns): when its event was
satisfied (scheduler), when its workers started, when their input was loaded,
when the first ring chunk was ready, when the last chunk was consumed, when
the epilogue was done and when the task finished.  From that this module
derives, per operator stage, where a task's time goes and how long the gap is
between the last task of one stage and the first task of the next (the cost
of a dependency hop inside the kernel).
"""
from __future__ import annotations

import statistics
from collections import defaultdict
from typing import Dict, List

KINDS = ("QKV", "ATTN", "OPROJ", "GATEUP", "DOWN", "LMHEAD")
PHASES = (("input_us", 1, 2), ("first_chunk_us", 2, 3), ("stream_us", 3, 4),
          ("epilogue_us", 4, 5), ("signal_us", 5, 6))


def summarize(trace_rows, tasks: List[dict]) -> Dict:
    """trace_rows: 8 words per queue entry (see mk_set_trace); tasks: the
    plan's task list."""
    recs = []
    for row in trace_rows:
        row = [int(v) for v in row]
        if row[6] == 0 or row[1] == 0:
            continue
        tid = row[7] & 0xFFFFFFFF
        t = tasks[tid]
        recs.append((t["kind"], t["layer"], row, row[7] >> 32))
    if not recs:
        return {}
    t0 = min(r[2][1] for r in recs)
    stage = defaultdict(list)
    for k, l, row, cta in recs:
        stage[(l, k)].append(row)
    order = sorted(stage, key=lambda key: min(x[1] for x in stage[key]))
    per_kind = defaultdict(lambda: defaultdict(list))
    prev_end = None
    for key in order:
        xs = stage[key]
        d = per_kind[KINDS[key[1]]]
        first_start = min(x[1] for x in xs)
        last_end = max(x[6] for x in xs)
        d["dur_us"].append(statistics.mean(x[6] - x[1] for x in xs) / 1e3)
        d["span_us"].append((last_end - first_start) / 1e3)
        d["skew_us"].append((max(x[1] for x in xs) - first_start) / 1e3)
        for name, a, b in PHASES:
            vals = [x[b] - x[a] for x in xs if x[a] and x[b]]
            if vals:
                d[name].append(statistics.mean(vals) / 1e3)
        if prev_end is not None:
            d["hop_us"].append((first_start - prev_end) / 1e3)
        prev_end = last_end
    total = (max(r[2][6] for r in recs) - t0) / 1e3
    out = {"step_us": total, "stages": len(order), "per_kind": {}}
    for kind, d in per_kind.items():
        out["per_kind"][kind] = {k: statistics.mean(v) for k, v in d.items() if v}
        out["per_kind"][kind]["count"] = len(d["dur_us"])
    busy = defaultdict(int)
    for k, l, row, cta in recs:
        busy[cta] += row[6] - row[1]
    out["mean_cta_busy_frac"] = statistics.mean(busy.values()) / 1e3 / total if total else None
    return out
