"""Per-task trace of one decode step: summaries and Chrome-trace export.

Input is what ``Decoder.trace()`` returns after a step run with tracing on:
the step's task descriptors and, per task, globaltimer stamps (producer
resolved / last stage issued, loader deps met / activation issued, consumer
picked up / has activation / math done / epilogue done) and the CTA that ran
it.
"""

from __future__ import annotations

import collections
import json
from typing import Dict

import numpy as np

OP_NAMES = {1: "rn", 2: "qkv", 3: "router", 4: "topk", 5: "attn", 6: "combine", 7: "oproj",
            8: "gateup", 9: "down", 10: "lmhead"}
D_OP, D_LAYER, D_A, D_B = 0, 1, 2, 3
(T_P_RESOLVED, T_P_ISSUED, T_L_DEPS, T_L_ACT, T_C_READY, T_C_ACT, T_C_MATH,
 T_C_END, T_CTA, T_C_WAITCYC, T_C_LOOPCYC, T_P_WAITCYC, T_K0, T_K1, T_K2, T_K3, T_K4,
 T_K5) = range(18)


def _times(stamps: np.ndarray) -> np.ndarray:
    """uint32 ns stamps -> float64 us relative to the earliest stamp.

    The stamps are the low 32 bits of a nanosecond timer, which wraps every
    ~4.3 s; a step is far shorter, so stamps that span more than half the
    range straddle one wrap, and the small (post-wrap) values are lifted by
    2^32 before the earliest stamp is taken."""
    st = stamps[:, :T_CTA].astype(np.int64)
    present = st != 0
    v = st.copy()
    if present.any() and st[present].max() - st[present].min() > (1 << 31):
        v[present & (st < (1 << 31))] += 1 << 32
    base = int(v[present].min()) if present.any() else 0
    out = (v - base).astype(np.float64) / 1e3
    out[~present] = np.nan
    return out


def summarize(desc, stamps) -> Dict:
    t = _times(stamps)
    cta = stamps[:, T_CTA].astype(np.int64) - 1
    per_op = collections.defaultdict(lambda: collections.defaultdict(list))
    for i in range(len(desc)):
        op = OP_NAMES.get(int(desc[i, D_OP]), "?")
        s = t[i]
        d = per_op[op]
        d["total"].append(s[T_C_END] - s[T_C_READY])
        d["act_wait"].append(s[T_C_ACT] - s[T_C_READY])
        if not np.isnan(s[T_C_MATH]):
            d["math"].append(s[T_C_MATH] - s[T_C_ACT])
            d["epilogue"].append(s[T_C_END] - s[T_C_MATH])
        d["deps_before_pickup"].append(s[T_C_READY] - s[T_L_DEPS])
        if stamps.shape[1] > T_P_WAITCYC and stamps[i, T_C_LOOPCYC]:
            ghz = 1.965e3   # cycles per us at the max SM clock
            d["loop_us"].append(stamps[i, T_C_LOOPCYC] / ghz)
            d["stage_wait_us"].append(stamps[i, T_C_WAITCYC] / ghz)
            d["producer_wait_us"].append(stamps[i, T_P_WAITCYC] / ghz)
        d["issued_before_pickup"].append(s[T_C_READY] - s[T_P_ISSUED])
    out = {"step_us": float(np.nanmax(t[:, T_C_END])), "ops": {}}
    for op, d in per_op.items():
        out["ops"][op] = {k: {"n": len(v), "mean": float(np.nanmean(v)),
                              "p50": float(np.nanmedian(v)), "max": float(np.nanmax(v))}
                          for k, v in d.items() if len(v) and not np.all(np.isnan(v))}
    gaps, busy = [], []
    for c in np.unique(cta[cta >= 0]):
        idx = np.where(cta == c)[0]
        idx = idx[np.argsort(t[idx, T_C_READY])]
        busy.append(np.nansum(t[idx, T_C_END] - t[idx, T_C_READY]))
        if len(idx) > 1:
            gaps.extend((t[idx[1:], T_C_READY] - t[idx[:-1], T_C_END]).tolist())
    out["gap_between_tasks_us"] = {"mean": float(np.nanmean(gaps)) if gaps else 0.0,
                                   "p50": float(np.nanmedian(gaps)) if gaps else 0.0}
    out["consumer_busy_frac"] = float(np.mean(busy) / out["step_us"]) if busy else 0.0
    ends = collections.defaultdict(lambda: -np.inf)
    for i in range(len(desc)):
        l = int(desc[i, D_LAYER])
        ends[l] = max(ends[l], t[i, T_C_END])
    out["layer_end_us"] = [ends[l] for l in sorted(ends)]
    if len(ends) > 2:
        out["layer_period_us"] = float(np.median(np.diff(out["layer_end_us"])))
    return out


def layer_timeline(desc, stamps, layer: int) -> Dict:
    """First pickup, last end, first/last deps-met time of each operation in
    one layer, relative to the layer's first pickup."""
    t = _times(stamps)
    ops = collections.defaultdict(lambda: [np.inf, -np.inf, np.inf, -np.inf, 0])
    for i in range(len(desc)):
        if int(desc[i, D_LAYER]) != layer:
            continue
        o = ops[OP_NAMES.get(int(desc[i, D_OP]), "?")]
        s = t[i]
        o[0] = min(o[0], s[T_C_READY])
        o[1] = max(o[1], s[T_C_END])
        o[2] = min(o[2], s[T_L_DEPS])
        o[3] = max(o[3], s[T_L_DEPS])
        o[4] += 1
    base = min(v[0] for v in ops.values())
    return {op: {"n": v[4], "pickup_first": v[0] - base, "end_last": v[1] - base,
                 "deps_first": v[2] - base, "deps_last": v[3] - base} for op, v in ops.items()}


def chrome_trace(desc, stamps, path: str) -> None:
    """Write a chrome://tracing JSON: one row per CTA, one slice per task."""
    t = _times(stamps)
    cta = stamps[:, T_CTA].astype(np.int64) - 1
    ev = []
    for i in range(len(desc)):
        s = t[i]
        if np.isnan(s[T_C_READY]) or np.isnan(s[T_C_END]):
            continue
        op = OP_NAMES.get(int(desc[i, D_OP]), "?")
        ev.append({"name": f"{op} L{int(desc[i, D_LAYER])}", "ph": "X", "pid": 0,
                   "tid": int(cta[i]), "ts": float(s[T_C_READY]),
                   "dur": float(max(0.0, s[T_C_END] - s[T_C_READY])),
                   "args": {"task": i, "a": int(desc[i, D_A]), "b": int(desc[i, D_B])}})
    with open(path, "w") as f:
        json.dump({"traceEvents": ev}, f)
