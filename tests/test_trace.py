"""Per-task trace tools on a hand-built trace (host logic only): the summary,
the per-layer timeline, the Chrome export and the 32-bit timer wrap."""

import json

import numpy as np
import pytest

from moe_persistent_cta_b200 import mk, trace as tr

OP = {name: code for code, name in tr.OP_NAMES.items()}


def make_trace(tasks, base_ns=1_000_000):
    """tasks: (op, layer, cta, {field: microseconds}) -> (desc, stamps) with the
    layout Decoder.trace() returns (globaltimer stamps in ns, CTA + 1)."""
    desc = np.zeros((len(tasks), 32), dtype=np.int32)
    stamps = np.zeros((len(tasks), mk.TRACE_WORDS), dtype=np.uint32)
    for i, (op, layer, cta, times) in enumerate(tasks):
        desc[i, tr.D_OP] = OP[op]
        desc[i, tr.D_LAYER] = layer
        for field, us in times.items():
            stamps[i, field] = (base_ns + int(round(us * 1000))) % (1 << 32)
        stamps[i, tr.T_CTA] = cta + 1
    return desc, stamps


def full(deps, ready, act, end, math=None):
    d = {tr.T_P_RESOLVED: deps - 1.0, tr.T_P_ISSUED: deps - 0.5, tr.T_L_DEPS: deps,
         tr.T_L_ACT: deps + 0.1, tr.T_C_READY: ready, tr.T_C_ACT: act, tr.T_C_END: end}
    if math is not None:
        d[tr.T_C_MATH] = math
    return d


TASKS = [
    ("rn", 0, 0, full(0.0, 0.5, 0.6, 3.0)),
    ("qkv", 0, 1, full(3.5, 4.0, 5.0, 9.0, math=7.0)),
    ("qkv", 0, 0, full(3.6, 3.5, 4.5, 8.0, math=6.5)),
    ("gateup", 0, 1, full(10.0, 11.0, 11.5, 15.0, math=13.0)),
    ("rn", 1, 0, full(15.5, 16.0, 16.2, 18.0)),
]


def test_summary_per_op_and_gaps():
    desc, stamps = make_trace(TASKS)
    s = tr.summarize(desc, stamps)
    # stamps are relative to the earliest one (the first task's producer stamp, -1 us)
    assert s["step_us"] == pytest.approx(19.0)
    qkv = s["ops"]["qkv"]
    assert qkv["total"]["n"] == 2
    assert qkv["total"]["mean"] == pytest.approx(((9.0 - 4.0) + (8.0 - 3.5)) / 2)
    assert qkv["math"]["mean"] == pytest.approx(((7.0 - 5.0) + (6.5 - 4.5)) / 2)
    assert qkv["epilogue"]["mean"] == pytest.approx(((9.0 - 7.0) + (8.0 - 6.5)) / 2)
    assert s["ops"]["rn"]["act_wait"]["mean"] == pytest.approx(((0.6 - 0.5) + (16.2 - 16.0)) / 2)
    assert "math" not in s["ops"]["rn"]   # tasks without a math stamp report none
    # CTA 0 runs rn(0) [0.5, 3.0], qkv [3.5, 8.0], rn(1) [16.0, 18.0]; CTA 1 one gap too
    gaps = sorted([3.5 - 3.0, 16.0 - 8.0, 11.0 - 9.0])
    assert s["gap_between_tasks_us"]["p50"] == pytest.approx(np.median(gaps))
    assert s["gap_between_tasks_us"]["mean"] == pytest.approx(np.mean(gaps))
    assert s["layer_end_us"] == pytest.approx([15.0 + 1.0, 18.0 + 1.0])


def test_layer_timeline_is_relative_to_first_pickup():
    desc, stamps = make_trace(TASKS)
    tl = tr.layer_timeline(desc, stamps, 0)
    assert set(tl) == {"rn", "qkv", "gateup"}
    assert tl["rn"]["pickup_first"] == pytest.approx(0.0)
    assert tl["qkv"]["n"] == 2
    assert tl["qkv"]["pickup_first"] == pytest.approx(3.5 - 0.5)
    assert tl["qkv"]["end_last"] == pytest.approx(9.0 - 0.5)
    assert tl["qkv"]["deps_first"] == pytest.approx(3.5 - 0.5)
    assert tl["qkv"]["deps_last"] == pytest.approx(3.6 - 0.5)
    assert tl["gateup"]["end_last"] == pytest.approx(15.0 - 0.5)


def test_timer_wrap_between_stamps():
    """The 32-bit nanosecond timer wraps every ~4.3 s; a step that straddles the
    wrap must still give increasing, correct times."""
    base = (1 << 32) - 2_000   # 2 us before the wrap
    desc, stamps = make_trace(TASKS, base_ns=base)
    assert stamps[:, tr.T_C_END].min() < stamps[:, tr.T_P_RESOLVED].max()   # wrapped
    s = tr.summarize(desc, stamps)
    assert s["step_us"] == pytest.approx(19.0)
    assert s["ops"]["qkv"]["total"]["mean"] == pytest.approx(4.75)


def test_missing_stamps_are_ignored():
    tasks = TASKS + [("down", 0, 2, {tr.T_P_RESOLVED: 12.0})]   # resolved, never run
    desc, stamps = make_trace(tasks)
    s = tr.summarize(desc, stamps)
    assert "total" not in s["ops"].get("down", {})   # no statistic from a task that never ran
    assert s["ops"]["qkv"]["total"]["n"] == 2
    assert s["step_us"] == pytest.approx(19.0)


def test_chrome_trace_export(tmp_path):
    tasks = TASKS + [("down", 0, 2, {tr.T_P_RESOLVED: 12.0})]
    desc, stamps = make_trace(tasks)
    path = tmp_path / "step.json"
    tr.chrome_trace(desc, stamps, str(path))
    ev = json.loads(path.read_text())["traceEvents"]
    assert len(ev) == len(TASKS)   # the task that never ran has no slice
    first = [e for e in ev if e["name"] == "gateup L0"][0]
    assert first["tid"] == 1
    assert first["ts"] == pytest.approx(11.0 + 1.0)
    assert first["dur"] == pytest.approx(4.0)
