"""Host schedule planner: structure, counter targets and deadlock freedom.

The planner's per-CTA lists must (a) contain every tile of every operation
exactly once, (b) give every counter exactly as many signalling tasks as its
per-step target, and (c) let a step finish when every CTA executes its list
in order and each task only waits on counters -- the property that lets the
persistent kernel spin on counters without deadlocking (every list is a
subsequence of one topological order, all CTAs co-resident).
"""

import collections

import numpy as np
import pytest

from moe_persistent_cta_b200 import configs, engine

D_OP, D_LAYER, D_A, D_B, D_C, D_D, D_FLAGS, D_NWAIT = 0, 1, 2, 3, 4, 5, 6, 7
D_W0, D_W0N, D_PW, D_PWN, D_NSIG, D_S0 = 8, 9, 12, 13, 14, 15
D_NSTAGE, D_ROW0, D_K0, D_KCH, D_R, D_NMAT, D_BSLOT, D_SEQ, D_X0 = 17, 18, 19, 20, 21, 22, 25, 26, 29
OP_RN, OP_QKV, OP_ROUTER, OP_TOPK, OP_ATTN, OP_COMBINE, OP_OPROJ, OP_GATEUP, OP_DOWN, OP_LM = range(1, 11)
F_LOAD_A, F_REL_A, F_LOAD_B, F_LAST, F_SINGLE = 1, 2, 4, 8, 16


def lists_of(counts, desc):
    return [desc[c, : counts[c]] for c in range(len(counts))]


def simulate(counts, desc, targets, epochs=2):
    """Run every CTA's list in order, a task completing as soon as its loader
    waits and its producer wait are met.  Returns final counter values."""
    n = len(counts)
    ctr = np.zeros(len(targets), dtype=np.int64)
    for ep in range(1, epochs + 1):
        pos = [0] * n
        progress = True
        while progress:
            progress = False
            for c in range(n):
                while pos[c] < counts[c]:
                    t = desc[c, pos[c]]
                    ok = True
                    for w in range(t[D_NWAIT]):
                        if ctr[t[D_W0 + 2 * w]] < ep * t[D_W0N + 2 * w]:
                            ok = False
                    if t[D_PW] >= 0 and ctr[t[D_PW]] < ep * t[D_PWN]:
                        ok = False
                    if not ok:
                        break
                    for s in range(t[D_NSIG]):
                        ctr[t[D_S0 + s]] += 1
                    pos[c] += 1
                    progress = True
        stuck = [c for c in range(n) if pos[c] < counts[c]]
        assert not stuck, f"epoch {ep}: CTAs {stuck[:5]} cannot make progress (deadlock)"
        assert np.array_equal(ctr, ep * targets.astype(np.int64))
    return ctr


@pytest.mark.parametrize("name,n_ctas,lens", [
    ("tiny", 148, [128]),
    ("tiny", 7, [128]),
    ("tiny", 3, [0]),
    ("tiny", 148, [5, 64, 65, 300]),
])
def test_tiny_plan_simulates(name, n_ctas, lens):
    shape = configs.TINY
    meta, counts, desc, targets = engine.plan_schedule(shape, n_ctas, lens)
    assert meta[0] == n_ctas
    assert counts.sum() == meta[2]
    simulate(counts, desc, targets)


def test_30b_b1_plan_structure():
    shape = configs.MOE30B
    meta, counts, desc, targets = engine.plan_schedule(shape, 148, [8192])
    simulate(counts, desc, targets, epochs=1)
    allt = np.concatenate(lists_of(counts, desc))
    ops = collections.Counter(allt[:, D_OP].tolist())
    L, d = shape["n_layers"], shape["d_model"]
    qkv_rows = (shape["n_q_heads"] + 2 * shape["n_kv_heads"]) * shape["head_dim"]
    assert ops[OP_RN] == (L + 1) * d // 64
    assert ops[OP_QKV] == L * qkv_rows // 16
    assert ops[OP_ROUTER] == L * shape["n_experts"] // 16
    assert ops[OP_TOPK] == L
    assert ops[OP_OPROJ] == L * shape["n_kv_heads"] * d // 64
    S = min(shape["n_experts"], shape["top_k"])
    assert ops[OP_GATEUP] == L * S * shape["d_ff"] // 16
    assert ops[OP_DOWN] == L * S * d // 64
    assert ops[OP_LM] == shape["vocab"] // 128
    # every (layer, tile) of QKV appears exactly once
    q = allt[allt[:, D_OP] == OP_QKV]
    keys = set(zip(q[:, D_LAYER].tolist(), q[:, D_ROW0].tolist()))
    assert len(keys) == len(q)
    # attention chunks cover all cached pages of every (layer, group)
    a = allt[allt[:, D_OP] == OP_ATTN]
    nc = a[0, D_D]
    ppc = a[0, 27]
    assert nc * ppc * 64 >= 8192 + 64
    assert len(a) == L * shape["n_kv_heads"] * nc
    # balance: the bytes each CTA streams are within a few percent
    assert counts.max() <= 2 * counts.min() + 64


def test_30b_b8_plan_simulates():
    shape = configs.MOE30B
    from moe_persistent_cta_b200 import synth
    lens = synth.seq_lengths(("uniform", 1024, 16384, 4), 8)
    meta, counts, desc, targets = engine.plan_schedule(shape, 148, lens)
    simulate(counts, desc, targets, epochs=1)
    assert meta[4] == 64   # expert slots = min(E, B*k)


def test_activation_slot_flags():
    """Slot A is (re)loaded exactly when the normalized-input level changes
    along a CTA's list and released after the last task of each run; every
    small-activation task loads and alternates its buffer."""
    meta, counts, desc, targets = engine.plan_schedule(configs.MOE30B, 148, [8192])
    a_ops = (OP_QKV, OP_ROUTER, OP_GATEUP, OP_LM)
    b_ops = (OP_ATTN, OP_OPROJ, OP_DOWN)
    for lst in lists_of(counts, desc):
        cur = None
        nb = 0
        last_a = None
        for i, t in enumerate(lst):
            assert t[D_SEQ] == i
            op = t[D_OP]
            if op in a_ops:
                level = t[D_LAYER]
                if level != cur:
                    assert t[D_FLAGS] & F_LOAD_A
                    if last_a is not None:
                        assert last_a[D_FLAGS] & F_REL_A
                    cur = level
                else:
                    assert not (t[D_FLAGS] & F_LOAD_A)
                last_a = t
            if op in b_ops:
                assert t[D_FLAGS] & F_LOAD_B
                assert t[D_BSLOT] == nb % 2
                nb += 1
            else:
                assert not (t[D_FLAGS] & F_LOAD_B)


def test_gemv_tiles_fill_whole_stages():
    """Every GEMV tile streams whole 16 KB stages: n_mat * R/16 * KCH units
    of 2 KB, a multiple of 8 per stage."""
    for shape in (configs.TINY, configs.MOE30B):
        meta, counts, desc, targets = engine.plan_schedule(shape, 148, [100])
        allt = np.concatenate(lists_of(counts, desc))
        g = allt[np.isin(allt[:, D_OP], [OP_QKV, OP_ROUTER, OP_OPROJ, OP_GATEUP, OP_DOWN, OP_LM])]
        units = g[:, D_NMAT] * (g[:, D_R] // 16) * g[:, D_KCH]
        assert np.all(units % 8 == 0)
        assert np.all(units // 8 == g[:, D_NSTAGE])
        mtn = g[:, D_NMAT] * (g[:, D_R] // 16)
        assert np.all(8 % mtn == 0)


def test_invalid_shapes_rejected():
    import ctypes
    from moe_persistent_cta_b200 import mk
    bad = dict(configs.TINY, head_dim=96)
    with pytest.raises(mk.MKError):
        engine.plan_schedule(bad, 148, [10])
    with pytest.raises(mk.MKError):
        engine.plan_schedule(configs.TINY, 148, [10] * 9)      # batch > 8
    with pytest.raises(mk.MKError):
        engine.plan_schedule(configs.TINY, 148, [-1])
