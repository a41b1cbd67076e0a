"""Host schedule planner: structure, counter targets and deadlock freedom.

The step is one task list; at run time every CTA takes the next task with an
atomic add, posts it to its in-order task FIFO and runs it.  The step cannot
deadlock if (a) every counter a task waits on is signalled only by tasks that
are earlier in the list (the earlier tasks were taken by running, co-resident
CTAs that finish their FIFOs in order) and (b) every counter's per-step target
equals the number of tasks that signal it.  These tests check both, plus the
list's structure, on CPU.
"""

import collections

import numpy as np
import pytest

from moe_persistent_cta_b200 import configs, engine, synth

D_OP, D_LAYER, D_A, D_B, D_C, D_D, D_FLAGS, D_NWAIT = 0, 1, 2, 3, 4, 5, 6, 7
D_W0, D_W0N, D_PW, D_PWN, D_NSIG, D_S0 = 8, 9, 12, 13, 14, 15
D_NSTAGE, D_ROW0, D_K0, D_KCH, D_R, D_NMAT, D_ACT, D_PPC, D_PHASE = 17, 18, 19, 20, 21, 22, 25, 27, 28
OP_RN, OP_QKV, OP_ROUTER, OP_TOPK, OP_ATTN, OP_COMBINE, OP_OPROJ, OP_GATEUP, OP_DOWN, OP_LM = range(1, 11)
NR_30B = 2048 // 64
ACT_NONE, ACT_A, ACT_B = 0, 1, 2


D_X0, D_X1, D_X2 = 29, 30, 31
F_COMBINE = 128   # last-arriver work: the attention merge of a (token, KV head)
F_ARGMAX = 512    # last-arriver work: a greedy step's tokens after the LM head
FUSED = F_COMBINE | F_ARGMAX


def signal_sets(desc, targets):
    """Per counter: (signals per step, tasks that may send them).  A task
    signals each counter of its list once; the tasks of a last-arriver group
    (same arrival counter D_X0) together signal their join counter D_X2 once,
    and any of them may be the sender."""
    count = collections.Counter()
    senders = collections.defaultdict(list)
    groups = collections.defaultdict(list)
    for i, t in enumerate(desc):
        for s in range(t[D_NSIG]):
            c = int(t[D_S0 + s])
            count[c] += 1
            senders[c].append(i)
        if t[D_FLAGS] & FUSED:
            groups[int(t[D_X0])].append(i)
    for a, members in groups.items():
        arrivals = {int(desc[i][D_X1]) for i in members}
        joins = {int(desc[i][D_X2]) for i in members}
        assert arrivals == {len(members)}, f"arrival counter {a}: {len(members)} arrive, {arrivals}"
        assert targets[a] == len(members)
        assert len(joins) == 1
        j = joins.pop()
        count[j] += 1
        senders[j].extend(members)
    return count, senders


def check_order_and_targets(desc, targets, n_ctas, grab):
    """(a) waits only on earlier senders, (b) targets == signals per step;
    then simulate a greedy dynamic execution on n_ctas CTAs."""
    count, senders = signal_sets(desc, targets)
    last_sig = {c: max(v) for c, v in senders.items()}
    for i, t in enumerate(desc):
        waits = [(int(t[D_W0 + 2 * w]), int(t[D_W0N + 2 * w])) for w in range(t[D_NWAIT])]
        if t[D_PW] >= 0:
            waits.append((int(t[D_PW]), int(t[D_PWN])))
        for c, need in waits:
            assert count[c] == need, f"task {i}: counter {c} gets {count[c]} signals, waits {need}"
            assert last_sig[c] < i, f"task {i} waits on counter {c} sent later (task {last_sig[c]})"
    for c, k in count.items():
        assert targets[c] == k
    assert targets[grab] == 0      # the dispenser restarts at 0 every launch
    # greedy dynamic execution: each CTA takes the next task when it has
    # finished its previous one; a task finishes when its waits are met
    remaining = {c: len(v) for c, v in senders.items()}
    done_time = collections.defaultdict(float)
    free = [0.0] * n_ctas
    finish = 0.0
    for i, t in enumerate(desc):
        c = int(np.argmin(free))
        start = free[c]
        waits = [int(t[D_W0 + 2 * w]) for w in range(t[D_NWAIT])]
        if t[D_PW] >= 0:
            waits.append(int(t[D_PW]))
        for w in waits:
            assert remaining[w] == 0      # every possible sender already taken earlier
            start = max(start, done_time[w])
        free[c] = start + 1.0
        finish = max(finish, free[c])
        sent = [int(t[D_S0 + s]) for s in range(t[D_NSIG])]
        if t[D_FLAGS] & FUSED:
            sent.append(int(t[D_X2]))
        for w in sent:
            remaining[w] -= 1
            done_time[w] = max(done_time[w], free[c])
    return finish


@pytest.mark.parametrize("n_ctas,lens", [(148, [128]), (7, [128]), (3, [0]),
                                         (148, [5, 64, 65, 300])])
def test_tiny_plan(n_ctas, lens):
    meta, desc, targets = engine.plan_schedule(configs.TINY, n_ctas, lens)
    assert meta[0] == len(desc)
    check_order_and_targets(desc, targets, n_ctas, meta[8])


def test_30b_b1_plan_structure():
    shape = configs.MOE30B
    meta, desc, targets = engine.plan_schedule(shape, 148, [8192])
    check_order_and_targets(desc, targets, 148, meta[8])
    ops = collections.Counter(desc[:, D_OP].tolist())
    L, d = shape["n_layers"], shape["d_model"]
    qkv_rows = (shape["n_q_heads"] + 2 * shape["n_kv_heads"]) * shape["head_dim"]
    assert ops[OP_QKV] == L * qkv_rows // 16
    # the norm tiles produce the router logits: no router tiles, and each
    # layer's top-k waits for all of the layer's norm tiles and signals the
    # counter the layer's expert tiles wait on
    assert ops[OP_ROUTER] == 0
    assert ops[OP_RN] == (L + 1) * d // 64
    assert ops[OP_TOPK] == L
    tk = desc[desc[:, D_OP] == OP_TOPK]
    assert np.all(tk[:, D_NWAIT] == 1) and np.all(tk[:, D_W0N] == d // 64)
    rn = desc[desc[:, D_OP] == OP_RN]
    # at batch 1 each expert tile's producer computes the layer's routing
    # itself once the layer's norm tiles are done: it waits on their counter
    gu = desc[desc[:, D_OP] == OP_GATEUP]
    for l in (0, 5, L - 1):
        norm_ctr = set(rn[rn[:, D_LAYER] == l][:, D_S0].tolist())
        assert set(gu[gu[:, D_LAYER] == l][:, D_PW].tolist()) == norm_ctr
        assert np.all(gu[gu[:, D_LAYER] == l][:, D_PWN] == d // 64)
    # a norm tile of a level that feeds a layer streams its router columns:
    # one ring stage per 128 experts; the final norm streams nothing
    E = shape["n_experts"]
    assert np.all(rn[rn[:, D_LAYER] < L][:, D_NSTAGE] == (E + 127) // 128)
    assert np.all(rn[rn[:, D_LAYER] == L][:, D_NSTAGE] == 0)
    # ... through its own layer's router tensor map (8 maps per layer, router third)
    D_MAP0 = 23
    lv = rn[rn[:, D_LAYER] < L]
    assert np.all(lv[:, D_MAP0] == lv[:, D_LAYER] * 8 + 2)
    for l in (0, 5):
        q = desc[(desc[:, D_OP] == OP_QKV) & (desc[:, D_LAYER] == l)]
        ctr = q[0, D_W0]
        senders = rn[(rn[:, D_LAYER] == l)]
        assert np.all(senders[:, D_S0] == ctr) and len(senders) == d // 64
    a_multi = desc[(desc[:, D_OP] == OP_ATTN) & (desc[:, D_D] > 1)]
    assert len(a_multi)
    fused_comb = bool(np.all(a_multi[:, D_FLAGS] & F_COMBINE))
    assert fused_comb or not np.any(a_multi[:, D_FLAGS] & F_COMBINE)
    assert ops[OP_COMBINE] == (0 if fused_comb else L * shape["n_kv_heads"])
    assert ops[OP_OPROJ] == L * shape["n_kv_heads"] * d // 64
    S = min(shape["n_experts"], shape["top_k"])
    assert ops[OP_GATEUP] == L * S * shape["d_ff"] // 16
    assert ops[OP_DOWN] == L * S * d // 64
    assert ops[OP_LM] == shape["vocab"] // 128
    lmt = desc[desc[:, D_OP] == OP_LM]
    assert np.all(lmt[:, D_FLAGS] & F_ARGMAX) and np.all(lmt[:, D_X1] == len(lmt))
    assert len(set(lmt[:, D_X0].tolist())) == 1 and np.all(lmt[:, D_NSIG] == 0)
    q = desc[desc[:, D_OP] == OP_QKV]
    assert len(set(zip(q[:, D_LAYER].tolist(), q[:, D_ROW0].tolist()))) == len(q)
    a = desc[desc[:, D_OP] == OP_ATTN]
    nc, ppc = a[0, D_D], a[0, D_PPC]
    assert nc * ppc * 64 >= 8192 + 64
    assert len(a) == L * shape["n_kv_heads"] * nc
    # each layer ends with tiles feeding the next norm
    for l in (0, 3, 47):
        ops = desc[desc[:, D_LAYER] == l][:, D_OP]
        assert ops[-1] in (OP_OPROJ, OP_DOWN)
    # every task of a layer is dispensed before the next layer's first
    # projection tile that reads its output
    for l in range(shape["n_layers"] - 1):
        last = np.where(desc[:, D_LAYER] == l)[0].max()
        nxt = np.where((desc[:, D_LAYER] == l + 1) & (desc[:, D_OP] != OP_RN))[0].min()
        assert last < nxt


def test_30b_b8_plan():
    shape = configs.MOE30B
    lens = synth.seq_lengths(("uniform", 1024, 16384, 4), 8)
    meta, desc, targets = engine.plan_schedule(shape, 148, lens)
    check_order_and_targets(desc, targets, 148, meta[8])
    assert meta[2] == 64   # expert slots = min(E, B*k)
    # at batch 8 the expert tiles' producers copy the top-k task's table:
    # they wait on the top-k's signal
    tk = desc[desc[:, D_OP] == OP_TOPK]
    for op in (OP_GATEUP, OP_DOWN):
        ex = desc[desc[:, D_OP] == op]
        for l in (0, 20):
            assert set(ex[ex[:, D_LAYER] == l][:, D_PW].tolist()) == \
                set(tk[tk[:, D_LAYER] == l][:, D_S0].tolist())
            assert np.all(ex[ex[:, D_LAYER] == l][:, D_PWN] == 1)


def test_activation_levels_never_decrease():
    """The runtime reuses slot A while consecutive A-tasks read the same
    level; that is only sound if levels never go back along the list."""
    for shape, lens in ((configs.TINY, [70, 3]), (configs.MOE30B, [8192])):
        meta, desc, targets = engine.plan_schedule(shape, 148, lens)
        a = desc[desc[:, D_ACT] == ACT_A]
        assert np.all(np.diff(a[:, D_LAYER]) >= 0)
        assert set(desc[desc[:, D_ACT] == ACT_A][:, D_OP]) <= {OP_QKV, OP_GATEUP, OP_LM}
        assert set(desc[desc[:, D_ACT] == ACT_B][:, D_OP]) <= {OP_ATTN, OP_OPROJ, OP_DOWN}


def test_gemv_tiles_fill_whole_stages():
    """Every GEMV tile streams whole 16 KB stages: n_mat * R/16 * KCH units
    of 2 KB, a multiple of 8 per stage."""
    for shape in (configs.TINY, configs.MOE30B):
        meta, desc, targets = engine.plan_schedule(shape, 148, [100])
        g = desc[np.isin(desc[:, D_OP], [OP_QKV, OP_OPROJ, OP_GATEUP, OP_DOWN, OP_LM])]
        units = g[:, D_NMAT] * (g[:, D_R] // 16) * g[:, D_KCH]
        assert np.all(units % 8 == 0)
        assert np.all(units // 8 == g[:, D_NSTAGE])
        mtn = g[:, D_NMAT] * (g[:, D_R] // 16)
        assert np.all(8 % mtn == 0)


def test_invalid_shapes_rejected():
    from moe_persistent_cta_b200 import mk
    with pytest.raises(mk.MKError):
        engine.plan_schedule(dict(configs.TINY, head_dim=96), 148, [10])
    with pytest.raises(mk.MKError):
        engine.plan_schedule(configs.TINY, 148, [10] * 9)      # batch > 8
    with pytest.raises(mk.MKError):
        engine.plan_schedule(configs.TINY, 148, [-1])
    with pytest.raises(mk.MKError):
        engine.plan_schedule(dict(configs.TINY, n_experts=10, top_k=2), 148, [10])   # E % 4


@pytest.mark.parametrize("lens", [[8192], [100, 2000, 5, 64, 9000, 300, 40, 7]])
def test_unused_slot_tiles_can_be_skipped(lens):
    """Expert tiles of unused slots are dropped by the producers, which jump
    the dispenser to D_C: one past the layer's last tile of the same
    operation.  That is only sound if those tiles are contiguous and
    slot-major (an unused slot is never followed by a used one), and if the
    counters their signals would have reached are the ones the top-k stands
    in for: the slot counter (n_ff gate/up tiles) and the down-tile row
    counters (one signal per slot)."""
    shape = configs.MOE30B
    meta, desc, targets = engine.plan_schedule(shape, 148, lens)
    S, n_ff, NR = meta[2], shape["d_ff"] // 16, shape["d_model"] // 64
    for op, per_slot in ((OP_GATEUP, n_ff), (OP_DOWN, NR)):
        idx = np.where(desc[:, D_OP] == op)[0]
        for l in (0, 17, shape["n_layers"] - 1):
            run = idx[desc[idx, D_LAYER] == l]
            assert len(run) == S * per_slot
            assert np.all(np.diff(run) == 1)                  # contiguous
            assert np.all(desc[run, D_C] == run[-1] + 1)      # jump past the run
            assert np.all(np.diff(desc[run, D_A]) >= 0)       # slot-major
    gu = desc[desc[:, D_OP] == OP_GATEUP]
    dn = desc[desc[:, D_OP] == OP_DOWN]
    # each slot counter is signalled by exactly its n_ff gate/up tiles and
    # waited on (for n_ff) by exactly its down tiles
    for l in (0, 30):
        for j in (0, S - 1):
            g = gu[(gu[:, D_LAYER] == l) & (gu[:, D_A] == j)]
            d = dn[(dn[:, D_LAYER] == l) & (dn[:, D_A] == j)]
            c = set(g[:, D_S0].tolist())
            assert len(c) == 1 and targets[c.pop()] == n_ff
            assert set(d[:, D_W0].tolist()) == set(g[:, D_S0].tolist())
            assert np.all(d[:, D_W0N] == n_ff)
        # each down-tile row counter gets one signal per slot plus the O-proj groups
        rows = dn[dn[:, D_LAYER] == l]
        for r in (0, NR - 1):
            c = set(rows[rows[:, D_B] == r][:, D_S0].tolist())
            assert len(c) == 1 and targets[c.pop()] == S + shape["n_kv_heads"]


def test_ring_depth_and_attention_work_area():
    """Shared memory of the 30B shape: at batch 1 the ring holds 10 stages and
    attention works in the scratch area; at batch 8 the 64 KB fp32
    activation buffer leaves room for 5 stages only because an attention
    chunk works in the rest of its own B buffer (sized for the down tiles'
    8 x 768 floats)."""
    m1, _, _ = engine.plan_schedule(configs.MOE30B, 148, [8192])
    m8, _, _ = engine.plan_schedule(configs.MOE30B, 148,
                                    [9291, 10503, 5128, 15912, 9509, 6887, 1439, 10393])
    assert (m1[10], m1[11]) == (10, 0)
    assert (m8[10], m8[11]) == (5, 1)
