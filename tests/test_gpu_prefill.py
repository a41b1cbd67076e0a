"""GPU parity of chunked prefill through the interpreter: the M prompt
tokens of one sequence run as M consecutive batch entries of one step (equal
seq_lens, positions seq_len + 0 .. M - 1, one page-table row).  The
definition they are checked against is causal attention over the sequence,
which the oracle computes as M decode steps in a row, each appending its
token's K/V before the next."""

import numpy as np
import pytest
import torch

import oracle
from moe_persistent_cta_b200 import configs, mk, synth
from tests.gpu_common import REL_L2, TinyRig, compare_logits
from tests.oracle_io import array_kv, array_weights, oracle_shape

pytestmark = pytest.mark.gpu

TIGHT = 2e-3   # as in the decode parity tests of the tiny model


def _layout(entries):
    """Per batch entry: cached prefix, position and owning sequence."""
    seq_lens, positions, owner = [], [], []
    for s, (prefix, m) in enumerate(entries):
        for g in range(m):
            seq_lens.append(prefix)
            positions.append(prefix + g)
            owner.append(s)
    return seq_lens, positions, owner


@pytest.mark.parametrize("entries", [
    [(61, 6)],                    # one group whose tokens cross a page boundary
    [(100, 1), (0, 4), (3, 1)],   # a group on an empty prefix between decode entries
    [(64, 2)],                    # batch 2: the two-token FMA tiles
    [(130, 8)],                   # eight prompt tokens, the largest group
    [(5, 3), (70, 5)],            # two groups in one batch
])
def test_prefill_group_matches_sequential_decode(entries):
    seq_lens, positions, owner = _layout(entries)
    rig = TinyRig(configs.TINY, seq_lens, seed=11)
    try:
        first = {}
        for b, s in enumerate(owner):
            first.setdefault(s, b)
        for b, s in enumerate(owner):
            rig.table[b] = rig.table[first[s]]
        tokens = [int(t) for t in rig.tokens]
        rig.dec.step(rig.i32(tokens), rig.i32(positions), rig.table.to(rig.dev),
                     rig.i32(seq_lens), rig.logits)
        rig.dec.check_ok()
        got = rig.logits.cpu().double().numpy()
        shape, W = oracle_shape(rig.shape), array_weights(rig.W)
        kv = array_kv(rig.k, rig.v)
        table = rig.table.numpy()
        for b in range(len(owner)):   # in batch order: a group's tokens in sequence order
            ref = oracle.decode_step(shape, W, kv, [tokens[b]], [positions[b]], [table[b]],
                                     append=True)[0]
            err, rel = compare_logits(got[b], ref)
            assert err <= TIGHT and rel <= REL_L2, (b, err, rel)
            assert int(np.argmax(got[b])) == int(np.argmax(ref)), b
        # the next token of every sequence reads all of the chunk's K/V from the pool
        nxt = [prefix + m for (prefix, m) in entries]
        rows = torch.stack([rig.table[first[s]] for s in range(len(entries))])
        rig.dec.build_schedule(nxt, rows.shape[1])
        nt = [int(t) for t in synth.make_tokens(len(entries), rig.shape["vocab"], 5)]
        lg = torch.empty((len(entries), rig.shape["vocab"]), dtype=torch.float32,
                         device=rig.dev)
        rig.dec.step(rig.i32(nt), rig.i32(nxt), rows.to(rig.dev), rig.i32(nxt), lg)
        rig.dec.check_ok()
        got2 = lg.cpu().double().numpy()
        ref2 = oracle.decode_step(shape, W, kv, nt, nxt, rows.numpy())
        for s in range(len(entries)):
            err, rel = compare_logits(got2[s], ref2[s])
            assert err <= TIGHT and rel <= REL_L2, (s, err, rel)
    finally:
        rig.close()


def test_prefill_group_unfused_equals_fused():
    """The per-phase launches run the same tasks: identical logits."""
    seq_lens, positions, _ = _layout([(40, 5)])
    rig = TinyRig(configs.TINY, seq_lens, seed=12)
    try:
        rig.table[1:] = rig.table[0]
        args = (rig.i32(rig.tokens), rig.i32(positions), rig.table.to(rig.dev),
                rig.i32(seq_lens))
        rig.dec.step(*args, rig.logits)
        rig.dec.check_ok()
        fused = rig.logits.cpu().numpy().copy()
        rig.dec.step(*args, rig.logits, unfused=True)
        rig.dec.check_ok()
        assert np.array_equal(fused, rig.logits.cpu().numpy())
    finally:
        rig.close()


@pytest.mark.parametrize("seq_lens,positions", [
    ([10, 10], [11, 11]),   # entry 0 claims a predecessor it does not have
    ([10, 20], [10, 21]),   # entry 1's predecessor is another sequence
    ([10, 10], [10, 12]),   # a gap in the group's positions
])
def test_broken_prefill_group_is_reported(seq_lens, positions):
    """Positions that do not form a prefill group stop the step with a
    device-side error (the kernel's own checks; no attention reads outside
    the batch), and the context stays usable."""
    rig = TinyRig(configs.TINY, seq_lens, seed=13)
    try:
        rig.dec.step(rig.i32(rig.tokens), rig.i32(positions), rig.table.to(rig.dev),
                     rig.i32(seq_lens), rig.logits)
        rc, detail = rig.dec.check()
        assert rc in (mk.MK_ERR_STATE, mk.MK_ERR_DEVICE), (rc, detail)
        rig.dec.build_schedule(seq_lens, rig.table.shape[1])
        got = rig.step()
        ref = rig.oracle_step()
        assert compare_logits(got, ref)[0] <= TIGHT
    finally:
        rig.close()
