"""Continuous batching on the GPU (tiny model): slots are refilled as
sequences stop, pages are allocated as sequences grow, the schedule is rebuilt
between steps, and every step's logits match the oracle run on the same KV
pools, tokens, lengths and page tables."""

import numpy as np
import pytest
import torch

import oracle
from moe_persistent_cta_b200 import configs, engine, synth
from moe_persistent_cta_b200.serving import PagePool, SlotScheduler, fill_prefix_kv
from tests.gpu_common import MAX_ABS, REL_L2, compare_logits, to_dev
from tests.oracle_io import array_kv, array_weights, oracle_shape

pytestmark = pytest.mark.gpu


def test_continuous_batching_matches_oracle_step_by_step():
    shape = configs.TINY
    dev = torch.device("cuda:0")
    slots, steps, max_pages = 3, 40, 8
    W = synth.make_weights(shape, 0, "cpu")
    Wd = to_dev(W, dev)
    n_pages = 3 * slots * max_pages
    k = torch.zeros((shape["n_layers"], n_pages, shape["n_kv_heads"], 64, shape["head_dim"]),
                    dtype=torch.bfloat16, device=dev)
    v = torch.zeros_like(k)
    dec = engine.Decoder(shape, Wd, k, v, max_batch=slots)
    rng = np.random.default_rng(11)
    gen = torch.Generator(device=dev).manual_seed(11)
    pool = PagePool(n_pages)
    sched = SlotScheduler(slots, pool, max_pages, rng, start_lo=5, start_hi=250, mean_new=6,
                          max_new=20, horizon=16)
    i32 = dict(dtype=torch.int32, device=dev)
    tokens = [0] * slots
    logits = torch.empty((slots, shape["vocab"]), dtype=torch.float32, device=dev)
    S, AW = oracle_shape(shape), array_weights(W)
    rebuilds = refills = 0
    try:
        for step in range(steps):
            for i in sched.fill():
                fill_prefix_kv(k, v, sched.seqs[i].pages, gen)
                tokens[i] = int(rng.integers(0, shape["vocab"]))
                refills += 1
            if sched.before_step():
                dec.build_schedule(sched.lens(), max_pages, plan_len=sched.planned())
                rebuilds += 1
            lens, table = sched.lens(), sched.page_table()
            kv = array_kv(k.cpu(), v.cpu())           # the pools as this step reads them
            dec.step(torch.tensor(tokens, **i32), torch.tensor(lens, **i32),
                     torch.from_numpy(table).to(dev), torch.tensor(lens, **i32), logits)
            dec.check_ok()
            got = logits.cpu().double().numpy()
            ref = oracle.decode_step(S, AW, kv, tokens, lens, table)
            err, rel = compare_logits(got, ref)
            assert err <= MAX_ABS and rel <= REL_L2, (step, err, rel)
            nxt = got.argmax(-1)
            assert np.array_equal(nxt, ref.argmax(-1)), step
            tokens = [int(t) for t in nxt]
            sched.after_step()
        assert refills > slots and rebuilds > 1
    finally:
        dec.close()


@pytest.mark.parametrize("horizon", [None, 16])
def test_greedy_chunks_match_stepwise_replay(horizon):
    """run_continuous launches the steps between two slot refills as one
    mk_decode_greedy call (tokens, positions and lengths advance on the
    device).  A replay of the same run, one mk_decode_step per step with a
    host argmax and the same seeded refills, must generate the same tokens:
    the arithmetic of every step is the same."""
    from moe_persistent_cta_b200 import serving
    shape = configs.TINY
    dev = torch.device("cuda:0")
    slots, steps, max_pages = 3, 40, 8
    W = synth.make_weights(shape, 0, "cpu")
    Wd = to_dev(W, dev)
    n_pages = 3 * slots * max_pages
    kshape = (shape["n_layers"], n_pages, shape["n_kv_heads"], 64, shape["head_dim"])
    common = dict(slots=slots, steps=steps, seed=21, start_lo=5, start_hi=250, mean_new=6,
                  max_new=steps, max_pages_per_seq=max_pages)
    k = torch.zeros(kshape, dtype=torch.bfloat16, device=dev)
    v = torch.zeros_like(k)
    dec = engine.Decoder(shape, Wd, k, v, max_batch=slots)
    try:
        r = serving.run_continuous(dec, shape, k, v, horizon=horizon, **common)
    finally:
        dec.close()
    assert r["generated"] == steps * slots and r["greedy_calls"] < steps
    # the replay: same draws in the same order, one step at a time
    k2 = torch.zeros(kshape, dtype=torch.bfloat16, device=dev)
    v2 = torch.zeros_like(k2)
    dec2 = engine.Decoder(shape, Wd, k2, v2, max_batch=slots)
    rng = np.random.default_rng(common["seed"])
    gen = torch.Generator(device=dev).manual_seed(common["seed"])
    sched = SlotScheduler(slots, PagePool(n_pages), max_pages, rng, 5, 250, 6, steps,
                          horizon=None)
    i32 = dict(dtype=torch.int32, device=dev)
    tokens = [0] * slots
    logits = torch.empty((slots, shape["vocab"]), dtype=torch.float32, device=dev)
    want = np.zeros((steps, slots), dtype=np.int64)
    try:
        for step in range(steps):
            refilled = sched.fill()
            for i in refilled:
                fill_prefix_kv(k2, v2, sched.seqs[i].pages, gen)
            for i, t in zip(refilled, [int(rng.integers(0, shape["vocab"])) for _ in refilled]):
                tokens[i] = t
            if sched.before_step():
                dec2.build_schedule(sched.lens(), max_pages, plan_len=sched.planned())
            lens, table = sched.lens(), sched.page_table()
            dec2.step(torch.tensor(tokens, **i32), torch.tensor(lens, **i32),
                      torch.from_numpy(table).to(dev), torch.tensor(lens, **i32), logits)
            dec2.check_ok()
            tokens = [int(t) for t in logits.argmax(-1).cpu()]
            want[step] = tokens
            sched.after_step()
    finally:
        dec2.close()
    if horizon is None:
        # one schedule for the whole run on both sides: bit-identical steps
        assert np.array_equal(r["tokens"], want)
    else:
        # rebuilt schedules cut attention into other chunks than the replay's
        # single schedule, so only the run itself is checked
        assert r["rebuilds"] > 1
        assert np.all((r["tokens"] >= 0) & (r["tokens"] < shape["vocab"]))
