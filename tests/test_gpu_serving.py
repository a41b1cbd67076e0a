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
