"""Continuous-batching host logic (no GPU): the page pool and the slot
scheduler keep page ownership consistent through refills and growth, and ask
for a schedule rebuild exactly when the batch changed or outgrew its plan."""

import numpy as np
import pytest

from moe_persistent_cta_b200.serving import PAGE, PagePool, SlotScheduler, pages_for


def check_invariants(sched, pool):
    owned = [p for s in sched.seqs if s is not None for p in s.pages]
    assert len(owned) == len(set(owned))                      # no page shared
    assert len(owned) + pool.free_count() == pool.n_pages     # none lost
    table = sched.page_table()
    for i, s in enumerate(sched.seqs):
        if s is None:
            continue
        assert len(s.pages) >= pages_for(s.cached)
        assert list(table[i, :len(s.pages)]) == s.pages
        assert np.all(table[i, len(s.pages):] == -1)


def test_pool_alloc_release_roundtrip():
    pool = PagePool(10)
    a = pool.alloc(4)
    b = pool.alloc(6)
    assert sorted(a + b) == list(range(10))
    with pytest.raises(MemoryError):
        pool.alloc(1)
    pool.release(a)
    assert pool.free_count() == 4
    assert sorted(pool.alloc(4)) == sorted(a)


def test_slot_scheduler_through_many_refills():
    rng = np.random.default_rng(5)
    pool = PagePool(400)
    sched = SlotScheduler(4, pool, max_pages_per_seq=40, rng=rng, start_lo=10, start_hi=900,
                          mean_new=6, max_new=64, horizon=16)
    rebuilds = 0
    for step in range(300):
        refilled = sched.fill()
        if step == 0:
            assert refilled == [0, 1, 2, 3]
        need = sched.before_step()
        assert need == (bool(refilled) or step == 0 or need)
        if need:
            plan = sched.planned()
            assert all(p >= s.cached for p, s in zip(plan, sched.seqs))
            rebuilds += 1
        # after a rebuild, every length is within its plan
        assert all(s.cached <= p for s, p in zip(sched.seqs, sched.plan_len))
        for s in sched.seqs:
            assert len(s.pages) >= pages_for(s.cached + 1)   # the new token's page exists
        check_invariants(sched, pool)
        before = [s.cached for s in sched.seqs]
        done = sched.after_step()
        for i, s in enumerate(sched.seqs):
            if i not in done:
                assert s.cached == before[i] + 1
    assert sched.generated == 300 * 4
    assert sched.finished > 20 and rebuilds >= sched.finished // 4
    check_invariants(sched, pool)


def test_rebuild_when_a_sequence_outgrows_its_plan():
    rng = np.random.default_rng(0)
    pool = PagePool(100)
    sched = SlotScheduler(1, pool, max_pages_per_seq=50, rng=rng, start_lo=100, start_hi=100,
                          mean_new=1e9, max_new=1000, horizon=8)
    sched.fill()
    assert sched.before_step()
    sched.planned()
    for k in range(9):                  # 100 .. 108 cached tokens: within the plan
        assert not sched.before_step()
        sched.after_step()
    assert sched.seqs[0].cached == 109
    assert sched.before_step()          # 109 > 108: outgrew the plan


def test_full_capacity_plan_needs_one_build():
    rng = np.random.default_rng(3)
    pool = PagePool(200)
    sched = SlotScheduler(3, pool, max_pages_per_seq=20, rng=rng, start_lo=10, start_hi=600,
                          mean_new=4, max_new=32, horizon=None)
    builds = 0
    for _ in range(200):
        sched.fill()
        if sched.before_step():
            assert sched.planned() == [20 * PAGE - 1] * 3
            builds += 1
        check_invariants(sched, pool)
        sched.after_step()
    assert builds == 1 and sched.finished > 30
