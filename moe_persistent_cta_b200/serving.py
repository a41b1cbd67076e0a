"""Continuous batching over the decode step: a paged-KV page allocator, slot
bookkeeping and the schedule-rebuild policy (host logic only).

The serving side the pages describe runs continuous batching with paged
attention and ragged sequence lengths, at most 8 sequences at a time, with
prefill done separately from the decode engine (aimodeling.com, "Cohere
megakernel engine: one CUDA file, 1.58x vLLM on H100", sections "From demo to
a full serving system" and "Caveats and takeaways").  Here every slot holds
one sequence; when a sequence stops, its pages go back to the pool and the
slot takes a new sequence, whose cached prefix is drawn synthetically into
freshly allocated pages (a stand-in for prefill, timed separately).  The
decode step itself is always the library's fused step.  A schedule depends
only on the batch size and the lengths it was planned for, not on the actual
lengths, so by default every slot is planned at its full page capacity once
and refills reuse the schedule; with a finite horizon the schedule is instead
rebuilt when a slot is refilled or a sequence outgrows its plan.
"""

from __future__ import annotations

import dataclasses
import time
from typing import Dict, List, Optional

import numpy as np
import torch

PAGE = 64


class PagePool:
    """Free list of physical KV pages (one id space shared by every layer's
    K and V pools)."""

    def __init__(self, n_pages: int):
        self.n_pages = n_pages
        self._free = list(range(n_pages - 1, -1, -1))

    def free_count(self) -> int:
        return len(self._free)

    def alloc(self, n: int) -> List[int]:
        if n > len(self._free):
            raise MemoryError(f"KV page pool exhausted: need {n}, have {len(self._free)}")
        out = [self._free.pop() for _ in range(n)]
        return out

    def release(self, pages: List[int]) -> None:
        self._free.extend(reversed(pages))


@dataclasses.dataclass
class Sequence:
    seq_id: int
    cached: int          # tokens in the KV cache before the next step
    remaining: int       # tokens still to generate
    pages: List[int]     # physical pages, in logical order


def pages_for(tokens: int) -> int:
    return (tokens + PAGE - 1) // PAGE


class SlotScheduler:
    """Host bookkeeping of the batch: which sequence each slot holds, its page
    table row, and when the schedule must be rebuilt.  No device work."""

    def __init__(self, slots: int, pool: PagePool, max_pages_per_seq: int, rng: np.random.Generator,
                 start_lo: int, start_hi: int, mean_new: float, max_new: int,
                 horizon: Optional[int] = 64):
        self.slots = slots
        self.pool = pool
        self.max_pages = max_pages_per_seq
        self.rng = rng
        self.start_lo, self.start_hi = start_lo, start_hi
        self.mean_new, self.max_new = mean_new, max_new
        self.horizon = horizon   # None: plan every slot at full capacity, once
        self.seqs: List[Optional[Sequence]] = [None] * slots
        self.plan_len: List[int] = [0] * slots
        self.next_id = 0
        self.need_rebuild = True
        self.generated = 0
        self.finished = 0

    def _new_sequence(self) -> Sequence:
        cached = int(self.rng.integers(self.start_lo, self.start_hi + 1))
        new = min(self.max_new, int(self.rng.geometric(1.0 / self.mean_new)))
        pages = self.pool.alloc(pages_for(cached + 1))
        s = Sequence(self.next_id, cached, new, pages)
        self.next_id += 1
        return s

    def fill(self) -> List[int]:
        """Give every empty slot a new sequence; returns the refilled slots."""
        refilled = []
        for i in range(self.slots):
            if self.seqs[i] is None:
                self.seqs[i] = self._new_sequence()
                refilled.append(i)
        if refilled and self.horizon is not None:
            self.need_rebuild = True
        return refilled

    def lens(self) -> List[int]:
        return [s.cached for s in self.seqs]

    def before_step(self) -> bool:
        """Make sure every sequence has the page its next token goes to;
        returns whether the schedule must be rebuilt first."""
        for i, s in enumerate(self.seqs):
            need = pages_for(s.cached + 1)
            if need > len(s.pages):
                s.pages.extend(self.pool.alloc(need - len(s.pages)))
            if need > self.max_pages:
                raise ValueError("sequence outgrew the page table")
            if s.cached > self.plan_len[i]:
                self.need_rebuild = True
        return self.need_rebuild

    def planned(self) -> List[int]:
        """Plan lengths for a rebuild: the current lengths plus the horizon,
        or every slot's full capacity."""
        cap = self.max_pages * PAGE - 1
        if self.horizon is None:
            self.plan_len = [cap] * self.slots
        else:
            self.plan_len = [min(s.cached + self.horizon, cap) for s in self.seqs]
        self.need_rebuild = False
        return list(self.plan_len)

    def page_table(self) -> np.ndarray:
        t = np.full((self.slots, self.max_pages), -1, dtype=np.int32)
        for i, s in enumerate(self.seqs):
            t[i, :len(s.pages)] = s.pages
        return t

    def after_step(self) -> List[int]:
        """Account the generated token of every slot; finished sequences give
        their pages back.  Returns the slots that finished."""
        done = []
        for i, s in enumerate(self.seqs):
            s.cached += 1
            s.remaining -= 1
            self.generated += 1
            if s.remaining <= 0:
                self.pool.release(s.pages)
                self.seqs[i] = None
                self.finished += 1
                done.append(i)
        return done


def fill_prefix_kv(k_pool: torch.Tensor, v_pool: torch.Tensor, pages: List[int], gen: torch.Generator):
    """Synthetic cached prefix of a new sequence: K and V ~ N(0, 1) in bf16 in
    the given pages of every layer (post-RoPE K, as the decode step expects)."""
    if not pages:
        return
    idx = torch.tensor(pages, dtype=torch.long, device=k_pool.device)
    L, _, Hkv, P, hd = k_pool.shape
    for l in range(L):
        k_pool[l].index_copy_(0, idx, torch.randn((len(pages), Hkv, P, hd), generator=gen,
                                                  device=k_pool.device).to(torch.bfloat16))
        v_pool[l].index_copy_(0, idx, torch.randn((len(pages), Hkv, P, hd), generator=gen,
                                                  device=k_pool.device).to(torch.bfloat16))


def run_continuous(dec, shape: Dict, k_pool: torch.Tensor, v_pool: torch.Tensor, slots: int,
                   steps: int, seed: int, start_lo: int, start_hi: int, mean_new: float,
                   max_new: int, max_pages_per_seq: int, stream=None,
                   horizon: Optional[int] = None) -> Dict:
    """Run `steps` greedy decode steps with slot refills.

    A sequence's stop length is drawn when it starts, so the host knows when
    the next slot frees up: it launches the greedy steps up to that point in
    one mk_decode_greedy call (tokens, positions and lengths advance on the
    device; no host round trip between steps), then refills the freed slots
    (page pool, synthetic prefix, token and length written to the device
    buffers on the same stream) and goes on.  Times are taken with CUDA
    events on the stream: the greedy steps (decode_s), the synthetic prefix
    fills (prefix_fill_s) and schedule rebuilds (rebuild_s, host).  Returns
    counts, times, the generated tokens [steps][slots] and the cached length
    of every slot at every step (for the KV bytes the steps read)."""
    dev = k_pool.device
    rng = np.random.default_rng(seed)
    gen = torch.Generator(device=dev).manual_seed(seed)
    pool = PagePool(int(k_pool.shape[1]))
    sched = SlotScheduler(slots, pool, max_pages_per_seq, rng, start_lo, start_hi, mean_new,
                          max_new, horizon=horizon)
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    i32 = dict(dtype=torch.int32, device=dev)
    tokens = torch.zeros(slots, **i32)
    lens_d = torch.zeros(slots, **i32)
    table_d = torch.zeros((slots, max_pages_per_seq), **i32)
    out = torch.full((steps, slots), -1, **i32)
    logits = torch.empty((slots, shape["vocab"]), dtype=torch.float32, device=dev)
    ev = []            # (kind, start event, end event)
    t_rebuild = 0.0
    rebuilds = 0
    lens_per_step = np.zeros((steps, slots), dtype=np.int64)
    done = 0
    with torch.cuda.stream(s):
        while done < steps:
            refilled = sched.fill()
            if refilled:
                e0 = torch.cuda.Event(enable_timing=True)
                e0.record(s)
                for i in refilled:
                    fill_prefix_kv(k_pool, v_pool, sched.seqs[i].pages, gen)
                e1 = torch.cuda.Event(enable_timing=True)
                e1.record(s)
                ev.append(("fill", e0, e1))
                # the refilled slots' first token and cached length, from a
                # fresh pinned buffer (torch keeps it until the copy has run)
                vals = [[int(rng.integers(0, shape["vocab"])) for _ in refilled],
                        [sched.seqs[i].cached for i in refilled]]
                hr = torch.tensor(vals, dtype=torch.int32).pin_memory().to(dev, non_blocking=True)
                idx = torch.tensor(refilled, dtype=torch.long).pin_memory().to(dev, non_blocking=True)
                tokens.index_copy_(0, idx, hr[0])
                lens_d.index_copy_(0, idx, hr[1])
            n = min(min(q.remaining for q in sched.seqs), steps - done)
            # pages for every token the next n steps append
            for q in sched.seqs:
                need = pages_for(q.cached + n)
                if need > len(q.pages):
                    q.pages.extend(pool.alloc(need - len(q.pages)))
                if need > max_pages_per_seq:
                    raise ValueError("sequence outgrew the page table")
            if sched.need_rebuild or any(q.cached + n - 1 > sched.plan_len[i]
                                         for i, q in enumerate(sched.seqs)):
                t0 = time.perf_counter()
                s.synchronize()
                dec.build_schedule(sched.lens(), max_pages_per_seq, plan_len=sched.planned())
                t_rebuild += time.perf_counter() - t0
                rebuilds += 1
            table_d.copy_(torch.from_numpy(sched.page_table()).pin_memory(), non_blocking=True)
            for j in range(n):
                lens_per_step[done + j] = [q.cached + j for q in sched.seqs]
            e0 = torch.cuda.Event(enable_timing=True)
            e0.record(s)
            dec.greedy(n, tokens, lens_d, table_d, lens_d, logits, out[done:done + n], stream=s)
            e1 = torch.cuda.Event(enable_timing=True)
            e1.record(s)
            ev.append(("decode", e0, e1))
            for _ in range(n):
                sched.after_step()
            done += n
    s.synchronize()
    dec.check_ok()
    t_decode = sum(a.elapsed_time(b) for k, a, b in ev if k == "decode") / 1e3
    t_fill = sum(a.elapsed_time(b) for k, a, b in ev if k == "fill") / 1e3
    return {"steps": steps, "slots": slots, "generated": sched.generated,
            "finished": sched.finished, "sequences": sched.next_id, "rebuilds": rebuilds,
            "decode_s": t_decode, "rebuild_s": t_rebuild, "prefix_fill_s": t_fill,
            "greedy_calls": sum(1 for k, _, _ in ev if k == "decode"),
            "tokens": out.cpu().numpy(), "lens_per_step": lens_per_step}
