"""Python-side handle on the native decode step (argument marshalling only).

``Decoder`` owns one ``mk_ctx``: it hands the library raw device pointers of
caller-owned torch tensors (weights, KV pools, step inputs, logits) and the
torch stream to launch on.  All computation happens in ``libmk.so``.
"""

from __future__ import annotations

import ctypes
from ctypes import byref, c_int32, c_void_p
from typing import Dict, Optional, Sequence

import numpy as np
import torch

from . import mk


def _ptr(t: torch.Tensor) -> int:
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


class Decoder:
    """One decode-step engine bound to a model and its paged KV pools."""

    def __init__(self, shape: Dict, weights: Dict, k_pool: torch.Tensor, v_pool: torch.Tensor,
                 max_batch: int, device: int = 0):
        self.shape = dict(shape)
        self.L = shape["n_layers"]
        self.max_batch = max_batch
        self.n_pages = int(k_pool.shape[1])
        cfg = mk.make_config(shape, max_batch, self.n_pages)
        L = self.L
        keep = []

        def arr(ts):
            a = mk.ptr_array([None if t is None else _ptr(t) for t in ts])
            keep.append(a)
            return a

        t = mk.mk_tensors()
        t.embed = _ptr(weights["embed"])
        t.lm_head = _ptr(weights["lm_head"])
        t.final_norm = _ptr(weights["final_norm"])
        t.attn_norm = arr(weights["attn_norm"])
        t.w_qkv = arr(weights["w_qkv"])
        t.w_o = arr(weights["w_o"])
        t.w_router = arr(weights["w_router"])
        rb = weights.get("router_bias")
        t.router_bias = arr(rb) if rb is not None else None
        t.w_gate = arr(weights["w_gate"])
        t.w_up = arr(weights["w_up"])
        t.w_down = arr(weights["w_down"])
        t.k_pool = arr([k_pool[l] for l in range(L)])
        t.v_pool = arr([v_pool[l] for l in range(L)])
        self._tensors = (weights, k_pool, v_pool)   # keep caller tensors alive
        ctx = c_void_p()
        mk.check_status(mk.lib.mk_create(byref(cfg), byref(t), int(device), byref(ctx)),
                        "mk_create")
        self._ctx = ctx
        self.batch = 0
        self.max_pages = 0

    # ------------------------------------------------------------------
    def build_schedule(self, seq_lens: Sequence[int], max_pages_per_seq: int,
                       plan_len: Optional[Sequence[int]] = None) -> None:
        B = len(seq_lens)
        sl = mk.int32_array(seq_lens)
        pl = mk.int32_array(plan_len) if plan_len is not None else None
        mk.check_status(mk.lib.mk_build_schedule(self._ctx, B, sl, pl, int(max_pages_per_seq)),
                        "mk_build_schedule")
        self.batch = B
        self.max_pages = int(max_pages_per_seq)

    def step(self, tokens: torch.Tensor, positions: torch.Tensor, page_table: torch.Tensor,
             seq_lens: torch.Tensor, logits: torch.Tensor, stream=None,
             unfused: bool = False) -> None:
        for t in (tokens, positions, page_table, seq_lens):
            if t.dtype != torch.int32 or not t.is_cuda:
                raise TypeError("step inputs must be int32 CUDA tensors")
        if logits.dtype != torch.float32 or not logits.is_cuda:
            raise TypeError("logits must be a float32 CUDA tensor")
        if page_table.shape[-1] != self.max_pages:
            raise ValueError("page_table row length differs from the schedule's")
        s = stream if stream is not None else torch.cuda.current_stream()
        fn = mk.lib.mk_decode_step_unfused if unfused else mk.lib.mk_decode_step
        st = fn(self._ctx, _ptr(tokens), _ptr(positions), _ptr(page_table), _ptr(seq_lens),
                _ptr(logits), c_void_p(s.cuda_stream))
        mk.check_status(st, "mk_decode_step")

    def greedy(self, n_steps: int, tokens: torch.Tensor, positions: torch.Tensor,
               page_table: torch.Tensor, seq_lens: torch.Tensor, logits: torch.Tensor,
               out_tokens: torch.Tensor, stream=None) -> None:
        """n_steps greedy steps on the device (mk_decode_greedy): tokens,
        positions and seq_lens are updated in place, out_tokens[i] receives
        step i's tokens.  Asynchronous."""
        for t in (tokens, positions, page_table, seq_lens, out_tokens):
            if t.dtype != torch.int32 or not t.is_cuda:
                raise TypeError("greedy inputs and outputs must be int32 CUDA tensors")
        if logits.dtype != torch.float32 or not logits.is_cuda:
            raise TypeError("logits must be a float32 CUDA tensor")
        if page_table.shape[-1] != self.max_pages:
            raise ValueError("page_table row length differs from the schedule's")
        if out_tokens.numel() < n_steps * self.batch:
            raise ValueError("out_tokens holds fewer than n_steps x batch tokens")
        s = stream if stream is not None else torch.cuda.current_stream()
        st = mk.lib.mk_decode_greedy(self._ctx, int(n_steps), _ptr(tokens), _ptr(positions),
                                     _ptr(page_table), _ptr(seq_lens), _ptr(logits),
                                     _ptr(out_tokens), c_void_p(s.cuda_stream))
        mk.check_status(st, "mk_decode_greedy")

    def check(self):
        """Synchronize and return (status, detail list)."""
        st = c_int32(0)
        detail = (c_int32 * 8)()
        rc = mk.lib.mk_check(self._ctx, byref(st), detail)
        return int(rc), [int(v) for v in detail]

    def check_ok(self) -> None:
        rc, detail = self.check()
        if rc != mk.MK_OK:
            raise mk.MKError(rc, "device status", detail)

    def selftest_timeout(self, timeout_ms: int = 10):
        """Run the failure-detection self-test; returns (status, detail list)."""
        st = c_int32(0)
        detail = (c_int32 * 8)()
        rc = mk.lib.mk_selftest_timeout(self._ctx, int(timeout_ms), byref(st), detail)
        return int(rc), [int(v) for v in detail]

    def set_trace(self, enable: bool) -> None:
        mk.check_status(mk.lib.mk_set_trace(self._ctx, int(bool(enable))), "mk_set_trace")

    def trace(self):
        """(desc [n_tasks][32], trace [n_tasks][18]) of the last traced step."""
        desc = self.debug(mk.MK_BUF_PLAN).reshape(-1, 32)
        stamps = self.debug(mk.MK_BUF_TRACE).reshape(-1, mk.TRACE_WORDS)
        return desc, stamps

    def set_timeout_ms(self, ms: int) -> None:
        mk.check_status(mk.lib.mk_set_timeout_ms(self._ctx, int(ms)), "mk_set_timeout_ms")

    def debug(self, which: int) -> np.ndarray:
        n = mk.lib.mk_debug_size(self._ctx, which)
        if n == 0:
            raise mk.MKError(mk.MK_ERR_STATE, "mk_debug_size")
        ints = (mk.MK_BUF_TOPK, mk.MK_BUF_NSLOTS, mk.MK_BUF_PLAN)
        dtype = np.int32 if which in ints else (np.uint32 if which == mk.MK_BUF_TRACE
                                                else np.float32)
        out = np.empty(n // 4, dtype=dtype)
        mk.check_status(mk.lib.mk_debug_read(self._ctx, which, out.ctypes.data_as(c_void_p), n),
                        "mk_debug_read")
        return out

    def close(self) -> None:
        if getattr(self, "_ctx", None):
            mk.lib.mk_destroy(self._ctx)
            self._ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def plan_schedule(shape: Dict, n_ctas: int, seq_lens: Sequence[int],
                  plan_len: Optional[Sequence[int]] = None, max_batch: int = 8,
                  n_pages: int = 1 << 20):
    """Host-only planner (no GPU): returns (meta, desc [n_tasks][32], targets)."""
    cfg = mk.make_config(shape, max_batch, n_pages)
    B = len(seq_lens)
    sl = mk.int32_array(seq_lens)
    pl = mk.int32_array(plan_len) if plan_len is not None else None
    meta = (c_int32 * 16)()
    mk.check_status(mk.lib.mk_plan_schedule(byref(cfg), n_ctas, B, sl, pl, meta, None, None),
                    "mk_plan_schedule")
    m = [int(v) for v in meta]
    n_tasks, n_counters = m[0], m[1]
    desc = np.zeros((n_tasks, 32), dtype=np.int32)
    targets = np.zeros(n_counters, dtype=np.int32)
    P = ctypes.POINTER(c_int32)
    mk.check_status(mk.lib.mk_plan_schedule(byref(cfg), n_ctas, B, sl, pl, meta,
                                            desc.ctypes.data_as(P), targets.ctypes.data_as(P)),
                    "mk_plan_schedule")
    return m, desc, targets
