"""Thin ctypes binding of the C ABI declared in ``include/mk.h``.

Argument marshalling only: every step of the decode path runs in the native
library's kernels.  Importing this module fails loudly when ``libmk.so`` is
missing; there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int, c_int32, c_size_t, c_void_p

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmk.so")

MK_OK, MK_ERR_INVALID, MK_ERR_CUDA, MK_ERR_OOM, MK_ERR_TIMEOUT = 0, 1, 2, 3, 4
MK_ERR_CAPACITY, MK_ERR_STATE, MK_ERR_DEVICE = 5, 6, 7

MK_BUF_X, MK_BUF_QKV, MK_BUF_ATTN_O, MK_BUF_RLOGITS, MK_BUF_TOPK = 0, 1, 2, 3, 4
MK_BUF_NSLOTS, MK_BUF_EXPERT_A, MK_BUF_MOE, MK_BUF_OPART = 5, 6, 7, 8
MK_BUF_TRACE, MK_BUF_PLAN = 9, 10
MK_STATIC_SCRATCH_MAX_BYTES = 32 * 1024 * 1024
TRACE_WORDS = 18

# every entry point the header declares (checked by the ABI test)
EXPORTS = (
    "mk_create", "mk_build_schedule", "mk_decode_step", "mk_decode_greedy",
    "mk_decode_step_unfused", "mk_decode_step_static",
    "mk_check", "mk_selftest_timeout", "mk_set_timeout_ms", "mk_set_trace", "mk_debug_read",
    "mk_debug_size",
    "mk_plan_schedule", "mk_strerror", "mk_destroy",
)


class MKError(RuntimeError):
    def __init__(self, status: int, what: str, detail=None):
        self.status = status
        self.detail = detail
        msg = f"{what}: {strerror(status)} ({status})"
        if detail is not None:
            msg += f" detail={list(detail)}"
        super().__init__(msg)


class mk_config(ctypes.Structure):
    _fields_ = [
        ("n_layers", c_int32), ("d_model", c_int32), ("n_q_heads", c_int32),
        ("n_kv_heads", c_int32), ("head_dim", c_int32), ("n_experts", c_int32),
        ("top_k", c_int32), ("d_ff", c_int32), ("vocab", c_int32), ("page_size", c_int32),
        ("max_batch", c_int32), ("n_pages", c_int32), ("rope_theta", c_float),
        ("rms_eps", c_float),
    ]


class mk_tensors(ctypes.Structure):
    _fields_ = [
        ("embed", c_void_p), ("lm_head", c_void_p), ("final_norm", c_void_p),
        ("attn_norm", POINTER(c_void_p)), ("w_qkv", POINTER(c_void_p)),
        ("w_o", POINTER(c_void_p)), ("w_router", POINTER(c_void_p)),
        ("router_bias", POINTER(c_void_p)), ("w_gate", POINTER(c_void_p)),
        ("w_up", POINTER(c_void_p)), ("w_down", POINTER(c_void_p)),
        ("k_pool", POINTER(c_void_p)), ("v_pool", POINTER(c_void_p)),
    ]


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"native library {_LIB_PATH} is missing: build it with "
            "`python -m moe_persistent_cta_b200.build` (there is no fallback path)")
    lib = ctypes.CDLL(_LIB_PATH)
    P = POINTER
    sig = {
        "mk_create": (c_int, [P(mk_config), P(mk_tensors), c_int, P(c_void_p)]),
        "mk_build_schedule": (c_int, [c_void_p, c_int, P(c_int32), P(c_int32), c_int32]),
        "mk_decode_step": (c_int, [c_void_p] + [c_void_p] * 5 + [c_void_p]),
        "mk_decode_greedy": (c_int, [c_void_p, c_int32] + [c_void_p] * 7),
        "mk_decode_step_unfused": (c_int, [c_void_p] + [c_void_p] * 5 + [c_void_p]),
        "mk_decode_step_static": (c_int, [c_void_p] + [c_void_p] * 5 + [c_void_p]),
        "mk_check": (c_int, [c_void_p, P(c_int32), P(c_int32)]),
        "mk_selftest_timeout": (c_int, [c_void_p, c_int32, P(c_int32), P(c_int32)]),
        "mk_set_timeout_ms": (c_int, [c_void_p, c_int32]),
        "mk_set_trace": (c_int, [c_void_p, c_int32]),
        "mk_debug_read": (c_int, [c_void_p, c_int, c_void_p, c_size_t]),
        "mk_debug_size": (c_size_t, [c_void_p, c_int]),
        "mk_plan_schedule": (c_int, [P(mk_config), c_int, c_int, P(c_int32), P(c_int32),
                                     P(c_int32), P(c_int32), P(c_int32)]),
        "mk_strerror": (c_char_p, [c_int]),
        "mk_destroy": (None, [c_void_p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def strerror(status: int) -> str:
    return lib.mk_strerror(int(status)).decode()


def check_status(status: int, what: str) -> None:
    if status != MK_OK:
        raise MKError(status, what)


def make_config(shape: dict, max_batch: int, n_pages: int) -> mk_config:
    return mk_config(
        shape["n_layers"], shape["d_model"], shape["n_q_heads"], shape["n_kv_heads"],
        shape["head_dim"], shape["n_experts"], shape["top_k"], shape["d_ff"], shape["vocab"],
        shape.get("page_size", 64), max_batch, n_pages, shape.get("rope_theta", 1.0e4),
        shape.get("rms_eps", 1.0e-6))


def int32_array(values):
    arr = (c_int32 * len(values))(*[int(v) for v in values])
    return arr


def ptr_array(ptrs):
    return (c_void_p * len(ptrs))(*[None if p is None else int(p) for p in ptrs])
