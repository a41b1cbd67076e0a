"""mk_decode_step_static: the decode step whose scratch sits in a fixed device
array, for callers that must not allocate device memory (a serving process
whose own pool already holds the free memory, or code that cannot afford an
allocation's implicit device synchronization).

Its logits must match mk_decode_step's on the same inputs, call after call:
the array keeps the previous call's contents, so two calls in a row also
check that everything that must start at zero is cleared.  This file is
collected last so that a run stopping at the first failure has already run
every other test.
"""

from ctypes import c_void_p

import numpy as np
import pytest
import torch

from moe_persistent_cta_b200 import configs, engine, mk
from tests.gpu_common import MAX_ABS, REL_L2, TinyRig, compare_logits

pytestmark = pytest.mark.gpu


def static_step(rig, logits):
    dev = rig.dev
    tok = rig.i32(rig.tokens)
    lens = rig.i32(rig.lens)
    table = rig.table.to(dev)
    stream = torch.cuda.current_stream()
    st = mk.lib.mk_decode_step_static(rig.dec._ctx, tok.data_ptr(), lens.data_ptr(),
                                      table.data_ptr(), lens.data_ptr(), logits.data_ptr(),
                                      c_void_p(stream.cuda_stream))
    mk.check_status(st, "mk_decode_step_static")
    rig.dec.check_ok()
    return logits.cpu().double().numpy()


@pytest.mark.parametrize("lens", [[128], [5, 70, 200]])
def test_static_scratch_step_matches_decode_step(lens):
    rig = TinyRig(configs.TINY, lens, seed=0)
    try:
        ref = rig.step()
        out = torch.full_like(rig.logits, float("nan"))
        for _ in range(2):
            got = static_step(rig, out)
            err, rel = compare_logits(got, ref)
            assert err <= MAX_ABS and rel <= REL_L2, (err, rel)
            assert np.array_equal(got.argmax(-1), ref.argmax(-1))
            out.fill_(float("nan"))
        # the context's own path is unaffected by the calls above
        again = rig.step()
        err, rel = compare_logits(again, ref)
        assert err <= MAX_ABS and rel <= REL_L2, (err, rel)
    finally:
        rig.close()


def test_static_scratch_rejects_oversized_schedules():
    """12 layers, 64 experts top-8, d_ff 768 at batch 8 needs about 38 MiB of
    step scratch (the expert activations alone take 12 x 64 x 8 x 768 x 4 B
    twice over), more than the array's 32 MiB: refused before any launch."""
    shape = dict(configs.TINY, n_layers=12, n_experts=64, top_k=8, d_ff=768)
    L, d, E, F, V = shape["n_layers"], shape["d_model"], 64, 768, shape["vocab"]
    hd, Hq, Hkv = shape["head_dim"], shape["n_q_heads"], shape["n_kv_heads"]
    dev = torch.device("cuda:0")
    bf = dict(dtype=torch.bfloat16, device=dev)
    W = {
        "embed": torch.zeros(V, d, **bf), "lm_head": torch.zeros(V, d, **bf),
        "final_norm": torch.ones(d, **bf),
        "attn_norm": [torch.ones(d, **bf) for _ in range(L)],
        "w_qkv": [torch.zeros((Hq + 2 * Hkv) * hd, d, **bf) for _ in range(L)],
        "w_o": [torch.zeros(d, Hq * hd, **bf) for _ in range(L)],
        "w_router": [torch.zeros(E, d, **bf) for _ in range(L)],
        "router_bias": None,
        "w_gate": [torch.empty(E, F, d, **bf) for _ in range(L)],
        "w_up": [torch.empty(E, F, d, **bf) for _ in range(L)],
        "w_down": [torch.empty(E, d, F, **bf) for _ in range(L)],
    }
    n_pages = 8 * 4
    kp = torch.zeros(L, n_pages, Hkv, 64, hd, **bf)
    vp = torch.zeros(L, n_pages, Hkv, 64, hd, **bf)
    dec = engine.Decoder(shape, W, kp, vp, max_batch=8)
    try:
        dec.build_schedule([100] * 8, 4)
        i32 = dict(dtype=torch.int32, device=dev)
        tok = torch.zeros(8, **i32)
        lens = torch.full((8,), 100, **i32)
        table = torch.arange(n_pages, **i32).reshape(8, 4)
        logits = torch.empty(8, V, dtype=torch.float32, device=dev)
        st = mk.lib.mk_decode_step_static(dec._ctx, tok.data_ptr(), lens.data_ptr(),
                                          table.data_ptr(), lens.data_ptr(), logits.data_ptr(),
                                          c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == mk.MK_ERR_CAPACITY
        assert dec.check()[0] == mk.MK_OK
    finally:
        dec.close()
