"""mk_decode_step_static: the decode step whose scratch sits in a fixed device
array, for callers that must not allocate device memory (a serving process
whose own pool already holds the free memory, or code that cannot afford an
allocation's implicit device synchronization).

Its logits must match mk_decode_step's on the same inputs, call after call
(the array keeps the previous call's contents, so two calls in a row also
check that everything that must start at zero is cleared), and the oracle's;
the device's free memory must not change across the calls; and the 30B-MoE
shape at batch 1 must fit the array.  This file is collected last so that a
run stopping at the first failure has already run every other test.
"""

import gc
from ctypes import c_void_p

import numpy as np
import pytest
import torch

from moe_persistent_cta_b200 import configs, engine, mk, synth
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
        oracle_logits = rig.oracle_step()
        out = torch.full_like(rig.logits, float("nan"))
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        for _ in range(2):
            got = static_step(rig, out)
            err, rel = compare_logits(got, ref)
            assert err <= MAX_ABS and rel <= REL_L2, (err, rel)
            assert np.array_equal(got.argmax(-1), ref.argmax(-1))
            err, rel = compare_logits(got, oracle_logits)
            assert err <= 2e-3 and rel <= REL_L2, (err, rel)
            out.fill_(float("nan"))
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        assert free1 == free0      # the calls allocated nothing
        # the context's own path is unaffected by the calls above
        again = rig.step()
        err, rel = compare_logits(again, ref)
        assert err <= MAX_ABS and rel <= REL_L2, (err, rel)
    finally:
        rig.close()


@pytest.mark.slow
def test_static_scratch_30b_batch1():
    """The 30B-MoE shape at batch 1 with an 8192-token cache fits the fixed
    array: two static steps in a row match mk_decode_step and the oracle's
    48-layer step (expert selection forced only inside the router tie band),
    with no change in free device memory."""
    from tests.test_gpu_30b import Run
    shape = configs.MOE30B
    W = synth.make_weights(shape, 0, "cuda:0", "uniform")
    r = Run(W, [8192])
    try:
        ref = r.logits.cpu().double().numpy()
        out = torch.full_like(r.logits, float("nan"))
        i32 = dict(dtype=torch.int32, device=r.dev)
        tok = torch.tensor(r.tokens, **i32)
        lens = torch.tensor(r.lens, **i32)
        table = r.table.to(r.dev)
        stream = torch.cuda.current_stream()
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        for _ in range(2):
            st = mk.lib.mk_decode_step_static(r.dec._ctx, tok.data_ptr(), lens.data_ptr(),
                                              table.data_ptr(), lens.data_ptr(), out.data_ptr(),
                                              c_void_p(stream.cuda_stream))
            mk.check_status(st, "mk_decode_step_static")
            r.dec.check_ok()
            got = out.cpu().double().numpy()
            err, rel = compare_logits(got, ref)
            assert err <= MAX_ABS and rel <= REL_L2, (err, rel)
            out.fill_(float("nan"))
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        assert free1 == free0
        oracle_logits, forced = r.whole_step(0)
        err, rel = compare_logits(got[0], oracle_logits)
        print(f"30B b1 static step vs oracle: max-abs {err:.3e} rel-L2 {rel:.3e}, forced {forced}")
        assert err <= MAX_ABS and rel <= REL_L2
        assert int(np.argmax(got[0])) == int(np.argmax(oracle_logits))
    finally:
        r.close()
        del W
        gc.collect()
        torch.cuda.empty_cache()


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
