"""Failure detection on the GPU without a fault: a wait that can never be
met runs out its deadline, the kernel reports MK_ERR_TIMEOUT through the
status word, and the context (and the GPU) keep working afterwards."""

import numpy as np
import pytest

from moe_persistent_cta_b200 import configs, mk
from tests.gpu_common import TinyRig

pytestmark = pytest.mark.gpu


def test_unsatisfiable_wait_times_out_and_the_step_still_runs():
    rig = TinyRig(configs.TINY, [128])
    try:
        ref = rig.step()
        rc, detail = rig.dec.selftest_timeout(10)
        assert rc == mk.MK_ERR_TIMEOUT
        assert detail[0] == mk.MK_ERR_TIMEOUT
        assert 0 <= detail[1] < 148           # the CTA that saw the deadline pass
        # status was cleared; the step's counters and outputs were untouched
        rc2, _ = rig.dec.check()
        assert rc2 == mk.MK_OK
        for _ in range(2):
            got = rig.step()
            assert np.array_equal(got, ref)
    finally:
        rig.close()


def test_selftest_needs_a_schedule():
    import torch
    from moe_persistent_cta_b200 import engine, synth
    shape = configs.TINY
    W = synth.make_weights(shape, 0, "cuda")
    k, v = synth.make_kv(shape, 4, 1, "cuda")
    dec = engine.Decoder(shape, W, k, v, max_batch=1)
    try:
        rc, _ = dec.selftest_timeout(10)
        assert rc == mk.MK_ERR_STATE
    finally:
        dec.close()
        del W, k, v
        torch.cuda.synchronize()
