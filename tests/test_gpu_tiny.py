"""GPU parity on the tiny model: the CUDA path vs the CPU oracle, element by
element, through the C ABI (sizes that span several tiles and ragged tails)."""

import numpy as np
import pytest
import torch

import oracle
from moe_persistent_cta_b200 import configs, mk
from tests.gpu_common import (MAX_ABS, REL_L2, TinyRig, compare_logits, router_gap)
from tests.oracle_io import array_kv, oracle_shape

pytestmark = pytest.mark.gpu

# Tighter internal bound than the contract: the hi/lo bf16 split keeps about
# 16 mantissa bits of every matmul input and all accumulation is fp32, so the
# tiny model agrees with the float64 oracle to ~1e-5.
TIGHT = 2e-3


@pytest.fixture(scope="module")
def rig():
    r = TinyRig(configs.TINY, [128], shuffled=False)
    yield r
    r.close()


def test_one_step_logits(rig):
    got = rig.step()
    ref = rig.oracle_step()
    err, rel = compare_logits(got, ref)
    assert err <= MAX_ABS and rel <= REL_L2
    assert err <= TIGHT, f"max_abs {err:.3e}"
    assert np.argmax(got[0]) == np.argmax(ref[0])


def test_intermediates_per_op(rig):
    """Per-operation parity from the step's own buffers: residual entering
    every layer, QKV, attention output, router logits and selection, expert
    activations, weighted expert outputs, O-proj partials."""
    rec = {}
    rig.step()
    rig.oracle_step(record=rec)
    shape = rig.shape
    L, B, d = shape["n_layers"], rig.B, shape["d_model"]
    Hq, Hkv, hd, E, K, F = (shape[x] for x in ("n_q_heads", "n_kv_heads", "head_dim",
                                               "n_experts", "top_k", "d_ff"))
    X = rig.dec.debug(mk.MK_BUF_X).reshape(L + 1, B, d)
    QKV = rig.dec.debug(mk.MK_BUF_QKV).reshape(L, B, -1)
    AO = rig.dec.debug(mk.MK_BUF_ATTN_O).reshape(L, B, Hq, hd)
    RL = rig.dec.debug(mk.MK_BUF_RLOGITS).reshape(L, B, E)
    TK = rig.dec.debug(mk.MK_BUF_TOPK)
    ids = TK[: L * B * K].reshape(L, B, K)
    wts = TK[L * B * K:].view(np.float32).reshape(L, B, K)
    OP = rig.dec.debug(mk.MK_BUF_OPART).reshape(L, Hkv, B, d)
    MO = rig.dec.debug(mk.MK_BUF_MOE).reshape(L, K, B, d)
    for l in range(L):
        r = rec[(l, 0)]
        assert np.allclose(X[l, 0], r["x_in"], atol=1e-4, rtol=1e-4)
        assert np.allclose(QKV[l, 0], r["qkv"], atol=1e-4, rtol=1e-4)
        assert np.allclose(AO[l, 0], r["o"], atol=1e-4, rtol=1e-4)
        assert np.allclose(RL[l, 0], r["router_logits"], atol=1e-4, rtol=1e-4)
        assert list(ids[l, 0]) == list(r["topk_idx"])
        assert np.allclose(wts[l, 0], r["topk_w"], atol=1e-5)
        assert np.allclose(OP[l, :, 0].sum(axis=0), r["attn_out"], atol=1e-4, rtol=1e-4)
        assert np.allclose(MO[l, :, 0].sum(axis=0), r["moe_out"], atol=1e-4, rtol=1e-4)
    assert np.allclose(X[L, 0], rec[(L - 1, 0)]["x_out"], atol=1e-4, rtol=1e-4)


def test_unfused_equals_fused(rig):
    a = rig.step()
    b = rig.step(unfused=True)
    assert np.array_equal(a, b)


def test_deterministic(rig):
    a = rig.step()
    b = rig.step()
    assert np.array_equal(a, b)


def bf16_neighbour(bits, toward_larger):
    """The bf16 bit pattern adjacent to `bits` in value, above or below."""
    b = bits.astype(np.int32)
    neg = (b & 0x8000) != 0
    step = np.where(toward_larger ^ neg, 1, -1)     # magnitude +1 moves away from zero
    return ((b + step) & 0xFFFF).astype(np.uint16)


def test_kv_append_matches_oracle_bits(rig):
    """The appended K and V are bf16 roundings of the projected (and, for K,
    rotated) values: a quantisation, so they must match bit for bit.  Both
    sides round to nearest even, but from different precisions (fp32 on the
    GPU, float64 in the oracle), so where the oracle's value lies within the
    GPU's measured projection error of the midpoint between two bf16 values
    either neighbour is a correct rounding; everywhere else the bits must be
    identical."""
    rec = {}
    rig.step()
    rig.oracle_step(record=rec)
    S = oracle_shape(rig.shape)
    L, hq, hkv, hd = S.n_layers, S.n_q_heads, S.n_kv_heads, S.head_dim
    qkv_gpu = rig.dec.debug(mk.MK_BUF_QKV).reshape(L, rig.B, -1).astype(np.float64)
    pos = rig.lens[0]
    page = int(rig.table[0][pos // 64])
    kd = rig.kd.view(torch.int16).cpu().numpy().view(np.uint16)
    vd = rig.vd.view(torch.int16).cpu().numpy().view(np.uint16)
    cos, sin = oracle.rope_cos_sin(pos, hd, S.rope_theta)
    n_amb = n_all = 0
    for l in range(L):
        r = rec[(l, 0)]
        delta = float(np.max(np.abs(qkv_gpu[l, 0] - r["qkv"])))
        k = r["qkv"][hq * hd:(hq + hkv) * hd].reshape(hkv, hd)
        v = r["qkv"][(hq + hkv) * hd:].reshape(hkv, hd)
        k_rot = oracle.apply_rope(k, cos, sin)
        for ours, ref, x, eps in ((kd[l, page, :, pos % 64, :], r["k_bits"], k_rot, 2 * delta),
                                  (vd[l, page, :, pos % 64, :], r["v_bits"], v, delta)):
            assert np.array_equal(ref, oracle.f64_to_bf16_bits(x))
            vb = oracle.bf16_bits_to_f64(ref)
            other = np.where(x > vb, bf16_neighbour(ref, True), bf16_neighbour(ref, False))
            mid = 0.5 * (vb + oracle.bf16_bits_to_f64(other))
            amb = (np.abs(x - mid) <= eps) & (x != vb)
            exact = ours == ref
            assert np.all(exact | (amb & (ours == other))), (l, int((~exact & ~amb).sum()))
            n_amb += int(amb.sum())
            n_all += x.size
    assert n_amb < 0.05 * n_all      # the band is narrow: almost every value is checked exactly


@pytest.mark.parametrize("lens,shuffled", [([5, 64, 200], True), ([0, 1, 63, 64, 65, 127, 128, 129], True)])
def test_ragged_batch(lens, shuffled):
    rig = TinyRig(configs.TINY, lens, seed=3, shuffled=shuffled)
    try:
        got = rig.step()
        ref = rig.oracle_step()
        err, rel = compare_logits(got, ref)
        assert err <= TIGHT and rel <= REL_L2, (err, rel)
        assert list(np.argmax(got, axis=1)) == list(np.argmax(ref, axis=1))
    finally:
        rig.close()


def test_wide_model_batch8_single_activation_buffer():
    """d_model 2048 at batch 8 leaves room for one activation-A buffer only:
    the first task of each new layer must still be picked up (it frees the
    buffer) before its activation is loaded."""
    shape = dict(configs.TINY, d_model=2048, n_q_heads=16, n_kv_heads=4, head_dim=128,
                 d_ff=768, n_experts=16, top_k=4)
    lens = [3, 64, 65, 130, 200, 17, 90, 127]
    rig = TinyRig(shape, lens, seed=5)
    try:
        got = rig.step()
        ref = rig.oracle_step()
        err, rel = compare_logits(got, ref)
        assert err <= TIGHT and rel <= REL_L2, (err, rel)
        assert list(np.argmax(got, axis=1)) == list(np.argmax(ref, axis=1))
    finally:
        rig.close()


@pytest.mark.parametrize("n_experts,top_k,lens", [(20, 4, [70, 3]), (192, 8, [40, 130, 65]),
                                                  (256, 8, [90])])
def test_router_stage_geometry(n_experts, top_k, lens):
    """The norm tiles stream their router columns in ring stages of 128
    expert rows: one partial stage (20 experts), two stages whose second runs
    past the last expert (192), two full stages (256).  Router logits match
    the oracle; the selection is the top-k of the kernel's own fp32 logits
    (value descending, index ascending) and the oracle's wherever its k-th /
    (k+1)-th gap is clear."""
    shape = dict(configs.TINY, n_experts=n_experts, top_k=top_k)
    rig = TinyRig(shape, lens, seed=7)
    try:
        got = rig.step()
        rec = {}
        ref = rig.oracle_step(record=rec)
        L, B, E, K = shape["n_layers"], rig.B, n_experts, top_k
        RL = rig.dec.debug(mk.MK_BUF_RLOGITS).reshape(L, B, E)
        TK = rig.dec.debug(mk.MK_BUF_TOPK)
        ids = TK[: L * B * K].reshape(L, B, K)
        clear = True
        for l in range(L):
            for b in range(B):
                r = rec[(l, b)]
                assert np.allclose(RL[l, b], r["router_logits"], atol=1e-4, rtol=1e-4), (l, b)
                own = sorted(range(E), key=lambda e: (-RL[l, b, e], e))[:K]
                assert list(ids[l, b]) == own, (l, b)
                if router_gap(r["router_logits"], K) > 1e-3:
                    assert sorted(ids[l, b].tolist()) == sorted(r["topk_idx"].tolist()), (l, b)
                else:
                    clear = False
        if clear:
            err, rel = compare_logits(got, ref)
            assert err <= TIGHT and rel <= REL_L2, (err, rel)
    finally:
        rig.close()


def test_zipf_routing_batch8():
    lens = [100, 200, 300, 400, 500, 600, 700, 800]
    rig = TinyRig(configs.TINY, lens, seed=5, routing="zipf")
    try:
        got = rig.step()
        rec = {}
        ref = rig.oracle_step(record=rec)
        err, rel = compare_logits(got, ref)
        assert err <= TIGHT and rel <= REL_L2, (err, rel)
        nslots = rig.dec.debug(mk.MK_BUF_NSLOTS)
        for l in range(rig.shape["n_layers"]):
            union = set()
            for b in range(len(lens)):
                union |= set(rec[(l, b)]["topk_idx"].tolist())
            assert nslots[l] == len(union)
    finally:
        rig.close()


def test_all_tokens_share_their_experts():
    """Every token of a batch of 8 routes to the same 8 experts (a router bias
    of 30 on a per-layer set of 8 of 64 experts, far above the logits'
    spread): each used slot holds all 8 tokens, the most a slot can hold, so
    the routing compaction places tokens at positions 0..7 and counts 8 per
    slot.  The step matches the oracle and every layer uses exactly 8 slots."""
    from moe_persistent_cta_b200 import synth
    shape = dict(configs.TINY, n_experts=64, top_k=8)
    W = synth.make_weights(shape, 11, "cpu", "uniform")
    gen = torch.Generator().manual_seed(12)
    biased = []
    W["router_bias"] = []
    for _ in range(shape["n_layers"]):
        chosen = torch.randperm(64, generator=gen)[:8]
        b = torch.zeros(64, dtype=torch.float32)
        b[chosen] = 30.0
        W["router_bias"].append(b)
        biased.append(set(chosen.tolist()))
    lens = [100, 200, 300, 400, 500, 600, 700, 800]
    rig = TinyRig(shape, lens, seed=11, weights=W)
    try:
        got = rig.step()
        rec = {}
        ref = rig.oracle_step(record=rec)
        err, rel = compare_logits(got, ref)
        assert err <= TIGHT and rel <= REL_L2, (err, rel)
        L, B, K = shape["n_layers"], len(lens), 8
        nslots = rig.dec.debug(mk.MK_BUF_NSLOTS)
        ids = rig.dec.debug(mk.MK_BUF_TOPK)[: L * B * K].reshape(L, B, K)
        for l in range(L):
            assert nslots[l] == 8, (l, nslots[l])
            for b in range(B):
                assert set(ids[l, b].tolist()) == biased[l], (l, b)
                assert set(rec[(l, b)]["topk_idx"].tolist()) == biased[l], (l, b)
    finally:
        rig.close()


def test_greedy_16_steps():
    """16 greedy steps: identical tokens, logits within tolerance each step,
    the GPU appending K/V into its own pool and the oracle into its copy."""
    rig = TinyRig(configs.TINY, [128], shuffled=False)
    try:
        kv = array_kv(rig.k, rig.v)
        import oracle as orc
        from tests.oracle_io import array_weights, oracle_shape
        ref_logits, fed = orc.greedy_decode(oracle_shape(rig.shape), array_weights(rig.W), kv,
                                            rig.tokens, rig.lens, rig.table.numpy(), 16)
        toks = list(rig.tokens)
        lens = list(rig.lens)
        for s in range(16):
            got = rig.step(toks, lens)
            assert toks == fed[s], f"step {s}: fed {toks} vs oracle {fed[s]}"
            err, rel = compare_logits(got, ref_logits[s])
            assert err <= TIGHT and rel <= REL_L2, (s, err, rel)
            toks = [int(np.argmax(got[b])) for b in range(rig.B)]
            lens = [x + 1 for x in lens]
    finally:
        rig.close()


def test_schedule_outgrown_is_reported():
    """A step at a length beyond the schedule's attention plan must latch
    MK_ERR_STATE on the device (no hang, context still usable)."""
    rig = TinyRig(configs.TINY, [100], shuffled=False, growth=256)
    try:
        rig.dec.build_schedule([100], rig.table.shape[1], plan_len=[100])
        rig.dec.step(rig.i32(rig.tokens), rig.i32([300]), rig.table.to(rig.dev),
                     rig.i32([300]), rig.logits)
        rc, detail = rig.dec.check()
        assert rc == mk.MK_ERR_STATE, (rc, detail)
        # the context recovers: a valid step right after passes
        rig.dec.build_schedule([100], rig.table.shape[1])
        got = rig.step(lens=[100])
        ref = rig.oracle_step(lens=[100])
        assert compare_logits(got, ref)[0] <= TIGHT
    finally:
        rig.close()
