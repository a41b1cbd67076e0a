"""Pins of the CPU oracle to things other than itself.

Each test checks one oracle function against a library routine, a closed
form, an invariant of the mathematics, or brute force, chosen so that a
plausible slip (a dropped term, a wrong sign or index, a transposed operand,
sequential instead of parallel branches) fails at least one of them.  The last
tests plant such slips in the oracle (on the CPU) and check that the
composition pin catches them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import decoder as od
from moe_persistent_cta_b200 import configs, roofline, synth
from tests.oracle_io import array_kv, array_weights, oracle_shape

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ bf16 ---
def test_bf16_round_matches_library_on_float32_inputs():
    rng = np.random.default_rng(0)
    x32 = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    # exact ties: bf16 value + half an ulp (even and odd mantissas)
    base = torch.randn(2000).to(torch.bfloat16)
    bits = base.view(torch.int16).numpy().view(np.uint16).astype(np.uint32) << 16
    ties = (bits + (1 << 15)).view(np.float32)
    x = np.concatenate([x32, ties])
    ours = oracle.f64_to_bf16_bits(x.astype(np.float64))
    lib = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, lib)


def test_bf16_widening_is_exact():
    t = torch.randn(5000).to(torch.bfloat16)
    ours = oracle.bf16_bits_to_f64(t.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(ours, t.to(torch.float64).numpy())


# --------------------------------------------------------------- RMSNorm ---
def test_rmsnorm_library_and_closed_form():
    rng = np.random.default_rng(1)
    h = rng.standard_normal(256)
    g = rng.uniform(0.5, 1.5, 256)
    lib = F.rms_norm(torch.from_numpy(h), (256,), weight=torch.from_numpy(g), eps=1e-6).numpy()
    assert np.allclose(oracle.rms_norm(h, g, 1e-6), lib, rtol=1e-13, atol=1e-13)
    c = -3.0
    out = oracle.rms_norm(np.full(64, c), np.ones(64), 1e-6)
    assert np.allclose(out, c / math.sqrt(c * c + 1e-6))
    # scale invariance (eps -> 0)
    assert np.allclose(oracle.rms_norm(7.5 * h, g, 0.0), oracle.rms_norm(h, g, 0.0))


# ------------------------------------------------------------------ RoPE ---
def test_rope_identity_norm_and_relative_position():
    rng = np.random.default_rng(2)
    hd = 128
    q, k = rng.standard_normal(hd), rng.standard_normal(hd)
    c0, s0 = oracle.rope_cos_sin(0, hd, 1e4)
    assert np.allclose(oracle.apply_rope(q, c0, s0), q)
    for pos in (1, 17, 8192, 262144):
        c, s = oracle.rope_cos_sin(pos, hd, 1e4)
        r = oracle.apply_rope(q, c, s)
        half = hd // 2
        # each rotated pair keeps its length
        assert np.allclose(r[:half] ** 2 + r[half:] ** 2, q[:half] ** 2 + q[half:] ** 2)
    # q(m).k(n) depends on m - n only
    def dot(m, n):
        cm, sm = oracle.rope_cos_sin(m, hd, 1e4)
        cn, sn = oracle.rope_cos_sin(n, hd, 1e4)
        return oracle.apply_rope(q, cm, sm) @ oracle.apply_rope(k, cn, sn)
    assert np.isclose(dot(10, 3), dot(1007, 1000))
    assert np.isclose(dot(5, 9), dot(105, 109))


def test_rope_matches_complex_rotation():
    """Rotate-half RoPE == multiplying z_i = x_i + i x_{i+hd/2} by e^{i pos w_i}."""
    rng = np.random.default_rng(3)
    hd, pos, theta = 64, 12345, 1e4
    x = rng.standard_normal(hd)
    w = theta ** (-np.arange(0, hd, 2) / hd)
    z = (x[: hd // 2] + 1j * x[hd // 2:]) * np.exp(1j * pos * w)
    c, s = oracle.rope_cos_sin(pos, hd, theta)
    r = oracle.apply_rope(x, c, s)
    assert np.allclose(r, np.concatenate([z.real, z.imag]))


# ------------------------------------------------------------- attention ---
def test_gqa_attention_matches_sdpa():
    rng = np.random.default_rng(4)
    Hq, Hkv, hd, T = 8, 2, 64, 37
    q = rng.standard_normal((Hq, hd))
    K = rng.standard_normal((T, Hkv, hd))
    V = rng.standard_normal((T, Hkv, hd))
    ours = oracle.gqa_decode_attention(q, K, V)
    tq = torch.from_numpy(q)[None, :, None, :]                     # [1, Hq, 1, hd]
    tk = torch.from_numpy(K).permute(1, 0, 2)[None]                # [1, Hkv, T, hd]
    tv = torch.from_numpy(V).permute(1, 0, 2)[None]
    lib = F.scaled_dot_product_attention(tq, tk, tv, enable_gqa=True)[0, :, 0, :]
    assert np.allclose(ours, lib.numpy(), rtol=1e-12, atol=1e-12)


def test_attention_single_key_and_uniform_keys():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((4, 32))
    K1 = rng.standard_normal((1, 2, 32))
    V1 = rng.standard_normal((1, 2, 32))
    o = oracle.gqa_decode_attention(q, K1, V1)
    assert np.allclose(o[0], V1[0, 0]) and np.allclose(o[3], V1[0, 1])
    K = np.repeat(rng.standard_normal((1, 2, 32)), 9, axis=0)
    V = rng.standard_normal((9, 2, 32))
    o = oracle.gqa_decode_attention(q, K, V)
    assert np.allclose(o[1], V[:, 0].mean(axis=0)) and np.allclose(o[2], V[:, 1].mean(axis=0))


def test_paged_gather_equals_contiguous():
    rng = np.random.default_rng(6)
    P, Hkv, S, hd = 12, 2, 64, 16
    seq = rng.standard_normal((P * S, Hkv, hd)).astype(np.float32)
    seq_bits = oracle.f64_to_bf16_bits(seq.astype(np.float64))
    perm = rng.permutation(P)
    pool = np.zeros((P, Hkv, S, hd), dtype=np.uint16)
    for lp in range(P):
        pool[perm[lp]] = seq_bits[lp * S:(lp + 1) * S].transpose(1, 0, 2)
    kv = oracle.ArrayKV([pool], [pool])
    for n in (1, 63, 64, 65, 700):
        got = oracle.gather_paged(kv, 0, "k", perm, n, S)
        assert np.array_equal(got, oracle.bf16_bits_to_f64(seq_bits[:n]))


# ---------------------------------------------------------------- router ---
def test_router_topk_equals_full_sort():
    rng = np.random.default_rng(7)
    for trial in range(200):
        E, k = 16, 4
        r = rng.integers(-3, 4, E).astype(np.float64) if trial % 2 else rng.standard_normal(E)
        idx, w = oracle.router_select(r, k)
        order = np.lexsort((np.arange(E), -r))          # value desc, then index asc
        assert np.array_equal(idx, order[:k])
        assert np.isclose(w.sum(), 1.0)
        ref = torch.softmax(torch.from_numpy(r[order[:k]]), dim=0).numpy()
        assert np.allclose(w, ref)
        idx2, w2 = oracle.router_select(r + 5.0, k)    # shift invariance
        assert np.array_equal(idx, idx2) and np.allclose(w, w2)


# ------------------------------------------------------------------- MoE ---
def _tiny(**over):
    shape = dict(configs.TINY, **over)
    return shape


def test_identical_experts_reduce_to_dense_mlp():
    shape = _tiny()
    W = synth.make_weights(shape, seed=11)
    for k in ("w_gate", "w_up", "w_down"):
        W[k] = [x[:1].repeat(x.shape[0], *([1] * (x.dim() - 1))) for x in W[k]]
    AW = array_weights(W)
    S = oracle_shape(dict(shape, top_k=shape["n_experts"]))
    n = np.random.default_rng(8).standard_normal(shape["d_model"])
    ours = oracle.moe_branch(S, AW, 0, n)
    g = W["w_gate"][0][0].double()
    u = W["w_up"][0][0].double()
    d = W["w_down"][0][0].double()
    tn = torch.from_numpy(n)
    lib = d @ (F.silu(g @ tn) * (u @ tn))
    assert np.allclose(ours, lib.numpy(), rtol=1e-10, atol=1e-12)


def test_one_hot_router_selects_that_expert():
    shape = _tiny(top_k=1)
    W = synth.make_weights(shape, seed=12)
    E = shape["n_experts"]
    W["router_bias"] = [torch.full((E,), -100.0) for _ in range(shape["n_layers"])]
    for l in range(shape["n_layers"]):
        W["router_bias"][l][5] = 100.0
    AW = array_weights(W)
    n = np.random.default_rng(9).standard_normal(shape["d_model"])
    rec = {}
    out = oracle.moe_branch(oracle_shape(shape), AW, 1, n, rec=rec)
    assert list(rec["topk_idx"]) == [5] and np.isclose(rec["topk_w"][0], 1.0)
    g, u, d = (W[k][1][5].double() for k in ("w_gate", "w_up", "w_down"))
    tn = torch.from_numpy(n)
    assert np.allclose(out, (d @ (F.silu(g @ tn) * (u @ tn))).numpy())


# ---------------------------------------------------------- whole model ---
def _tiny_case(seed=0, lens=(128,), shuffled=False):
    shape = configs.TINY
    W = synth.make_weights(shape, seed=seed)
    table, n_pages = synth.make_page_tables(list(lens), not shuffled, seed + 3)
    k, v = synth.make_kv(shape, n_pages, seed + 1)
    toks = synth.make_tokens(len(lens), shape["vocab"], seed + 2)
    return shape, W, k, v, table, toks, list(lens)


def torch_reference_step(shape, W, k, v, table, toks, lens):
    """Independent float64 restatement with torch library routines
    (rms_norm, scaled_dot_product_attention with GQA, topk, silu, complex
    rotation), batched instead of looped."""
    L, d, Hq, Hkv, hd = (shape[x] for x in ("n_layers", "d_model", "n_q_heads", "n_kv_heads",
                                             "head_dim"))
    E, K, eps, theta = shape["n_experts"], shape["top_k"], shape["rms_eps"], shape["rope_theta"]
    out = []
    for b, tok in enumerate(toks):
        pos = lens[b]
        x = W["embed"][tok].double()
        inv = theta ** (-torch.arange(0, hd, 2, dtype=torch.float64) / hd)
        rot = torch.polar(torch.ones(hd // 2, dtype=torch.float64), pos * inv)
        t = torch.arange(pos)
        pages = table[b][t // 64].long()
        for l in range(L):
            n = F.rms_norm(x, (d,), weight=W["attn_norm"][l].double(), eps=eps)
            qkv = W["w_qkv"][l].double() @ n
            q = qkv[: Hq * hd].view(Hq, hd)
            kk = qkv[Hq * hd:(Hq + Hkv) * hd].view(Hkv, hd)
            vv = qkv[(Hq + Hkv) * hd:].view(Hkv, hd)

            def rope(z):
                c = torch.complex(z[:, : hd // 2], z[:, hd // 2:]) * rot
                return torch.cat([c.real, c.imag], dim=1)

            q, kk = rope(q), rope(kk)
            kk = kk.float().to(torch.bfloat16).double()
            vv = vv.float().to(torch.bfloat16).double()
            Kc = k[l][pages, :, t % 64, :].double()              # [T, Hkv, hd]
            Vc = v[l][pages, :, t % 64, :].double()
            Ks = torch.cat([Kc, kk[None]], 0).permute(1, 0, 2)[None]
            Vs = torch.cat([Vc, vv[None]], 0).permute(1, 0, 2)[None]
            o = F.scaled_dot_product_attention(q[None, :, None, :], Ks, Vs, enable_gqa=True)
            attn = W["w_o"][l].double() @ o[0, :, 0, :].reshape(-1)
            r = W["w_router"][l].double() @ n
            if W.get("router_bias") is not None:
                r = r + W["router_bias"][l].double()
            top = torch.topk(r, K)
            wts = torch.softmax(top.values, 0)
            moe = torch.zeros(d, dtype=torch.float64)
            for j in range(K):
                e = int(top.indices[j])
                g = W["w_gate"][l][e].double() @ n
                u = W["w_up"][l][e].double() @ n
                moe += wts[j] * (W["w_down"][l][e].double() @ (F.silu(g) * u))
            x = x + attn + moe
        xf = F.rms_norm(x, (d,), weight=W["final_norm"].double(), eps=eps)
        out.append((W["lm_head"].double() @ xf).numpy())
    return np.stack(out)


@pytest.mark.parametrize("lens,shuffled", [((128,), False), ((5, 64, 200), True), ((0,), False)])
def test_tiny_step_matches_library_restatement(lens, shuffled):
    shape, W, k, v, table, toks, lens = _tiny_case(lens=lens, shuffled=shuffled)
    got = oracle.decode_step(oracle_shape(shape), array_weights(W), array_kv(k, v), toks, lens,
                             table.numpy())
    ref = torch_reference_step(shape, W, k, v, table, toks, lens)
    assert np.allclose(got, ref, rtol=1e-9, atol=1e-9)


def torch_reference_prefill(shape, W, k, v, row, prefix, prompt):
    """Causal prefill of `prompt` after `prefix` cached tokens, restated in
    batched form with torch library routines: all prompt tokens projected at
    once, RoPE at each token's own position, and one masked
    scaled_dot_product_attention in which token i sees the prefix and prompt
    tokens 0 .. i.  Returns float64 logits [M][V]."""
    L, d, Hq, Hkv, hd = (shape[x] for x in ("n_layers", "d_model", "n_q_heads", "n_kv_heads",
                                             "head_dim"))
    K, eps, theta = shape["top_k"], shape["rms_eps"], shape["rope_theta"]
    M = len(prompt)
    x = W["embed"][torch.tensor(prompt)].double()                       # [M, d]
    pos = torch.arange(prefix, prefix + M, dtype=torch.float64)
    inv = theta ** (-torch.arange(0, hd, 2, dtype=torch.float64) / hd)
    rot = torch.polar(torch.ones(M, hd // 2, dtype=torch.float64), pos[:, None] * inv[None])
    t = torch.arange(prefix)
    pages = row[t // 64].long()
    allowed = torch.ones(M, prefix + M, dtype=torch.bool)
    allowed[:, prefix:] = torch.tril(torch.ones(M, M, dtype=torch.bool))

    def rope(z):                                                         # [M, H, hd]
        c = torch.complex(z[..., : hd // 2], z[..., hd // 2:]) * rot[:, None, :]
        return torch.cat([c.real, c.imag], dim=-1)

    for l in range(L):
        n = F.rms_norm(x, (d,), weight=W["attn_norm"][l].double(), eps=eps)
        qkv = n @ W["w_qkv"][l].double().T
        q = rope(qkv[:, : Hq * hd].view(M, Hq, hd))
        kk = rope(qkv[:, Hq * hd:(Hq + Hkv) * hd].view(M, Hkv, hd))
        vv = qkv[:, (Hq + Hkv) * hd:].view(M, Hkv, hd)
        kk = kk.float().to(torch.bfloat16).double()
        vv = vv.float().to(torch.bfloat16).double()
        Ks = torch.cat([k[l][pages, :, t % 64, :].double(), kk], 0).permute(1, 0, 2)[None]
        Vs = torch.cat([v[l][pages, :, t % 64, :].double(), vv], 0).permute(1, 0, 2)[None]
        o = F.scaled_dot_product_attention(q.permute(1, 0, 2)[None], Ks, Vs,
                                           attn_mask=allowed, enable_gqa=True)
        attn = o[0].permute(1, 0, 2).reshape(M, Hq * hd) @ W["w_o"][l].double().T
        r = n @ W["w_router"][l].double().T
        if W.get("router_bias") is not None:
            r = r + W["router_bias"][l].double()
        top = torch.topk(r, K, dim=1)
        wts = torch.softmax(top.values, 1)
        moe = torch.zeros(M, d, dtype=torch.float64)
        for i in range(M):
            for j in range(K):
                e = int(top.indices[i, j])
                g = W["w_gate"][l][e].double() @ n[i]
                u = W["w_up"][l][e].double() @ n[i]
                moe[i] += wts[i, j] * (W["w_down"][l][e].double() @ (F.silu(g) * u))
        x = x + attn + moe
    xf = F.rms_norm(x, (d,), weight=W["final_norm"].double(), eps=eps)
    return (xf @ W["lm_head"].double().T).numpy()


@pytest.mark.parametrize("prefix,m", [(0, 4), (61, 5), (128, 3)])
def test_sequential_decode_is_causal_prefill(prefix, m):
    """The prefill definition the GPU's prefill groups are checked against:
    M decode steps in a row, each appending its token's K/V, give the logits
    of a causal prefill of the M tokens written in batched form."""
    shape, W, k, v, table, toks, lens = _tiny_case(lens=(prefix,), shuffled=True)
    prompt = [int(x) for x in synth.make_tokens(m, shape["vocab"], 21)]
    S, AW, KV = oracle_shape(shape), array_weights(W), array_kv(k, v)
    row = table[0].numpy()
    got = np.stack([oracle.decode_step(S, AW, KV, [prompt[j]], [prefix + j], [row],
                                       append=True)[0] for j in range(m)])
    ref = torch_reference_prefill(shape, W, k, v, table[0], prefix, prompt)
    assert np.allclose(got, ref, rtol=1e-9, atol=1e-9)


def test_layer_is_sum_of_branches():
    shape, W, k, v, table, toks, lens = _tiny_case()
    S, AW, KV = oracle_shape(shape), array_weights(W), array_kv(k, v)
    x = np.random.default_rng(10).standard_normal(shape["d_model"])
    both, _, _ = oracle.parallel_layer(S, AW, KV, 0, x, lens[0], table[0].numpy(), lens[0])
    a, _, _ = oracle.parallel_layer(S, AW, KV, 0, x, lens[0], table[0].numpy(), lens[0],
                                    branches=(True, False))
    m, _, _ = oracle.parallel_layer(S, AW, KV, 0, x, lens[0], table[0].numpy(), lens[0],
                                    branches=(False, True))
    assert np.allclose(both - x, (a - x) + (m - x), rtol=1e-12, atol=1e-12)


def test_zero_branches_closed_form():
    """With W_o = 0 and every expert's down projection 0 the residual stream
    never changes: logits = W_lm . RMSNorm(embed[token])."""
    shape, W, k, v, table, toks, lens = _tiny_case()
    W["w_o"] = [torch.zeros_like(t) for t in W["w_o"]]
    W["w_down"] = [torch.zeros_like(t) for t in W["w_down"]]
    got = oracle.decode_step(oracle_shape(shape), array_weights(W), array_kv(k, v), toks, lens,
                             table.numpy())
    e = W["embed"][toks[0]].double()
    ref = W["lm_head"].double() @ F.rms_norm(e, (shape["d_model"],), eps=shape["rms_eps"])
    assert np.allclose(got[0], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_greedy_appends_the_step_kv():
    shape, W, k, v, table, toks, lens = _tiny_case()
    S, AW = oracle_shape(shape), array_weights(W)
    KV = array_kv(k, v)
    rec = {}
    oracle.decode_step(S, AW, array_kv(k, v), toks, lens, table.numpy(), record=rec)
    logits, fed = oracle.greedy_decode(S, AW, KV, toks, lens, table.numpy(), 3)
    pos = lens[0]
    page = int(table[0][pos // 64])
    for l in range(shape["n_layers"]):
        assert np.array_equal(KV.k[l][page, :, pos % 64, :], rec[(l, 0)]["k_bits"])
        assert np.array_equal(KV.v[l][page, :, pos % 64, :], rec[(l, 0)]["v_bits"])
    assert fed[1][0] == int(np.argmax(logits[0][0]))
    again, _ = oracle.greedy_decode(S, AW, array_kv(k, v), toks, lens, table.numpy(), 3)
    assert np.array_equal(logits, again)


# ------------------------------------------- planted mistakes are caught ---
def _composition_close(monkeypatch, target, replacement):
    shape, W, k, v, table, toks, lens = _tiny_case(lens=(70,), shuffled=True)
    monkeypatch.setattr(od, target, replacement)
    got = od.decode_step(oracle_shape(shape), array_weights(W), array_kv(k, v), toks, lens,
                         table.numpy())
    ref = torch_reference_step(shape, W, k, v, table, toks, lens)
    return np.allclose(got, ref, rtol=1e-6, atol=1e-6)


def test_planted_rope_sign_error_is_caught(monkeypatch):
    def bad_rope(x, cos, sin):
        half = x.shape[-1] // 2
        x1, x2 = x[..., :half], x[..., half:]
        return np.concatenate([x1 * cos + x2 * sin, x2 * cos - x1 * sin], axis=-1)
    assert not _composition_close(monkeypatch, "apply_rope", bad_rope)


def test_planted_gqa_mapping_error_is_caught(monkeypatch):
    def bad_attn(q, keys, values):
        hq, hd = q.shape
        hkv = keys.shape[1]
        o = np.zeros((hq, hd))
        for h in range(hq):
            g = h % hkv                               # interleaved instead of grouped
            s = keys[:, g, :] @ q[h] / np.sqrt(hd)
            p = np.exp(s - s.max())
            o[h] = (p / p.sum()) @ values[:, g, :]
        return o
    assert not _composition_close(monkeypatch, "gqa_decode_attention", bad_attn)


def test_planted_router_weighting_error_is_caught(monkeypatch):
    orig = od.router_select

    def bad_select(r, k, forced=None):
        idx, w = orig(r, k, forced)
        return idx, np.full_like(w, 1.0 / len(w))    # drops the softmax
    assert not _composition_close(monkeypatch, "router_select", bad_select)


def test_planted_norm_error_is_caught(monkeypatch):
    def bad_norm(h, gamma, eps):
        return h / np.sqrt(np.sum(h * h) + eps) * gamma   # sum instead of mean
    assert not _composition_close(monkeypatch, "rms_norm", bad_norm)


# --------------------------------------------------------------- roofline ---
def test_roofline_reproduces_pages_figures():
    g = json.load(open(os.path.join(GOLDEN, "sol_pages.json")))
    sol = roofline.sol_tok_s(g["hbm_bytes_per_s"], g["weight_bytes"] + g["kv_bytes_8k"])
    assert abs(sol - g["sol_tok_s"]) / g["sol_tok_s"] < 0.01
    assert abs(g["megakernel_tok_s"] / sol - g["megakernel_frac_of_sol"]) < 0.01
    assert abs(g["vllm_tok_s"] / sol - g["vllm_frac_of_sol"]) < 0.01
    assert abs(g["megakernel_tok_s"] / g["vllm_tok_s"] - g["speedup"]) < 0.01


def test_step_bytes_30b_b1():
    sb = roofline.step_bytes(configs.MOE30B, [8192], [8] * 48)
    assert abs(sb["weights"] / 1e9 - 5.277) < 0.01
    assert abs(sb["kv"] / 1e9 - 0.805) < 0.01
