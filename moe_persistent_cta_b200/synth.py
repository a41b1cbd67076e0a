"""Seeded synthetic inputs: weights, paged KV cache, page tables, tokens.

This module holds no arithmetic of the decode method; it only draws the
inputs that both the native path and the CPU oracle consume.  Every draw uses
torch's seeded generators in a fixed order:

* weights ~ N(0, 0.02) rounded to bf16 (router weights use the workload's
  router scale), RMSNorm gains = 1;
* Zipf routing: per layer a seeded permutation of the experts and a router
  bias b_e = ln p_e with p_e proportional to rank^-s;
* KV cache ~ N(0, 1) in bf16, [n_pages][Hkv][64][hd] per layer;
* page tables: logical pages of each sequence mapped to a seeded random
  permutation of the physical pages (or the identity for "contiguous");
* tokens uniform over the vocabulary.

Small models are drawn on the CPU (so the bytes are identical on every
machine); large ones are drawn directly on the GPU.
"""

from __future__ import annotations

import math
from typing import Dict, List, Optional

import torch

WEIGHT_STD = 0.02
GUMBEL_STD = math.pi / math.sqrt(6.0)


def _randn_bf16(shape, gen, device, std):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    t.mul_(std)
    return t.to(torch.bfloat16)


def router_std(shape: dict, routing: str) -> float:
    if routing == "zipf":
        # logit noise ~ Gumbel-like spread around the Zipf bias
        return GUMBEL_STD / math.sqrt(shape["d_model"])
    return WEIGHT_STD


def zipf_bias(shape: dict, s: float, seed: int) -> List[torch.Tensor]:
    """Per-layer router bias b_e = ln p_e, p_e ~ rank^-s over a seeded permutation."""
    E = shape["n_experts"]
    gen = torch.Generator(device="cpu").manual_seed(seed)
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    p = ranks.pow(-s)
    p = p / p.sum()
    logp = torch.log(p).to(torch.float32)
    out = []
    for _ in range(shape["n_layers"]):
        perm = torch.randperm(E, generator=gen)
        b = torch.empty(E, dtype=torch.float32)
        b[perm] = logp
        out.append(b)
    return out


def make_weights(shape: dict, seed: int = 0, device: str = "cpu", routing: str = "uniform",
                 zipf_s: float = 1.1) -> Dict[str, object]:
    """Draw the model.  Returns a dict of bf16 torch tensors on ``device``:
    embed, lm_head, final_norm and per-layer lists attn_norm, w_qkv, w_o,
    w_router, router_bias (float32 or None), w_gate, w_up, w_down."""
    L, d, V = shape["n_layers"], shape["d_model"], shape["vocab"]
    hd, Hq, Hkv = shape["head_dim"], shape["n_q_heads"], shape["n_kv_heads"]
    E, F = shape["n_experts"], shape["d_ff"]
    gen = torch.Generator(device=device).manual_seed(seed)
    W: Dict[str, object] = {}
    W["embed"] = _randn_bf16((V, d), gen, device, WEIGHT_STD)
    W["lm_head"] = _randn_bf16((V, d), gen, device, WEIGHT_STD)
    W["final_norm"] = torch.ones(d, dtype=torch.bfloat16, device=device)
    keys = ("attn_norm", "w_qkv", "w_o", "w_router", "w_gate", "w_up", "w_down")
    for k in keys:
        W[k] = []
    for _ in range(L):
        W["attn_norm"].append(torch.ones(d, dtype=torch.bfloat16, device=device))
        W["w_qkv"].append(_randn_bf16(((Hq + 2 * Hkv) * hd, d), gen, device, WEIGHT_STD))
        W["w_o"].append(_randn_bf16((d, Hq * hd), gen, device, WEIGHT_STD))
        W["w_gate"].append(_randn_bf16((E, F, d), gen, device, WEIGHT_STD))
        W["w_up"].append(_randn_bf16((E, F, d), gen, device, WEIGHT_STD))
        W["w_down"].append(_randn_bf16((E, d, F), gen, device, WEIGHT_STD))
    W["w_router"], W["router_bias"] = make_router(shape, seed, device, routing, zipf_s)
    return W


def make_router(shape: dict, seed: int = 0, device: str = "cpu", routing: str = "uniform",
                zipf_s: float = 1.1):
    """Router weights (their own seeded stream, so models that differ only in
    routing share every other tensor) and the per-layer bias (None for
    uniform routing)."""
    gen = torch.Generator(device=device).manual_seed(seed + 500)
    rstd = router_std(shape, routing)
    w = [_randn_bf16((shape["n_experts"], shape["d_model"]), gen, device, rstd)
         for _ in range(shape["n_layers"])]
    bias = None
    if routing == "zipf":
        bias = [b.to(device) for b in zipf_bias(shape, zipf_s, seed + 1000)]
    return w, bias


def seq_lengths(spec, batch: int) -> List[int]:
    if isinstance(spec, (list, tuple)) and spec and spec[0] == "uniform":
        _, lo, hi, seed = spec
        gen = torch.Generator(device="cpu").manual_seed(seed)
        return [int(v) for v in torch.randint(lo, hi + 1, (batch,), generator=gen)]
    return [int(v) for v in spec][:batch]


def pages_needed(seq_len: int, growth: int = 64, page: int = 64) -> int:
    """Pages that hold seq_len cached tokens plus `growth` future tokens."""
    return (seq_len + growth + page - 1) // page


def make_page_tables(seq_lens: List[int], contiguous: bool, seed: int, growth: int = 64,
                     page: int = 64, extra_pages: int = 0):
    """Returns (page_table int32 [B][max_pages] with -1 padding, n_pages)."""
    need = [pages_needed(s, growth, page) for s in seq_lens]
    n_pages = sum(need) + extra_pages
    max_pages = max(need)
    if contiguous:
        phys = torch.arange(n_pages, dtype=torch.int32)
    else:
        gen = torch.Generator(device="cpu").manual_seed(seed)
        phys = torch.randperm(n_pages, generator=gen).to(torch.int32)
    table = torch.full((len(seq_lens), max_pages), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = phys[off:off + n]
        off += n
    return table, n_pages


def make_kv(shape: dict, n_pages: int, seed: int, device: str = "cpu"):
    """K and V pools, each [L][n_pages][Hkv][64][hd] bf16 ~ N(0, 1)."""
    L, Hkv, hd = shape["n_layers"], shape["n_kv_heads"], shape["head_dim"]
    gen = torch.Generator(device=device).manual_seed(seed)
    k = torch.empty((L, n_pages, Hkv, 64, hd), dtype=torch.bfloat16, device=device)
    v = torch.empty_like(k)
    for l in range(L):
        k[l] = _randn_bf16((n_pages, Hkv, 64, hd), gen, device, 1.0)
        v[l] = _randn_bf16((n_pages, Hkv, 64, hd), gen, device, 1.0)
    return k, v


def make_tokens(batch: int, vocab: int, seed: int) -> List[int]:
    gen = torch.Generator(device="cpu").manual_seed(seed)
    return [int(t) for t in torch.randint(0, vocab, (batch,), generator=gen)]


def make_workload(wl: dict, device: str = "cpu", model_device: Optional[str] = None):
    """Everything one decode step needs, drawn from the workload's seeds."""
    shape = wl["shape"]
    B = wl["batch"]
    lens = seq_lengths(wl["seq_lens"], B)
    table, n_pages = make_page_tables(lens, wl.get("contiguous", False), wl["page_seed"])
    mdev = model_device or device
    W = make_weights(shape, wl["weight_seed"], mdev, wl.get("routing", "uniform"),
                     wl.get("zipf_s", 1.1))
    k, v = make_kv(shape, n_pages, wl["kv_seed"], mdev)
    toks = make_tokens(B, shape["vocab"], wl["token_seed"])
    return dict(shape=shape, weights=W, k=k, v=v, page_table=table, n_pages=n_pages,
                seq_lens=lens, tokens=toks, batch=B)
