"""Adapters from the seeded torch inputs to the oracle's accessors (tests only)."""

from __future__ import annotations

import numpy as np
import torch

from oracle import ArrayKV, ArrayWeights, ModelShape


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_shape(shape: dict) -> ModelShape:
    return ModelShape(n_layers=shape["n_layers"], d_model=shape["d_model"],
                      n_q_heads=shape["n_q_heads"], n_kv_heads=shape["n_kv_heads"],
                      head_dim=shape["head_dim"], n_experts=shape["n_experts"],
                      top_k=shape["top_k"], d_ff=shape["d_ff"], vocab=shape["vocab"],
                      page_size=shape.get("page_size", 64),
                      rope_theta=shape.get("rope_theta", 1.0e4),
                      rms_eps=shape.get("rms_eps", 1.0e-6))


def array_weights(W: dict) -> ArrayWeights:
    """Whole model in host memory (small models)."""
    t = {
        "embed": u16(W["embed"]), "lm_head": u16(W["lm_head"]),
        "final_norm": u16(W["final_norm"]),
    }
    for k in ("attn_norm", "w_qkv", "w_o", "w_router", "w_gate", "w_up", "w_down"):
        t[k] = [u16(x) for x in W[k]]
    rb = W.get("router_bias")
    t["router_bias"] = None if rb is None else [x.detach().float().cpu().numpy() for x in rb]
    return ArrayWeights(t)


class TorchWeights:
    """Lazy accessor over torch tensors (possibly on the GPU): each call
    copies one tensor to host memory."""

    def __init__(self, W: dict):
        self.W = W

    def embed_row(self, token):
        return u16(self.W["embed"][token])

    def lm_head_rows(self, r0, r1):
        return u16(self.W["lm_head"][r0:r1])

    def final_norm(self):
        return u16(self.W["final_norm"])

    def attn_norm(self, l):
        return u16(self.W["attn_norm"][l])

    def w_qkv(self, l):
        return u16(self.W["w_qkv"][l])

    def w_o(self, l):
        return u16(self.W["w_o"][l])

    def w_router(self, l):
        return u16(self.W["w_router"][l])

    def router_bias(self, l):
        rb = self.W.get("router_bias")
        return None if rb is None else rb[l].detach().float().cpu().numpy()

    def expert(self, l, e):
        return (u16(self.W["w_gate"][l][e]), u16(self.W["w_up"][l][e]),
                u16(self.W["w_down"][l][e]))


class TorchKV:
    """Lazy accessor over torch KV pools [L][n_pages][Hkv][64][hd]."""

    def __init__(self, k: torch.Tensor, v: torch.Tensor):
        self.k, self.v = k, v

    def pages(self, l, kind, page_ids):
        pool = self.k if kind == "k" else self.v
        idx = torch.as_tensor(list(page_ids), dtype=torch.long, device=pool.device)
        return u16(pool[l].index_select(0, idx))


def array_kv(k: torch.Tensor, v: torch.Tensor) -> ArrayKV:
    L = k.shape[0]
    return ArrayKV([u16(k[l]) for l in range(L)], [u16(v[l]) for l in range(L)])
