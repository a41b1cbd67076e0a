"""HBM roofline of the decode step.

A decode step at small batch must stream the active weights plus the KV
cache it attends over; its speed of light is bandwidth / those bytes
(agenticcommons.xyz, "Cohere North Mini Code megakernel serving engine",
section "Why decode is slow").
"""

from __future__ import annotations

from typing import Sequence

from .configs import kv_bytes_read, weight_bytes_active


def sol_tok_s(bandwidth_bytes_s: float, bytes_per_step: float, batch: int = 1) -> float:
    """Tokens/s at the roofline: batch tokens per step, one step per
    bytes_per_step / bandwidth seconds."""
    return batch * bandwidth_bytes_s / bytes_per_step


def step_bytes(shape: dict, seq_lens: Sequence[int], experts_per_layer: Sequence[int]) -> dict:
    """Algorithmic bytes of one step: active weights (the experts the batch
    touches in each layer), the embedding rows, and the KV read."""
    w = weight_bytes_active(shape, experts_per_layer)
    emb = len(seq_lens) * shape["d_model"] * 2
    kv = kv_bytes_read(shape, seq_lens)
    return dict(weights=w + emb, kv=kv, total=w + emb + kv)
