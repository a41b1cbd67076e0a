"""Model shapes and synthetic workloads.

The 30B-MoE shape and the workload mix (batch 1 and 8, ragged 1K-16K
contexts, 256K context, continuous batching) are the stand-ins for the pages'
North Mini Code serving runs (agenticcommons.xyz, "Cohere North Mini Code
megakernel serving engine", section "Why decode is slow": 30B total / a few B
active parameters, BF16, 8K context, batch 1 to 8, up to 256K context).  All
inputs are seeded and synthetic (generators in ``synth``).
"""

from __future__ import annotations

TINY = dict(n_layers=2, d_model=256, n_q_heads=4, n_kv_heads=2, head_dim=64, n_experts=8,
            top_k=2, d_ff=512, vocab=1024, page_size=64, rope_theta=1.0e4, rms_eps=1.0e-6)

MOE30B = dict(n_layers=48, d_model=2048, n_q_heads=16, n_kv_heads=4, head_dim=128,
              n_experts=128, top_k=8, d_ff=768, vocab=151552, page_size=64, rope_theta=1.0e4,
              rms_eps=1.0e-6)

# Workloads.  ``seq_lens`` is either a list or ("uniform", lo, hi, seed).
WORKLOADS = {
    "tiny": dict(shape=TINY, batch=1, seq_lens=[128], routing="uniform", contiguous=True,
                 weight_seed=0, kv_seed=1, token_seed=2, page_seed=3),
    "moe30b_b1": dict(shape=MOE30B, batch=1, seq_lens=[8192], routing="uniform",
                      contiguous=False, weight_seed=0, kv_seed=1, token_seed=2, page_seed=3),
    "moe30b_b8_zipf": dict(shape=MOE30B, batch=8, seq_lens=("uniform", 1024, 16384, 4),
                           routing="zipf", zipf_s=1.1, contiguous=False, weight_seed=0,
                           kv_seed=1, token_seed=2, page_seed=3),
    "moe30b_b1_256k": dict(shape=MOE30B, batch=1, seq_lens=[262144], routing="uniform",
                           contiguous=False, weight_seed=0, kv_seed=1, token_seed=2,
                           page_seed=3),
}

# continuous batching run: 8 slots, 512 steps, start lengths U[512, 32768],
# lengths geometric with mean 128, Zipf routing
CONTINUOUS = dict(shape=MOE30B, slots=8, steps=512, start_lo=512, start_hi=32768,
                  mean_new=128, routing="zipf", zipf_s=1.1, seed=5)


def weight_bytes_active(shape: dict, experts_per_layer) -> int:
    """Algorithmic weight bytes one step must read (bf16): attention, router,
    norms, the experts actually touched, LM head, final norm."""
    d, hd = shape["d_model"], shape["head_dim"]
    qkv = (shape["n_q_heads"] + 2 * shape["n_kv_heads"]) * hd * d
    wo = d * shape["n_q_heads"] * hd
    router = shape["n_experts"] * d
    expert = 3 * shape["d_ff"] * d
    total = 0
    for u in experts_per_layer:
        total += 2 * (qkv + wo + router + d + u * expert)
    total += 2 * (shape["vocab"] * d + d)
    return total


def kv_bytes_read(shape: dict, seq_lens) -> int:
    """KV bytes read by attention: every cached token plus the new one, K and
    V, all layers, all KV heads (bf16)."""
    per_tok = shape["n_layers"] * 2 * shape["n_kv_heads"] * shape["head_dim"] * 2
    return sum((int(s) + 1) * per_tok for s in seq_lens)
