"""CPU oracle for the decode step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` may import this package.  The product path (the C-ABI library and
its Python binding) never imports, calls or links anything here.
"""

from .decoder import (  # noqa: F401
    ModelShape,
    ArrayWeights,
    ArrayKV,
    bf16_bits_to_f64,
    f64_to_bf16_bits,
    rms_norm,
    rope_cos_sin,
    apply_rope,
    gather_paged,
    gqa_decode_attention,
    router_select,
    swiglu_expert,
    moe_branch,
    attention_branch,
    parallel_layer,
    decode_step,
    greedy_decode,
)
