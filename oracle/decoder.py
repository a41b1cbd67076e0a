"""Plain float64 CPU oracle for one decode step of a parallel-layer MoE decoder.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` may use it.  It shares no code with the CUDA path.

What it computes is the plain definition of the forward pass the megakernel
must reproduce (the pages claim the fused engine changes speed, not results:
agenticcommons "Cohere North Mini Code megakernel serving engine", summary and
section "Why decode is slow"; aimodeling "Cohere megakernel engine: one CUDA
file, 1.58x vLLM on H100", section "From demo to a full serving system").

Model (per token b, residual x in float64):
  x_0 = embed[token]
  for each layer l (parallel transformer layer: attention and the MoE FFN
  read the same RMSNorm'd input and are merged by a residual add; agenticcommons
  post, section "Three sources of speedup", item 1; aimodeling article, section
  "One persistent kernel for the whole decode step"):
      n   = RMSNorm(x_l; gamma_l)
      x_{l+1} = x_l + Attn_l(n) + MoE_l(n)
  logits = W_lm . RMSNorm(x_L; gamma_final)

Readings where the pages are silent:
  * RMSNorm: h / sqrt(mean(h^2) + eps) * gamma, eps = 1e-6.
  * RoPE: rotate-half pairs (i, i + hd/2), angle = pos * theta^(-2i/hd).
  * Cached K is post-RoPE; the new token's K and V are rounded to bf16 before
    attention reads them, exactly as they are stored in the cache.
  * Attention: GQA, q-head h uses kv-head h // (Hq/Hkv); scale 1/sqrt(hd);
    keys are the seq_len cached tokens plus the new one.
  * Router: r = W_r n + bias; top-k by (r descending, expert index ascending);
    weights = softmax over the k selected logits; no capacity limit.
  * Expert: down(silu(gate n) * up n), silu(z) = z / (1 + exp(-z)).
  * Weights, embeddings and the KV cache are bf16; every activation is f64.

Weights and cache are read through small accessor objects so that the same
code runs on a tiny in-memory model and on a 30B-shaped model whose tensors
live elsewhere (the accessor fetches one tensor at a time).  Accessors return
raw bf16 bit patterns (uint16); the conversion to float64 happens here.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np


# ----------------------------------------------------------------------------
# shape
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class ModelShape:
    n_layers: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_experts: int
    top_k: int
    d_ff: int
    vocab: int
    page_size: int = 64
    rope_theta: float = 1.0e4
    rms_eps: float = 1.0e-6

    @property
    def qkv_rows(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim


# ----------------------------------------------------------------------------
# bf16 <-> float64 (bit-level definitions)
# ----------------------------------------------------------------------------
def bf16_bits_to_f64(bits) -> np.ndarray:
    """bf16 is the upper 16 bits of an IEEE binary32; widen exactly."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x) -> np.ndarray:
    """Round float64 to the nearest bf16 (ties to even), return the bits.

    Rounds the float64 value directly to 8 significant bits (no detour
    through binary32, so there is no double rounding).  Finite normal
    inputs only, which is all the decoder produces.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                   # x = m * 2**e, 0.5 <= |m| < 1
    # bf16 keeps 8 significant bits: |m| * 2**8 in [128, 256)
    r = np.rint(m * 256.0)               # np.rint rounds half to even
    y = np.ldexp(r, e - 8)
    f32 = y.astype(np.float32)           # exact: y has <= 8 significant bits
    bits = (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    return bits


# ----------------------------------------------------------------------------
# accessors
# ----------------------------------------------------------------------------
class ArrayWeights:
    """Weights held in host memory as bf16 bit patterns (numpy uint16).

    Expected keys: ``embed`` [V][d], ``lm_head`` [V][d], ``final_norm`` [d],
    and per layer l the lists ``attn_norm`` [d], ``w_qkv`` [(Hq+2Hkv)hd][d]
    (rows: q heads, then k heads, then v heads), ``w_o`` [d][Hq hd],
    ``w_router`` [E][d], ``router_bias`` (float32 [E] or None),
    ``w_gate`` [E][F][d], ``w_up`` [E][F][d], ``w_down`` [E][d][F].
    """

    def __init__(self, tensors: Dict[str, object]):
        self.t = tensors

    def embed_row(self, token: int) -> np.ndarray:
        return self.t["embed"][token]

    def lm_head_rows(self, r0: int, r1: int) -> np.ndarray:
        return self.t["lm_head"][r0:r1]

    def final_norm(self) -> np.ndarray:
        return self.t["final_norm"]

    def attn_norm(self, l: int) -> np.ndarray:
        return self.t["attn_norm"][l]

    def w_qkv(self, l: int) -> np.ndarray:
        return self.t["w_qkv"][l]

    def w_o(self, l: int) -> np.ndarray:
        return self.t["w_o"][l]

    def w_router(self, l: int) -> np.ndarray:
        return self.t["w_router"][l]

    def router_bias(self, l: int):
        rb = self.t.get("router_bias")
        return None if rb is None else rb[l]

    def expert(self, l: int, e: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
        return self.t["w_gate"][l][e], self.t["w_up"][l][e], self.t["w_down"][l][e]


class ArrayKV:
    """Paged KV pools in host memory: per layer ``k[l]``, ``v[l]`` are uint16
    arrays shaped [n_pages][Hkv][page_size][hd] (bf16 bits)."""

    def __init__(self, k_pools: Sequence[np.ndarray], v_pools: Sequence[np.ndarray]):
        self.k = [np.array(p, dtype=np.uint16, copy=True) for p in k_pools]
        self.v = [np.array(p, dtype=np.uint16, copy=True) for p in v_pools]

    def pages(self, l: int, kind: str, page_ids) -> np.ndarray:
        pool = self.k[l] if kind == "k" else self.v[l]
        return pool[np.asarray(page_ids, dtype=np.int64)]

    def write_token(self, l: int, page: int, slot: int, k_bits, v_bits) -> None:
        self.k[l][page, :, slot, :] = k_bits
        self.v[l][page, :, slot, :] = v_bits


# ----------------------------------------------------------------------------
# the operations, one function each
# ----------------------------------------------------------------------------
def rms_norm(h: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """h / sqrt(mean(h^2) + eps) * gamma (fused residual add + RMSNorm joins
    the two branches: agenticcommons post, "Three sources of speedup", item 1)."""
    h = np.asarray(h, dtype=np.float64)
    return h / np.sqrt(np.mean(h * h) + eps) * np.asarray(gamma, dtype=np.float64)


def rope_cos_sin(pos: int, head_dim: int, theta: float) -> Tuple[np.ndarray, np.ndarray]:
    """cos/sin of angle_i = pos * theta^(-2i/hd), i < hd/2."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / head_dim)
    ang = float(pos) * inv_freq
    return np.cos(ang), np.sin(ang)


def apply_rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE on the last axis: pairs (i, i + hd/2)."""
    half = x.shape[-1] // 2
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def gather_paged(kv, l: int, kind: str, page_table_row, n_tokens: int,
                 page_size: int) -> np.ndarray:
    """Logical token t of a sequence lives in physical page
    page_table_row[t // page_size], slot t % page_size.  Returns the first
    n_tokens tokens as float64 [n_tokens][Hkv][hd]."""
    n_pages = (n_tokens + page_size - 1) // page_size
    if n_pages == 0:
        return None
    pages = kv.pages(l, kind, list(page_table_row[:n_pages]))     # [P][Hkv][S][hd]
    seq = np.transpose(pages, (0, 2, 1, 3)).reshape(n_pages * page_size,
                                                    pages.shape[1], pages.shape[3])
    return bf16_bits_to_f64(seq[:n_tokens])


def gqa_decode_attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray) -> np.ndarray:
    """q [Hq][hd], keys/values [T][Hkv][hd] -> o [Hq][hd].
    Softmax(q.k / sqrt(hd)) over all T keys; q-head h reads kv-head
    h // (Hq / Hkv)."""
    hq, hd = q.shape
    hkv = keys.shape[1]
    group = hq // hkv
    o = np.zeros((hq, hd), dtype=np.float64)
    for h in range(hq):
        g = h // group
        s = keys[:, g, :] @ q[h] / np.sqrt(hd)
        s = s - np.max(s)
        p = np.exp(s)
        p = p / np.sum(p)
        o[h] = p @ values[:, g, :]
    return o


def router_select(r: np.ndarray, k: int, forced: Optional[Sequence[int]] = None):
    """Top-k experts by (logit descending, index ascending) and their weights,
    a softmax over the selected logits.  ``forced`` replaces the selection
    (used when a near-tie may legitimately resolve either way)."""
    r = np.asarray(r, dtype=np.float64)
    if forced is None:
        order = sorted(range(r.shape[0]), key=lambda e: (-r[e], e))
        idx = np.array(order[:k], dtype=np.int64)
    else:
        idx = np.array(list(forced), dtype=np.int64)
    sel = r[idx]
    w = np.exp(sel - np.max(sel))
    w = w / np.sum(w)
    return idx, w


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def swiglu_expert(n: np.ndarray, gate_bits, up_bits, down_bits) -> np.ndarray:
    """down . (silu(gate . n) * (up . n))."""
    g = bf16_bits_to_f64(gate_bits) @ n
    u = bf16_bits_to_f64(up_bits) @ n
    a = silu(g) * u
    return bf16_bits_to_f64(down_bits) @ a, a


def attention_branch(shape: ModelShape, W, kv, l: int, n: np.ndarray, pos: int,
                     page_table_row, seq_len: int, rec: Optional[dict] = None):
    """QKV projection, RoPE at ``pos``, bf16 K/V append, paged GQA attention
    over the seq_len cached tokens plus the new one, output projection."""
    hq, hkv, hd = shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    qkv = bf16_bits_to_f64(W.w_qkv(l)) @ n
    q = qkv[: hq * hd].reshape(hq, hd)
    k = qkv[hq * hd: (hq + hkv) * hd].reshape(hkv, hd)
    v = qkv[(hq + hkv) * hd:].reshape(hkv, hd)
    cos, sin = rope_cos_sin(pos, hd, shape.rope_theta)
    q_rot = apply_rope(q, cos, sin)
    k_rot = apply_rope(k, cos, sin)
    k_bits = f64_to_bf16_bits(k_rot)
    v_bits = f64_to_bf16_bits(v)
    cached_k = gather_paged(kv, l, "k", page_table_row, seq_len, shape.page_size)
    cached_v = gather_paged(kv, l, "v", page_table_row, seq_len, shape.page_size)
    new_k = bf16_bits_to_f64(k_bits)[None]
    new_v = bf16_bits_to_f64(v_bits)[None]
    keys = new_k if cached_k is None else np.concatenate([cached_k, new_k], axis=0)
    vals = new_v if cached_v is None else np.concatenate([cached_v, new_v], axis=0)
    o = gqa_decode_attention(q_rot, keys, vals)
    out = bf16_bits_to_f64(W.w_o(l)) @ o.reshape(-1)
    if rec is not None:
        rec.update(qkv=qkv, q_rot=q_rot, k_bits=k_bits, v_bits=v_bits, o=o, attn_out=out)
    return out, k_bits, v_bits


def moe_branch(shape: ModelShape, W, l: int, n: np.ndarray,
               forced: Optional[Sequence[int]] = None, rec: Optional[dict] = None):
    """Router logits (+ bias), top-k + softmax, weighted sum of SwiGLU experts."""
    r = bf16_bits_to_f64(W.w_router(l)) @ n
    bias = W.router_bias(l)
    if bias is not None:
        r = r + np.asarray(bias, dtype=np.float64)
    idx, w = router_select(r, shape.top_k, forced)
    out = np.zeros(shape.d_model, dtype=np.float64)
    acts = []
    for j in range(len(idx)):
        y, a = swiglu_expert(n, *W.expert(l, int(idx[j])))
        out = out + w[j] * y
        acts.append(a)
    if rec is not None:
        rec.update(router_logits=r, topk_idx=idx, topk_w=w, expert_act=acts, moe_out=out)
    return out


def parallel_layer(shape: ModelShape, W, kv, l: int, x: np.ndarray, pos: int,
                   page_table_row, seq_len: int, forced=None, rec: Optional[dict] = None,
                   branches: Tuple[bool, bool] = (True, True)):
    """x + Attn(RMSNorm(x)) + MoE(RMSNorm(x)): both branches read the same
    normalized input.  ``branches`` switches a branch off (it then adds 0)."""
    n = rms_norm(x, bf16_bits_to_f64(W.attn_norm(l)), shape.rms_eps)
    attn, k_bits, v_bits = attention_branch(shape, W, kv, l, n, pos, page_table_row,
                                            seq_len, rec)
    moe = moe_branch(shape, W, l, n, forced, rec)
    if not branches[0]:
        attn = np.zeros_like(attn)
    if not branches[1]:
        moe = np.zeros_like(moe)
    x_next = x + attn + moe
    if rec is not None:
        rec.update(x_in=x, xn=n, x_out=x_next)
    return x_next, k_bits, v_bits


def final_logits(shape: ModelShape, W, x: np.ndarray, rows_per_block: int = 8192,
                 rec: Optional[dict] = None) -> np.ndarray:
    """logits = W_lm . RMSNorm(x; gamma_final)."""
    xf = rms_norm(x, bf16_bits_to_f64(W.final_norm()), shape.rms_eps)
    out = np.empty(shape.vocab, dtype=np.float64)
    for r0 in range(0, shape.vocab, rows_per_block):
        r1 = min(shape.vocab, r0 + rows_per_block)
        out[r0:r1] = bf16_bits_to_f64(W.lm_head_rows(r0, r1)) @ xf
    if rec is not None:
        rec["xf"] = xf
    return out


def decode_step(shape: ModelShape, W, kv, tokens: Sequence[int], seq_lens: Sequence[int],
                page_tables, forced: Optional[Dict[Tuple[int, int], Sequence[int]]] = None,
                record: Optional[Dict[Tuple[int, int], dict]] = None,
                layers: Optional[int] = None, append: bool = False) -> np.ndarray:
    """One decode step for a batch of independent sequences.

    tokens[b] is the token fed at position seq_lens[b] (the number of tokens
    already cached for sequence b).  Returns float64 logits [B][V].  With
    ``append`` the new K/V are written into ``kv`` (which must then be an
    oracle-owned cache such as ArrayKV).  ``layers`` limits the number of
    layers run (a bounded sample; the LM head is then skipped and the
    residual after those layers is returned instead of logits).
    """
    B = len(tokens)
    L = shape.n_layers if layers is None else layers
    xs = []
    new_kv = []
    for b in range(B):
        x = bf16_bits_to_f64(W.embed_row(int(tokens[b])))
        per_layer = []
        for l in range(L):
            rec = None
            if record is not None:
                rec = record.setdefault((l, b), {})
            fz = None if forced is None else forced.get((l, b))
            x, kb, vb = parallel_layer(shape, W, kv, l, x, int(seq_lens[b]), page_tables[b],
                                       int(seq_lens[b]), fz, rec)
            per_layer.append((kb, vb))
        xs.append(x)
        new_kv.append(per_layer)
    if append:
        for b in range(B):
            pos = int(seq_lens[b])
            page = int(page_tables[b][pos // shape.page_size])
            for l in range(L):
                kb, vb = new_kv[b][l]
                kv.write_token(l, page, pos % shape.page_size, kb, vb)
    if layers is not None and layers < shape.n_layers:
        return np.stack(xs)
    out = np.stack([final_logits(shape, W, x,
                                 rec=None if record is None else record.setdefault(("final", b), {}))
                    for b, x in enumerate(xs)])
    return out


def greedy_decode(shape: ModelShape, W, kv, tokens: Sequence[int], seq_lens: Sequence[int],
                  page_tables, n_steps: int):
    """Feed ``tokens``, then n_steps-1 greedy continuations (argmax, lowest
    index on ties).  Mutates ``kv`` (oracle-owned).  Returns (logits per step
    [n_steps][B][V], token ids fed per step [n_steps][B])."""
    toks = [int(t) for t in tokens]
    lens = [int(s) for s in seq_lens]
    all_logits, fed = [], []
    for _ in range(n_steps):
        logits = decode_step(shape, W, kv, toks, lens, page_tables, append=True)
        all_logits.append(logits)
        fed.append(list(toks))
        toks = [int(np.argmax(logits[b])) for b in range(len(toks))]
        lens = [s + 1 for s in lens]
    return np.stack(all_logits), fed
