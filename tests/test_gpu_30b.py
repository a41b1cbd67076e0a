"""GPU parity at the full 30B-MoE shape (48 layers, d 2048, 128 experts top-8,
vocab 151552), in the launch configuration bench.py times.

* batch 1, 8192-token paged KV, near-uniform routing: the whole step against
  the oracle (every layer, final logits), selection forced only where the
  oracle's k-th/(k+1)-th router gap is under 1e-3, plus teacher-forced
  single-layer checks (the oracle layer applied to the GPU's own layer input);
* batch 8, ragged 1K-16K lengths, Zipf routing: the oracle's whole 48-layer
  step for every token (expert selection identical at every layer outside the
  tie band, final logits), plus teacher-forced layers 0, 24 and 47;
* batch 1, 262144-token KV: teacher-forced layers (split-KV attention with
  ~37 chunks per KV group and the combine) and the LM head.
"""

import gc

import numpy as np
import pytest
import torch

import oracle
from moe_persistent_cta_b200 import configs, engine, mk, synth
from tests.gpu_common import MAX_ABS, REL_L2, ROUTER_TIE, compare_logits, router_gap
from tests.oracle_io import TorchKV, TorchWeights, oracle_shape

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SHAPE = configs.MOE30B
LAYER_ATOL = 2e-3        # one layer's output, teacher-forced
LOGIT_TIGHT = 1e-2       # whole 48-layer step (tighter than the 5e-2 contract)


@pytest.fixture(scope="module")
def model():
    dev = "cuda:0"
    W = synth.make_weights(SHAPE, 0, dev, "uniform")
    yield W
    del W
    gc.collect()
    torch.cuda.empty_cache()


class Run:
    """One GPU step; `positions` defaults to the lengths (decode).  A prefill
    group (positions = lengths + 0 .. M - 1) shares the first entry's
    page-table row."""

    def __init__(self, W, lens, seed=0, growth=64, positions=None):
        self.W = W
        self.lens = list(lens)
        self.B = len(lens)
        self.pos = list(positions) if positions is not None else list(lens)
        self.dev = torch.device("cuda:0")
        self.table, self.n_pages = synth.make_page_tables(self.lens, False, seed + 3,
                                                          growth=growth)
        if positions is not None:
            self.table[1:] = self.table[0]
        self.k, self.v = synth.make_kv(SHAPE, self.n_pages, seed + 1, "cuda:0")
        self.tokens = synth.make_tokens(self.B, SHAPE["vocab"], seed + 2)
        self.dec = engine.Decoder(SHAPE, W, self.k, self.v, max_batch=self.B)
        self.dec.build_schedule(self.lens, self.table.shape[1])
        i32 = dict(dtype=torch.int32, device=self.dev)
        self.logits = torch.empty((self.B, SHAPE["vocab"]), dtype=torch.float32, device=self.dev)
        self.dec.step(torch.tensor(self.tokens, **i32), torch.tensor(self.pos, **i32),
                      self.table.to(self.dev), torch.tensor(self.lens, **i32), self.logits)
        self.dec.check_ok()
        L, d, E, K = SHAPE["n_layers"], SHAPE["d_model"], SHAPE["n_experts"], SHAPE["top_k"]
        self.X = self.dec.debug(mk.MK_BUF_X).reshape(L + 1, self.B, d).astype(np.float64)
        self.RL = self.dec.debug(mk.MK_BUF_RLOGITS).reshape(L, self.B, E)
        tk = self.dec.debug(mk.MK_BUF_TOPK)
        self.ids = tk[: L * self.B * K].reshape(L, self.B, K)
        self.S = oracle_shape(SHAPE)
        self.WA = TorchWeights(W)
        self.KV = TorchKV(self.k, self.v)

    def close(self):
        self.dec.close()
        del self.k, self.v
        gc.collect()
        torch.cuda.empty_cache()

    def layer(self, l, b, x_in):
        """Oracle layer l on x_in; the selection is the oracle's own unless it
        differs from the GPU's inside the near-tie band.  Returns (x_out,
        record, forced?)."""
        rec = {}
        pt = self.table[b].numpy()
        x_out, _, _ = oracle.parallel_layer(self.S, self.WA, self.KV, l, x_in, self.pos[b], pt,
                                            self.pos[b], rec=rec)
        gpu_sel = [int(e) for e in self.ids[l, b]]
        if gpu_sel != [int(e) for e in rec["topk_idx"]]:
            gap = router_gap(rec["router_logits"], SHAPE["top_k"])
            assert gap < ROUTER_TIE, f"layer {l} token {b}: selection differs, gap {gap:.2e}"
            rec = {}
            x_out, _, _ = oracle.parallel_layer(self.S, self.WA, self.KV, l, x_in, self.pos[b],
                                                pt, self.pos[b], forced=gpu_sel, rec=rec)
            return x_out, rec, True
        return x_out, rec, False

    def teacher_forced(self, layers, tokens):
        worst = 0.0
        for l in layers:
            for b in tokens:
                x_out, rec, _ = self.layer(l, b, self.X[l, b])
                err = float(np.max(np.abs(self.X[l + 1, b] - x_out)))
                rerr = float(np.max(np.abs(self.RL[l, b] - rec["router_logits"])))
                worst = max(worst, err)
                assert err <= LAYER_ATOL, f"layer {l} token {b}: max-abs {err:.3e}"
                assert rerr <= 1e-3, f"layer {l} token {b}: router logits {rerr:.3e}"
        return worst

    def whole_step(self, b):
        """The oracle's own 48-layer pass for token b (selection forced only
        inside the near-tie band) and its logits.  Prints how far the GPU's
        residual stream is from the oracle's at each layer."""
        x = oracle.bf16_bits_to_f64(self.WA.embed_row(self.tokens[b]))
        forced = 0
        drift = []
        try:
            for l in range(SHAPE["n_layers"]):
                x, _, f = self.layer(l, b, x)
                forced += int(f)
                drift.append(float(np.max(np.abs(self.X[l + 1, b] - x))))
        finally:
            print(f"token {b}: residual drift GPU vs oracle every 4th layer: "
                  + " ".join(f"{v:.1e}" for v in drift[::4]))
        return oracle.decoder.final_logits(self.S, self.WA, x), forced


def test_30b_b1_whole_step(model):
    r = Run(model, [8192])
    try:
        ref, forced = r.whole_step(0)
        got = r.logits[0].cpu().double().numpy()
        err, rel = compare_logits(got, ref)
        print(f"30B b1: logits max-abs {err:.3e} rel-L2 {rel:.3e}, forced layers {forced}")
        assert err <= MAX_ABS and rel <= REL_L2
        assert err <= LOGIT_TIGHT
        assert int(np.argmax(got)) == int(np.argmax(ref))
        worst = r.teacher_forced(range(SHAPE["n_layers"]), [0])
        print(f"30B b1: teacher-forced layer max-abs {worst:.3e}")
        nslots = r.dec.debug(mk.MK_BUF_NSLOTS)
        assert np.all(nslots == SHAPE["top_k"])
    finally:
        r.close()


def test_30b_b8_zipf(model):
    W = dict(model)
    W["w_router"], W["router_bias"] = synth.make_router(SHAPE, 0, "cuda:0", "zipf", 1.1)
    lens = synth.seq_lengths(("uniform", 1024, 16384, 4), 8)
    r = Run(W, lens)
    try:
        worst = r.teacher_forced([0, 24, 47], range(8))
        print(f"30B b8 zipf: teacher-forced layer max-abs {worst:.3e}")
        for b in range(8):
            ref, forced = r.whole_step(b)
            got = r.logits[b].cpu().double().numpy()
            err, rel = compare_logits(got, ref)
            print(f"30B b8 zipf token {b}: logits max-abs {err:.3e} rel-L2 {rel:.3e}, "
                  f"forced {forced}")
            assert err <= MAX_ABS and rel <= REL_L2
            assert int(np.argmax(got)) == int(np.argmax(ref))
        nslots = r.dec.debug(mk.MK_BUF_NSLOTS)
        print(f"30B b8 zipf: experts touched per layer mean {nslots.mean():.1f}")
        assert np.all(nslots >= SHAPE["top_k"]) and np.all(nslots <= 64)
    finally:
        r.close()


def test_30b_b1_256k(model):
    r = Run(model, [262144])
    try:
        worst = r.teacher_forced([0, 47], [0])
        print(f"30B b1 256K: teacher-forced layer max-abs {worst:.3e}")
        ref = oracle.decoder.final_logits(r.S, r.WA, r.X[SHAPE["n_layers"], 0])
        got = r.logits[0].cpu().double().numpy()
        err, rel = compare_logits(got, ref)
        print(f"30B b1 256K: LM head from the GPU residual max-abs {err:.3e} rel-L2 {rel:.3e}")
        assert err <= 1e-3 and rel <= 1e-4
    finally:
        r.close()


def test_30b_prefill_chunk8(model):
    """Eight prompt tokens after an 8192-token prefix in one step (a prefill
    group, as bench.py times it).  The oracle reads the KV pool as the GPU
    step left it, so token g at position 8192 + g attends to the prefix and
    to the group's g earlier tokens, appended by the step: every token's
    layers 0, 24 and 47 teacher-forced, and the oracle's whole 48-layer pass
    for the first and the last token."""
    prefix = 8192
    r = Run(model, [prefix] * 8, positions=[prefix + g for g in range(8)])
    try:
        worst = r.teacher_forced([0, 24, 47], range(8))
        print(f"30B prefill chunk 8: teacher-forced layer max-abs {worst:.3e}")
        for b in (0, 7):
            ref, forced = r.whole_step(b)
            got = r.logits[b].cpu().double().numpy()
            err, rel = compare_logits(got, ref)
            print(f"30B prefill token {b}: logits max-abs {err:.3e} rel-L2 {rel:.3e}, "
                  f"forced {forced}")
            assert err <= MAX_ABS and rel <= REL_L2
            assert err <= LOGIT_TIGHT
            assert int(np.argmax(got)) == int(np.argmax(ref))
    finally:
        r.close()
