"""Shared helpers for the GPU parity tests."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from moe_persistent_cta_b200 import engine, synth
from tests.oracle_io import array_kv, array_weights, oracle_shape

# Pass thresholds of the method's contract (logits): max-abs and relative L2.
MAX_ABS = 5e-2
REL_L2 = 1e-2
# Near-tie band in which either expert choice is correct.
ROUTER_TIE = 1e-3


def to_dev(W, dev):
    out = {}
    for k, v in W.items():
        if isinstance(v, list):
            out[k] = [t.to(dev) for t in v]
        elif v is None:
            out[k] = None
        else:
            out[k] = v.to(dev)
    return out


class TinyRig:
    """A small model drawn on the CPU, copied to the GPU, with a Decoder."""

    def __init__(self, shape, lens, seed=0, shuffled=True, routing="uniform", zipf_s=1.1,
                 growth=64, weights=None):
        self.shape = shape
        self.lens = list(lens)
        self.B = len(lens)
        self.dev = torch.device("cuda:0")
        self.W = weights if weights is not None else synth.make_weights(shape, seed, "cpu",
                                                                        routing, zipf_s)
        self.table, self.n_pages = synth.make_page_tables(self.lens, not shuffled, seed + 3,
                                                          growth=growth)
        self.k, self.v = synth.make_kv(shape, self.n_pages, seed + 1)
        self.tokens = synth.make_tokens(self.B, shape["vocab"], seed + 2)
        self.Wd = to_dev(self.W, self.dev)
        self.kd, self.vd = self.k.to(self.dev), self.v.to(self.dev)
        self.dec = engine.Decoder(shape, self.Wd, self.kd, self.vd, max_batch=self.B)
        self.dec.build_schedule(self.lens, self.table.shape[1])
        self.logits = torch.empty((self.B, shape["vocab"]), dtype=torch.float32,
                                  device=self.dev)

    def i32(self, vals):
        return torch.tensor(list(vals), dtype=torch.int32, device=self.dev)

    def step(self, tokens=None, lens=None, unfused=False):
        tokens = self.tokens if tokens is None else tokens
        lens = self.lens if lens is None else lens
        self.dec.step(self.i32(tokens), self.i32(lens), self.table.to(self.dev),
                      self.i32(lens), self.logits, unfused=unfused)
        self.dec.check_ok()
        return self.logits.cpu().double().numpy()

    def oracle_step(self, tokens=None, lens=None, kv=None, record=None, forced=None):
        tokens = self.tokens if tokens is None else tokens
        lens = self.lens if lens is None else lens
        kv = kv if kv is not None else array_kv(self.k, self.v)
        return oracle.decode_step(oracle_shape(self.shape), array_weights(self.W), kv, tokens,
                                  lens, self.table.numpy(), record=record, forced=forced)

    def close(self):
        self.dec.close()


def compare_logits(got, ref):
    err = float(np.max(np.abs(got - ref)))
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    return err, rel


def router_gap(logits_row, k):
    """Gap between the k-th and (k+1)-th largest router logits."""
    s = np.sort(np.asarray(logits_row))[::-1]
    return float(s[k - 1] - s[k]) if len(s) > k else float("inf")
