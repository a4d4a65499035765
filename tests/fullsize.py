"""Session-wide state of the full-size parity tests.

One Beam layer is shared by every full-size test: its 20 GB of bf16 expert weights on the GPU and
one host copy for the oracle, its FP8 and NVFP4 checkpoints (GPU codes and host copies), each
workload's inputs, the oracle's routing of each workload and the oracle's outputs on each workload's
token sample.  Each is built once per session, on first use, so that no test copies the layer back
from the GPU or re-runs the oracle on work another test already did.

Token samples (oracle outputs are compared on these; routing and dispatch on every token):
  decode   all 256 tokens
  prefill  512 seeded tokens
  skew     4096 seeded tokens
  long     4096 seeded tokens plus every outlier row (655)
The FP8 and NVFP4 checkpoints are compared on decode (all tokens) and prefill (256 seeded tokens), on
the converter paths and on the native FP8 path ("mxfp8": MXFP8 activations too).
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

import beam_synth as bs
import oracle
from tests import parity

SAMPLE = {"decode": None, "prefill": 512, "skew": 4096, "long": 4096}
W4A4_EPS = 3e-5  # tolerance of the 4-bit path's near-boundary envelope (tests/test_gpu_w4a4.py)
SAMPLE_LOWP = {"decode": None, "prefill": 256}
FULL = ("decode", "prefill", "skew", "long")


def sample(name: str, fmt: str = "bf16") -> np.ndarray:
    wl = bs.get(name)
    n = (SAMPLE if fmt == "bf16" else SAMPLE_LOWP)[name]
    if n is None:
        return np.arange(wl.T)
    return bs.sample_tokens(wl, n, include=bs.outlier_rows(wl))


def _host_bits(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


class Bank:
    def __init__(self):
        self.wl = bs.WORKLOADS["prefill"]
        self.gpu = bs.make_experts(self.wl, device="cuda")
        self._host = None
        self._fp8 = None
        self._fp8_host = None
        self._nv4 = None
        self._nv4_host = None
        self._cases: Dict[str, parity.Case] = {}
        self._y: Dict[tuple, np.ndarray] = {}

    # ---- weights ------------------------------------------------------------------------------
    def host(self):
        if self._host is None:
            self._host = tuple(_host_bits(t) for t in self.gpu)
        return self._host

    def fp8(self):
        if self._fp8 is None:
            self._fp8 = bs.quantize_experts(*self.gpu)
        return self._fp8

    def nvfp4(self):
        if self._nv4 is None:
            self._nv4 = bs.quantize_experts_nvfp4(*self.gpu)
        return self._nv4

    def fetch(self, fmt: str):
        """fetch(e) of the oracle: one expert's weights (bf16 bits, or FP64 for NVFP4) on the host.
        "mxfp8" (the native FP8 path) reads the FP8 checkpoint like "fp8"."""
        if fmt == "mxfp8":
            fmt = "fp8"
        if fmt == "w4a4":
            fmt = "nvfp4"
        if fmt == "bf16":
            h = self.host()
            return lambda e: (h[0][e], h[1][e], h[2][e])
        if fmt == "fp8":
            if self._fp8_host is None:
                self._fp8_host = {k: v.cpu().numpy() for k, v in self.fp8().items()}
            w = self._fp8_host
            return lambda e: tuple(oracle.dequant_mxfp8(w["q_" + n][e], w["s_" + n][e]) for n in ("gate", "up", "down"))
        if self._nv4_host is None:
            self._nv4_host = {k: v.cpu().numpy() for k, v in self.nvfp4().items()}
        w = self._nv4_host
        return lambda e: tuple(oracle.dequant_nvfp4(w["q_" + n][e], w["s_" + n][e], float(w["g_" + n][e]))
                               for n in ("gate", "up", "down"))

    # ---- workloads ----------------------------------------------------------------------------
    def case(self, name: str) -> parity.Case:
        if name not in self._cases:
            c = parity.Case(bs.get(name), weights=self.gpu)
            c.fetch = lambda e: self.fetch("bf16")(e)  # host copy on first use
            self._cases[name] = c
        return self._cases[name]

    def y_of(self, fmt: str, name: str):
        """y_of(ids, w, tokens): the oracle's expert half on `tokens` of workload `name`."""
        c = self.case(name)
        run = _RUN[fmt]
        fetch = self.fetch(fmt)

        def y_of(ids, w, tokens):
            return run(np.ascontiguousarray(c.x_bits[tokens]), ids[tokens], w[tokens], fetch, c.layer["n_experts"],
                       c.layer["routed_scale"])
        return y_of

    def oracle_y(self, fmt: str, name: str) -> np.ndarray:
        """The oracle's outputs on the token sample of `name`, on the oracle's own routing (for "w4a4",
        the pair (outputs, envelope)).  The first request of a format computes every workload of
        that format in one pass over the experts."""
        key = (fmt, name)
        if key not in self._y:
            names = FULL if fmt == "bf16" else tuple(SAMPLE_LOWP)
            xs, ids, ws, spans = [], [], [], []
            at = 0
            for n in names:
                c = self.case(n)
                r = c.oracle_route()
                tok = sample(n, fmt)
                xs.append(c.x_bits[tok])
                ids.append(r["ids"][tok])
                ws.append(r["weight"][tok])
                spans.append((n, at, at + len(tok)))
                at += len(tok)
            x = np.ascontiguousarray(np.concatenate(xs))
            run = _RUN[fmt]
            L = self.wl.layer
            args = (x, np.concatenate(ids), np.concatenate(ws), self.fetch(fmt), L["n_experts"], L["routed_scale"])
            if fmt == "w4a4":  # with the envelope of h's near-boundary quantisation decisions
                y, env = run(*args, eps=W4A4_EPS)
                for n, a, b in spans:
                    self._y[(fmt, n)] = (y[a:b], env[a:b])
                return self._y[key]
            y = run(*args)
            for n, a, b in spans:
                self._y[(fmt, n)] = y[a:b]
        return self._y[key]


# the oracle's expert half per weight format
_RUN = {"bf16": oracle.experts_tokens, "fp8": oracle.experts_tokens, "nvfp4": oracle.experts_tokens_f64,
        "mxfp8": oracle.experts_tokens_mx8, "w4a4": oracle.experts_tokens_w4a4}

_BANK: Optional[Bank] = None


def bank() -> Bank:
    global _BANK
    if _BANK is None:
        _BANK = Bank()
    return _BANK
