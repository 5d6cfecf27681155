"""Seeded synthetic inputs for the KLA workloads.

This module only draws random numbers; it holds none of the method's
arithmetic and is shared by the CUDA path's tests/benchmark and by the oracle
checks.  Every tensor is produced on the host by NumPy's PCG64 generator with a
fixed seed, in the order q, k, v, key scale, g, eta, h0, and then cast with
round-to-nearest-even to the workload's I/O dtype.

Workloads (the distributions are the ones the method's evaluation is described
with: 0.4B-scale layer shapes, contexts up to 65K, decode against a 32K-token
prefilled state):

``tiny``         B=1 T=256 H=2 d=64, fp32 I/O; q,k,v ~ N(0,1) (keys not
                 normalised); g = -softplus(N(2,1)); eta = sigmoid(N(0,1)).
``prefill_4k``   B=8 T=4096 H=8 d=128, bf16; q,v ~ N(0,1); k = s*z with
                 z ~ N(0,I) and a per-token scale s ~ LogUniform(0.25, 4);
                 g = -softplus(N(3,1)); eta = sigmoid(N(0,1)).
``prefill_65k``  B=1 T=65536 H=16 d=128, bf16; as ``prefill_4k`` plus strong
                 forgets: with probability 1% per (b, t), shared by all heads,
                 g ~ U(-5, -2).
``stress``       B=4 T=8192 H=32 d=64, bf16; k = rho * z/|z| with the norm
                 rho ~ LogUniform(1e-2, 1e2); eta ~ U(0, 2); g = 0 with
                 probability 1/2 else -softplus(N(1, 2)); h0 ~ N(0, 0.1^2).
``decode``       B=64 H=16 d=128; one new token per sequence per step (bf16
                 q,k,v; g, eta as ``prefill_4k``); the state is what a
                 32768-token prefix of ``prefill_4k``-distributed tokens
                 leaves.  Only the last ``prefix_tokens`` tokens of that
                 prefix are drawn: whatever the earlier tokens wrote reaches
                 the final state multiplied by the product of alpha over the
                 kept tokens (and by erase factors of norm <= 1).  With
                 g = -softplus(N(3,1)) that product over 128 tokens is below
                 1e-100, so the state equals the 32K-prefix state to fp64
                 precision.

eps = 1e-6 and chunk C = 64 everywhere.

Per-channel gates (the KDA form) replace g by one log-gate per key channel,
drawn by :func:`channel_gates`: g = -softplus(N(3, 1.5)) i.i.d. per channel,
so most channels forget slowly (alpha ~ 0.95) and a tail forgets fast.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional

import numpy as np
import torch

EPS = 1e-6
CHUNK = 64


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: str  # "bf16" or "fp32": dtype of q, k, v, o
    seed: int
    kind: str   # distribution family: "tiny", "layer", "long", "stress"

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def scaled(self, **kw) -> "Workload":
        """Same distributions with other sizes or seed (for parity tests)."""
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 256, 2, 64, 64, "fp32", 1000, "tiny"),
    "prefill_4k": Workload("prefill_4k", 8, 4096, 8, 128, 128, "bf16", 1001, "layer"),
    "prefill_65k": Workload("prefill_65k", 1, 65536, 16, 128, 128, "bf16", 1002, "long"),
    "stress": Workload("stress", 4, 8192, 32, 64, 64, "bf16", 1004, "stress"),
}


@dataclass(frozen=True)
class DecodeWorkload:
    name: str = "decode"
    B: int = 64
    H: int = 16
    dk: int = 128
    dv: int = 128
    dtype: str = "bf16"
    seed: int = 1003
    context: int = 32768       # prefilled context length the state stands for
    prefix_tokens: int = 128   # trailing prefix tokens actually drawn
    steps: int = 1000

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def scaled(self, **kw) -> "DecodeWorkload":
        return replace(self, **kw)


DECODE = DecodeWorkload()


def _softplus(x):
    return np.logaddexp(0.0, x)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _cast(x: np.ndarray, dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dtype)


def _draw_tokens(rng, kind, B, T, H, dk, dv):
    """q, k, v (float32 numpy), g, eta, following the family's recipe."""
    shp = (B, T, H)
    q = rng.standard_normal(shp + (dk,), dtype=np.float32)
    z = rng.standard_normal(shp + (dk,), dtype=np.float32)
    v = rng.standard_normal(shp + (dv,), dtype=np.float32)
    if kind == "tiny":
        k = z
        g = -_softplus(rng.normal(2.0, 1.0, shp))
        eta = _sigmoid(rng.standard_normal(shp))
    elif kind in ("layer", "long"):
        s = np.exp(rng.uniform(np.log(0.25), np.log(4.0), shp))
        k = z * s[..., None].astype(np.float32)
        g = -_softplus(rng.normal(3.0, 1.0, shp))
        eta = _sigmoid(rng.standard_normal(shp))
        if kind == "long":
            strong = rng.random((B, T)) < 0.01
            gs = rng.uniform(-5.0, -2.0, (B, T))
            g = np.where(strong[..., None], gs[..., None], g)
    elif kind == "stress":
        rho = np.exp(rng.uniform(np.log(1e-2), np.log(1e2), shp))
        nz = np.sqrt((z.astype(np.float64) ** 2).sum(-1))
        k = (z / np.maximum(nz, 1e-30)[..., None] * rho[..., None]).astype(np.float32)
        zero_gate = rng.random(shp) < 0.5
        gd = -_softplus(rng.normal(1.0, 2.0, shp))
        g = np.where(zero_gate, 0.0, gd)
        eta = rng.uniform(0.0, 2.0, shp)
    else:
        raise ValueError(kind)
    return q, k, v, g.astype(np.float32), eta.astype(np.float32)


def channel_gates(shape, seed: int) -> torch.Tensor:
    """Per-key-channel log-gates of the given shape (last axis = channel),
    fp32: g = -softplus(N(3, 1.5)), drawn from their own seeded stream."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return torch.from_numpy((-_softplus(rng.normal(3.0, 1.5, shape))).astype(np.float32))


def make_prefill(w: Workload, with_h0: Optional[bool] = None):
    """Inputs of a prefill workload as host tensors.

    Returns a dict with q, k, v (``w.dtype``), g, eta (fp32, [B,T,H]),
    h0 (fp32 [B,H,dk,dv] or None), eps and chunk.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed))
    q, k, v, g, eta = _draw_tokens(rng, w.kind, w.B, w.T, w.H, w.dk, w.dv)
    if with_h0 is None:
        with_h0 = w.kind == "stress"
    h0 = None
    if with_h0:
        h0 = torch.from_numpy(
            rng.normal(0.0, 0.1, (w.B, w.H, w.dk, w.dv)).astype(np.float32))
    dt = w.torch_dtype
    return dict(q=_cast(q, dt), k=_cast(k, dt), v=_cast(v, dt),
                g=torch.from_numpy(g), eta=torch.from_numpy(eta), h0=h0,
                eps=EPS, chunk=CHUNK)


def make_decode(w: DecodeWorkload = DECODE, steps: Optional[int] = None):
    """Inputs of the decode workload as host tensors.

    ``prefix``: the trailing ``prefix_tokens`` tokens of the prefilled context
    (q, k, v, g, eta shaped [B, P, H, d] / [B, P, H]); ``steps``: the new
    tokens, q, k, v [S, B, H, d] and g, eta [S, B, H].
    """
    n = w.steps if steps is None else steps
    rng = np.random.Generator(np.random.PCG64(w.seed))
    pq, pk, pv, pg, pe = _draw_tokens(rng, "layer", w.B, w.prefix_tokens, w.H, w.dk, w.dv)
    sq, sk, sv, sg, se = _draw_tokens(rng, "layer", w.B, n, w.H, w.dk, w.dv)
    dt = w.torch_dtype
    tr = lambda x: np.ascontiguousarray(np.swapaxes(x, 0, 1))  # [B,S,..] -> [S,B,..]
    prefix = dict(q=_cast(pq, dt), k=_cast(pk, dt), v=_cast(pv, dt),
                  g=torch.from_numpy(pg), eta=torch.from_numpy(pe))
    steps_ = dict(q=_cast(tr(sq), dt), k=_cast(tr(sk), dt), v=_cast(tr(sv), dt),
                  g=torch.from_numpy(tr(sg)), eta=torch.from_numpy(tr(se)))
    return dict(prefix=prefix, steps=steps_, eps=EPS)
