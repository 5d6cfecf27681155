"""Chunkwise (UT / WY) form of the KLA recurrence in fp64 NumPy -- TEST UTILITY.

Part of the oracle package and, like it, only for the tests.  It evaluates
the chunkwise parallel algorithm of "Deep Dive into KDA", section 3
(inter-chunk state update and intra-chunk output), specialised to a scalar
gate, with the intermediates U and W -- which that section names but does not
define -- given by the plainest reading consistent with it:

  Within a chunk of C tokens starting from state h_n (h = S^T, [dk, dv]),
  G_r = sum_{j <= r} g_j (chunk-local, inclusive), and u_r defined by
  h_r = alpha_r h_{r-1} + k_r u_r^T, unrolling gives

      (I + A) u = diag(beta) V - diag(beta e^G) K h_n,
      A_rs = beta_r (k_r . k_s) e^{G_r - G_s}   for s < r, else 0,

  so with T = (I + A)^{-1}, W = T diag(beta e^G) K and U = T diag(beta) V:

      V'      = U - W h_n                                   (= u)
      O       = diag(e^G) Q h_n + (Q K^T * M) V',  M_rs = e^{G_r - G_s}, s <= r
      h_{n+1} = e^{G_{C-1}} h_n + sum_s e^{G_{C-1} - G_s} k_s V'_s^T.

  These are the section's Gamma (*) Q S, Tril((Gamma (*) Q)(K / Gamma)^T) and
  (Gamma (*) K)^T terms; the decay ratios are always formed as masked
  differences of G (never K / Gamma), the log-domain advice of the same page
  (section 3 and section 5).

A ragged tail is padded with g = 0, beta = 0 and zero vectors, which is an
exact identity step.  It is pinned against the token recurrence in the tests
for C in {1, 2, 4, 8, 64}; it exposes T, W, U, V' and the per-chunk states so
GPU stages can be checked one by one.
"""
from __future__ import annotations

import numpy as np

from . import f64


def _chunk_head(q, k, v, g, beta, h, C, keep):
    """One head.  q,k [T,dk]; v [T,dv]; g,beta [T]; h [dk,dv] (copied)."""
    T, dk = k.shape
    dv = v.shape[1]
    nchunks = (T + C - 1) // C
    Tp = nchunks * C
    pad = Tp - T
    if pad:
        q = np.concatenate([q, np.zeros((pad, dk))])
        k = np.concatenate([k, np.zeros((pad, dk))])
        v = np.concatenate([v, np.zeros((pad, dv))])
        g = np.concatenate([g, np.zeros(pad)])
        beta = np.concatenate([beta, np.zeros(pad)])
    h = h.copy()
    o = np.zeros((Tp, dv))
    inter = [] if keep else None
    r_idx = np.arange(C)[:, None]
    s_idx = np.arange(C)[None, :]
    strict = s_idx < r_idx
    incl = s_idx <= r_idx
    for n in range(nchunks):
        sl = slice(n * C, (n + 1) * C)
        Q, K, V, gb, bb = q[sl], k[sl], v[sl], g[sl], beta[sl]
        G = np.cumsum(gb)
        D = G[:, None] - G[None, :]
        dec_strict = np.exp(np.where(strict, D, 0.0)) * strict
        dec_incl = np.exp(np.where(incl, D, 0.0)) * incl
        A = bb[:, None] * (K @ K.T) * dec_strict
        Tm = np.linalg.inv(np.eye(C) + A)
        W = Tm @ ((bb * np.exp(G))[:, None] * K)
        U = Tm @ (bb[:, None] * V)
        Vp = U - W @ h
        O = np.exp(G)[:, None] * (Q @ h) + ((Q @ K.T) * dec_incl) @ Vp
        Kt = np.exp(G[-1] - G)[:, None] * K
        if keep:
            inter.append(dict(T=Tm, W=W, U=U, Vp=Vp, h=h.copy(), G=G, A=A))
        h = np.exp(G[-1]) * h + Kt.T @ Vp
        o[sl] = O
    return o[:T], h, inter


def forward(q, k, v, g, beta, h0=None, C: int = 64, keep: bool = False):
    """Chunk-form gated delta rule (beta given).  Returns (o, hT[, inter])."""
    q, k, v, g, beta, h0 = map(f64, (q, k, v, g, beta, h0))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    hT = np.zeros((B, H, dk, dv))
    inters = {}
    for b in range(B):
        for hh in range(H):
            h = h0[b, hh] if h0 is not None else np.zeros((dk, dv))
            ob, hb, it = _chunk_head(q[b, :, hh], k[b, :, hh], v[b, :, hh],
                                     g[b, :, hh], beta[b, :, hh], h, C, keep)
            o[b, :, hh] = ob
            hT[b, hh] = hb
            if keep:
                inters[(b, hh)] = it
    if keep:
        return o, hT, inters
    return o, hT
