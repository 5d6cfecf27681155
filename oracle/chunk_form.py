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

The module also holds the reverse mode of the same chunk form (the
chunkwise adjoint, derived below since the pages print no backward), and
the chunk form of the per-channel-gate rule with its reverse mode, all
pinned against the oracle's token loops for C in {1, 3, 8, 64}.
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


# ---------------------------------------------------------------- reverse mode
#
# The pages print no backward.  Differentiating the chunk form above by hand
# (loss L with dL/do and dL/dh_T given) splits it into one reverse chain over
# the chunks and independent per-chunk terms.  With Gam_rs = e^{G_r - G_s},
# gam = e^G, gC = e^{G_{C-1}}, Qt = diag(gam) Q, Kt = diag(gC / gam) K, the
# strict (s < r) and inclusive (s <= r) masks, and dH the adjoint of the
# state after the chunk:
#
#   dV' = P^T dO + Kt dH                     (V' enters O and h_{n+1})
#   dh_n = gC dH + Qt^T dO - W^T dV'         (the chain, chunk by chunk)
#   dP = (dO V'^T) masked inclusive;  dQ = diag(gam) dO h_n^T + (dP * Gam) K
#   dW = -dV' h_n^T;  dU = dV';  dT = dW (diag(beta gam) K)^T + dU (diag(beta) V)^T
#   dA = -strict(T^T dT T^T)                 (T = (I + A)^{-1})
#   dK = (dP * Gam)^T Q + diag(gC / gam) V' dH^T + diag(beta gam) T^T dW
#        + diag(beta) (dA * Gam) K + (diag(beta) (dA * Gam))^T K
#   dV = diag(beta) T^T dU
#   dbeta = gam * rowdot(T^T dW, K) + rowdot(T^T dU, V) + rowsum(dA * Gam * K K^T)
#   dG = rowsum - colsum of (dA * A) and of (dP * P) + rowdot(dO, Qt h_n)
#        + beta gam rowdot(T^T dW, K) - rowdot(V' dH^T, Kt),
#   dG_{C-1} += sum rowdot(V' dH^T, Kt) + gC <dH, h_n>,
#   dg = reverse in-chunk cumsum of dG (G_r = sum_{j <= r} g_j).
#
# It is pinned in the tests against the token-loop gradients of the oracle
# (themselves pinned by finite differences) for several chunk lengths.

def _chunk_head_backward(q, k, v, g, beta, h, do, dh, C):
    """One head, beta given.  Returns dq, dk, dv, dg, dbeta, dh0."""
    T, dk = k.shape
    dv = v.shape[1]
    nchunks = (T + C - 1) // C
    pad = nchunks * C - T
    if pad:  # identity steps, as in the forward; their gradients are dropped
        z = lambda a, w: np.concatenate([a, np.zeros((pad, w))])
        q, k, v, do = z(q, dk), z(k, dk), z(v, dv), z(do, dv)
        g = np.concatenate([g, np.zeros(pad)])
        beta = np.concatenate([beta, np.zeros(pad)])
    r_idx = np.arange(C)[:, None]
    s_idx = np.arange(C)[None, :]
    strict = s_idx < r_idx
    incl = s_idx <= r_idx
    # forward, keeping what the reverse pass reads
    saved = []
    h = h.copy()
    for n in range(nchunks):
        sl = slice(n * C, (n + 1) * C)
        Q, K, V, bb = q[sl], k[sl], v[sl], beta[sl]
        G = np.cumsum(g[sl])
        D = G[:, None] - G[None, :]
        Gam = np.exp(np.where(incl, D, 0.0)) * incl
        A = bb[:, None] * (K @ K.T) * Gam * strict
        Tm = np.linalg.inv(np.eye(C) + A)
        gam = np.exp(G)
        W = Tm @ ((bb * gam)[:, None] * K)
        Vp = Tm @ (bb[:, None] * V) - W @ h
        P = (Q @ K.T) * Gam
        Kt = np.exp(G[-1] - G)[:, None] * K
        saved.append((h.copy(), G, Gam, A, Tm, gam, W, Vp, P, Kt))
        h = np.exp(G[-1]) * h + Kt.T @ Vp
    out_q, out_k, out_v = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    out_g, out_b = np.zeros(len(g)), np.zeros(len(g))
    dH = dh.copy()
    for n in range(nchunks - 1, -1, -1):
        sl = slice(n * C, (n + 1) * C)
        Q, K, V, bb, dO = q[sl], k[sl], v[sl], beta[sl], do[sl]
        hn, G, Gam, A, Tm, gam, W, Vp, P, Kt = saved[n]
        gC = np.exp(G[-1])
        Qt = gam[:, None] * Q
        dVp = P.T @ dO + Kt @ dH
        dP = (dO @ Vp.T) * incl
        dPG = dP * Gam
        dKt = Vp @ dH.T
        TdW = Tm.T @ (-dVp @ hn.T)
        TdU = Tm.T @ dVp
        dT = (-dVp @ hn.T) @ ((bb * gam)[:, None] * K).T + dVp @ (bb[:, None] * V).T
        dA = -(Tm.T @ dT @ Tm.T) * strict
        E = dA * Gam
        out_q[sl] = gam[:, None] * (dO @ hn.T) + dPG @ K
        out_k[sl] = (dPG.T @ Q + np.exp(G[-1] - G)[:, None] * dKt + (bb * gam)[:, None] * TdW
                     + bb[:, None] * (E @ K) + (bb[:, None] * E).T @ K)
        out_v[sl] = bb[:, None] * TdU
        out_b[sl] = (gam * (TdW * K).sum(1) + (TdU * V).sum(1) + (E * (K @ K.T)).sum(1))
        FA, FP = dA * A, dP * P
        dG = (FA.sum(1) - FA.sum(0) + FP.sum(1) - FP.sum(0) + (dO * (Qt @ hn)).sum(1)
              + bb * gam * (TdW * K).sum(1) - (dKt * Kt).sum(1))
        dG[-1] += (dKt * Kt).sum() + gC * (dH * hn).sum()
        out_g[sl] = np.cumsum(dG[::-1])[::-1]
        dH = gC * dH + Qt.T @ dO - W.T @ dVp
    return out_q[:T], out_k[:T], out_v[:T], out_g[:T], out_b[:T], dH


def gated_delta_backward(q, k, v, g, beta, h0, do, dhT, C: int = 64):
    """Chunk-form gradients of the gated delta rule (beta given) for
    dL/do = do and dL/dh_T = dhT.  Returns dq, dk, dv, dg, dbeta, dh0 (fp64)."""
    q, k, v, g, beta, do = map(f64, (q, k, v, g, beta, do))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    h0 = np.zeros((B, H, dk, dv)) if h0 is None else f64(h0)
    dhT = np.zeros((B, H, dk, dv)) if dhT is None else f64(dhT)
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dg=np.zeros((B, T, H)), dbeta=np.zeros((B, T, H)), dh0=np.zeros((B, H, dk, dv)))
    for b in range(B):
        for hh in range(H):
            r = _chunk_head_backward(q[b, :, hh], k[b, :, hh], v[b, :, hh], g[b, :, hh],
                                     beta[b, :, hh], h0[b, hh], do[b, :, hh], dhT[b, hh], C)
            for name, x in zip(("dq", "dk", "dv", "dg", "dbeta"), r[:5]):
                out[name][b, :, hh] = x
            out["dh0"][b, hh] = r[5]
    return out


def backward(q, k, v, g, eta, eps: float, h0, do, dhT, C: int = 64):
    """Chunk-form gradients of KLA (beta = eta / (||k||^2 + eps), "Kaczmarz
    Linear Attention", Abstract): the gated-delta gradients above, then the
    step size's chain rule, deta = dbeta / (||k||^2 + eps) and
    dk -= 2 dbeta eta k / (||k||^2 + eps)^2.  Returns dq, dk, dv, dg, deta,
    dh0 (fp64)."""
    k64, eta64 = f64(k), f64(eta)
    den = (k64 * k64).sum(-1) + eps
    out = gated_delta_backward(q, k64, v, g, eta64 / den, h0, do, dhT, C)
    dbeta = out.pop("dbeta")
    out["deta"] = dbeta / den
    out["dk"] = out["dk"] - (2.0 * dbeta * eta64 / den ** 2)[..., None] * k64
    return out


# ---------------------------------------------------------------- per-channel gate
#
# The chunk form of the per-channel-gate rule ("Deep Dive into KDA", section
# 2.3, decay before the erase): one log-gate per key channel, G [C, dk] its
# in-chunk cumsum, and E[r, s, i] = e^{G_ri - G_si} for s <= r (never above
# 1).  Unrolling the recurrence over a chunk from h_n gives
#
#   A_rs = beta_r sum_i k_ri k_si E_rsi  (s < r),   T = (I + A)^{-1}
#   W = T diag(beta) (K o e^G),  U = T diag(beta) V,  V' = U - W h_n
#   O = (Q o e^G) h_n + P V',   P_rs = sum_i q_ri k_si E_rsi  (s <= r)
#   h_{n+1} = Diag(e^{G_last}) h_n + (K o e^{G_last - G})^T V'
#
# and its reverse mode (dH the adjoint of h_{n+1}; every per-channel decay
# passes its gradient to G channel by channel, dg being the reverse
# in-chunk cumsum of dG per channel):
#
#   dV' = P^T dO + Kt dH,  dh_n = Diag(e^{G_last}) dH + Qg^T dO - W^T dV'
#   dP = (dO V'^T) masked inclusive,  dW = -dV' h_n^T,  dU = dV'
#   dKg = diag(beta) T^T dW,  dV = diag(beta) T^T dU
#   dT = dW (diag(beta) Kg)^T + dU (diag(beta) V)^T,  dA = -strict(T^T dT T^T)
#   dbeta = rowdot(T^T dW, Kg) + rowdot(T^T dU, V) + rowsum(dA * KKE)
#   through KKE_rs = sum_i k_ri k_si E_rsi (weight beta_r dA_rs) and
#   QKE_rs = sum_i q_ri k_si E_rsi (weight dP_rs): the products' gradients
#   to the rows, + to G_ri and - to G_si of each term;
#   Qg = Q o e^G, Kg = K o e^G, Kt = K o e^{G_last - G} and the state decay:
#   elementwise, with Kt's and the decay's share of G_last on row C - 1.

def _kda_chunk_head(q, k, v, g, beta, h, do, dh, C):
    """One head, beta given, per-channel gate g [T, dk]: the outputs, the
    final state and (with do, dh given) the gradients."""
    T, dk = k.shape
    dv = v.shape[1]
    nchunks = (T + C - 1) // C
    pad = nchunks * C - T
    if pad:
        z = lambda a, w: np.concatenate([a, np.zeros((pad, w))])
        q, k, v, g = z(q, dk), z(k, dk), z(v, dv), z(g, dk)
        do = z(do, dv) if do is not None else None
        beta = np.concatenate([beta, np.zeros(pad)])
    incl = np.tril(np.ones((C, C), dtype=bool))
    strict = np.tril(np.ones((C, C), dtype=bool), -1)
    o = np.zeros((nchunks * C, dv))
    saved = []
    h = h.copy()
    for n in range(nchunks):
        sl = slice(n * C, (n + 1) * C)
        Q, K, V, bb = q[sl], k[sl], v[sl], beta[sl]
        G = np.cumsum(g[sl], axis=0)
        D = G[:, None, :] - G[None, :, :]                      # [r, s, i]
        E = np.exp(np.where(incl[:, :, None], D, 0.0)) * incl[:, :, None]
        KKE = np.einsum("ri,si,rsi->rs", K, K, E)
        QKE = np.einsum("ri,si,rsi->rs", Q, K, E)
        A = bb[:, None] * KKE * strict
        Tm = np.linalg.inv(np.eye(C) + A)
        eG, eL = np.exp(G), np.exp(G[-1])
        Kg, Qg, Kt = K * eG, Q * eG, K * np.exp(G[-1][None, :] - G)
        W = Tm @ (bb[:, None] * Kg)
        Vp = Tm @ (bb[:, None] * V) - W @ h
        o[sl] = Qg @ h + QKE @ Vp
        saved.append((h.copy(), G, E, KKE, QKE, Tm, Kg, Qg, Kt, W, Vp))
        h = eL[:, None] * h + Kt.T @ Vp
    if do is None:
        return o[:T], h
    dq_, dk_, dv_ = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dg_, db_ = np.zeros_like(g), np.zeros(len(beta))
    dH = dh.copy()
    for n in range(nchunks - 1, -1, -1):
        sl = slice(n * C, (n + 1) * C)
        Q, K, V, bb, dO = q[sl], k[sl], v[sl], beta[sl], do[sl]
        hn, G, E, KKE, QKE, Tm, Kg, Qg, Kt, W, Vp = saved[n]
        eG, eL = np.exp(G), np.exp(G[-1])
        P = QKE * incl
        dVp = P.T @ dO + Kt @ dH
        dP = (dO @ Vp.T) * incl
        dW = -dVp @ hn.T
        TdW, TdU = Tm.T @ dW, Tm.T @ dVp
        dT = dW @ (bb[:, None] * Kg).T + dVp @ (bb[:, None] * V).T
        dA = -(Tm.T @ dT @ Tm.T) * strict
        dKKE = bb[:, None] * dA
        dQ = np.einsum("rs,si,rsi->ri", dP, K, E) + (dO @ hn.T) * eG
        dK = (np.einsum("rs,si,rsi->ri", dKKE, K, E) + np.einsum("rs,ri,rsi->si", dKKE, K, E)
              + np.einsum("rs,ri,rsi->si", dP, Q, E))
        dKg = bb[:, None] * TdW
        dKt = Vp @ dH.T
        dK += dKg * eG + dKt * np.exp(G[-1][None, :] - G)
        # G: the per-channel decays inside KKE and QKE, then the elementwise ones
        FK = np.einsum("rs,ri,si,rsi->rsi", dKKE, K, K, E)
        FQ = np.einsum("rs,ri,si,rsi->rsi", dP, Q, K, E)
        dG = FK.sum(1) - FK.sum(0) + FQ.sum(1) - FQ.sum(0)
        dG += (dO @ hn.T) * Qg + dKg * Kg - dKt * Kt
        dG[-1] += (dKt * Kt).sum(0) + eL * (dH * hn).sum(1)
        dq_[sl], dk_[sl] = dQ, dK
        dv_[sl] = bb[:, None] * TdU
        db_[sl] = (TdW * Kg).sum(1) + (TdU * V).sum(1) + (dA * KKE).sum(1)
        dg_[sl] = np.cumsum(dG[::-1], axis=0)[::-1]
        dH = eL[:, None] * dH + Qg.T @ dO - W.T @ dVp
    return dq_[:T], dk_[:T], dv_[:T], dg_[:T], db_[:T], dH


def _kda_args(q, k, v, g, beta, h0):
    q, k, v, g, beta = map(f64, (q, k, v, g, beta))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    h0 = np.zeros((B, H, dk, dv)) if h0 is None else f64(h0)
    return q, k, v, g, beta, h0, B, T, H, dk, dv


def kda_forward(q, k, v, g, beta, h0=None, C: int = 64):
    """Chunk-form per-channel-gate rule (beta given, g [B,T,H,dk]).
    Returns (o, hT) in fp64."""
    q, k, v, g, beta, h0, B, T, H, dk, dv = _kda_args(q, k, v, g, beta, h0)
    o, hT = np.zeros((B, T, H, dv)), np.zeros((B, H, dk, dv))
    for b in range(B):
        for hh in range(H):
            o[b, :, hh], hT[b, hh] = _kda_chunk_head(
                q[b, :, hh], k[b, :, hh], v[b, :, hh], g[b, :, hh], beta[b, :, hh], h0[b, hh],
                None, None, C)
    return o, hT


def kda_backward_beta(q, k, v, g, beta, h0, do, dhT, C: int = 64):
    """Chunk-form gradients of the per-channel-gate rule (beta given) for
    dL/do = do and dL/dh_T = dhT.  Returns dq, dk, dv, dg [B,T,H,dk], dbeta,
    dh0 (fp64)."""
    q, k, v, g, beta, h0, B, T, H, dk, dv = _kda_args(q, k, v, g, beta, h0)
    do = f64(do)
    dhT = np.zeros((B, H, dk, dv)) if dhT is None else f64(dhT)
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dg=np.zeros_like(g), dbeta=np.zeros((B, T, H)), dh0=np.zeros((B, H, dk, dv)))
    for b in range(B):
        for hh in range(H):
            r = _kda_chunk_head(q[b, :, hh], k[b, :, hh], v[b, :, hh], g[b, :, hh],
                                beta[b, :, hh], h0[b, hh], do[b, :, hh], dhT[b, hh], C)
            for name, x in zip(("dq", "dk", "dv", "dg", "dbeta"), r[:5]):
                out[name][b, :, hh] = x
            out["dh0"][b, hh] = r[5]
    return out
