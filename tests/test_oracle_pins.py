"""Pins for the fp64 oracle: checks against what the pages and the mathematics
fix, none of which re-types the oracle's own loop.

  * hand-worked exact steps (tests/golden/hand_worked.txt),
  * the Kaczmarz projection identity (KLA Abstract: beta from the key norm),
  * pure decay when eta = 0,
  * the DeltaNet special case ("Deep Dive into KDA", section 2.1) in the
    S-orientation,
  * explicit product-of-matrices unrolling for T <= 8,
  * a scalar closed form (geometric series),
  * exact recall with orthonormal keys,
  * linearity in (V, h0) and continuation across a split,
  * the chunkwise form ("Deep Dive into KDA", section 3) for several C.
"""
import os

import numpy as np
import pytest

import oracle
from oracle import chunk_form

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.txt")


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _rand_problem(seed, B=1, T=12, H=2, dk=8, dv=6, gate=True, h0=True):
    r = _rng(seed)
    q = r.standard_normal((B, T, H, dk))
    k = r.standard_normal((B, T, H, dk)) * np.exp(r.uniform(-1, 1, (B, T, H, 1)))
    v = r.standard_normal((B, T, H, dv))
    g = -np.log1p(np.exp(r.normal(0.5, 1.0, (B, T, H)))) if gate else np.zeros((B, T, H))
    eta = r.uniform(0.1, 1.9, (B, T, H))
    hh = r.standard_normal((B, H, dk, dv)) * 0.3 if h0 else None
    return q, k, v, g, eta, hh


def _rel(a, b):
    return oracle.rel_l2(a, b)


# ----------------------------------------------------------------- golden
def _parse_golden(path):
    cases, cur = {}, None
    for raw in open(path):
        line = raw.split("#", 1)[0].strip()
        if not line:
            continue
        if line.startswith("[case"):
            cur = line[len("[case"):].strip(" ]")
            cases[cur] = {}
            continue
        key, val = (s.strip() for s in line.split("=", 1))
        if val == "none":
            cases[cur][key] = None
        elif key in ("dk", "dv"):
            cases[cur][key] = int(val)
        elif key == "eps":
            cases[cur][key] = float(val)
        else:
            rows = [[float(x) for x in row.split()] for row in val.split(";")]
            cases[cur][key] = np.array(rows)
    return cases


def test_golden_hand_worked():
    cases = _parse_golden(GOLDEN)
    assert len(cases) == 3
    for name, c in cases.items():
        dk, dv = c["dk"], c["dv"]
        k = c["k"].reshape(-1, dk)
        T = k.shape[0]
        sh = lambda x, d: x.reshape(1, T, 1, d)
        g = c["g"].reshape(1, T, 1)
        eta = c["eta"].reshape(1, T, 1)
        h0 = None if c["h0"] is None else c["h0"].reshape(1, 1, dk, dv)
        o, hT = oracle.forward(sh(c["q"], dk), sh(k, dk), sh(c["v"], dv), g, eta,
                               c["eps"], h0)
        np.testing.assert_allclose(o.reshape(T, dv), c["o"].reshape(T, dv),
                                   rtol=1e-14, atol=1e-14, err_msg=name)
        np.testing.assert_allclose(hT.reshape(dk, dv), c["hT"].reshape(dk, dv),
                                   rtol=1e-14, atol=1e-14, err_msg=name)


# ------------------------------------------------------------- projection
@pytest.mark.parametrize("eps", [1e-6, 1e-16])
def test_kaczmarz_projection(eps):
    """alpha = eta = 1: S_t k_t - v_t = eps/(|k_t|^2+eps) (S_{t-1} k_t - v_t)."""
    q, k, v, g, eta, h0 = _rand_problem(11, B=1, T=10, H=1, dk=16, dv=5)
    g[:] = 0.0
    eta[:] = 1.0
    q = k.copy()  # o_t = S_t k_t
    o, _ = oracle.forward(q, k, v, g, eta, eps, h0)
    for t in range(10):
        if t == 0:
            prev = h0[0, 0]
        else:
            _, hp = oracle.forward(q[:, :t], k[:, :t], v[:, :t], g[:, :t],
                                   eta[:, :t], eps, h0)
            prev = hp[0, 0]
        kt, vt = k[0, t, 0], v[0, t, 0]
        res_prev = prev.T @ kt - vt
        res = o[0, t, 0] - vt
        n2 = float(kt @ kt)
        np.testing.assert_allclose(res, eps / (n2 + eps) * res_prev,
                                   rtol=1e-6, atol=1e-12 * np.linalg.norm(vt))
        assert np.linalg.norm(res) <= max(1e-10 * np.linalg.norm(vt),
                                          2 * eps / n2 * np.linalg.norm(res_prev))


# ------------------------------------------------------------- pure decay
def test_pure_decay_eta_zero():
    q, k, v, g, eta, h0 = _rand_problem(12, T=20)
    eta[:] = 0.0
    o, hT = oracle.forward(q, k, v, g, eta, 1e-6, h0)
    cum = np.cumsum(g, axis=1)  # [B,T,H]
    for b in range(q.shape[0]):
        for h in range(q.shape[2]):
            for t in range(q.shape[1]):
                exp_o = np.exp(cum[b, t, h]) * (h0[b, h].T @ q[b, t, h])
                assert _rel(o[b, t, h], exp_o) < 1e-13
            np.testing.assert_allclose(hT[b, h], np.exp(cum[b, -1, h]) * h0[b, h],
                                       rtol=1e-13)


# --------------------------------------------------------------- DeltaNet
def test_deltanet_special_case():
    """g = 0 and a constant beta: S_t = S_{t-1} - beta (S_{t-1} k_t - v_t) k_t^T,
    evaluated on S = h^T (dv x dk), the other orientation."""
    q, k, v, g, eta, h0 = _rand_problem(13, T=15, dk=7, dv=9)
    g[:] = 0.0
    beta = np.full(g.shape, 0.37)
    o, hT = oracle.gated_delta(q, k, v, g, beta, h0)
    B, T, H, _ = q.shape
    for b in range(B):
        for h in range(H):
            S = h0[b, h].T.copy()
            for t in range(T):
                kt, vt = k[b, t, h], v[b, t, h]
                S = S - 0.37 * np.outer(S @ kt - vt, kt)
                np.testing.assert_allclose(o[b, t, h], S @ q[b, t, h], rtol=1e-12,
                                           atol=1e-12)
            np.testing.assert_allclose(hT[b, h], S.T, rtol=1e-12, atol=1e-12)


def test_kla_is_gdn_with_key_norm_beta():
    q, k, v, g, eta, h0 = _rand_problem(14, T=9)
    eps = 1e-3
    beta = eta / ((k * k).sum(-1) + eps)
    o1, h1 = oracle.forward(q, k, v, g, eta, eps, h0)
    o2, h2 = oracle.gated_delta(q, k, v, g, beta, h0)
    assert _rel(o1, o2) < 1e-14 and _rel(h1, h2) < 1e-14
    np.testing.assert_allclose(oracle.beta(k, eta, eps), beta, rtol=1e-15)


# ------------------------------------------------------------- unrolling
@pytest.mark.parametrize("d", [4, 64])
@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_product_unrolling(T, d):
    """S_T = S_0 prod_t M_t + sum_t beta_t v_t k_t^T prod_{j>t} M_j with
    M_t = alpha_t (I - beta_t k_t k_t^T), as explicit d x d matrices."""
    q, k, v, g, eta, h0 = _rand_problem(100 + T + d, B=1, T=T, H=1, dk=d, dv=d)
    eps = 1e-6
    o, hT = oracle.forward(q, k, v, g, eta, eps, h0)
    kk, vv, qq = k[0, :, 0], v[0, :, 0], q[0, :, 0]
    beta = eta[0, :, 0] / ((kk * kk).sum(-1) + eps)
    alpha = np.exp(g[0, :, 0])
    M = [alpha[t] * (np.eye(d) - beta[t] * np.outer(kk[t], kk[t])) for t in range(T)]
    S0 = h0[0, 0].T
    for t_end in range(1, T + 1):
        P = np.eye(d)
        for t in range(t_end):
            P = P @ M[t]
        S = S0 @ P
        for t in range(t_end):
            R = np.eye(d)
            for j in range(t + 1, t_end):
                R = R @ M[j]
            S = S + beta[t] * np.outer(vv[t], kk[t]) @ R
        np.testing.assert_allclose(o[0, t_end - 1, 0], S @ qq[t_end - 1],
                                   rtol=1e-10, atol=1e-11)
        if t_end == T:
            assert _rel(hT[0, 0], S.T) < 1e-12


# ----------------------------------------------------------- closed form
def test_scalar_geometric_series():
    """d = 1 with constant inputs: h_t = a h_{t-1} + c, a = alpha (1 - beta k^2),
    c = beta k v, so h_T = a^T h_0 + c (1 - a^T) / (1 - a)."""
    T, kk, vv, qq, gg, ee, eps, hh0 = 37, 1.7, -0.6, 0.9, -0.2, 0.8, 1e-3, 2.5
    ones = np.ones((1, T, 1, 1))
    o, hT = oracle.forward(ones * qq, ones * kk, ones * vv, np.full((1, T, 1), gg),
                           np.full((1, T, 1), ee), eps, np.full((1, 1, 1, 1), hh0))
    beta = ee / (kk * kk + eps)
    a = np.exp(gg) * (1 - beta * kk * kk)
    c = beta * kk * vv
    t = np.arange(1, T + 1)
    h_t = a ** t * hh0 + c * (1 - a ** t) / (1 - a)
    np.testing.assert_allclose(o[0, :, 0, 0], h_t * qq, rtol=1e-13)
    np.testing.assert_allclose(hT[0, 0, 0, 0], h_t[-1], rtol=1e-13)


def test_orthonormal_keys_exact_recall():
    """alpha = eta = 1, eps = 0 and orthonormal keys: every written pair is
    recalled exactly, S_T k_i = v_i for all i."""
    d, dv = 16, 5
    r = _rng(15)
    Qm, _ = np.linalg.qr(r.standard_normal((d, d)))
    k = Qm.T.reshape(1, d, 1, d)           # rows are orthonormal keys
    v = r.standard_normal((1, d, 1, dv))
    g = np.zeros((1, d, 1))
    eta = np.ones((1, d, 1))
    o, hT = oracle.forward(k, k, v, g, eta, 0.0, None)
    np.testing.assert_allclose(o[0, :, 0], v[0, :, 0], atol=1e-12)
    np.testing.assert_allclose(k[0, :, 0] @ hT[0, 0], v[0, :, 0], atol=1e-12)


# ---------------------------------------------------- linearity/continuation
def test_linear_in_values_and_state():
    q, k, v, g, eta, h0 = _rand_problem(16, T=11)
    _, _, v2, _, _, h02 = _rand_problem(17, T=11)
    a, b = 0.7, -1.3
    o1, s1 = oracle.forward(q, k, v, g, eta, 1e-6, h0)
    o2, s2 = oracle.forward(q, k, v2, g, eta, 1e-6, h02)
    o3, s3 = oracle.forward(q, k, a * v + b * v2, g, eta, 1e-6, a * h0 + b * h02)
    assert _rel(o3, a * o1 + b * o2) < 1e-12
    assert _rel(s3, a * s1 + b * s2) < 1e-12


def test_continuation_and_decode_handoff():
    q, k, v, g, eta, h0 = _rand_problem(18, T=24)
    o, hT = oracle.forward(q, k, v, g, eta, 1e-6, h0)
    oa, ha = oracle.forward(q[:, :10], k[:, :10], v[:, :10], g[:, :10], eta[:, :10], 1e-6, h0)
    ob, hb = oracle.forward(q[:, 10:], k[:, 10:], v[:, 10:], g[:, 10:], eta[:, 10:], 1e-6, ha)
    assert _rel(np.concatenate([oa, ob], axis=1), o) < 1e-13
    assert _rel(hb, hT) < 1e-13
    # decode of the last token from the state the first T-1 tokens leave
    _, hp = oracle.forward(q[:, :-1], k[:, :-1], v[:, :-1], g[:, :-1], eta[:, :-1], 1e-6, h0)
    od, sd = oracle.decode_step(q[:, -1], k[:, -1], v[:, -1], g[:, -1], eta[:, -1], 1e-6, hp)
    assert _rel(od, o[:, -1]) < 1e-13 and _rel(sd, hT) < 1e-13


# ----------------------------------------------------------- chunk form
@pytest.mark.parametrize("C", [1, 2, 4, 8, 64])
def test_chunk_form_matches_recurrence(C):
    q, k, v, g, eta, h0 = _rand_problem(19, B=2, T=150, H=2, dk=8, dv=6)
    eps = 1e-6
    beta = oracle.beta(k, eta, eps)
    o, hT = oracle.forward(q, k, v, g, eta, eps, h0)
    oc, hc = chunk_form.forward(q, k, v, g, beta, h0, C=C)
    assert _rel(oc, o) < 1e-12
    assert _rel(hc, hT) < 1e-12


def test_chunk_form_strong_gates_no_overflow():
    """Strong forgetting (g ~ -3 per token, the 0.4B-layer recipe) makes
    e^{G} underflow inside a chunk; the masked log-difference form must stay
    finite and agree with the recurrence."""
    q, k, v, g, eta, h0 = _rand_problem(20, B=1, T=130, H=1, dk=8, dv=8)
    g = -np.log1p(np.exp(_rng(21).normal(3.0, 1.0, g.shape))) * 10
    beta = oracle.beta(k, eta, 1e-6)
    o, hT = oracle.forward(q, k, v, g, eta, 1e-6, h0)
    oc, hc = chunk_form.forward(q, k, v, g, beta, h0, C=64)
    assert np.isfinite(oc).all() and np.isfinite(hc).all()
    assert _rel(oc, o) < 1e-12
    assert _rel(hc, hT) < 1e-10 or np.abs(hc - hT).max() < 1e-300
