"""Pins for the oracle's per-channel-gate recurrence (KDA form, "Deep Dive
into KDA", section 2.3, with the KLA step size): checks against what the
pages and the mathematics fix, none of which re-types the oracle's loop.

  * hand-worked exact steps (tests/golden/kda_hand_worked.txt),
  * a gate equal on every channel is the scalar gate: the result equals the
    separately pinned scalar-gate oracle,
  * the Kaczmarz projection identity holds for any per-channel gate when the
    erase reads the decayed state (it fails for erase-then-decay),
  * pure per-channel decay when eta = 0 (closed form; the gate scales rows of
    h, the key side),
  * a channel that decays to zero with a zero key entry stays zero,
  * linearity in (V, h0) and continuation across a split.
"""
import os

import numpy as np
import pytest

import oracle
from test_oracle_pins import _parse_golden

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kda_hand_worked.txt")


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _problem(seed, B=1, T=12, H=2, dk=8, dv=6, h0=True):
    r = _rng(seed)
    q = r.standard_normal((B, T, H, dk))
    k = r.standard_normal((B, T, H, dk)) * np.exp(r.uniform(-1, 1, (B, T, H, 1)))
    v = r.standard_normal((B, T, H, dv))
    g = -np.log1p(np.exp(r.normal(0.0, 1.5, (B, T, H, dk))))  # per channel
    eta = r.uniform(0.1, 1.9, (B, T, H))
    hh = r.standard_normal((B, H, dk, dv)) * 0.3 if h0 else None
    return q, k, v, g, eta, hh


def test_golden_hand_worked():
    cases = _parse_golden(GOLDEN)
    assert len(cases) == 3
    for name, c in cases.items():
        dk, dv = c["dk"], c["dv"]
        k = c["k"].reshape(-1, dk)
        T = k.shape[0]
        sh = lambda x, d: x.reshape(1, T, 1, d)
        g = c["g"].reshape(1, T, 1, dk)
        eta = c["eta"].reshape(1, T, 1)
        h0 = None if c["h0"] is None else c["h0"].reshape(1, 1, dk, dv)
        o, hT = oracle.kda_forward(sh(c["q"], dk), sh(k, dk), sh(c["v"], dv), g, eta,
                                   c["eps"], h0)
        np.testing.assert_allclose(o.reshape(T, dv), c["o"].reshape(T, dv),
                                   rtol=1e-14, atol=1e-14, err_msg=name)
        np.testing.assert_allclose(hT.reshape(dk, dv), c["hT"].reshape(dk, dv),
                                   rtol=1e-14, atol=1e-14, err_msg=name)


def test_uniform_gate_is_the_scalar_gate():
    q, k, v, g, eta, h0 = _problem(21, T=17)
    gs = g[..., 0]  # one value per token, copied to every channel
    gv = np.repeat(gs[..., None], k.shape[-1], axis=-1)
    o1, h1 = oracle.kda_forward(q, k, v, gv, eta, 1e-6, h0)
    o2, h2 = oracle.forward(q, k, v, gs, eta, 1e-6, h0)
    assert oracle.rel_l2(o1, o2) < 1e-13 and oracle.rel_l2(h1, h2) < 1e-13


@pytest.mark.parametrize("eps", [1e-6, 1e-16])
def test_kaczmarz_projection_any_channel_gate(eps):
    """eta = 1: after every token S_t k_t = v_t up to eps/(|k|^2+eps) of the
    residual of the decayed state, whatever the per-channel gates."""
    q, k, v, g, eta, h0 = _problem(22, B=1, T=10, H=1, dk=16, dv=5)
    eta[:] = 1.0
    o, _ = oracle.kda_forward(k, k, v, g, eta, eps, h0)  # q = k: o_t = S_t k_t
    for t in range(10):
        n2 = float(k[0, t, 0] @ k[0, t, 0])
        res = np.linalg.norm(o[0, t, 0] - v[0, t, 0])
        assert res <= 1e-10 * np.linalg.norm(v[0, t, 0]) + 50 * eps / n2


def test_pure_channel_decay_eta_zero():
    """eta = 0: h_t = Diag(exp(sum of g)) h0 row by row (key side)."""
    q, k, v, g, eta, h0 = _problem(23, T=15, dk=6, dv=6)
    eta[:] = 0.0
    o, hT = oracle.kda_forward(q, k, v, g, eta, 1e-6, h0)
    cum = np.cumsum(g, axis=1)  # [B,T,H,dk]
    for h in range(q.shape[2]):
        for t in range(q.shape[1]):
            ht = np.exp(cum[0, t, h])[:, None] * h0[0, h]
            assert oracle.rel_l2(o[0, t, h], ht.T @ q[0, t, h]) < 1e-13
        np.testing.assert_allclose(hT[0, h], np.exp(cum[0, -1, h])[:, None] * h0[0, h],
                                   rtol=1e-13)


def test_wiped_channel_stays_zero():
    q, k, v, g, eta, h0 = _problem(24, T=9)
    g[0, 4, :, 3] = -800.0  # channel 3 decays to exactly zero at token 4
    k[0, 4:, :, 3] = 0.0    # ... and is never written again
    _, hT = oracle.kda_forward(q, k, v, g, eta, 1e-6, h0)
    assert np.all(hT[0, :, 3, :] == 0.0)
    assert np.all(np.abs(hT[0, :, :3, :]) > 0)


def test_linear_in_values_and_state_and_continuation():
    q, k, v, g, eta, h0 = _problem(25, T=14)
    _, _, v2, _, _, h02 = _problem(26, T=14)
    a, b = 0.7, -1.3
    o1, h1 = oracle.kda_forward(q, k, v, g, eta, 1e-6, h0)
    o2, h2 = oracle.kda_forward(q, k, v2, g, eta, 1e-6, h02)
    o3, h3 = oracle.kda_forward(q, k, a * v + b * v2, g, eta, 1e-6, a * h0 + b * h02)
    assert oracle.rel_l2(o3, a * o1 + b * o2) < 1e-12
    assert oracle.rel_l2(h3, a * h1 + b * h2) < 1e-12
    # split after 5 tokens, the first part's final state starts the second
    oa, ha = oracle.kda_forward(q[:, :5], k[:, :5], v[:, :5], g[:, :5], eta[:, :5], 1e-6, h0)
    ob, hb = oracle.kda_forward(q[:, 5:], k[:, 5:], v[:, 5:], g[:, 5:], eta[:, 5:], 1e-6, ha)
    assert oracle.rel_l2(np.concatenate([oa, ob], axis=1), o1) < 1e-13
    assert oracle.rel_l2(hb, h1) < 1e-13
