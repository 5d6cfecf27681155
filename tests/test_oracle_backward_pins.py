"""Pins for the oracle's gradients of KLA (reverse mode through the token
loop; the pages print no backward algorithm): central finite differences
of the separately pinned forward oracle, the Euler identities of the two
linear dependences (o is linear in q; (o, h_T) jointly linear in (v, h0)),
and a one-token closed form."""
import numpy as np
import pytest

import oracle


def _problem(seed, B=1, T=7, H=2, dk=5, dv=4, gate=True):
    r = np.random.Generator(np.random.PCG64(seed))
    q = r.standard_normal((B, T, H, dk))
    k = r.standard_normal((B, T, H, dk)) * np.exp(r.uniform(-0.7, 0.7, (B, T, H, 1)))
    v = r.standard_normal((B, T, H, dv))
    g = -np.log1p(np.exp(r.normal(0.5, 1.0, (B, T, H)))) if gate else np.zeros((B, T, H))
    eta = r.uniform(0.2, 1.8, (B, T, H))
    h0 = r.standard_normal((B, H, dk, dv)) * 0.3
    dout = r.standard_normal((B, T, H, dv))
    dhT = r.standard_normal((B, H, dk, dv))
    return dict(q=q, k=k, v=v, g=g, eta=eta, h0=h0), dout, dhT


def _loss(x, eps, dout, dhT):
    o, hT = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["eta"], eps, x["h0"])
    return float((o * dout).sum() + (hT * dhT).sum())


@pytest.mark.parametrize("eps", [1e-6, 0.5])
def test_gradients_match_finite_differences(eps):
    x, dout, dhT = _problem(31)
    gr = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["eta"], eps, x["h0"], dout, dhT)
    r = np.random.Generator(np.random.PCG64(32))
    names = dict(q="dq", k="dk", v="dv", g="dg", eta="deta", h0="dh0")
    for name, gname in names.items():
        for trial in range(2):
            d = r.standard_normal(x[name].shape)
            h = 1e-6
            xp = dict(x); xp[name] = x[name] + h * d
            xm = dict(x); xm[name] = x[name] - h * d
            fd = (_loss(xp, eps, dout, dhT) - _loss(xm, eps, dout, dhT)) / (2 * h)
            an = float((gr[gname] * d).sum())
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_euler_identities():
    x, dout, dhT = _problem(33, T=9)
    eps = 1e-6
    gr = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["eta"], eps, x["h0"], dout, dhT)
    o, hT = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["eta"], eps, x["h0"])
    lo = float((o * dout).sum())
    lh = float((hT * dhT).sum())
    assert abs(float((gr["dq"] * x["q"]).sum()) - lo) < 1e-10 * max(1.0, abs(lo))
    lin = float((gr["dv"] * x["v"]).sum() + (gr["dh0"] * x["h0"]).sum())
    assert abs(lin - (lo + lh)) < 1e-10 * max(1.0, abs(lo + lh))


def test_one_token_closed_form():
    """T = 1, h0 = 0: o = beta (k . q) v, so dv = beta (k . q) dout and
    dq = beta (v . dout) k."""
    x, dout, _ = _problem(34, T=1, H=1)
    x["h0"] = np.zeros_like(x["h0"])
    eps = 0.25
    gr = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["eta"], eps, None, dout, None)
    k = x["k"][0, 0, 0]; q = x["q"][0, 0, 0]; v = x["v"][0, 0, 0]; do = dout[0, 0, 0]
    beta = x["eta"][0, 0, 0] / (k @ k + eps)
    np.testing.assert_allclose(gr["dv"][0, 0, 0], beta * (k @ q) * do, rtol=1e-12)
    np.testing.assert_allclose(gr["dq"][0, 0, 0], beta * (v @ do) * k, rtol=1e-12)
    assert abs(gr["dg"][0, 0, 0]) < 1e-12  # alpha multiplies the zero state only


def test_gated_delta_gradients_match_finite_differences():
    """The gated delta form (beta given): its gradients against central
    differences of the separately pinned gated_delta forward."""
    x, dout, dhT = _problem(35, T=6)
    r = np.random.Generator(np.random.PCG64(36))
    x["beta"] = r.uniform(0.1, 1.9, x["eta"].shape)
    gr = oracle.gated_delta_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], dout,
                                     dhT)

    def loss(y):
        o, hT = oracle.gated_delta(y["q"], y["k"], y["v"], y["g"], y["beta"], y["h0"])
        return float((o * dout).sum() + (hT * dhT).sum())

    names = dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", h0="dh0")
    for name, gname in names.items():
        d = r.standard_normal(x[name].shape)
        h = 1e-6
        xp = dict(x); xp[name] = x[name] + h * d
        xm = dict(x); xm[name] = x[name] - h * d
        fd = (loss(xp) - loss(xm)) / (2 * h)
        an = float((gr[gname] * d).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def _kda_problem(seed, T=6, H=2, dk=5, dv=4):
    x, dout, dhT = _problem(seed, T=T, H=H, dk=dk, dv=dv)
    r = np.random.Generator(np.random.PCG64(seed + 100))
    x["gv"] = -np.log1p(np.exp(r.normal(0.5, 1.5, x["k"].shape)))  # per key channel
    x["beta"] = r.uniform(0.1, 1.9, x["eta"].shape)
    return x, dout, dhT


@pytest.mark.parametrize("form", ["beta", "kla"])
def test_kda_gradients_match_finite_differences(form):
    """Per-channel gate: gradients against central differences of the pinned
    per-channel-gate forward, for beta given and for the KLA step size."""
    x, dout, dhT = _kda_problem(37)
    eps = 1e-6
    step = "beta" if form == "beta" else "eta"
    if form == "beta":
        gr = oracle.kda_backward_beta(x["q"], x["k"], x["v"], x["gv"], x["beta"], x["h0"], dout,
                                      dhT)
    else:
        gr = oracle.kda_backward(x["q"], x["k"], x["v"], x["gv"], x["eta"], eps, x["h0"], dout,
                                 dhT)

    def loss(y):
        if form == "beta":
            o, hT = oracle.kda(y["q"], y["k"], y["v"], y["gv"], y["beta"], y["h0"])
        else:
            o, hT = oracle.kda_forward(y["q"], y["k"], y["v"], y["gv"], y["eta"], eps, y["h0"])
        return float((o * dout).sum() + (hT * dhT).sum())

    r = np.random.Generator(np.random.PCG64(38))
    names = dict(q="dq", k="dk", v="dv", gv="dg", h0="dh0")
    names[step] = "dbeta" if form == "beta" else "deta"
    for name, gname in names.items():
        d = r.standard_normal(x[name].shape)
        h = 1e-6
        xp = dict(x); xp[name] = x[name] + h * d
        xm = dict(x); xm[name] = x[name] - h * d
        fd = (loss(xp) - loss(xm)) / (2 * h)
        an = float((gr[gname] * d).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_kda_gradients_reduce_to_scalar_gate():
    """A per-channel gate equal on every channel is the scalar gate: the
    per-channel gradients equal the gated delta ones, and the channel sum of
    dg is the scalar dg."""
    x, dout, dhT = _kda_problem(39)
    gv = np.repeat(x["g"][..., None], x["k"].shape[-1], axis=-1)
    a = oracle.kda_backward_beta(x["q"], x["k"], x["v"], gv, x["beta"], x["h0"], dout, dhT)
    b = oracle.gated_delta_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], dout,
                                    dhT)
    for n in ("dq", "dk", "dv", "dbeta", "dh0"):
        np.testing.assert_allclose(a[n], b[n], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(a["dg"].sum(-1), b["dg"], rtol=1e-10, atol=1e-12)


# ---- the chunkwise adjoint (the algebra the GPU backward kernels follow),
# evaluated in fp64 by oracle.chunk_form and held to the token-loop gradients
# above: chunk lengths 1 (no intra-chunk coupling), 3 and 8 (ragged chunks)
# and 64 (the GPU's), a sequence that ends inside a chunk, and gates strong
# enough that e^G underflows inside a chunk.

from oracle import chunk_form  # noqa: E402


@pytest.mark.parametrize("C", [1, 3, 8, 64])
def test_chunk_form_backward_matches_token_loop(C):
    x, dout, dhT = _problem(41, B=2, T=150, H=2, dk=6, dv=5)
    eps = 1e-6
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["eta"], eps, x["h0"], dout, dhT)
    got = chunk_form.backward(x["q"], x["k"], x["v"], x["g"], x["eta"], eps, x["h0"], dout, dhT,
                              C=C)
    for n in ("dq", "dk", "dv", "dg", "deta", "dh0"):
        assert oracle.rel_l2(got[n], ref[n]) < 1e-12, (C, n)


def test_chunk_form_backward_gated_delta_and_strong_gates():
    x, dout, dhT = _problem(42, T=130, dk=6, dv=5)
    r = np.random.Generator(np.random.PCG64(43))
    x["g"] = np.where(r.uniform(size=x["g"].shape) < 0.3, -40.0, x["g"])  # e^G underflows
    beta = r.uniform(0.05, 1.5, x["g"].shape)
    ref = oracle.gated_delta_backward(x["q"], x["k"], x["v"], x["g"], beta, x["h0"], dout, dhT)
    got = chunk_form.gated_delta_backward(x["q"], x["k"], x["v"], x["g"], beta, x["h0"], dout,
                                          dhT, C=64)
    for n in ("dq", "dk", "dv", "dg", "dbeta", "dh0"):
        assert np.all(np.isfinite(got[n])), n
        assert oracle.rel_l2(got[n], ref[n]) < 1e-11, n


def _kda_chunk_problem(seed, T=150, dk=6, dv=5, strong=False):
    r = np.random.Generator(np.random.PCG64(seed))
    B, H = 1, 2
    q = r.standard_normal((B, T, H, dk))
    k = r.standard_normal((B, T, H, dk)) * 0.6
    v = r.standard_normal((B, T, H, dv))
    g = -np.log1p(np.exp(r.normal(1.0, 1.5, (B, T, H, dk))))
    if strong:  # some channels wiped: e^G underflows inside a chunk
        g = np.where(r.uniform(size=g.shape) < 0.3, -40.0, g)
    beta = r.uniform(0.1, 1.2, (B, T, H))
    h0 = r.standard_normal((B, H, dk, dv)) * 0.3
    return q, k, v, g, beta, h0, r.standard_normal((B, T, H, dv)), r.standard_normal(h0.shape)


@pytest.mark.parametrize("C", [1, 3, 8, 64])
def test_kda_chunk_form_matches_token_loop(C):
    """The per-channel-gate chunk form (the algebra of the per-channel prep
    kernel) and its reverse mode, against the token-loop oracle."""
    q, k, v, g, beta, h0, do, dhT = _kda_chunk_problem(51)
    o_ref, h_ref = oracle.kda(q, k, v, g, beta, h0)
    o, hT = chunk_form.kda_forward(q, k, v, g, beta, h0, C=C)
    assert oracle.rel_l2(o, o_ref) < 1e-12 and oracle.rel_l2(hT, h_ref) < 1e-12
    ref = oracle.kda_backward_beta(q, k, v, g, beta, h0, do, dhT)
    got = chunk_form.kda_backward_beta(q, k, v, g, beta, h0, do, dhT, C=C)
    for n in ("dq", "dk", "dv", "dg", "dbeta", "dh0"):
        assert oracle.rel_l2(got[n], ref[n]) < 1e-12, (C, n)


def test_kda_chunk_form_strong_channel_gates():
    q, k, v, g, beta, h0, do, dhT = _kda_chunk_problem(52, T=130, strong=True)
    ref = oracle.kda_backward_beta(q, k, v, g, beta, h0, do, dhT)
    got = chunk_form.kda_backward_beta(q, k, v, g, beta, h0, do, dhT, C=64)
    for n in ("dq", "dk", "dv", "dg", "dbeta", "dh0"):
        assert np.all(np.isfinite(got[n])), n
        assert oracle.rel_l2(got[n], ref[n]) < 1e-11, n
