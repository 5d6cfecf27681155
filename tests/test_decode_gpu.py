"""Decode step (kla_decode_step) against the fp64 oracle, on the GPU."""
import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_kla_b200 import api, inputs

from helpers import TOL, cuda, oracle_decode_state, rel

pytestmark = pytest.mark.gpu


def _run(w, nsteps, dtype_name):
    d = inputs.make_decode(w, steps=nsteps)
    S0 = oracle_decode_state(d)
    S = cuda(S0.clone())
    Sref = oracle.f64(S0)
    st = d["steps"]
    errs_o, errs_dS = [], []
    for i in range(nsteps):
        q, k, v, g, e = (cuda(st[n][i]) for n in ("q", "k", "v", "g", "eta"))
        S_prev = S.clone()
        o = api.decode_step(q, k, v, g, e, S, eps=d["eps"])
        o_ref, Sref_new = oracle.decode_step(st["q"][i], st["k"][i], st["v"][i],
                                             st["g"][i], st["eta"][i], d["eps"], Sref)
        errs_o.append(rel(o, o_ref))
        # the change of the state this step (stricter than S itself)
        a = np.exp(oracle.f64(st["g"][i]))[..., None, None]
        dS = oracle.f64(S) - a * oracle.f64(S_prev)
        dS_ref = Sref_new - a * Sref
        errs_dS.append(rel(dS, dS_ref))
        Sref = Sref_new
    torch.cuda.synchronize()
    return max(errs_o), rel(S, Sref), max(errs_dS)


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_small(dt, d):
    w = inputs.DECODE.scaled(B=3, H=5, dk=d, dv=d, dtype=dt, prefix_tokens=40)
    eo, eS, edS = _run(w, 6, dt)
    assert eo < TOL[dt] and eS < TOL[dt] and edS < TOL[dt], (eo, eS, edS)


def test_decode_full_size_state():
    """B=64, H=16, d=128 with the 32K-prefix state, 3 steps."""
    eo, eS, edS = _run(inputs.DECODE, 3, "bf16")
    assert eo < 1e-2 and eS < 1e-2 and edS < 1e-2, (eo, eS, edS)


def test_decode_thousand_steps():
    """1000 consecutive in-place steps against 1000 oracle steps."""
    w = inputs.DECODE.scaled(B=2, H=2, prefix_tokens=32)
    eo, eS, edS = _run(w, 1000, "bf16")
    assert eo < 1e-2 and eS < 1e-2 and edS < 1e-2, (eo, eS, edS)


def test_decode_fp32_tight():
    """fp32 I/O: every operation is fp32, the bar is 1e-4."""
    w = inputs.DECODE.scaled(B=4, H=4, dtype="fp32", prefix_tokens=32)
    eo, eS, edS = _run(w, 20, "fp32")
    assert eo < 1e-4 and eS < 1e-4 and edS < 1e-4, (eo, eS, edS)


def test_decode_degenerate_tokens():
    """Zero keys (beta = eta / eps: no write lands), eta = 0 (pure decay),
    g = 0 (no decay) and g = -40 (the state is wiped), per (b, h)."""
    w = inputs.DECODE.scaled(B=4, H=4, prefix_tokens=32)
    d = inputs.make_decode(w, steps=4)
    st = d["steps"]
    st["k"][0, 0] = 0
    st["eta"][1, 1] = 0.0
    st["g"][2, 2] = 0.0
    st["g"][3, 3] = -40.0
    S0 = oracle_decode_state(d)
    S = cuda(S0.clone())
    Sref = oracle.f64(S0)
    for i in range(4):
        q, k, v, g, e = (cuda(st[n][i]) for n in ("q", "k", "v", "g", "eta"))
        o = api.decode_step(q, k, v, g, e, S, eps=d["eps"])
        o_ref, Sref = oracle.decode_step(st["q"][i], st["k"][i], st["v"][i], st["g"][i],
                                         st["eta"][i], d["eps"], Sref)
        assert np.isfinite(oracle.f64(o)).all()
        assert rel(o, o_ref) < TOL["bf16"]
    torch.cuda.synchronize()
    assert rel(S, Sref) < TOL["bf16"]
