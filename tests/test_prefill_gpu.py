"""Prefill (kla_chunk_fwd / kla_recurrent_fwd) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_kla_b200 import api, inputs

from helpers import TOL, cuda, rel, worst_head_rel

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS


def _check(w, fn, with_h0=None, tol=None):
    x = inputs.make_prefill(w, with_h0=with_h0)
    xc = cuda(x)
    o, hT = fn(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"], xc["h0"])
    torch.cuda.synchronize()
    o_ref, h_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    tol = TOL[w.dtype] if tol is None else tol
    eo, eh = rel(o, o_ref), rel(hT, h_ref)
    assert np.isfinite(oracle.f64(o)).all()
    assert eo < tol and eh < tol, (w, eo, eh, worst_head_rel(o, o_ref))
    return eo, eh


# ------------------------------------------------------- token-serial path
def test_recurrent_tiny_fp32():
    _check(W["tiny"], api.recurrent_fwd)


@pytest.mark.parametrize("T", [1, 63, 65, 200])
def test_recurrent_bf16_layer(T):
    _check(W["prefill_4k"].scaled(B=2, T=T, H=3), api.recurrent_fwd)


def test_recurrent_stress_d64_with_h0():
    _check(W["stress"].scaled(B=1, T=300, H=4), api.recurrent_fwd)


def test_tiny_through_chunk_entry_point_fp32():
    """fp32 I/O through kla_chunk_fwd (the token-serial kernel serves it)."""
    _check(W["tiny"], api.chunk_fwd)


def test_empty_sequence_copies_state():
    w = W["stress"].scaled(B=1, T=0, H=2)
    x = cuda(inputs.make_prefill(w, with_h0=True))
    o, hT = api.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    torch.cuda.synchronize()
    assert torch.equal(hT, x["h0"]) and o.numel() == 0


def test_state_alias_in_place():
    w = W["prefill_4k"].scaled(B=1, T=70, H=2)
    x = inputs.make_prefill(w, with_h0=True)
    xc = cuda(x)
    h = xc["h0"].clone()
    api.recurrent_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"], h, hT=h)
    torch.cuda.synchronize()
    _, h_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    assert rel(h, h_ref) < 1e-2
