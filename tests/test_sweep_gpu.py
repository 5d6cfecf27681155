"""A seeded sweep of random small problems through every product entry
point, each against the fp64 oracle on the GPU: shapes (B, T, H, d), I/O
type, initial state, the three forms of the recurrence (KLA step size,
beta given, per-channel gate), the decode step and both backward paths.
The configurations are drawn from one fixed seed, so the sweep is the same
on every run; each case's parameters are in its test id."""
import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_kla_b200 import api, inputs

from helpers import TOL, cuda, rel

pytestmark = pytest.mark.gpu

N_CASES = 24


def _cases():
    r = np.random.Generator(np.random.PCG64(2024))
    out = []
    for i in range(N_CASES):
        out.append(dict(idx=i,
                        B=int(r.integers(1, 4)),
                        T=int(r.choice([1, 5, 63, 64, 65, 127, 129, 200, 257, 320])),
                        H=int(r.integers(1, 4)),
                        d=int(r.choice([64, 128])),
                        dt=str(r.choice(["bf16", "bf16", "fp32"])),
                        h0=bool(r.integers(0, 2)),
                        kind=str(r.choice(["layer", "stress", "long"]))))
    return out


CASES = _cases()


def _name(c):
    return "i{idx}-B{B}-T{T}-H{H}-d{d}-{dt}-h0{h0}-{kind}".format(**c)


def _problem(c, seed_shift=0):
    name = {"layer": "prefill_4k", "stress": "stress", "long": "prefill_65k"}[c["kind"]]
    w = inputs.WORKLOADS[name].scaled(B=c["B"], T=c["T"], H=c["H"], dk=c["d"], dv=c["d"],
                                      dtype=c["dt"], seed=5000 + c["idx"] + seed_shift)
    return w, inputs.make_prefill(w, with_h0=c["h0"])


def _upstream(w, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    do = torch.from_numpy(rng.standard_normal((w.B, w.T, w.H, w.dv)).astype(np.float32))
    dhT = torch.from_numpy(rng.standard_normal((w.B, w.H, w.dk, w.dv)).astype(np.float32))
    return do.to(w.torch_dtype), dhT


@pytest.mark.parametrize("c", CASES, ids=_name)
def test_sweep_prefill(c):
    w, x = _problem(c)
    xc = cuda(x)
    o, hT = api.chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"], xc["h0"])
    api.check_device_error()
    o_ref, h_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    tol = TOL[c["dt"]]
    assert rel(o.cpu(), o_ref) < tol and rel(hT.cpu(), h_ref) < tol


@pytest.mark.parametrize("c", CASES, ids=_name)
def test_sweep_gated_delta_and_channel_gate(c):
    w, x = _problem(c, 100)
    rng = np.random.Generator(np.random.PCG64(6000 + c["idx"]))
    beta = torch.from_numpy(rng.uniform(0.05, 1.5, x["g"].shape).astype(np.float32))
    kf = x["k"].float()
    k = (kf / kf.norm(dim=-1, keepdim=True).clamp_min(1e-6)).to(x["k"].dtype)
    xc = cuda(x)
    o, hT = api.gdn_chunk_fwd(xc["q"], cuda(k), xc["v"], xc["g"], cuda(beta), xc["h0"])
    o_ref, h_ref = oracle.gated_delta(x["q"], k, x["v"], x["g"], beta, x["h0"])
    tol = TOL[c["dt"]]
    assert rel(o.cpu(), o_ref) < tol and rel(hT.cpu(), h_ref) < tol
    gv = inputs.channel_gates((w.B, w.T, w.H, w.dk), 7000 + c["idx"])
    o, hT = api.kda_chunk_fwd(xc["q"], xc["k"], xc["v"], cuda(gv), xc["eta"], x["eps"],
                              xc["h0"])
    api.check_device_error()
    o_ref, h_ref = oracle.kda_forward(x["q"], x["k"], x["v"], gv, x["eta"], x["eps"], x["h0"])
    assert rel(o.cpu(), o_ref) < tol and rel(hT.cpu(), h_ref) < tol


@pytest.mark.parametrize("c", CASES, ids=_name)
def test_sweep_decode(c):
    w = inputs.DECODE.scaled(B=c["B"], H=c["H"], dk=c["d"], dv=c["d"], dtype=c["dt"],
                             prefix_tokens=16, seed=8000 + c["idx"])
    d = inputs.make_decode(w, steps=3)
    S0 = torch.from_numpy(np.random.Generator(np.random.PCG64(8100 + c["idx"]))
                          .normal(0.0, 0.3, (w.B, w.H, w.dk, w.dv)).astype(np.float32))
    S = cuda(S0.clone())
    Sref = oracle.f64(S0)
    st = d["steps"]
    for i in range(3):
        args = [st[n][i] for n in ("q", "k", "v", "g", "eta")]
        o = api.decode_step(*(cuda(a) for a in args), S, eps=d["eps"])
        o_ref, Sref = oracle.decode_step(*args, d["eps"], Sref)
        assert rel(o.cpu(), o_ref) < TOL[c["dt"]]
    assert rel(S.cpu(), Sref) < TOL[c["dt"]]


@pytest.mark.parametrize("c", CASES, ids=_name)
def test_sweep_backward(c):
    """The chunkwise backward (bf16: chunk kernels; fp32: token-serial) and
    the token-serial one, against the oracle's gradients."""
    w, x = _problem(c, 200)
    do, dhT = _upstream(w, 9000 + c["idx"])
    xc = cuda(x)
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"], do, dhT)
    names = ("dq", "dk", "dv", "dg", "deta") + (("dh0",) if c["h0"] else ())
    for fn, tol in ((api.chunk_bwd, TOL["bf16"] if c["dt"] == "bf16" else TOL["fp32"]),
                    (api.recurrent_bwd, TOL["fp32"])):
        out = fn(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], cuda(do), x["eps"], xc["h0"],
                 cuda(dhT))
        api.check_device_error()
        errs = {n: rel(out[n].cpu(), ref[n]) for n in names}
        assert all(e < tol for e in errs.values()), (fn.__name__, errs)
