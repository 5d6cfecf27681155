"""Gated DeltaNet mode (beta given per token) against the oracle's gated
delta rule, on the GPU: the chunk kernels (bf16), the token-serial kernel
(fp32 I/O) and the decode step.  KLA is this rule with beta_t =
eta_t / (||k_t||^2 + eps) ("Kaczmarz Linear Attention", Abstract)."""
import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_kla_b200 import api, inputs

from helpers import TOL, cuda, rel

pytestmark = pytest.mark.gpu


def _beta(shape, seed):
    # a GDN-style step size in (0, 1): sigmoid of a Gaussian
    rng = np.random.Generator(np.random.PCG64(seed))
    return torch.from_numpy((1.0 / (1.0 + np.exp(-rng.normal(size=shape)))).astype(np.float32))


@pytest.mark.parametrize("name,B,T,H,dt", [("prefill_4k", 2, 200, 2, "bf16"),
                                           ("stress", 2, 130, 2, "bf16"),
                                           ("tiny", 2, 150, 2, "fp32"),
                                           # long and few heads: the cut state chain
                                           ("prefill_4k", 1, 3000, 1, "bf16")])
def test_gdn_prefill(name, B, T, H, dt):
    w = inputs.WORKLOADS[name].scaled(B=B, T=T, H=H, dtype=dt)
    x = inputs.make_prefill(w)
    # GDN is used with normalised keys; keep them at unit norm
    kf = x["k"].float()
    k = (kf / kf.norm(dim=-1, keepdim=True).clamp_min(1e-6)).to(x["k"].dtype)
    beta = _beta(x["g"].shape, 11)
    xc = cuda(x)
    o, hT = api.gdn_chunk_fwd(xc["q"], cuda(k), xc["v"], xc["g"], cuda(beta), xc["h0"])
    api.check_device_error()
    o_ref, h_ref = oracle.gated_delta(x["q"], k, x["v"], x["g"], beta, x["h0"])
    assert rel(o.cpu(), o_ref) < TOL[dt] and rel(hT.cpu(), h_ref) < TOL[dt]


def test_gdn_and_kla_agree_when_beta_is_the_kla_step():
    """GDN with beta = eta / (||k||^2 + eps) is KLA: same kernels, same result
    up to the rounding of the one division."""
    w = inputs.WORKLOADS["prefill_4k"].scaled(B=1, T=190, H=2)
    x = inputs.make_prefill(w)
    n2 = (x["k"].double() ** 2).sum(-1)
    beta = (x["eta"].double() / (n2 + x["eps"])).float()
    xc = cuda(x)
    o1, h1 = api.chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"], None)
    o2, h2 = api.gdn_chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], cuda(beta), None)
    torch.cuda.synchronize()
    assert rel(o2.cpu(), o1.cpu()) < 1e-2 and rel(h2.cpu(), h1.cpu()) < 1e-2


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_gdn_decode(dt):
    w = inputs.DECODE.scaled(B=3, H=4, dtype=dt, prefix_tokens=24)
    d = inputs.make_decode(w, steps=5)
    rng = np.random.Generator(np.random.PCG64(5))
    S0 = torch.from_numpy(rng.normal(0, 0.1, (w.B, w.H, w.dk, w.dv)).astype(np.float32))
    S = cuda(S0.clone())
    Sref = oracle.f64(S0)
    st = d["steps"]
    kf = st["k"].float()  # unit keys keep the GDN step stable
    st["k"] = (kf / kf.norm(dim=-1, keepdim=True).clamp_min(1e-6)).to(st["k"].dtype)
    for i in range(5):
        beta = _beta((w.B, w.H), 100 + i)
        q, k, v, g = (cuda(st[n][i]) for n in ("q", "k", "v", "g"))
        o = api.gdn_decode_step(q, k, v, g, cuda(beta), S)
        o_ref, Sref = oracle.gated_delta(st["q"][i][:, None], st["k"][i][:, None],
                                         st["v"][i][:, None], st["g"][i][:, None],
                                         beta[:, None], Sref)
        assert rel(o, o_ref[:, 0]) < TOL[dt]
    torch.cuda.synchronize()
    assert rel(S, Sref) < TOL[dt]
