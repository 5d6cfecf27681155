"""kla_chunk_fwd_host: the prefill from host buffers with the copies
pipelined against the kernels, against the fp64 oracle and against the
device-buffer entry point, over batch sizes that exercise every piece/slot
arrangement (fewer pieces than slots, slot reuse, a short last piece)."""
import pytest
import torch

import oracle
from delta_rule_linear_kla_b200 import api, inputs

from helpers import TOL, cuda, rel

pytestmark = pytest.mark.gpu


def _pinned(x):
    return {k: (v.pin_memory() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


@pytest.mark.parametrize("name,B,T,H,dt,h0", [("prefill_4k", 1, 150, 2, "bf16", False),
                                              ("prefill_4k", 3, 200, 2, "bf16", True),
                                              ("stress", 9, 130, 2, "bf16", True),
                                              ("tiny", 4, 70, 2, "fp32", True)])
def test_host_prefill(name, B, T, H, dt, h0):
    w = inputs.WORKLOADS[name].scaled(B=B, T=T, H=H, dtype=dt, seed=61)
    x = _pinned(inputs.make_prefill(w, with_h0=h0))
    o, hT = api.chunk_fwd_host(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    torch.cuda.synchronize()
    api.check_device_error()
    assert not o.is_cuda and not hT.is_cuda
    o_ref, h_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    assert rel(o, o_ref) < TOL[dt] and rel(hT, h_ref) < TOL[dt]
    xc = cuda(x)
    o2, h2 = api.chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"], xc["h0"])
    torch.cuda.synchronize()
    assert rel(o, o2.cpu()) < 2e-3 and rel(hT, h2.cpu()) < 2e-3


def test_host_prefill_repeated_calls_share_staging():
    """Back-to-back calls on one stream with one staging buffer and new
    inputs each time: every call's outputs belong to its own inputs."""
    outs = []
    w0 = inputs.WORKLOADS["stress"].scaled(B=5, T=100, H=2)
    need = api.chunk_fwd_host_staging_size(5, 100, 2, w0.dk, w0.dv)
    staging = torch.empty(need, dtype=torch.uint8, device="cuda")
    xs = [_pinned(inputs.make_prefill(w0.scaled(seed=70 + i))) for i in range(3)]
    for x in xs:
        outs.append(api.chunk_fwd_host(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"],
                                       x["h0"], staging=staging))
    torch.cuda.synchronize()
    for x, (o, hT) in zip(xs, outs):
        o_ref, h_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"],
                                      x["h0"])
        assert rel(o, o_ref) < TOL["bf16"] and rel(hT, h_ref) < TOL["bf16"]


def test_host_prefill_many_pieces_reuse_slots():
    """Large enough to be cut into four pieces of two sequences (slots are
    reused): equal to the device-buffer call to rounding, and to the oracle
    on a sampled head of the last piece."""
    w = inputs.WORKLOADS["prefill_4k"].scaled(B=8, T=8192, H=8, seed=63)
    x = _pinned(inputs.make_prefill(w, with_h0=True))
    o, hT = api.chunk_fwd_host(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    torch.cuda.synchronize()
    api.check_device_error()
    xc = cuda(x)
    o2, h2 = api.chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"], xc["h0"])
    torch.cuda.synchronize()
    assert rel(o, o2.cpu()) < 2e-3 and rel(hT, h2.cpu()) < 2e-3
    b, h = 7, 5
    sl = lambda t: t[b:b + 1, :, h:h + 1]
    o_ref, h_ref = oracle.forward(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["g"]), sl(x["eta"]),
                                  x["eps"], x["h0"][b:b + 1, h:h + 1])
    assert rel(o[b:b + 1, :, h:h + 1], o_ref) < TOL["bf16"]
    assert rel(hT[b:b + 1, h:h + 1], h_ref) < TOL["bf16"]
