"""No kernel of the library uses atomics or a reduction order that depends
on scheduling: repeated calls agree bit for bit.  The chunkwise backward
(both head sizes) and the per-channel-gate chunk prefill, each called twice
on the same inputs."""
import numpy as np
import pytest
import torch

from delta_rule_linear_kla_b200 import api, inputs

from helpers import cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,T", [("prefill_4k", 200), ("stress", 130)])
def test_chunk_backward_bitwise_repeatable(name, T):
    w = inputs.WORKLOADS[name].scaled(B=1, T=T, H=2, seed=81)
    x = cuda(inputs.make_prefill(w, with_h0=True))
    rng = np.random.Generator(np.random.PCG64(82))
    do = cuda(torch.from_numpy(rng.standard_normal((w.B, w.T, w.H, w.dv)).astype(np.float32))
              .to(w.torch_dtype))
    dhT = cuda(torch.from_numpy(rng.standard_normal((w.B, w.H, w.dk, w.dv)).astype(np.float32)))
    run = lambda: api.chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["eta"], do, x["eps"], x["h0"],
                                dhT)
    a, b = run(), run()
    api.check_device_error()
    for n in ("dq", "dk", "dv", "dg", "deta", "dh0"):
        assert torch.equal(a[n], b[n]), n


def test_per_channel_gate_chunk_prefill_bitwise_repeatable():
    w = inputs.WORKLOADS["prefill_4k"].scaled(B=1, T=200, H=2, seed=83)
    x = cuda(inputs.make_prefill(w, with_h0=True))
    gv = cuda(inputs.channel_gates((w.B, w.T, w.H, w.dk), 84))
    run = lambda: api.kda_chunk_fwd(x["q"], x["k"], x["v"], gv, x["eta"], x["eps"], x["h0"])
    (o1, h1), (o2, h2) = run(), run()
    api.check_device_error()
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
