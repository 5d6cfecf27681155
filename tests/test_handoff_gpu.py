"""Hand-offs between the prefill and the decode step, on the GPU.

"Deep Dive into KDA", section 3: only the d_k x d_v state crosses a chunk
boundary, so the state a prefill leaves is all a continuation needs:
  * decode of token T+1 from the prefill's h_T equals the prefill of T+1
    tokens (its last output row and its final state);
  * a prefill split at any token (inside a chunk or on a boundary) and
    continued from the first part's h_T equals the unsplit prefill.
Both sides are also compared with the fp64 oracle run over the whole
sequence."""
import pytest
import torch

import oracle
from delta_rule_linear_kla_b200 import api, inputs

from helpers import assert_parity, assert_state_parity, cuda, rel

pytestmark = pytest.mark.gpu


def _cut(x, t0, t1):
    return {k: (v[:, t0:t1].contiguous() if isinstance(v, torch.Tensor) and k != "h0" else v)
            for k, v in x.items()}


@pytest.mark.parametrize("name,T,h0", [("prefill_4k", 200, False), ("prefill_4k", 128, True),
                                       ("stress", 77, True), ("prefill_65k", 1000, False)])
def test_decode_continues_prefill(name, T, h0):
    w = inputs.WORKLOADS[name].scaled(B=2, T=T + 1, H=3, seed=61)
    x = inputs.make_prefill(w, with_h0=h0)
    xc = cuda(x)
    head = _cut(xc, 0, T)
    _, S = api.chunk_fwd(head["q"], head["k"], head["v"], head["g"], head["eta"], x["eps"],
                         xc["h0"])
    tok = {k: xc[k][:, T].contiguous() for k in ("q", "k", "v", "g", "eta")}
    o_dec = api.decode_step(tok["q"], tok["k"], tok["v"], tok["g"], tok["eta"], S, x["eps"])
    o_all, h_all = api.chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"],
                                 xc["h0"])
    api.check_device_error()
    o_ref, h_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    # the decode path and the one-call prefill both match the oracle ...
    assert rel(o_dec.cpu(), o_ref[:, T]) < 1e-2
    assert_state_parity(S.cpu(), h_ref, "bf16")
    assert rel(o_all[:, T].cpu(), o_ref[:, T]) < 1e-2
    assert_state_parity(h_all.cpu(), h_ref, "bf16")
    # ... and each other
    assert rel(o_dec.cpu(), o_all[:, T].cpu()) < 1e-2 and rel(S.cpu(), h_all.cpu()) < 1e-2


@pytest.mark.parametrize("name,T,split", [("prefill_4k", 300, 100), ("prefill_4k", 256, 128),
                                          ("stress", 400, 1), ("stress", 300, 299)])
def test_split_prefill_continues_exactly(name, T, split):
    w = inputs.WORKLOADS[name].scaled(B=2, T=T, H=2, seed=63)
    x = inputs.make_prefill(w, with_h0=True)
    xc = cuda(x)
    a, b = _cut(xc, 0, split), _cut(xc, split, T)
    o1, h1 = api.chunk_fwd(a["q"], a["k"], a["v"], a["g"], a["eta"], x["eps"], xc["h0"])
    o2, h2 = api.chunk_fwd(b["q"], b["k"], b["v"], b["g"], b["eta"], x["eps"], h1)
    api.check_device_error()
    o = torch.cat([o1, o2], dim=1).cpu()
    o_ref, h_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    assert_parity(o, o_ref, "bf16")
    assert_state_parity(h2.cpu(), h_ref, "bf16")
