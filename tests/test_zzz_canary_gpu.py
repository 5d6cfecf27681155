"""Out-of-bounds writes, without a sanitizer: every output and workspace
buffer handed to the library sits inside a larger allocation whose borders
hold a byte pattern, and after the call the borders must be unchanged (and
the results still match the oracle).  Outputs, states and workspaces of the
prefill (uncut and cut state chain, both head sizes, fp32 I/O), the
per-channel-gate prefill, the decode step and the backward."""
import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_kla_b200 import api, inputs

from helpers import TOL, Padded, cuda, rel

pytestmark = pytest.mark.gpu


def _prefill(name, B, T, H, seed=61):
    w = inputs.WORKLOADS[name].scaled(B=B, T=T, H=H, seed=seed)
    return w, inputs.make_prefill(w, with_h0=True)


@pytest.mark.parametrize("name,B,T,H", [("prefill_4k", 1, 200, 2),   # ragged tail, d = 128
                                        ("prefill_4k", 1, 4000, 2),  # state chain cut
                                        ("stress", 2, 130, 2),       # d = 64
                                        ("tiny", 1, 100, 2)])        # fp32 I/O
def test_prefill_writes_stay_inside(name, B, T, H):
    w, x = _prefill(name, B, T, H)
    xc = cuda(x)
    o = Padded((B, T, H, w.dv), w.torch_dtype, "cuda")
    hT = Padded((B, H, w.dk, w.dv), torch.float32, "cuda")
    need = api.chunk_fwd_workspace_size(B, T, H, w.dk, w.dv, w.torch_dtype)
    ws = Padded((need,), torch.uint8, "cuda") if need else None
    api.chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"], xc["h0"], o=o.t,
                  hT=hT.t, workspace=None if ws is None else ws.t)
    api.check_device_error()
    torch.cuda.synchronize()
    assert o.intact() and hT.intact() and (ws is None or ws.intact())
    o_ref, h_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    assert rel(o.t.cpu(), o_ref) < TOL[w.dtype] and rel(hT.t.cpu(), h_ref) < TOL[w.dtype]


def test_per_channel_gate_prefill_writes_stay_inside():
    w, x = _prefill("prefill_4k", 1, 150, 2)
    gv = inputs.channel_gates((w.B, w.T, w.H, w.dk), 62)
    xc = cuda(x)
    o = Padded((w.B, w.T, w.H, w.dv), w.torch_dtype, "cuda")
    hT = Padded((w.B, w.H, w.dk, w.dv), torch.float32, "cuda")
    need = api.kda_chunk_fwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv, w.torch_dtype)
    ws = Padded((need,), torch.uint8, "cuda")
    api.kda_chunk_fwd(xc["q"], xc["k"], xc["v"], cuda(gv), xc["eta"], x["eps"], xc["h0"],
                      o=o.t, hT=hT.t, workspace=ws.t)
    api.check_device_error()
    torch.cuda.synchronize()
    assert o.intact() and hT.intact() and ws.intact()
    o_ref, h_ref = oracle.kda_forward(x["q"], x["k"], x["v"], gv, x["eta"], x["eps"], x["h0"])
    assert rel(o.t.cpu(), o_ref) < TOL["bf16"] and rel(hT.t.cpu(), h_ref) < TOL["bf16"]


@pytest.mark.parametrize("d,dt", [(128, "bf16"), (64, "bf16"), (128, "fp32")])
def test_decode_writes_stay_inside(d, dt):
    w = inputs.DECODE.scaled(B=3, H=2, dk=d, dv=d, dtype=dt, prefix_tokens=16, seed=63)
    dec = inputs.make_decode(w, steps=1)
    S0 = torch.from_numpy(np.random.Generator(np.random.PCG64(64))
                          .normal(0.0, 0.3, (w.B, w.H, d, d)).astype(np.float32))
    S = Padded((w.B, w.H, d, d), torch.float32, "cuda")
    S.t.copy_(S0.cuda())
    o = Padded((w.B, w.H, d), w.torch_dtype, "cuda")
    args = [dec["steps"][n][0] for n in ("q", "k", "v", "g", "eta")]
    api.decode_step(*(cuda(a) for a in args), S.t, eps=dec["eps"], o=o.t)
    api.check_device_error()
    torch.cuda.synchronize()
    assert S.intact() and o.intact()
    o_ref, S_ref = oracle.decode_step(*args, dec["eps"], oracle.f64(S0))
    assert rel(o.t.cpu(), o_ref) < TOL[dt] and rel(S.t.cpu(), S_ref) < TOL[dt]


@pytest.mark.parametrize("name,T,fn", [("prefill_4k", 200, "chunk_bwd"),
                                       ("stress", 130, "chunk_bwd"),
                                       ("prefill_4k", 70, "recurrent_bwd")])
def test_backward_workspace_stays_inside(name, T, fn):
    w, x = _prefill(name, 1, T, 2)
    rng = np.random.Generator(np.random.PCG64(65))
    do = torch.from_numpy(rng.standard_normal((w.B, w.T, w.H, w.dv)).astype(np.float32))
    do = do.to(w.torch_dtype)
    dhT = torch.from_numpy(rng.standard_normal((w.B, w.H, w.dk, w.dv)).astype(np.float32))
    size = (api.chunk_bwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv, w.torch_dtype)
            if fn == "chunk_bwd" else api.recurrent_bwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv))
    ws = Padded((size,), torch.uint8, "cuda")
    xc = cuda(x)
    out = getattr(api, fn)(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], cuda(do), x["eps"],
                           xc["h0"], cuda(dhT), workspace=ws.t)
    api.check_device_error()
    torch.cuda.synchronize()
    assert ws.intact()
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"], do, dhT)
    tol = TOL["bf16"] if fn == "chunk_bwd" else TOL["fp32"]
    for n in ("dq", "dk", "dv", "dg", "deta", "dh0"):
        assert rel(out[n].cpu(), ref[n]) < tol, n
