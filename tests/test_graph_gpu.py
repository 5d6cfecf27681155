"""The prefill and decode calls inside CUDA graphs: captured once on static
buffers (every call only enqueues kernels on the caller's stream, never
synchronises or allocates), replayed with new inputs copied in, and equal to
the same calls made directly."""
import pytest
import torch

from delta_rule_linear_kla_b200 import api, inputs

from helpers import cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,B,T,H", [("prefill_4k", 2, 200, 2),     # uncut chain
                                        ("prefill_4k", 1, 4000, 2)])  # cut chain (3 launches)
def test_prefill_graph_replay(name, B, T, H):
    w = inputs.WORKLOADS[name].scaled(B=B, T=T, H=H, seed=111)
    x0 = cuda(inputs.make_prefill(w, with_h0=True))
    x1 = cuda(inputs.make_prefill(w.scaled(seed=112), with_h0=True))
    ws = torch.empty(api.chunk_fwd_workspace_size(B, T, H, w.dk, w.dv), dtype=torch.uint8,
                     device="cuda")
    buf = {k: v.clone() for k, v in x0.items() if isinstance(v, torch.Tensor)}
    o = torch.empty((B, T, H, w.dv), dtype=torch.bfloat16, device="cuda")
    hT = torch.empty((B, H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    run = lambda: api.chunk_fwd(buf["q"], buf["k"], buf["v"], buf["g"], buf["eta"], x0["eps"],
                                buf["h0"], o=o, hT=hT, workspace=ws)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()  # first call outside the capture (one-time kernel attributes)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run()
    for x in (x1, x0):
        for k in buf:
            buf[k].copy_(x[k])
        graph.replay()
        torch.cuda.synchronize()
        o_ref, h_ref = api.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"],
                                     workspace=torch.empty_like(ws))
        api.check_device_error()
        assert torch.equal(o, o_ref) and torch.equal(hT, h_ref)


def test_decode_graph_of_many_steps():
    w = inputs.DECODE.scaled(B=4, H=2, prefix_tokens=24)
    d = inputs.make_decode(w, steps=8)
    st = {k: cuda(v) for k, v in d["steps"].items()}
    S0 = torch.randn(w.B, w.H, w.dk, w.dv, device="cuda") * 0.1
    S = S0.clone()
    outs = [torch.empty((w.B, w.H, w.dv), dtype=torch.bfloat16, device="cuda") for _ in range(8)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        api.decode_step(st["q"][0], st["k"][0], st["v"][0], st["g"][0], st["eta"][0],
                        S.clone(), d["eps"])
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(8):
            api.decode_step(st["q"][i], st["k"][i], st["v"][i], st["g"][i], st["eta"][i], S,
                            d["eps"], o=outs[i])
    S.copy_(S0)
    graph.replay()
    torch.cuda.synchronize()
    S2 = S0.clone()
    for i in range(8):
        o = api.decode_step(st["q"][i], st["k"][i], st["v"][i], st["g"][i], st["eta"][i], S2,
                            d["eps"])
        assert torch.equal(o, outs[i])
    torch.cuda.synchronize()
    assert torch.equal(S, S2)


def test_backward_graph_replay():
    """The chunkwise backward (forward chunk prefill with its state output,
    three backward kernels) captured once and replayed on new inputs equals
    the direct call bit for bit."""
    w = inputs.WORKLOADS["prefill_4k"].scaled(B=1, T=300, H=2, seed=113)
    x0 = cuda(inputs.make_prefill(w, with_h0=True))
    x1 = cuda(inputs.make_prefill(w.scaled(seed=114), with_h0=True))
    gen = torch.Generator(device="cpu").manual_seed(115)
    do0 = torch.randn((1, 300, 2, w.dv), generator=gen).bfloat16().cuda()
    do1 = torch.randn((1, 300, 2, w.dv), generator=gen).bfloat16().cuda()
    ws = torch.empty(api.chunk_bwd_workspace_size(1, 300, 2, w.dk, w.dv), dtype=torch.uint8,
                     device="cuda")
    buf = {k: v.clone() for k, v in x0.items() if isinstance(v, torch.Tensor)}
    dbuf = do0.clone()
    run = lambda: api.chunk_bwd(buf["q"], buf["k"], buf["v"], buf["g"], buf["eta"], dbuf,
                                x0["eps"], buf["h0"], workspace=ws)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()  # first call outside the capture (one-time kernel attributes)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out = run()
    for x, do in ((x1, do1), (x0, do0)):
        for k in buf:
            buf[k].copy_(x[k])
        dbuf.copy_(do)
        graph.replay()
        torch.cuda.synchronize()
        ref = api.chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["eta"], do, x["eps"], x["h0"],
                            workspace=torch.empty_like(ws))
        api.check_device_error()
        for n in ("dq", "dk", "dv", "dg", "deta", "dh0"):
            assert torch.equal(out[n], ref[n]), n
