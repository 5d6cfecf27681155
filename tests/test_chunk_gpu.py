"""tcgen05 chunkwise prefill (kla_chunk_fwd, bf16) against the fp64 oracle.

Small shapes are compared element by element over the whole output; the
full-size workloads run in the same launch configuration the benchmark times
and are compared on sampled heads (each head is an independent recurrence,
so the oracle can evaluate a few heads on their own)."""
import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_kla_b200 import api, inputs

from helpers import assert_parity, assert_state_parity, cuda, rel

pytestmark = pytest.mark.gpu
W = inputs.WORKLOADS
TOL = 1e-2


def _run(w, with_h0=None):
    x = inputs.make_prefill(w, with_h0=with_h0)
    xc = cuda(x)
    o, hT = api.chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"], xc["h0"])
    api.check_device_error()
    return x, o.cpu(), hT.cpu()


def _full_check(w, with_h0=None):
    x, o, hT = _run(w, with_h0)
    o_ref, h_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    assert np.isfinite(oracle.f64(o)).all() and np.isfinite(oracle.f64(hT)).all()
    assert_parity(o, o_ref, "bf16")
    assert_state_parity(hT, h_ref, "bf16")


@pytest.mark.parametrize("T", [1, 17, 64, 65, 130, 256])
def test_layer_shapes_d128(T):
    _full_check(W["prefill_4k"].scaled(B=2, T=T, H=2))


@pytest.mark.parametrize("T", [1, 63, 64, 200])
def test_with_initial_state_d128(T):
    _full_check(W["prefill_4k"].scaled(B=1, T=T, H=3, seed=7), with_h0=True)


@pytest.mark.parametrize("T", [1, 64, 129, 300])
def test_stress_shapes_d64(T):
    _full_check(W["stress"].scaled(B=2, T=T, H=3))


def test_long_gates_small():
    _full_check(W["prefill_65k"].scaled(T=700, H=2))


def _ut_bytes(w):
    return w.B * w.H * ((w.T + 63) // 64) * 16384


# Few heads and long sequences: the state chain is cut into segments that run
# in parallel (transitions, start states, then outputs per segment).  The
# shapes give several segments of at least 8 chunks and a ragged tail.
SEGMENTED = [("prefill_4k", 1, 4000, 2, True), ("stress", 2, 2000, 1, False),
             ("stress", 1, 1536, 1, True), ("prefill_65k", 1, 2500, 3, True)]


@pytest.mark.parametrize("name,B,T,H,h0", SEGMENTED)
def test_segmented_chain(name, B, T, H, h0):
    w = W[name].scaled(B=B, T=T, H=H, seed=17)
    assert api.chunk_fwd_segments(w.B, w.T, w.H, w.dk, w.dv) > 1
    _full_check(w, with_h0=h0)


@pytest.mark.parametrize("name,B,T,H,h0", SEGMENTED[:2])
def test_segmented_equals_uncut_chain(name, B, T, H, h0):
    """The same factors through the cut chain (full workspace) and the uncut
    one (a workspace holding the factors only) agree to rounding."""
    w = W[name].scaled(B=B, T=T, H=H, seed=19)
    x = cuda(inputs.make_prefill(w, with_h0=h0))
    ws = api.chunk_ut_transform(x["k"], x["g"], x["eta"], x["eps"])
    o1, h1 = api.chunk_state_fwd(x["q"], x["k"], x["v"], x["g"], ws, x["h0"])
    o2, h2 = api.chunk_state_fwd(x["q"], x["k"], x["v"], x["g"], ws[:_ut_bytes(w)], x["h0"])
    api.check_device_error()
    assert rel(o1.cpu(), o2.cpu()) < 2e-3 and rel(h1.cpu(), h2.cpu()) < 2e-3


def test_final_state_only_and_alias():
    w = W["stress"].scaled(B=1, T=150, H=2)
    x = inputs.make_prefill(w)
    xc = cuda(x)
    h = xc["h0"].clone()
    o, hT = api.chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"], h, hT=h)
    torch.cuda.synchronize()
    assert hT.data_ptr() == h.data_ptr()
    _, h_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    assert rel(h, h_ref) < TOL
    o2, none = api.chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"],
                             xc["h0"], return_state=False)
    torch.cuda.synchronize()
    assert none is None and torch.equal(o2, o)


def test_two_stages_equal_one_call():
    """kla_chunk_ut_transform then kla_chunk_state_fwd is the same computation
    as kla_chunk_fwd (bit for bit), including a ragged tail and h0."""
    w = W["stress"].scaled(B=2, T=200, H=3)
    x = inputs.make_prefill(w)
    xc = cuda(x)
    o1, h1 = api.chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"], xc["h0"])
    ws = api.chunk_ut_transform(xc["k"], xc["g"], xc["eta"], x["eps"])
    o2, h2 = api.chunk_state_fwd(xc["q"], xc["k"], xc["v"], xc["g"], ws, xc["h0"])
    api.check_device_error()
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


def test_deterministic():
    w = W["prefill_4k"].scaled(B=1, T=300, H=2)
    _, o1, h1 = _run(w)
    _, o2, h2 = _run(w)
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


def _sampled(w, heads, with_h0=None):
    """Full-size launch; oracle on the listed (b, h) heads only."""
    x, o, hT = _run(w, with_h0)
    errs = []
    for (b, h) in heads:
        sl = lambda t: t[b:b + 1, :, h:h + 1]
        h0 = None if x["h0"] is None else x["h0"][b:b + 1, h:h + 1]
        o_ref, h_ref = oracle.forward(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["g"]),
                                      sl(x["eta"]), x["eps"], h0)
        # whole head, and every 64-token chunk of it
        r = assert_parity(o[b:b + 1, :, h:h + 1], o_ref, "bf16")
        eh, _ = assert_state_parity(hT[b:b + 1, h:h + 1], h_ref, "bf16")
        errs.append((b, h, r["whole"], r["worst_chunk"][0], eh))
    return errs


def test_full_size_layer_4k_sampled():
    _sampled(W["prefill_4k"], [(0, 0), (3, 5), (7, 7)])


def test_full_size_stress_sampled():
    _sampled(W["stress"], [(0, 0), (1, 17), (3, 31)])


def test_full_size_long_65k_sampled():
    _sampled(W["prefill_65k"], [(0, 3), (0, 15)])


def test_matches_token_serial_all_heads_4k():
    """Property at full size over every head: the chunkwise kernel and the
    token-serial kernel evaluate the same recurrence."""
    w = W["prefill_4k"]
    x = cuda(inputs.make_prefill(w))
    o1, h1 = api.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"])
    o2, h2 = api.recurrent_fwd(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"])
    torch.cuda.synchronize()
    assert rel(o1, o2) < TOL and rel(h1, h2) < TOL


def _degenerate(w, seed):
    """Inputs of workload ``w`` with degenerate tokens mixed in: zero keys
    (beta = eta / eps), eta = 0 (pure decay), g = 0 (no decay), a forget
    strong enough to wipe the state (g = -40), zero queries and values."""
    x = inputs.make_prefill(w)
    rng = np.random.Generator(np.random.PCG64(seed))
    B, T, H = x["g"].shape
    pick = lambda p: torch.from_numpy(rng.random((B, T, H)) < p)
    zk, ze, zg, wipe, zq, zv = (pick(p) for p in (0.05, 0.05, 0.1, 0.01, 0.05, 0.05))
    x["k"][zk] = 0
    x["q"][zq] = 0
    x["v"][zv] = 0
    x["eta"][ze] = 0.0
    x["g"][zg] = 0.0
    x["g"][wipe] = -40.0
    return x


@pytest.mark.parametrize("name,T", [("prefill_4k", 300), ("stress", 257)])
def test_degenerate_tokens(name, T):
    w = W[name].scaled(B=1, T=T, H=2)
    x = _degenerate(w, 7)
    xc = cuda(x)
    o, hT = api.chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"], xc["h0"])
    api.check_device_error()
    o_ref, h_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    assert np.isfinite(oracle.f64(o.cpu())).all() and np.isfinite(oracle.f64(hT.cpu())).all()
    assert_parity(o.cpu(), o_ref, "bf16")
    assert_state_parity(hT.cpu(), h_ref, "bf16")


def test_all_keys_zero_is_pure_decay():
    """Every key zero: no write ever lands, h_T = e^{sum g} h0 exactly as the
    recurrence says, and o_t = e^{G_t} h0^T q_t."""
    w = W["stress"].scaled(B=1, T=130, H=2)
    x = inputs.make_prefill(w)
    x["k"].zero_()
    xc = cuda(x)
    o, hT = api.chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"], xc["h0"])
    api.check_device_error()
    o_ref, h_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    assert rel(o.cpu(), o_ref) < TOL and rel(hT.cpu(), h_ref) < TOL


@pytest.mark.parametrize("B,T,H", [(2, 300, 2),     # uncut chain
                                   (1, 4000, 2)])  # cut chain
def test_chunk_start_states(B, T, H):
    """kla_chunk_fwd_states: the state at the start of every chunk equals the
    oracle's state after the first 64 n tokens; o and h_T are bitwise those
    of kla_chunk_fwd."""
    w = inputs.WORKLOADS["prefill_4k"].scaled(B=B, T=T, H=H)
    x = inputs.make_prefill(w, with_h0=True)
    xc = cuda(x)
    o, hT, hs = api.chunk_fwd_states(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"],
                                     xc["h0"])
    o2, h2 = api.chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"], xc["h0"])
    api.check_device_error()
    assert torch.equal(o, o2) and torch.equal(hT, h2)
    nck = (T + 63) // 64
    assert hs.shape == (B, H, nck, w.dk, w.dv)
    hs = hs.cpu()
    for n in sorted({0, 1, nck // 2, nck - 1}):
        if n == 0:
            ref = oracle.f64(x["h0"])
        else:
            sl = lambda t: t[:, :64 * n]
            _, ref = oracle.forward(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["g"]), sl(x["eta"]),
                                    x["eps"], x["h0"])
        assert rel(hs[:, :, n], ref) < TOL, n


def test_side_stream_matches_current_stream():
    """A call given a side stream allocates its temporaries (outputs,
    workspace) on that stream and returns the same result as on the current
    stream; more allocations on the current stream right after the call (the
    caching allocator may hand them a freed temporary only once the side
    stream's kernels are done with it) leave the result unchanged."""
    w = W["prefill_4k"].scaled(B=2, T=700, H=2, seed=71)
    x = cuda(inputs.make_prefill(w, with_h0=True))
    o1, h1 = api.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    o2, h2 = api.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"],
                           stream=side)
    junk = [torch.full((1 << 20,), 7, dtype=torch.uint8, device="cuda") for _ in range(64)]
    torch.cuda.current_stream().wait_stream(side)
    api.check_device_error()
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
    del junk


@pytest.mark.parametrize("name,B,T,H,h0", SEGMENTED)
def test_cut_chain_overlapped_ut_equals_staged(name, B, T, H, h0):
    """The cut chain as kla_chunk_fwd runs it (the UT kernel for the chunks
    of the first segments, then pass 1 beside UT lanes that make the last
    segment's factors) equals the staged calls (kla_chunk_ut_transform for
    every chunk, then kla_chunk_state_fwd on the same workspace) bit for bit:
    the factors do not depend on which kernel makes them."""
    w = W[name].scaled(B=B, T=T, H=H, seed=19)
    x = cuda(inputs.make_prefill(w, with_h0=h0))
    nws = api.chunk_fwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv)
    assert api.chunk_fwd_segments(w.B, w.T, w.H, w.dk, w.dv, ws_bytes=nws) > 1
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    o1, h1 = api.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"],
                           workspace=ws)
    ws2 = torch.empty(nws, dtype=torch.uint8, device="cuda")
    api.chunk_ut_transform(x["k"], x["g"], x["eta"], x["eps"], workspace=ws2)
    o2, h2 = api.chunk_state_fwd(x["q"], x["k"], x["v"], x["g"], ws2, x["h0"])
    api.check_device_error()
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
