"""Per-channel gate (KDA form, "Deep Dive into KDA", section 2.3, with the
KLA step size or beta given) on the GPU against the fp64 oracle: the
token-serial prefill kernel (bf16 and fp32 I/O) and the decode step."""
import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_kla_b200 import api, inputs

from helpers import TOL, assert_parity, assert_state_parity, cuda, rel

pytestmark = pytest.mark.gpu


def _prefill_inputs(name, B, T, H, dt, seed, with_h0=True):
    w = inputs.WORKLOADS[name].scaled(B=B, T=T, H=H, dtype=dt, seed=seed)
    x = inputs.make_prefill(w, with_h0=with_h0)
    x["gv"] = inputs.channel_gates((B, T, H, w.dk), seed + 1)
    return w, x


@pytest.mark.parametrize("name,T,dt", [("prefill_4k", 1, "bf16"), ("prefill_4k", 130, "bf16"),
                                       ("stress", 97, "bf16"), ("tiny", 150, "fp32"),
                                       ("prefill_4k", 70, "fp32")])
def test_kda_prefill(name, T, dt):
    w, x = _prefill_inputs(name, 2, T, 2, dt, 41)
    xc = cuda(x)
    o, hT = api.kda_fwd(xc["q"], xc["k"], xc["v"], xc["gv"], xc["eta"], x["eps"], xc["h0"])
    api.check_device_error()
    o_ref, h_ref = oracle.kda_forward(x["q"], x["k"], x["v"], x["gv"], x["eta"], x["eps"],
                                      x["h0"])
    assert rel(o.cpu(), o_ref) < TOL[dt] and rel(hT.cpu(), h_ref) < TOL[dt]


def test_kda_prefill_beta_given():
    w, x = _prefill_inputs("prefill_4k", 1, 90, 3, "bf16", 43)
    kf = x["k"].float()
    k = (kf / kf.norm(dim=-1, keepdim=True).clamp_min(1e-6)).to(x["k"].dtype)
    rng = np.random.Generator(np.random.PCG64(44))
    beta = torch.from_numpy((1 / (1 + np.exp(-rng.normal(size=(1, 90, 3))))).astype(np.float32))
    xc = cuda(x)
    o, hT = api.kda_fwd_beta(xc["q"], cuda(k), xc["v"], xc["gv"], cuda(beta), xc["h0"])
    api.check_device_error()
    o_ref, h_ref = oracle.kda(x["q"], k, x["v"], x["gv"], beta, x["h0"])
    assert rel(o.cpu(), o_ref) < TOL["bf16"] and rel(hT.cpu(), h_ref) < TOL["bf16"]


def test_uniform_channel_gate_equals_scalar_gate_kernel():
    """A gate equal on every channel is the scalar gate: the per-channel
    token-serial kernel agrees with the scalar one to fp32 rounding."""
    w, x = _prefill_inputs("tiny", 1, 200, 2, "fp32", 45)
    gv = x["g"][..., None].expand(-1, -1, -1, w.dk).contiguous()
    xc = cuda(x)
    o1, h1 = api.kda_fwd(xc["q"], xc["k"], xc["v"], cuda(gv), xc["eta"], x["eps"], xc["h0"])
    o2, h2 = api.recurrent_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], x["eps"],
                               xc["h0"])
    torch.cuda.synchronize()
    assert rel(o1.cpu(), o2.cpu()) < 1e-5 and rel(h1.cpu(), h2.cpu()) < 1e-5


def test_kda_prefill_wiped_channels_and_empty():
    """Channels whose gate wipes them (g = -200: a = 0) and a zero-length
    prefill (hT = h0)."""
    w, x = _prefill_inputs("prefill_4k", 1, 80, 2, "fp32", 47)
    x["gv"][0, 10:20, :, ::7] = -200.0
    xc = cuda(x)
    o, hT = api.kda_fwd(xc["q"], xc["k"], xc["v"], xc["gv"], xc["eta"], x["eps"], xc["h0"])
    api.check_device_error()
    o_ref, h_ref = oracle.kda_forward(x["q"], x["k"], x["v"], x["gv"], x["eta"], x["eps"],
                                      x["h0"])
    assert rel(o.cpu(), o_ref) < TOL["fp32"] and rel(hT.cpu(), h_ref) < TOL["fp32"]
    q0 = xc["q"][:, :0].contiguous()
    _, h_empty = api.kda_fwd(q0, q0, xc["v"][:, :0].contiguous(),
                             xc["gv"][:, :0].contiguous(), xc["eta"][:, :0].contiguous(),
                             x["eps"], xc["h0"])
    torch.cuda.synchronize()
    assert torch.equal(h_empty, xc["h0"])


@pytest.mark.parametrize("dt,d", [("bf16", 128), ("fp32", 128), ("bf16", 64)])
def test_kda_decode(dt, d):
    w = inputs.DECODE.scaled(B=3, H=4, dk=d, dv=d, dtype=dt, prefix_tokens=24)
    dd = inputs.make_decode(w, steps=5)
    st = dd["steps"]
    gv = inputs.channel_gates((5, w.B, w.H, d), 49)
    rng = np.random.Generator(np.random.PCG64(50))
    S0 = torch.from_numpy(rng.normal(0, 0.1, (w.B, w.H, d, d)).astype(np.float32))
    S = cuda(S0.clone())
    Sref = oracle.f64(S0)
    for i in range(5):
        args = [st[n][i] for n in ("q", "k", "v")]
        o = api.kda_decode_step(*(cuda(a) for a in args), cuda(gv[i]), cuda(st["eta"][i]), S,
                                dd["eps"])
        o_ref, Sref = oracle.kda_decode_step(*args, gv[i], st["eta"][i], dd["eps"], Sref)
        assert rel(o.cpu(), o_ref) < TOL[dt]
    api.check_device_error()
    assert rel(S.cpu(), Sref) < TOL["fp32"]


def test_kda_decode_beta_given():
    w = inputs.DECODE.scaled(B=2, H=3, dtype="bf16", prefix_tokens=24)
    dd = inputs.make_decode(w, steps=3)
    st = dd["steps"]
    gv = inputs.channel_gates((3, w.B, w.H, w.dk), 51)
    rng = np.random.Generator(np.random.PCG64(52))
    beta = torch.from_numpy(rng.uniform(0.0, 1.0, (3, w.B, w.H)).astype(np.float32))
    S = cuda(torch.zeros(w.B, w.H, w.dk, w.dv))
    Sref = np.zeros((w.B, w.H, w.dk, w.dv))
    for i in range(3):
        args = [st[n][i] for n in ("q", "k", "v")]
        o = api.kda_decode_step_beta(*(cuda(a) for a in args), cuda(gv[i]), cuda(beta[i]), S)
        o_ref, Sref = oracle.kda(*(a[:, None] for a in args), gv[i][:, None], beta[i][:, None],
                                 Sref)
        assert rel(o.cpu(), o_ref[:, 0]) < TOL["bf16"]
    torch.cuda.synchronize()
    assert rel(S.cpu(), Sref) < TOL["fp32"]


# ------------------------------------------------- chunk path (tensor cores)
@pytest.mark.parametrize("name,B,T,H,h0", [("prefill_4k", 2, 130, 2, True),
                                           ("prefill_4k", 1, 1, 2, False),
                                           ("prefill_4k", 1, 64, 3, True),
                                           ("stress", 2, 97, 3, True),
                                           ("stress", 1, 300, 2, False)])
def test_kda_chunk_prefill(name, B, T, H, h0):
    w, x = _prefill_inputs(name, B, T, H, "bf16", 91, with_h0=h0)
    xc = cuda(x)
    o, hT = api.kda_chunk_fwd(xc["q"], xc["k"], xc["v"], xc["gv"], xc["eta"], x["eps"],
                              xc["h0"])
    api.check_device_error()
    o_ref, h_ref = oracle.kda_forward(x["q"], x["k"], x["v"], x["gv"], x["eta"], x["eps"],
                                      x["h0"])
    assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()
    assert_parity(o.cpu(), o_ref, "bf16")
    assert_state_parity(hT.cpu(), h_ref, "bf16")


def test_kda_chunk_strong_and_zero_gates():
    """Channels that wipe the state (g down to -60 per token), channels that
    never decay (g = 0) and mixtures inside one chunk: every decay factor the
    chunk path forms is e^{difference} <= 1, so nothing overflows."""
    w, x = _prefill_inputs("prefill_4k", 1, 200, 2, "bf16", 93, with_h0=True)
    gv = x["gv"]
    gv[..., :16] = 0.0
    gv[0, 30:40, :, 16:48] = -60.0
    gv[0, :, :, 100:] = -8.0
    xc = cuda(x)
    o, hT = api.kda_chunk_fwd(xc["q"], xc["k"], xc["v"], xc["gv"], xc["eta"], x["eps"],
                              xc["h0"])
    api.check_device_error()
    o_ref, h_ref = oracle.kda_forward(x["q"], x["k"], x["v"], gv, x["eta"], x["eps"], x["h0"])
    assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()
    assert_parity(o.cpu(), o_ref, "bf16")
    assert_state_parity(hT.cpu(), h_ref, "bf16")


def test_kda_chunk_beta_given_and_fp32():
    w, x = _prefill_inputs("prefill_4k", 2, 150, 2, "bf16", 95, with_h0=True)
    rng = np.random.Generator(np.random.PCG64(96))
    beta = torch.from_numpy(rng.uniform(0.0, 1.0, (2, 150, 2)).astype(np.float32))
    kf = x["k"].float()
    k = (kf / kf.norm(dim=-1, keepdim=True).clamp_min(1e-6)).to(torch.bfloat16)
    xc = cuda(x)
    o, hT = api.kda_chunk_fwd_beta(xc["q"], cuda(k), xc["v"], xc["gv"], cuda(beta), xc["h0"])
    api.check_device_error()
    o_ref, h_ref = oracle.kda(x["q"], k, x["v"], x["gv"], beta, x["h0"])
    assert rel(o.cpu(), o_ref) < TOL["bf16"] and rel(hT.cpu(), h_ref) < TOL["bf16"]
    # fp32 I/O goes to the token-serial kernel through the same entry point
    w2, x2 = _prefill_inputs("tiny", 1, 90, 2, "fp32", 97, with_h0=True)
    x2c = cuda(x2)
    o2, h2 = api.kda_chunk_fwd(x2c["q"], x2c["k"], x2c["v"], x2c["gv"], x2c["eta"], x2["eps"],
                               x2c["h0"])
    torch.cuda.synchronize()
    o2_ref, h2_ref = oracle.kda_forward(x2["q"], x2["k"], x2["v"], x2["gv"], x2["eta"],
                                        x2["eps"], x2["h0"])
    assert rel(o2.cpu(), o2_ref) < TOL["fp32"] and rel(h2.cpu(), h2_ref) < TOL["fp32"]


def test_kda_chunk_few_heads_long_sequence():
    """Few heads, long sequence (a shape the scalar-gate chain cuts into
    segments): the per-channel form runs its chain uncut, and its workspace
    holds the per-chunk tiles only."""
    w, x = _prefill_inputs("prefill_4k", 1, 4000, 2, "bf16", 99, with_h0=True)
    assert api.chunk_fwd_segments(1, 4000, 2, w.dk, w.dv) > 1
    tiles = 1 * 2 * ((4000 + 63) // 64) * (16384 + 3 * 2 * 8192 + 1024)
    assert api.kda_chunk_fwd_workspace_size(1, 4000, 2, w.dk, w.dv) == tiles
    xc = cuda(x)
    o, hT = api.kda_chunk_fwd(xc["q"], xc["k"], xc["v"], xc["gv"], xc["eta"], x["eps"],
                              xc["h0"])
    api.check_device_error()
    o_ref, h_ref = oracle.kda_forward(x["q"], x["k"], x["v"], x["gv"], x["eta"], x["eps"],
                                      x["h0"])
    assert_parity(o.cpu(), o_ref, "bf16")
    assert_state_parity(hT.cpu(), h_ref, "bf16")


@pytest.mark.parametrize("name,heads", [("prefill_4k", [(0, 0), (4, 3), (7, 7)]),
                                        ("stress", [(0, 0), (2, 19), (3, 31)])])
def test_kda_chunk_full_size_oracle_sampled(name, heads):
    """The full-size per-channel-gate chunk prefill, in the launch
    configuration the benchmark times (every chunk of every head through the
    factor kernel and the chain), against the fp64 oracle on sampled heads:
    each head is an independent recurrence the oracle can run alone."""
    w = inputs.WORKLOADS[name]
    x = inputs.make_prefill(w)
    gv = inputs.channel_gates((w.B, w.T, w.H, w.dk), w.seed + 11)
    xc = cuda(x)
    o, hT = api.kda_chunk_fwd(xc["q"], xc["k"], xc["v"], cuda(gv), xc["eta"], x["eps"],
                              xc["h0"])
    api.check_device_error()
    o, hT = o.cpu(), hT.cpu()
    for (b, h) in heads:
        sl = lambda t: t[b:b + 1, :, h:h + 1]
        h0 = None if x["h0"] is None else x["h0"][b:b + 1, h:h + 1]
        o_ref, h_ref = oracle.kda_forward(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(gv),
                                          sl(x["eta"]), x["eps"], h0)
        assert_parity(sl(o), o_ref, "bf16")
        assert_state_parity(hT[b:b + 1, h:h + 1], h_ref, "bf16")


def test_kda_chunk_matches_token_serial_4k_sampled():
    """The full 4K shape in the benchmark's launch configuration: the chunk
    path against the token-serial kernel on every head (same recurrence)."""
    w = inputs.WORKLOADS["prefill_4k"]
    x = cuda(inputs.make_prefill(w))
    gv = cuda(inputs.channel_gates((w.B, w.T, w.H, w.dk), w.seed + 11))
    o1, h1 = api.kda_chunk_fwd(x["q"], x["k"], x["v"], gv, x["eta"], x["eps"])
    o2, h2 = api.kda_fwd(x["q"], x["k"], x["v"], gv, x["eta"], x["eps"])
    api.check_device_error()
    assert rel(o1, o2) < TOL["bf16"] and rel(h1, h2) < TOL["bf16"]
