"""Backward of the prefill (kla_recurrent_bwd, kla_gdn_recurrent_bwd) on the
GPU against the oracle's reverse-mode gradients of the token loop (which are
pinned by finite differences of the forward oracle).  The kernels compute in
fp32 on inputs that the oracle widens exactly, so the fp32 bar applies to
bf16 I/O as well."""
import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_kla_b200 import api, inputs

from helpers import cuda, rel

pytestmark = pytest.mark.gpu

TOL_BWD = 1e-4
GRADS = ("dq", "dk", "dv", "dg", "deta", "dh0")


def _upstream(w, seed, with_dhT=True):
    """dL/do in the I/O dtype and dL/dh_T (fp32), seeded N(0, 1)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    do = torch.from_numpy(rng.standard_normal((w.B, w.T, w.H, w.dv)).astype(np.float32))
    dhT = None
    if with_dhT:
        dhT = torch.from_numpy(rng.standard_normal((w.B, w.H, w.dk, w.dv)).astype(np.float32))
    return do.to(w.torch_dtype), dhT


def _check(out, ref, names=GRADS, tol=TOL_BWD):
    errs = {n: rel(out[n].cpu(), ref[n]) for n in names}
    print(" ".join("%s=%.1e" % kv for kv in errs.items()))
    assert all(e < tol for e in errs.values()), errs


@pytest.mark.parametrize("name,B,T,H,dt,with_h0,with_dhT", [
    ("tiny", 2, 200, 2, "fp32", True, True),          # 4 blocks, ragged last one
    ("prefill_4k", 1, 300, 2, "bf16", False, True),
    ("prefill_4k", 2, 129, 3, "fp32", True, False),
    ("stress", 1, 257, 2, "bf16", True, True),        # key norms 1e-2 .. 1e2, eta up to 2
    ("prefill_65k", 1, 700, 2, "bf16", False, True),  # strong forgets
])
def test_kla_backward(name, B, T, H, dt, with_h0, with_dhT):
    w = inputs.WORKLOADS[name].scaled(B=B, T=T, H=H, dtype=dt)
    x = inputs.make_prefill(w, with_h0=with_h0)
    do, dhT = _upstream(w, 77, with_dhT)
    xc = cuda(x)
    out = api.recurrent_bwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], cuda(do), x["eps"],
                            xc["h0"], cuda(dhT))
    api.check_device_error()
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"], do, dhT)
    _check(out, ref)


@pytest.mark.parametrize("T", [1, 7, 8, 9, 63, 64, 65, 128])
def test_kla_backward_lengths(T):
    """Block and sub-block edges: one token, one partial sub-block, exact
    sub-blocks and blocks, one token past them."""
    w = inputs.WORKLOADS["prefill_4k"].scaled(B=1, T=T, H=2, dk=64, dv=64)
    x = inputs.make_prefill(w, with_h0=True)
    do, dhT = _upstream(w, 78)
    xc = cuda(x)
    out = api.recurrent_bwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], cuda(do), x["eps"],
                            xc["h0"], cuda(dhT))
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"], do, dhT)
    _check(out, ref)


def test_kla_backward_empty_sequence():
    """T = 0: dL/dh0 = dL/dh_T, nothing else to compute."""
    dhT = torch.randn(2, 3, 64, 64, device="cuda")
    q = torch.empty(2, 0, 3, 64, dtype=torch.bfloat16, device="cuda")
    g = torch.empty(2, 0, 3, device="cuda")
    out = api.recurrent_bwd(q, q, q, g, g, q, 1e-6, None, dhT)
    torch.cuda.synchronize()
    assert torch.equal(out["dh0"], dhT)


def test_gdn_backward():
    w = inputs.WORKLOADS["prefill_4k"].scaled(B=2, T=150, H=2)
    x = inputs.make_prefill(w, with_h0=True)
    kf = x["k"].float()
    k = (kf / kf.norm(dim=-1, keepdim=True)).to(x["k"].dtype)
    rng = np.random.Generator(np.random.PCG64(79))
    beta = torch.from_numpy(rng.uniform(0.05, 1.95, x["g"].shape).astype(np.float32))
    do, dhT = _upstream(w, 80)
    xc = cuda(x)
    out = api.gdn_recurrent_bwd(xc["q"], cuda(k), xc["v"], xc["g"], cuda(beta), cuda(do),
                                xc["h0"], cuda(dhT))
    ref = oracle.gated_delta_backward(x["q"], k, x["v"], x["g"], beta, x["h0"], do, dhT)
    _check(out, ref, names=("dq", "dk", "dv", "dg", "dbeta", "dh0"))


def test_backward_deterministic_and_optional_outputs():
    """No atomics: two calls agree bitwise; grad_h0 may be skipped."""
    w = inputs.WORKLOADS["prefill_4k"].scaled(B=1, T=100, H=2)
    x = cuda(inputs.make_prefill(w))
    do, _ = _upstream(w, 81, False)
    do = cuda(do)
    a = api.recurrent_bwd(x["q"], x["k"], x["v"], x["g"], x["eta"], do, x["eps"])
    b = api.recurrent_bwd(x["q"], x["k"], x["v"], x["g"], x["eta"], do, x["eps"], need_h0=False)
    torch.cuda.synchronize()
    assert b["dh0"] is None
    for n in ("dq", "dk", "dv", "dg", "deta"):
        assert torch.equal(a[n], b[n]), n


def test_backward_full_size_sampled_heads():
    """The 4K layer (B=8 T=4096 H=8 d=128, bf16) in one call; the oracle's
    gradients of two sampled heads (heads are independent)."""
    w = inputs.WORKLOADS["prefill_4k"]
    x = inputs.make_prefill(w)
    do, dhT = _upstream(w, 82)
    xc = cuda(x)
    out = api.recurrent_bwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], cuda(do), x["eps"],
                            None, cuda(dhT))
    api.check_device_error()
    for b, h in ((3, 5), (7, 0)):
        sl = lambda t: t[b:b + 1, :, h:h + 1]
        ref = oracle.backward(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["g"]), sl(x["eta"]),
                              x["eps"], None, sl(do), dhT[b:b + 1, h:h + 1])
        got = {n: sl(out[n].cpu()) for n in ("dq", "dk", "dv", "dg", "deta")}
        got["dh0"] = out["dh0"][b:b + 1, h:h + 1].cpu()
        _check(got, ref)


@pytest.mark.parametrize("name,B,T,H,dt,with_h0,strong", [
    ("prefill_4k", 1, 200, 2, "bf16", False, False),
    ("tiny", 2, 130, 2, "fp32", True, False),
    ("prefill_4k", 1, 65, 2, "bf16", True, True),   # some channels wiped (g = -60)
    ("stress", 1, 100, 2, "bf16", True, False),
])
def test_kda_backward(name, B, T, H, dt, with_h0, strong):
    """Per-channel gate, KLA step size: against the oracle's per-channel-gate
    gradients (pinned by finite differences and by the equal-channel
    reduction to the scalar gate)."""
    w = inputs.WORKLOADS[name].scaled(B=B, T=T, H=H, dtype=dt)
    x = inputs.make_prefill(w, with_h0=with_h0)
    gv = inputs.channel_gates((B, T, H, w.dk), 83)
    if strong:
        gv[:, ::7, :, ::5] = -60.0
    do, dhT = _upstream(w, 84)
    xc = cuda(x)
    out = api.kda_recurrent_bwd(xc["q"], xc["k"], xc["v"], cuda(gv), xc["eta"], cuda(do),
                                x["eps"], xc["h0"], cuda(dhT))
    api.check_device_error()
    ref = oracle.kda_backward(x["q"], x["k"], x["v"], gv, x["eta"], x["eps"], x["h0"], do, dhT)
    _check(out, ref)


def test_kda_backward_beta():
    w = inputs.WORKLOADS["prefill_4k"].scaled(B=2, T=140, H=2, dk=64, dv=64)
    x = inputs.make_prefill(w, with_h0=True)
    kf = x["k"].float()
    k = (kf / kf.norm(dim=-1, keepdim=True)).to(x["k"].dtype)
    gv = inputs.channel_gates((2, 140, 2, 64), 85)
    rng = np.random.Generator(np.random.PCG64(86))
    beta = torch.from_numpy(rng.uniform(0.05, 1.95, x["g"].shape).astype(np.float32))
    do, dhT = _upstream(w, 87)
    xc = cuda(x)
    out = api.kda_recurrent_bwd_beta(xc["q"], cuda(k), xc["v"], cuda(gv), cuda(beta), cuda(do),
                                     xc["h0"], cuda(dhT))
    ref = oracle.kda_backward_beta(x["q"], k, x["v"], gv, beta, x["h0"], do, dhT)
    _check(out, ref, names=("dq", "dk", "dv", "dg", "dbeta", "dh0"))


def test_kda_backward_equal_channels_is_scalar_gate():
    """The same per-token gate on every channel: the per-channel kernels give
    the scalar-gate gradients (dg summed over channels)."""
    w = inputs.WORKLOADS["prefill_4k"].scaled(B=1, T=150, H=2)
    x = cuda(inputs.make_prefill(w))
    do, _ = _upstream(w, 88, False)
    do = cuda(do)
    gv = x["g"][..., None].expand(-1, -1, -1, w.dk).contiguous()
    a = api.kda_recurrent_bwd(x["q"], x["k"], x["v"], gv, x["eta"], do, x["eps"])
    b = api.recurrent_bwd(x["q"], x["k"], x["v"], x["g"], x["eta"], do, x["eps"])
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "deta", "dh0"):
        assert rel(a[n].cpu(), b[n].cpu()) < 1e-5, n
    assert rel(a["dg"].sum(-1).cpu(), b["dg"].cpu()) < 1e-5


# ---- chunkwise backward (kla_chunk_bwd): bf16, d = 128 on the chunk kernels
# (tf32 tensor-core products), so the bf16 bar applies
TOL_CHUNK = 1e-2


@pytest.mark.parametrize("name,B,T,H,with_h0,with_dhT", [
    ("prefill_4k", 1, 150, 2, True, True),     # 3 chunks, ragged last one
    ("prefill_4k", 2, 64, 3, False, True),     # exactly one chunk
    ("prefill_4k", 1, 1, 2, True, True),       # one token
    ("prefill_4k", 1, 257, 1, False, False),   # one token past 4 chunks
    ("prefill_65k", 1, 700, 2, False, True),   # strong forgets
    ("stress", 1, 200, 3, True, True),         # d = 64: key norms 1e-2 .. 1e2, eta up to 2
    ("stress", 2, 64, 2, True, False),
])
def test_chunk_backward(name, B, T, H, with_h0, with_dhT):
    w = inputs.WORKLOADS[name].scaled(B=B, T=T, H=H)
    x = inputs.make_prefill(w, with_h0=with_h0)
    do, dhT = _upstream(w, 90, with_dhT)
    xc = cuda(x)
    out = api.chunk_bwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], cuda(do), x["eps"],
                        xc["h0"], cuda(dhT))
    api.check_device_error()
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"], do, dhT)
    _check(out, ref, tol=TOL_CHUNK)


def test_gdn_chunk_backward():
    w = inputs.WORKLOADS["prefill_4k"].scaled(B=2, T=130, H=2)
    x = inputs.make_prefill(w, with_h0=True)
    kf = x["k"].float()
    k = (kf / kf.norm(dim=-1, keepdim=True)).to(x["k"].dtype)
    rng = np.random.Generator(np.random.PCG64(91))
    beta = torch.from_numpy(rng.uniform(0.05, 1.95, x["g"].shape).astype(np.float32))
    do, dhT = _upstream(w, 92)
    xc = cuda(x)
    out = api.gdn_chunk_bwd(xc["q"], cuda(k), xc["v"], xc["g"], cuda(beta), cuda(do), xc["h0"],
                            cuda(dhT))
    ref = oracle.gated_delta_backward(x["q"], k, x["v"], x["g"], beta, x["h0"], do, dhT)
    _check(out, ref, names=("dq", "dk", "dv", "dg", "dbeta", "dh0"), tol=TOL_CHUNK)


def test_chunk_backward_other_shapes_run_token_serial():
    """fp32 I/O and d = 64 take the token-serial kernels through the same
    entry point (the fp32 bar then holds)."""
    w = inputs.WORKLOADS["tiny"].scaled(B=1, T=100, H=2)
    x = inputs.make_prefill(w, with_h0=True)
    do, dhT = _upstream(w, 93)
    xc = cuda(x)
    out = api.chunk_bwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], cuda(do), x["eps"],
                        xc["h0"], cuda(dhT))
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"], do, dhT)
    _check(out, ref)


def test_chunk_backward_full_size_sampled_heads():
    """The 4K layer (B=8 T=4096 H=8 d=128, bf16) in one call on the chunk
    kernels; the oracle's gradients of two sampled heads."""
    w = inputs.WORKLOADS["prefill_4k"]
    x = inputs.make_prefill(w)
    do, dhT = _upstream(w, 94)
    xc = cuda(x)
    out = api.chunk_bwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["eta"], cuda(do), x["eps"],
                        None, cuda(dhT))
    api.check_device_error()
    for b, h in ((2, 6), (5, 1)):
        sl = lambda t: t[b:b + 1, :, h:h + 1]
        ref = oracle.backward(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["g"]), sl(x["eta"]),
                              x["eps"], None, sl(do), dhT[b:b + 1, h:h + 1])
        got = {n: sl(out[n].cpu()) for n in ("dq", "dk", "dv", "dg", "deta")}
        got["dh0"] = out["dh0"][b:b + 1, h:h + 1].cpu()
        _check(got, ref, tol=TOL_CHUNK)


def test_autograd_binding_matches_oracle_gradients():
    """kla_prefill under torch.autograd: a loss <o, do> + <hT, dhT> gives the
    oracle's gradients (bf16 inputs receive their gradients in bf16)."""
    from delta_rule_linear_kla_b200 import kla_prefill
    w = inputs.WORKLOADS["prefill_4k"].scaled(B=1, T=160, H=2)
    x = inputs.make_prefill(w, with_h0=True)
    do, dhT = _upstream(w, 95)
    leaves = {n: cuda(x[n]).requires_grad_(True) for n in ("q", "k", "v", "g", "eta", "h0")}
    o, hT = kla_prefill(leaves["q"], leaves["k"], leaves["v"], leaves["g"], leaves["eta"],
                        x["eps"], leaves["h0"])
    loss = (o.float() * cuda(do).float()).sum() + (hT * cuda(dhT)).sum()
    loss.backward()
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"], do, dhT)
    names = dict(q="dq", k="dk", v="dv", g="dg", eta="deta", h0="dh0")
    for n, rn in names.items():
        got = leaves[n].grad
        assert got.dtype == leaves[n].dtype
        err = rel(got.float().cpu(), ref[rn])
        # bf16 gradients add their own rounding (2^-9) to the kernels' error
        assert err < TOL_CHUNK, (n, err)
