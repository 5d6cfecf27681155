"""kla_chunk_fwd_noalloc: the prefill for callers that cannot allocate.

Some integrations own all device memory through another allocator, or may
not allocate once they are running, so they cannot pass kla_chunk_fwd a
workspace.  The no-allocation entry point runs the same prefill with a fixed
scratch array built into libkla.so.  These tests call it through the C ABI
and compare it with kla_chunk_fwd given a torch-allocated workspace of the
same size as that array (so both run the same kernels with the same segment
count, and the results must be identical bit for bit), on two calls in a
row with different inputs, so a stale array from the first call would show
up in the second.  One shape cuts the state chain into segments, the path
that keeps segment states in the array.  Each result is also checked
against the fp64 oracle.  This file is collected last on purpose.
"""
import pytest
import torch

import oracle
from delta_rule_linear_kla_b200 import _native, api, inputs
from helpers import assert_parity, assert_state_parity

OK, UNSUPPORTED = 0, 2
MAX_CHUNKS = 1024
SCRATCH_BYTES = MAX_CHUNKS * 16384


def _call(lib, x, o, hT, B, T, H, d, dtype_code=0):
    return lib.kla_chunk_fwd_noalloc(
        x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), x["g"].data_ptr(),
        x["eta"].data_ptr(), x["eps"], x["h0"].data_ptr(), o.data_ptr(), hT.data_ptr(),
        B, T, H, d, d, dtype_code, torch.cuda.current_stream().cuda_stream)


def _run_twice(w_of_seed, expect_cut):
    lib = _native.lib()
    for seed in (31, 32):  # two calls in a row
        w = w_of_seed(seed)
        xh = inputs.make_prefill(w, with_h0=True)
        x = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in xh.items()}
        d = w.dk
        nseg = api.chunk_fwd_segments(w.B, w.T, w.H, d, d, torch.bfloat16, SCRATCH_BYTES)
        assert (nseg > 1) == expect_cut, nseg
        ws = torch.empty(SCRATCH_BYTES, dtype=torch.uint8, device="cuda")
        o_ref, h_ref = api.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"],
                                     x["h0"], workspace=ws)
        o = torch.full_like(o_ref, float("nan"))
        hT = torch.full_like(h_ref, float("nan"))
        assert _call(lib, x, o, hT, w.B, w.T, w.H, d) == OK
        torch.cuda.synchronize()
        # same kernels, same inputs, same segment count: identical results
        assert torch.equal(o, o_ref) and torch.equal(hT, h_ref)
        o64, h64 = oracle.forward(xh["q"], xh["k"], xh["v"], xh["g"], xh["eta"], xh["eps"],
                                  xh["h0"])
        assert_parity(o.cpu(), o64, "bf16")
        assert_state_parity(hT.cpu(), h64, "bf16")


@pytest.mark.gpu
@pytest.mark.parametrize("d", [128, 64])
def test_noalloc_matches_workspace_entry_point_twice(d):
    base = inputs.WORKLOADS["prefill_4k" if d == 128 else "stress"]
    _run_twice(lambda seed: base.scaled(B=2, T=300, H=3, seed=seed), expect_cut=False)


@pytest.mark.gpu
def test_noalloc_cut_chain_twice():
    """64 chunks of one head: the chain is cut into segments whose states
    live in the shared array after the factors."""
    base = inputs.WORKLOADS["prefill_4k"]
    _run_twice(lambda seed: base.scaled(B=1, T=4096, H=1, seed=seed), expect_cut=True)


@pytest.mark.gpu
def test_noalloc_fp32_has_no_chunk_limit():
    """fp32 I/O runs the token-serial kernel, which needs no scratch: more
    chunks than the bf16 limit are accepted and match the oracle."""
    lib = _native.lib()
    w = inputs.WORKLOADS["tiny"].scaled(B=1, H=1, T=64 * (MAX_CHUNKS + 1), seed=33)
    xh = inputs.make_prefill(w, with_h0=True)
    x = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in xh.items()}
    o = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device="cuda")
    hT = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    assert _call(lib, x, o, hT, w.B, w.T, w.H, w.dk, dtype_code=1) == OK
    torch.cuda.synchronize()
    o64, h64 = oracle.forward(xh["q"], xh["k"], xh["v"], xh["g"], xh["eta"], xh["eps"],
                              xh["h0"])
    assert_parity(o.cpu(), o64, "fp32")
    assert_state_parity(hT.cpu(), h64, "fp32")


def test_noalloc_rejects_more_chunks_than_its_scratch():
    """Over the limit a bf16 call fails with KLA_ERR_UNSUPPORTED before any
    CUDA call (so this runs without a GPU), also where the chunk count only
    exceeds the limit in 64-bit arithmetic."""
    lib = _native.lib()
    A = 1 << 20  # never dereferenced: the size check comes first
    T = 64 * 1025  # 1025 chunks > KLA_NOALLOC_MAX_CHUNKS (1024)
    st = lib.kla_chunk_fwd_noalloc(A, 2 * A, 3 * A, 4 * A, 5 * A, 1e-6, None, 6 * A, None,
                                   1, T, 1, 128, 128, 0, None)
    assert st == UNSUPPORTED
    st = lib.kla_chunk_fwd_noalloc(A, 2 * A, 3 * A, 4 * A, 5 * A, 1e-6, None, 6 * A, None,
                                   2, 64 * 512 + 1, 1, 64, 64, 0, None)
    assert st == UNSUPPORTED
    # T within 63 of INT_MAX: ceil(T / 64) must not wrap
    st = lib.kla_chunk_fwd_noalloc(A, 2 * A, 3 * A, 4 * A, 5 * A, 1e-6, None, 6 * A, None,
                                   1, 2**31 - 10, 1, 64, 64, 0, None)
    assert st == UNSUPPORTED
