"""kla_chunk_fwd_noalloc: the prefill for callers that cannot allocate.

Some integrations own all device memory through another allocator, or may
not allocate once they are running, so they cannot pass kla_chunk_fwd a
workspace.  The no-allocation entry point runs the same prefill with a fixed
scratch array built into libkla.so.  These tests call it through the C ABI
and compare it with kla_chunk_fwd (given a torch-allocated workspace) on two
calls in a row with different inputs, so a stale array from the first call
would show up in the second.  This file is collected last on purpose.
"""
import pytest
import torch

from delta_rule_linear_kla_b200 import _native, api, inputs

OK, UNSUPPORTED = 0, 2
TOL = 1e-2


def _call(lib, x, o, hT, B, T, H, d):
    return lib.kla_chunk_fwd_noalloc(
        x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), x["g"].data_ptr(),
        x["eta"].data_ptr(), x["eps"], x["h0"].data_ptr(), o.data_ptr(), hT.data_ptr(),
        B, T, H, d, d, 0, torch.cuda.current_stream().cuda_stream)


def _rel(a, b):
    a, b = a.double(), b.double()
    return float((a - b).norm() / b.norm())


@pytest.mark.gpu
@pytest.mark.parametrize("d", [128, 64])
def test_noalloc_matches_workspace_entry_point_twice(d):
    lib = _native.lib()
    base = inputs.WORKLOADS["prefill_4k" if d == 128 else "stress"]
    for seed in (31, 32):  # two calls in a row
        w = base.scaled(B=2, T=300, H=3, seed=seed)
        x = {k: (v.cuda() if isinstance(v, torch.Tensor) else v)
             for k, v in inputs.make_prefill(w, with_h0=True).items()}
        o_ref, h_ref = api.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["eta"], x["eps"], x["h0"])
        o = torch.full_like(o_ref, float("nan"))
        hT = torch.full_like(h_ref, float("nan"))
        assert _call(lib, x, o, hT, w.B, w.T, w.H, d) == OK
        torch.cuda.synchronize()
        assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()
        assert _rel(o, o_ref) < TOL and _rel(hT, h_ref) < TOL


def test_noalloc_rejects_more_chunks_than_its_scratch():
    """Over the limit the call fails with KLA_ERR_UNSUPPORTED before any
    CUDA call (so this runs without a GPU)."""
    lib = _native.lib()
    A = 1 << 20  # never dereferenced: the size check comes first
    T = 64 * 1025  # 1025 chunks > KLA_NOALLOC_MAX_CHUNKS (1024)
    st = lib.kla_chunk_fwd_noalloc(A, 2 * A, 3 * A, 4 * A, 5 * A, 1e-6, None, 6 * A, None,
                                   1, T, 1, 128, 128, 0, None)
    assert st == UNSUPPORTED
    st = lib.kla_chunk_fwd_noalloc(A, 2 * A, 3 * A, 4 * A, 5 * A, 1e-6, None, 6 * A, None,
                                   2, 64 * 512 + 1, 1, 64, 64, 0, None)
    assert st == UNSUPPORTED
