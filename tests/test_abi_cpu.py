"""The C ABI on a machine without a GPU: the library loads, exports every
entry point include/kla.h declares, and rejects bad arguments on the host
before any CUDA call (no compute call is made here)."""
import ctypes

import pytest

from delta_rule_linear_kla_b200 import _native
from delta_rule_linear_kla_b200 import build as kbuild

OK, INVALID, UNSUPPORTED = 0, 1, 2
A = 1 << 20  # fake, 16-byte-aligned device addresses: never dereferenced here


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return _native.lib()


def test_exports_every_declared_symbol(lib):
    names = _native.header_symbols()
    assert len(names) >= 7
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_native.SIGNATURES)


def test_status_strings(lib):
    for s in range(5):
        assert lib.kla_status_string(s)
    assert lib.kla_status_string(99) == b"unknown status"
    assert lib.kla_version() >= 100


def _fwd(lib, q=A, k=2 * A, v=3 * A, g=4 * A, eta=5 * A, eps=1e-6, h0=None, o=6 * A,
         hT=None, B=1, T=128, H=2, dk=128, dv=128, chunk=64, dtype=0, ws=None, wsb=0):
    return lib.kla_chunk_fwd(q, k, v, g, eta, eps, h0, o, hT, B, T, H, dk, dv, chunk,
                             dtype, ws, wsb, None)


def test_prefill_rejects_bad_arguments(lib):
    assert _fwd(lib, q=None) == INVALID
    assert _fwd(lib, o=None) == INVALID
    assert _fwd(lib, k=2 * A + 8) == INVALID          # misaligned
    assert _fwd(lib, B=0) == INVALID
    assert _fwd(lib, T=-1) == INVALID
    assert _fwd(lib, dtype=7) == INVALID
    assert _fwd(lib, eps=-1.0) == INVALID
    assert _fwd(lib, eps=float("nan")) == INVALID
    assert _fwd(lib, o=A + 256) == INVALID             # o overlaps q
    assert _fwd(lib, h0=7 * A, hT=7 * A + 1024) == INVALID  # partial state overlap
    assert _fwd(lib, dk=96, dv=96) == UNSUPPORTED
    assert _fwd(lib, dk=128, dv=64) == UNSUPPORTED
    assert _fwd(lib, chunk=32) == UNSUPPORTED
    assert lib.kla_recurrent_fwd(None, 2 * A, 3 * A, 4 * A, 5 * A, 1e-6, None, 6 * A,
                                 None, 1, 4, 1, 64, 64, 1, None) == INVALID
    assert lib.kla_recurrent_fwd(A, 2 * A, 3 * A, 4 * A, 5 * A, 1e-6, None, 6 * A,
                                 None, 1, 4, 1, 32, 32, 1, None) == UNSUPPORTED


def test_prefill_stages_reject_bad_arguments(lib):
    ws, wsb = 8 * A, 1 << 22
    ut = lambda **kw: lib.kla_chunk_ut_transform(
        kw.get("k", 2 * A), kw.get("g", 4 * A), kw.get("eta", 5 * A), kw.get("eps", 1e-6),
        kw.get("B", 1), kw.get("T", 128), kw.get("H", 2), kw.get("dk", 128),
        kw.get("dtype", 0), kw.get("ws", ws), kw.get("wsb", wsb), None)
    assert ut(k=None) == INVALID
    assert ut(T=0) == INVALID
    assert ut(ws=None) == INVALID
    assert ut(wsb=16) == INVALID                       # workspace too small
    assert ut(ws=2 * A + 64) == INVALID                # workspace overlaps k
    assert ut(dk=96) == UNSUPPORTED
    assert ut(dtype=1) == UNSUPPORTED                  # fp32 I/O has no stages
    st = lambda **kw: lib.kla_chunk_state_fwd(
        kw.get("q", A), kw.get("k", 2 * A), kw.get("v", 3 * A), kw.get("g", 4 * A),
        kw.get("h0", None), kw.get("o", 6 * A), kw.get("hT", None), kw.get("B", 1),
        kw.get("T", 128), kw.get("H", 2), kw.get("dk", 128), kw.get("dv", 128),
        kw.get("dtype", 0), kw.get("ws", ws), kw.get("wsb", wsb), None)
    assert st(q=None) == INVALID
    assert st(o=A + 256) == INVALID                    # o overlaps q
    assert st(o=ws + 1024) == INVALID                  # o overlaps the workspace
    assert st(wsb=16) == INVALID
    assert st(dk=128, dv=64) == UNSUPPORTED
    assert st(dtype=1) == UNSUPPORTED


def test_gdn_entry_points_reject_bad_arguments(lib):
    gdn = lambda **kw: lib.kla_gdn_chunk_fwd(
        kw.get("q", A), kw.get("k", 2 * A), kw.get("v", 3 * A), kw.get("g", 4 * A),
        kw.get("beta", 5 * A), None, kw.get("o", 6 * A), None, 1, kw.get("T", 128), 2,
        kw.get("dk", 128), kw.get("dv", 128), kw.get("chunk", 64), kw.get("dtype", 0),
        None, 0, None)
    assert gdn(beta=None) == INVALID
    assert gdn(o=A + 256) == INVALID                   # o overlaps q
    assert gdn(dk=96, dv=96) == UNSUPPORTED
    assert gdn(chunk=32) == UNSUPPORTED
    assert gdn(dtype=0) == INVALID                     # bf16 needs a workspace
    args = [A, 2 * A, 3 * A, 4 * A, 5 * A, 6 * A, 7 * A, 2, 3, 128, 128, 0, None]
    bad = list(args); bad[4] = None
    assert lib.kla_gdn_decode_step(*bad) == INVALID
    bad = list(args); bad[9], bad[10] = 80, 80
    assert lib.kla_gdn_decode_step(*bad) == UNSUPPORTED


def test_kda_entry_points_reject_bad_arguments(lib):
    """Per-channel gate: g is [B][T][H][dk] (prefill) / [B][H][dk] (decode)."""
    kda = lambda **kw: lib.kla_kda_fwd(
        kw.get("q", A), kw.get("k", 2 * A), kw.get("v", 3 * A), kw.get("g", 4 * A),
        kw.get("eta", 5 * A), kw.get("eps", 1e-6), None, kw.get("o", 6 * A), kw.get("hT", None),
        1, kw.get("T", 128), 2, kw.get("dk", 128), kw.get("dv", 128), kw.get("dtype", 0), None)
    assert kda(g=None) == INVALID
    assert kda(eps=-1.0) == INVALID
    assert kda(dk=96, dv=96) == UNSUPPORTED
    # 1 x 128 x 2 x 128 fp32 gates = 128 KiB: o placed inside that range
    assert kda(o=4 * A + 64 * 1024) == INVALID
    assert kda(hT=4 * A + 64 * 1024) == INVALID        # written state over the gates
    assert lib.kla_kda_fwd_beta(A, 2 * A, 3 * A, 4 * A, None, None, 6 * A, None, 1, 4, 1,
                                64, 64, 1, None) == INVALID
    args = [A, 2 * A, 3 * A, 4 * A, 5 * A, 1e-6, 6 * A, 7 * A, 2, 3, 128, 128, 0, None]
    bad = list(args); bad[7] = 4 * A + 2048          # o inside the 3 KiB of gates
    assert lib.kla_kda_decode_step(*bad) == INVALID
    bad = list(args); bad[5] = -1.0
    assert lib.kla_kda_decode_step(*bad) == INVALID
    bad = list(args); bad[10], bad[11] = 80, 80
    assert lib.kla_kda_decode_step(*bad) == UNSUPPORTED
    bargs = [A, 2 * A, 3 * A, 4 * A, None, 6 * A, 7 * A, 2, 3, 128, 128, 0, None]
    assert lib.kla_kda_decode_step_beta(*bargs) == INVALID


def test_host_prefill_rejects_bad_arguments(lib):
    """kla_chunk_fwd_host: host pointers, a device staging buffer; every
    check below returns before any CUDA call."""
    need = lib.kla_chunk_fwd_host_staging_size(3, 100, 2, 64, 64, 0)
    assert need > 0
    assert lib.kla_chunk_fwd_host_staging_size(3, 0, 2, 64, 64, 0) == 0
    assert lib.kla_chunk_fwd_host_staging_size(3, 100, 2, 64, 64, 5) == 0
    host = lambda **kw: lib.kla_chunk_fwd_host(
        kw.get("q", A), kw.get("k", 2 * A), kw.get("v", 3 * A), kw.get("g", 4 * A),
        kw.get("eta", 5 * A), kw.get("eps", 1e-6), None, kw.get("o", 6 * A), None, 3,
        kw.get("T", 100), 2, kw.get("dk", 64), kw.get("dv", 64), 0, kw.get("st", 64 * A),
        kw.get("stb", need), None)
    assert host(q=None) == INVALID
    assert host(o=None) == INVALID
    assert host(T=0) == INVALID
    assert host(eps=-1.0) == INVALID
    assert host(st=64 * A + 16) == INVALID             # staging not 256-byte aligned
    assert host(stb=need - 1) == INVALID               # staging too small
    assert host(st=None) == INVALID
    assert host(dk=96, dv=96) == UNSUPPORTED


def test_decode_rejects_bad_arguments(lib):
    args = [A, 2 * A, 3 * A, 4 * A, 5 * A, 1e-6, 6 * A, 7 * A, 2, 3, 128, 128, 0, None]
    bad = list(args); bad[6] = None
    assert lib.kla_decode_step(*bad) == INVALID
    bad = list(args); bad[7] = 6 * A + 64            # o inside S
    assert lib.kla_decode_step(*bad) == INVALID
    bad = list(args); bad[10], bad[11] = 80, 80
    assert lib.kla_decode_step(*bad) == UNSUPPORTED
    bad = list(args); bad[8] = 0
    assert lib.kla_decode_step(*bad) == INVALID


def _ut_bytes(B, T, H):
    return B * H * ((T + 63) // 64) * 16384  # two 64 x 64 bf16 factors per chunk


def test_selftest_rejects_bad_limits(lib):
    assert lib.kla_selftest_wait_timeout(0, None) == INVALID
    assert lib.kla_selftest_wait_timeout(10001, None) == INVALID


def test_workspace_query(lib):
    # an uncut chain: the per-chunk factors alone (a short batch, the
    # 0.4B-scale layer, more state CTAs than SMs)
    assert lib.kla_chunk_fwd_workspace_size(2, 1000, 4, 128, 128, 0) == _ut_bytes(2, 1000, 4)
    assert lib.kla_chunk_fwd_workspace_size(8, 4096, 8, 128, 128, 0) == _ut_bytes(8, 4096, 8)
    assert lib.kla_chunk_fwd_workspace_size(16, 4096, 8, 128, 128, 0) == _ut_bytes(16, 4096, 8)
    # the single launch is not taken for any shape: its factors are always
    # formed by a launch of their own
    full = lambda *a: lib.kla_chunk_fwd_workspace_size(*a, 128, 128, 0)
    for B, T, H, d in ((2, 1000, 4, 128), (8, 4096, 8, 128), (16, 4096, 8, 128),
                       (1, 65536, 16, 128), (2, 777, 8, 64), (1, 64, 1, 128)):
        for dt in (0, 1):
            assert lib.kla_chunk_fwd_single_launch(B, T, H, d, d, dt, 1 << 40) == 0
    assert lib.kla_chunk_fwd_single_launch(2, 1000, 4, 128, 128, 0, full(2, 1000, 4)) == 0
    # few heads and a long sequence: per-segment states (E, start state,
    # transition) follow the factors, for between 2 and 64 segments
    n = lib.kla_chunk_fwd_workspace_size(1, 65536, 16, 128, 128, 0)
    per_seg = 16 * (2 * 128 * 128 + 128 * 128) * 4
    extra = n - _ut_bytes(1, 65536, 16)
    assert extra > 0 and extra % per_seg == 0 and 2 <= extra // per_seg <= 64
    assert lib.kla_chunk_fwd_segments(1, 65536, 16, 128, 128, 0, n) == extra // per_seg
    # the cost model's choices at the benchmark shapes: three segments at 65K
    # (on a B200 the fastest of 1..16 segments: 1.29 ms against 1.84 ms for
    # two and 1.50 ms for four), the 4K layer and the stress shape uncut
    assert extra // per_seg == 3
    assert lib.kla_chunk_fwd_segments(4, 8192, 32, 64, 64, 0, 1 << 40) == 1
    assert lib.kla_chunk_fwd_segments(1, 65536, 16, 128, 128, 0, n - 16) == 1  # no room: uncut
    assert lib.kla_chunk_fwd_segments(8, 4096, 8, 128, 128, 0, 1 << 40) == 1
    assert lib.kla_chunk_fwd_segments(1, 65536, 16, 128, 128, 1, n) == 0  # fp32 I/O
    assert lib.kla_chunk_fwd_segments(1, 65536, 16, 96, 96, 0, n) == 0
    # short sequences are never cut (segments keep at least 8 chunks)
    assert lib.kla_chunk_fwd_workspace_size(1, 64 * 15, 1, 64, 64, 0) == _ut_bytes(1, 960, 1)
    assert lib.kla_chunk_fwd_workspace_size(1, 65536, 16, 128, 128, 1) == 0  # fp32: none


def test_prefill_workspace_checks(lib):
    ws = 8 * A
    assert _fwd(lib, ws=ws, wsb=_ut_bytes(1, 128, 2) - 16) == INVALID  # factors do not fit
    assert _fwd(lib, ws=2 * A, wsb=1 << 22) == INVALID                 # overlaps k
    # a cut chain (B=1, T=1536, H=1, d=64): the factors end right where o
    # starts, so only the segment states past them would overlap o
    T, d = 1536, 64
    full = lib.kla_chunk_fwd_workspace_size(1, T, 1, d, d, 0)
    ut = _ut_bytes(1, T, 1)
    assert full > ut
    assert _fwd(lib, ws=6 * A - ut, wsb=full, T=T, H=1, dk=d, dv=d) == INVALID


def _bwd(lib, q=A, k=2 * A, v=3 * A, g=4 * A, eta=5 * A, eps=1e-6, h0=None, go=6 * A,
         ghT=None, gq=7 * A, gk=8 * A, gv=9 * A, gg=10 * A, geta=11 * A, gh0=None, B=1, T=128,
         H=2, dk=128, dv=128, dtype=0, ws=64 * A, wsb=None):
    if wsb is None:
        wsb = lib.kla_recurrent_bwd_workspace_size(B, T, H, dk, dv)
    return lib.kla_recurrent_bwd(q, k, v, g, eta, eps, h0, go, ghT, gq, gk, gv, gg, geta, gh0,
                                 B, T, H, dk, dv, dtype, ws, wsb, None)


def test_backward_rejects_bad_arguments(lib):
    # the fake buffers above are 1 MiB apart: big enough for these sizes
    need = lib.kla_recurrent_bwd_workspace_size(1, 128, 2, 128, 128)
    assert need > 2 * 2 * 128 * 128 * 4  # two checkpoints for each of the two heads
    assert lib.kla_recurrent_bwd_workspace_size(1, 128, 2, 96, 96) == 0
    assert _bwd(lib, dk=96, dv=96) == UNSUPPORTED
    assert _bwd(lib, wsb=need - 1) == INVALID
    assert _bwd(lib, ws=None) == INVALID
    assert _bwd(lib, eps=-1.0) == INVALID
    assert _bwd(lib, B=0) == INVALID
    assert _bwd(lib, dtype=7) == INVALID
    assert _bwd(lib, gq=None) == INVALID
    assert _bwd(lib, go=None) == INVALID
    assert _bwd(lib, q=A + 4) == INVALID          # misaligned
    assert _bwd(lib, gk=7 * A) == INVALID         # two gradients in one buffer
    assert _bwd(lib, gv=3 * A) == INVALID         # a gradient over an input
    assert _bwd(lib, ws=2 * A) == INVALID         # workspace over an input
    assert _bwd(lib, gh0=64 * A + 4096) == INVALID  # dh0 inside the workspace
    # T == 0 with nothing to write: valid, no CUDA call
    assert _bwd(lib, T=0, ws=None, wsb=0) == OK
    # the gated delta variant takes the same checks (beta for eta, no eps)
    assert lib.kla_gdn_recurrent_bwd(A, 2 * A, 3 * A, 4 * A, 5 * A, None, 6 * A, None, 7 * A,
                                     7 * A, 9 * A, 10 * A, 11 * A, None, 1, 128, 2, 128, 128,
                                     0, 64 * A, need, None) == INVALID


def test_kda_backward_rejects_bad_arguments(lib):
    need = lib.kla_kda_recurrent_bwd_workspace_size(1, 128, 2, 128, 128)
    assert need > lib.kla_recurrent_bwd_workspace_size(1, 128, 2, 128, 128)
    args = [A, 2 * A, 3 * A, 4 * A, 5 * A, 1e-6, None, 6 * A, None, 7 * A, 8 * A, 9 * A,
            10 * A, 11 * A, None, 1, 128, 2, 128, 128, 0, 64 * A, need, None]
    bad = list(args); bad[22] = need - 1
    assert lib.kla_kda_recurrent_bwd(*bad) == INVALID
    bad = list(args); bad[12] = 4 * A + 64  # grad_g ([B,T,H,dk] fp32) over g
    assert lib.kla_kda_recurrent_bwd(*bad) == INVALID
    beta_args = args[:5] + args[6:]
    bad = list(beta_args); bad[17] = 96; bad[18] = 96
    assert lib.kla_kda_recurrent_bwd_beta(*bad) == UNSUPPORTED


def test_chunk_backward_rejects_bad_arguments(lib):
    """kla_chunk_bwd: the chunk kernels' workspace for bf16 (d = 64, 128),
    the token-serial one for fp32 I/O; the same argument checks as the
    token-serial entry points (no CUDA call is made for these)."""
    need = lib.kla_chunk_bwd_workspace_size(1, 128, 2, 128, 128, 0)
    # per chunk: h_n, dH (64 KiB each), T (16 KiB), V', dV', W, X (32 KiB each), Y (64 KiB)
    assert need >= 4 * (2 * 65536 + 16384 + 4 * 32768 + 65536)
    assert lib.kla_chunk_bwd_workspace_size(1, 128, 2, 64, 64, 0) < need
    assert lib.kla_chunk_bwd_workspace_size(1, 128, 2, 128, 128, 1) == \
        lib.kla_recurrent_bwd_workspace_size(1, 128, 2, 128, 128)
    assert lib.kla_chunk_bwd_workspace_size(1, 128, 2, 96, 96, 0) == 0
    args = [A, 2 * A, 3 * A, 4 * A, 5 * A, 1e-6, None, 6 * A, None, 7 * A, 8 * A, 9 * A,
            10 * A, 11 * A, None, 1, 128, 2, 128, 128, 0, 64 * A, need, None]
    bad = list(args); bad[22] = need - 1
    assert lib.kla_chunk_bwd(*bad) == INVALID
    bad = list(args); bad[5] = -1.0
    assert lib.kla_chunk_bwd(*bad) == INVALID
    bad = list(args); bad[9] = 3 * A  # grad_q over v
    assert lib.kla_chunk_bwd(*bad) == INVALID
    bad = list(args); bad[18] = 96; bad[19] = 96
    assert lib.kla_chunk_bwd(*bad) == UNSUPPORTED
    gdn = args[:5] + args[6:]
    bad = list(gdn); bad[20] = None  # no workspace
    assert lib.kla_gdn_chunk_bwd(*bad) == INVALID
    assert lib.kla_gdn_chunk_bwd(*(gdn[:14] + [0] + gdn[15:])) == INVALID  # B = 0


def test_chunk_fwd_states_rejects_bad_arguments(lib):
    ws = lib.kla_chunk_fwd_workspace_size(1, 128, 2, 128, 128, 0)
    args = [A, 2 * A, 3 * A, 4 * A, 5 * A, 1e-6, None, None, None, 7 * A,
            1, 128, 2, 128, 128, 0, 16 * A, ws, None]
    bad = list(args); bad[9] = A  # states over q
    assert lib.kla_chunk_fwd_states(*bad) == INVALID
    bad = list(args); bad[9] = None
    assert lib.kla_chunk_fwd_states(*bad) == INVALID
    bad = list(args); bad[15] = 1
    assert lib.kla_chunk_fwd_states(*bad) == UNSUPPORTED  # fp32 I/O
    bad = list(args); bad[17] = _ut_bytes(1, 128, 2) - 1  # the factors do not fit
    assert lib.kla_chunk_fwd_states(*bad) == INVALID
    bad = list(args); bad[11] = 0
    assert lib.kla_chunk_fwd_states(*bad) == INVALID  # T = 0
