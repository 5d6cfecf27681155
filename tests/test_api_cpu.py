"""The Python binding is marshalling only: every compute entry point refuses
host (CPU) tensors with a clear error instead of computing anything on the
CPU, and the workspace queries answer without a GPU."""
import pytest
import torch

from delta_rule_linear_kla_b200 import api, inputs, kla_prefill

W = inputs.WORKLOADS["prefill_4k"].scaled(B=1, T=70, H=2)


def _x():
    x = inputs.make_prefill(W)
    gv = torch.zeros((W.B, W.T, W.H, W.dk))
    do = torch.zeros_like(x["v"])
    S = torch.zeros((W.B, W.H, W.dk, W.dv))
    t = lambda a: a[:, 0]
    return x, gv, do, S, t


CALLS = {
    "chunk_fwd": lambda x, gv, do, S, t: api.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["eta"]),
    "chunk_fwd_states": lambda x, gv, do, S, t: api.chunk_fwd_states(x["q"], x["k"], x["v"],
                                                                     x["g"], x["eta"]),
    "chunk_ut_transform": lambda x, gv, do, S, t: api.chunk_ut_transform(x["k"], x["g"], x["eta"]),
    "recurrent_fwd": lambda x, gv, do, S, t: api.recurrent_fwd(x["q"], x["k"], x["v"], x["g"],
                                                               x["eta"]),
    "gdn_chunk_fwd": lambda x, gv, do, S, t: api.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["g"],
                                                               x["eta"]),
    "kda_chunk_fwd": lambda x, gv, do, S, t: api.kda_chunk_fwd(x["q"], x["k"], x["v"], gv,
                                                               x["eta"]),
    "kda_fwd": lambda x, gv, do, S, t: api.kda_fwd(x["q"], x["k"], x["v"], gv, x["eta"]),
    "decode_step": lambda x, gv, do, S, t: api.decode_step(t(x["q"]), t(x["k"]), t(x["v"]),
                                                           t(x["g"]), t(x["eta"]), S),
    "gdn_decode_step": lambda x, gv, do, S, t: api.gdn_decode_step(t(x["q"]), t(x["k"]),
                                                                   t(x["v"]), t(x["g"]),
                                                                   t(x["eta"]), S),
    "kda_decode_step": lambda x, gv, do, S, t: api.kda_decode_step(t(x["q"]), t(x["k"]),
                                                                   t(x["v"]), t(gv), t(x["eta"]),
                                                                   S),
    "chunk_bwd": lambda x, gv, do, S, t: api.chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["eta"],
                                                       do),
    "gdn_chunk_bwd": lambda x, gv, do, S, t: api.gdn_chunk_bwd(x["q"], x["k"], x["v"], x["g"],
                                                               x["eta"], do),
    "recurrent_bwd": lambda x, gv, do, S, t: api.recurrent_bwd(x["q"], x["k"], x["v"], x["g"],
                                                               x["eta"], do),
    "kda_recurrent_bwd": lambda x, gv, do, S, t: api.kda_recurrent_bwd(x["q"], x["k"], x["v"],
                                                                       gv, x["eta"], do),
    "kla_prefill": lambda x, gv, do, S, t: kla_prefill(x["q"], x["k"], x["v"], x["g"], x["eta"]),
}


@pytest.mark.parametrize("name", sorted(CALLS))
def test_host_tensors_are_refused(name):
    with pytest.raises(ValueError, match="CUDA"):
        CALLS[name](*_x())


def test_workspace_queries_need_no_gpu():
    d = dict(B=2, T=300, H=3, dk=128, dv=128)
    # the factors (16 KiB per chunk); the chain is uncut at this length
    assert api.chunk_fwd_workspace_size(**d) == 2 * 3 * 5 * 16384
    assert not api.chunk_fwd_single_launch(**d)
    assert api.chunk_bwd_workspace_size(**d) > api.chunk_fwd_workspace_size(**d)
    assert api.recurrent_bwd_workspace_size(**d) > 0
    assert api.kda_chunk_fwd_workspace_size(**d) > 0
    assert api.chunk_bwd_workspace_size(2, 300, 3, 128, 64) == 0  # d_k != d_v: unsupported


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without libkla.so there is no other path: the first call that needs
    the library raises."""
    from delta_rule_linear_kla_b200 import _native
    monkeypatch.setattr(_native, "LIB_PATH", str(tmp_path / "libkla.so"))
    monkeypatch.setattr(_native, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        api.chunk_fwd_workspace_size(1, 64, 1, 128, 128)
