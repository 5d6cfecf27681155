"""Python binding of the KLA C ABI (include/kla.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libkla.so.  Tensors must live on the current CUDA device; outputs
are allocated here with torch (the library itself never allocates).
"""
from __future__ import annotations

import contextlib
from typing import Optional, Tuple

import torch

from . import _native

KLA_BF16, KLA_FP32 = 0, 1
CHUNK = 64
_DT = {torch.bfloat16: KLA_BF16, torch.float32: KLA_FP32}


class KLAError(RuntimeError):
    """A non-OK kla_status returned by the library."""

    def __init__(self, status: int, where: str):
        msg = _native.lib().kla_status_string(status).decode()
        super().__init__("%s: %s (status %d)" % (where, msg, status))
        self.status = status


def _check(status: int, where: str):
    if status != 0:
        raise KLAError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _need(t, name, dtype=None, shape=None, dev=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if dev is not None and t.device != dev:
        raise ValueError("%s is on %s, the call's other tensors on %s" % (name, t.device, dev))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


@contextlib.contextmanager
def _on(ref, stream):
    """Device and stream of one call: ``ref``'s device is made current (the
    library sizes its TMA maps and error word for the current device) and
    ``stream`` (default: that device's current stream) becomes torch's
    current stream, so every temporary allocated inside (outputs,
    workspaces) belongs to the stream the kernels run on.  The caching
    allocator then only reuses a freed temporary for work ordered after
    those kernels.  Yields the raw stream handle for the C call."""
    _need(ref, "q")
    dev = ref.device
    with torch.cuda.device(dev):
        s = torch.cuda.current_stream(dev) if stream is None else stream
        if s.device != dev:
            raise ValueError("stream is on %s, the tensors on %s" % (s.device, dev))
        with torch.cuda.stream(s):
            yield s.cuda_stream


def chunk_fwd_workspace_size(B: int, T: int, H: int, dk: int, dv: int,
                             dtype: torch.dtype = torch.bfloat16) -> int:
    return int(_native.lib().kla_chunk_fwd_workspace_size(B, T, H, dk, dv, _DT[dtype]))


def chunk_fwd_segments(B: int, T: int, H: int, dk: int, dv: int,
                       dtype: torch.dtype = torch.bfloat16, ws_bytes: Optional[int] = None) -> int:
    """Segments the bf16 state chain runs in (1 = uncut, 0 = not the chunk
    path); ws_bytes defaults to the full workspace size."""
    if ws_bytes is None:
        ws_bytes = chunk_fwd_workspace_size(B, T, H, dk, dv, dtype)
    return int(_native.lib().kla_chunk_fwd_segments(B, T, H, dk, dv, _DT[dtype], ws_bytes))


def chunk_fwd_single_launch(B: int, T: int, H: int, dk: int, dv: int,
                            dtype: torch.dtype = torch.bfloat16,
                            ws_bytes: Optional[int] = None) -> bool:
    """Whether the bf16 prefill of this shape runs as one kernel launch
    (kla_chunk_fwd_single_launch); ws_bytes defaults to the full workspace
    size.  False for every shape at present: the single launch is built but
    not taken."""
    if ws_bytes is None:
        ws_bytes = chunk_fwd_workspace_size(B, T, H, dk, dv, dtype)
    return bool(_native.lib().kla_chunk_fwd_single_launch(B, T, H, dk, dv, _DT[dtype],
                                                          ws_bytes))


def _prefill_args(q, k, v, g, eta, h0, o, hT, return_state):
    _need(q, "q")
    if q.dtype not in _DT:
        raise ValueError("q, k, v must be bfloat16 or float32")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    d = q.device
    _need(k, "k", q.dtype, (B, T, H, dk), d)
    _need(v, "v", q.dtype, (B, T, H, dv), d)
    _need(g, "g", torch.float32, (B, T, H), d)
    _need(eta, "eta", torch.float32, (B, T, H), d)
    _need(h0, "h0", torch.float32, (B, H, dk, dv), d)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=d)
    _need(o, "o", q.dtype, (B, T, H, dv), d)
    if hT is None and return_state:
        hT = torch.empty((B, H, dk, dv), dtype=torch.float32, device=d)
    _need(hT, "hT", torch.float32, (B, H, dk, dv), d)
    return B, T, H, dk, dv, o, hT


def chunk_fwd(q, k, v, g, eta, eps: float = 1e-6, h0=None, *, o=None, hT=None,
              return_state: bool = True, workspace=None,
              stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunkwise KLA prefill (kla_chunk_fwd).  Returns (o, hT)."""
    with _on(q, stream) as s:
        B, T, H, dk, dv, o, hT = _prefill_args(q, k, v, g, eta, h0, o, hT, return_state)
        need = chunk_fwd_workspace_size(B, T, H, dk, dv, q.dtype)
        if need and workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        _need(workspace, "workspace", torch.uint8, dev=q.device)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = _native.lib().kla_chunk_fwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(eta), float(eps), _ptr(h0),
            _ptr(o), _ptr(hT), B, T, H, dk, dv, CHUNK, _DT[q.dtype], _ptr(workspace),
            ws_bytes, s)
    _check(st, "kla_chunk_fwd")
    return o, hT


def chunk_fwd_states(q, k, v, g, eta, eps: float = 1e-6, h0=None, *, outputs: bool = True,
                     workspace=None, stream=None):
    """bf16 chunk prefill that also returns the state at the start of every
    chunk (kla_chunk_fwd_states).  Returns (o, hT, hs) with hs
    [B, H, ceil(T / 64), dk, dv] fp32; o and hT are None if not outputs."""
    with _on(q, stream) as s:
        B, T, H, dk, dv, o, hT = _prefill_args(q, k, v, g, eta, h0, None, None, outputs)
        if not outputs:
            o = None
        hs = torch.empty((B, H, (T + CHUNK - 1) // CHUNK, dk, dv), dtype=torch.float32,
                         device=q.device)
        need = chunk_fwd_workspace_size(B, T, H, dk, dv, q.dtype)
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
        _need(workspace, "workspace", torch.uint8, dev=q.device)
        ws_bytes = workspace.numel() * workspace.element_size()
        st = _native.lib().kla_chunk_fwd_states(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(eta), float(eps), _ptr(h0), _ptr(o),
            _ptr(hT), _ptr(hs), B, T, H, dk, dv, _DT[q.dtype], _ptr(workspace), ws_bytes, s)
    _check(st, "kla_chunk_fwd_states")
    return o, hT, hs


def _workspace(workspace, B, T, H, dk, dv, dtype, device):
    need = chunk_fwd_workspace_size(B, T, H, dk, dv, dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
    _need(workspace, "workspace", torch.uint8, dev=device)
    return workspace, workspace.numel() * workspace.element_size()


def chunk_ut_transform(k, g, eta, eps: float = 1e-6, *, workspace=None, stream=None):
    """First stage of the bf16 chunk prefill (kla_chunk_ut_transform): the
    per-chunk factors T diag(beta), T diag(beta e^G) into the workspace,
    which is returned."""
    _need(k, "k", torch.bfloat16)
    B, T, H, dk = k.shape
    _need(g, "g", torch.float32, (B, T, H), k.device)
    _need(eta, "eta", torch.float32, (B, T, H), k.device)
    with _on(k, stream) as s:
        workspace, ws_bytes = _workspace(workspace, B, T, H, dk, dk, k.dtype, k.device)
        st = _native.lib().kla_chunk_ut_transform(
            _ptr(k), _ptr(g), _ptr(eta), float(eps), B, T, H, dk, KLA_BF16, _ptr(workspace),
            ws_bytes, s)
    _check(st, "kla_chunk_ut_transform")
    return workspace


def chunk_ut_bound_check(k, g, eta, eps: float = 1e-6, *, workspace=None, stream=None):
    """kla_chunk_ut_transform with the debug check of its factors
    (kla_chunk_ut_bound_check).  Returns (workspace, ratio_max) with
    ratio_max a one-element fp32 CUDA tensor: the largest ratio of
    |T_rs| ||k_r|| / ||k_s|| to eta'_r e^{G_r - G_s} over the factors'
    entries.  A ratio above 1.25 also sets the device error word
    (check_device_error then raises KLAError with KLA_ERR_BOUND)."""
    _need(k, "k", torch.bfloat16)
    B, T, H, dk = k.shape
    _need(g, "g", torch.float32, (B, T, H), k.device)
    _need(eta, "eta", torch.float32, (B, T, H), k.device)
    with _on(k, stream) as s:
        workspace, ws_bytes = _workspace(workspace, B, T, H, dk, dk, k.dtype, k.device)
        ratio = torch.empty(4, dtype=torch.float32, device=k.device)  # 16-byte aligned
        st = _native.lib().kla_chunk_ut_bound_check(
            _ptr(k), _ptr(g), _ptr(eta), float(eps), B, T, H, dk, KLA_BF16, _ptr(workspace),
            ws_bytes, _ptr(ratio), s)
    _check(st, "kla_chunk_ut_bound_check")
    return workspace, ratio[:1]


def chunk_state_fwd(q, k, v, g, workspace, h0=None, *, o=None, hT=None,
                    return_state: bool = True, stream=None):
    """Second stage of the bf16 chunk prefill (kla_chunk_state_fwd): the
    state recurrence and outputs from a workspace made by chunk_ut_transform
    of the same k and g.  Returns (o, hT)."""
    with _on(q, stream) as s:
        B, T, H, dk, dv, o, hT = _prefill_args(q, k, v, g, g, h0, o, hT, return_state)
        if workspace is None:
            raise ValueError("workspace must be a CUDA tensor")
        _need(workspace, "workspace", torch.uint8, dev=q.device)
        ws_bytes = workspace.numel() * workspace.element_size()
        st = _native.lib().kla_chunk_state_fwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(h0), _ptr(o), _ptr(hT), B, T, H, dk, dv,
            _DT[q.dtype], _ptr(workspace), ws_bytes, s)
    _check(st, "kla_chunk_state_fwd")
    return o, hT


def recurrent_fwd(q, k, v, g, eta, eps: float = 1e-6, h0=None, *, o=None, hT=None,
                  return_state: bool = True, stream=None):
    """Token-serial KLA prefill on CUDA cores (kla_recurrent_fwd)."""
    with _on(q, stream) as s:
        B, T, H, dk, dv, o, hT = _prefill_args(q, k, v, g, eta, h0, o, hT, return_state)
        st = _native.lib().kla_recurrent_fwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(eta), float(eps), _ptr(h0),
            _ptr(o), _ptr(hT), B, T, H, dk, dv, _DT[q.dtype], s)
    _check(st, "kla_recurrent_fwd")
    return o, hT


def recurrent_bwd_workspace_size(B: int, T: int, H: int, dk: int, dv: int) -> int:
    return int(_native.lib().kla_recurrent_bwd_workspace_size(B, T, H, dk, dv))


def kda_recurrent_bwd_workspace_size(B: int, T: int, H: int, dk: int, dv: int) -> int:
    return int(_native.lib().kla_kda_recurrent_bwd_workspace_size(B, T, H, dk, dv))


def chunk_bwd_workspace_size(B: int, T: int, H: int, dk: int, dv: int,
                             dtype: torch.dtype = torch.bfloat16) -> int:
    return int(_native.lib().kla_chunk_bwd_workspace_size(B, T, H, dk, dv, _DT[dtype]))


def _bwd(fn, name, q, k, v, g, step, eps, h0, grad_o, grad_hT, need_h0, workspace, stream,
         vector_gate=False, chunked=False):
    _need(q, "q")
    if q.dtype not in _DT:
        raise ValueError("q, k, v must be bfloat16 or float32")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    d = q.device
    _need(k, "k", q.dtype, (B, T, H, dk), d)
    _need(v, "v", q.dtype, (B, T, H, dv), d)
    gshape = (B, T, H, dk) if vector_gate else (B, T, H)
    _need(g, "g", torch.float32, gshape, d)
    _need(step, "eta/beta", torch.float32, (B, T, H), d)
    _need(h0, "h0", torch.float32, (B, H, dk, dv), d)
    _need(grad_o, "grad_o", q.dtype, (B, T, H, dv), d)
    _need(grad_hT, "grad_hT", torch.float32, (B, H, dk, dv), d)
    with _on(q, stream) as s:
        return _bwd_launch(fn, name, q, k, v, g, step, eps, h0, grad_o, grad_hT, need_h0,
                           workspace, s, gshape, vector_gate, chunked)


def _bwd_launch(fn, name, q, k, v, g, step, eps, h0, grad_o, grad_hT, need_h0, workspace, s,
                gshape, vector_gate, chunked):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    f32 = dict(dtype=torch.float32, device=q.device)
    out = dict(dq=torch.empty((B, T, H, dk), **f32), dk=torch.empty((B, T, H, dk), **f32),
               dv=torch.empty((B, T, H, dv), **f32), dg=torch.empty(gshape, **f32),
               dstep=torch.empty((B, T, H), **f32),
               dh0=torch.empty((B, H, dk, dv), **f32) if need_h0 else None)
    if chunked:
        need = chunk_bwd_workspace_size(B, T, H, dk, dv, q.dtype)
    else:
        need = (kda_recurrent_bwd_workspace_size if vector_gate
                else recurrent_bwd_workspace_size)(B, T, H, dk, dv)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace", torch.uint8, dev=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(step)]
    if eps is not None:
        args.append(float(eps))
    args += [_ptr(h0), _ptr(grad_o), _ptr(grad_hT), _ptr(out["dq"]), _ptr(out["dk"]),
             _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dstep"]), _ptr(out["dh0"]),
             B, T, H, dk, dv, _DT[q.dtype], _ptr(workspace), ws_bytes, s]
    _check(fn(*args), name)
    return out


def recurrent_bwd(q, k, v, g, eta, grad_o, eps: float = 1e-6, h0=None, grad_hT=None, *,
                  need_h0: bool = True, workspace=None, stream=None):
    """Gradients of the KLA prefill for dL/do = grad_o and dL/dh_T = grad_hT
    (None = 0), token-serial fp32 (kla_recurrent_bwd).  Returns a dict of
    fp32 tensors dq, dk, dv, dg, deta, dh0 (None unless need_h0)."""
    out = _bwd(_native.lib().kla_recurrent_bwd, "kla_recurrent_bwd", q, k, v, g, eta, eps, h0,
               grad_o, grad_hT, need_h0, workspace, stream)
    out["deta"] = out.pop("dstep")
    return out


def chunk_bwd(q, k, v, g, eta, grad_o, eps: float = 1e-6, h0=None, grad_hT=None, *,
              need_h0: bool = True, workspace=None, stream=None):
    """Gradients of the KLA prefill from the chunk form (kla_chunk_bwd):
    dq, dk, dv, dg, deta, dh0 (fp32).  bf16 with d = 128 runs the chunkwise
    tensor-core kernels, everything else the token-serial ones."""
    out = _bwd(_native.lib().kla_chunk_bwd, "kla_chunk_bwd", q, k, v, g, eta, eps, h0, grad_o,
               grad_hT, need_h0, workspace, stream, chunked=True)
    out["deta"] = out.pop("dstep")
    return out


def gdn_chunk_bwd(q, k, v, g, beta, grad_o, h0=None, grad_hT=None, *, need_h0: bool = True,
                  workspace=None, stream=None):
    """The same with beta given per token (kla_gdn_chunk_bwd)."""
    out = _bwd(_native.lib().kla_gdn_chunk_bwd, "kla_gdn_chunk_bwd", q, k, v, g, beta, None, h0,
               grad_o, grad_hT, need_h0, workspace, stream, chunked=True)
    out["dbeta"] = out.pop("dstep")
    return out


def kda_recurrent_bwd(q, k, v, g, eta, grad_o, eps: float = 1e-6, h0=None, grad_hT=None, *,
                      need_h0: bool = True, workspace=None, stream=None):
    """Gradients of the per-channel-gate prefill (g [B,T,H,dk]), KLA step
    size (kla_kda_recurrent_bwd): dq, dk, dv, dg [B,T,H,dk], deta, dh0."""
    out = _bwd(_native.lib().kla_kda_recurrent_bwd, "kla_kda_recurrent_bwd", q, k, v, g, eta,
               eps, h0, grad_o, grad_hT, need_h0, workspace, stream, vector_gate=True)
    out["deta"] = out.pop("dstep")
    return out


def kda_recurrent_bwd_beta(q, k, v, g, beta, grad_o, h0=None, grad_hT=None, *,
                           need_h0: bool = True, workspace=None, stream=None):
    """The same with beta given per token (kla_kda_recurrent_bwd_beta):
    dq, dk, dv, dg, dbeta, dh0."""
    out = _bwd(_native.lib().kla_kda_recurrent_bwd_beta, "kla_kda_recurrent_bwd_beta", q, k, v,
               g, beta, None, h0, grad_o, grad_hT, need_h0, workspace, stream, vector_gate=True)
    out["dbeta"] = out.pop("dstep")
    return out


def gdn_recurrent_bwd(q, k, v, g, beta, grad_o, h0=None, grad_hT=None, *, need_h0: bool = True,
                      workspace=None, stream=None):
    """Gradients of the gated delta rule prefill (beta given per token):
    dq, dk, dv, dg, dbeta, dh0 (kla_gdn_recurrent_bwd)."""
    out = _bwd(_native.lib().kla_gdn_recurrent_bwd, "kla_gdn_recurrent_bwd", q, k, v, g, beta,
               None, h0, grad_o, grad_hT, need_h0, workspace, stream)
    out["dbeta"] = out.pop("dstep")
    return out


def decode_step(q, k, v, g, eta, S, eps: float = 1e-6, *, o=None, stream=None):
    """One decode token per sequence; S [B,H,dk,dv] fp32 is updated in place.
    Returns o [B,H,dv]."""
    _need(q, "q")
    if q.dtype not in _DT:
        raise ValueError("q, k, v must be bfloat16 or float32")
    B, H, dk = q.shape
    dv = v.shape[-1]
    d = q.device
    _need(k, "k", q.dtype, (B, H, dk), d)
    _need(v, "v", q.dtype, (B, H, dv), d)
    _need(g, "g", torch.float32, (B, H), d)
    _need(eta, "eta", torch.float32, (B, H), d)
    _need(S, "S", torch.float32, (B, H, dk, dv), d)
    with _on(q, stream) as s:
        if o is None:
            o = torch.empty((B, H, dv), dtype=q.dtype, device=d)
        _need(o, "o", q.dtype, (B, H, dv), d)
        st = _native.lib().kla_decode_step(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(eta), float(eps), _ptr(S), _ptr(o),
            B, H, dk, dv, _DT[q.dtype], s)
    _check(st, "kla_decode_step")
    return o


def gdn_chunk_fwd(q, k, v, g, beta, h0=None, *, o=None, hT=None, return_state: bool = True,
                  workspace=None, stream=None):
    """Gated DeltaNet prefill (kla_gdn_chunk_fwd): beta [B,T,H] fp32 is the
    step size itself.  Returns (o, hT)."""
    with _on(q, stream) as s:
        B, T, H, dk, dv, o, hT = _prefill_args(q, k, v, g, beta, h0, o, hT, return_state)
        need = chunk_fwd_workspace_size(B, T, H, dk, dv, q.dtype)
        if need and workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        _need(workspace, "workspace", torch.uint8, dev=q.device)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = _native.lib().kla_gdn_chunk_fwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(o), _ptr(hT),
            B, T, H, dk, dv, CHUNK, _DT[q.dtype], _ptr(workspace), ws_bytes, s)
    _check(st, "kla_gdn_chunk_fwd")
    return o, hT


def gdn_decode_step(q, k, v, g, beta, S, *, o=None, stream=None):
    """One Gated DeltaNet decode token per sequence (kla_gdn_decode_step);
    S is updated in place.  Returns o [B,H,dv]."""
    _need(q, "q")
    if q.dtype not in _DT:
        raise ValueError("q, k, v must be bfloat16 or float32")
    B, H, dk = q.shape
    dv = v.shape[-1]
    d = q.device
    _need(k, "k", q.dtype, (B, H, dk), d)
    _need(v, "v", q.dtype, (B, H, dv), d)
    _need(g, "g", torch.float32, (B, H), d)
    _need(beta, "beta", torch.float32, (B, H), d)
    _need(S, "S", torch.float32, (B, H, dk, dv), d)
    with _on(q, stream) as s:
        if o is None:
            o = torch.empty((B, H, dv), dtype=q.dtype, device=d)
        _need(o, "o", q.dtype, (B, H, dv), d)
        st = _native.lib().kla_gdn_decode_step(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o), B, H, dk, dv,
            _DT[q.dtype], s)
    _check(st, "kla_gdn_decode_step")
    return o


def _need_host(t, name, dtype, shape):
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise ValueError("%s must be a host (CPU) tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError("%s must be %s of shape %s" % (name, dtype, tuple(shape)))


def chunk_fwd_host_staging_size(B: int, T: int, H: int, dk: int, dv: int,
                                dtype: torch.dtype = torch.bfloat16) -> int:
    return int(_native.lib().kla_chunk_fwd_host_staging_size(B, T, H, dk, dv, _DT[dtype]))


def chunk_fwd_host(q, k, v, g, eta, eps: float = 1e-6, h0=None, *, o=None, hT=None,
                   return_state: bool = True, staging=None, device=None, stream=None):
    """Prefill from host tensors (kla_chunk_fwd_host): the copies to and
    from the device are pipelined against the kernels.  Inputs and outputs
    are CPU tensors (pin them for the copies to overlap; outputs allocated
    here are pinned).  Only enqueues work: synchronise ``stream`` before
    reading o, hT.  Returns (o, hT)."""
    if q.dtype not in _DT:
        raise ValueError("q, k, v must be bfloat16 or float32")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for t, n, dt, sh in ((q, "q", q.dtype, (B, T, H, dk)), (k, "k", q.dtype, (B, T, H, dk)),
                         (v, "v", q.dtype, (B, T, H, dv)), (g, "g", torch.float32, (B, T, H)),
                         (eta, "eta", torch.float32, (B, T, H)),
                         (h0, "h0", torch.float32, (B, H, dk, dv))):
        _need_host(t, n, dt, sh)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, pin_memory=True)
    _need_host(o, "o", q.dtype, (B, T, H, dv))
    if hT is None and return_state:
        hT = torch.empty((B, H, dk, dv), dtype=torch.float32, pin_memory=True)
    _need_host(hT, "hT", torch.float32, (B, H, dk, dv))
    if device is None:
        device = staging.device if staging is not None else (
            stream.device if stream is not None else
            torch.device("cuda", torch.cuda.current_device()))
    dev = torch.device(device)
    need = chunk_fwd_host_staging_size(B, T, H, dk, dv, q.dtype)
    with torch.cuda.device(dev):
        s = torch.cuda.current_stream(dev) if stream is None else stream
        if s.device != dev:
            raise ValueError("stream is on %s, the staging buffer on %s" % (s.device, dev))
        with torch.cuda.stream(s):
            if staging is None:
                staging = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
            _need(staging, "staging", torch.uint8, dev=dev)
            st = _native.lib().kla_chunk_fwd_host(
                _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(eta), float(eps), _ptr(h0), _ptr(o),
                _ptr(hT), B, T, H, dk, dv, _DT[q.dtype], _ptr(staging),
                staging.numel() * staging.element_size(), s.cuda_stream)
    _check(st, "kla_chunk_fwd_host")
    return o, hT


def _kda_prefill(fn, name, q, k, v, g, step, eps, h0, o, hT, return_state, stream):
    # the per-token arguments as for chunk_fwd; g is checked on its own
    with _on(q, stream) as s:
        B, T, H, dk, dv, o, hT = _prefill_args(q, k, v, None, step, h0, o, hT, return_state)
        if g is None:
            raise ValueError("g must be a CUDA tensor")
        _need(g, "g", torch.float32, (B, T, H, dk), q.device)
        args = [_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(step)]
        if eps is not None:
            args.append(float(eps))
        st = fn(*args, _ptr(h0), _ptr(o), _ptr(hT), B, T, H, dk, dv, _DT[q.dtype], s)
    _check(st, name)
    return o, hT


def kda_fwd(q, k, v, g, eta, eps: float = 1e-6, h0=None, *, o=None, hT=None,
            return_state: bool = True, stream=None):
    """KLA prefill with a per-channel gate (kla_kda_fwd): g [B,T,H,dk] fp32,
    one log-gate per key channel.  Returns (o, hT)."""
    return _kda_prefill(_native.lib().kla_kda_fwd, "kla_kda_fwd", q, k, v, g, eta, eps, h0,
                        o, hT, return_state, stream)


def kda_fwd_beta(q, k, v, g, beta, h0=None, *, o=None, hT=None, return_state: bool = True,
                 stream=None):
    """Per-channel-gated prefill with beta given per token (kla_kda_fwd_beta)."""
    return _kda_prefill(_native.lib().kla_kda_fwd_beta, "kla_kda_fwd_beta", q, k, v, g, beta,
                        None, h0, o, hT, return_state, stream)


def kda_chunk_fwd_workspace_size(B: int, T: int, H: int, dk: int, dv: int,
                                 dtype: torch.dtype = torch.bfloat16) -> int:
    return int(_native.lib().kla_kda_chunk_fwd_workspace_size(B, T, H, dk, dv, _DT[dtype]))


def _kda_chunk(fn, name, q, k, v, g, step, eps, h0, o, hT, return_state, workspace, stream):
    with _on(q, stream) as s:
        B, T, H, dk, dv, o, hT = _prefill_args(q, k, v, None, step, h0, o, hT, return_state)
        if g is None:
            raise ValueError("g must be a CUDA tensor")
        _need(g, "g", torch.float32, (B, T, H, dk), q.device)
        need = kda_chunk_fwd_workspace_size(B, T, H, dk, dv, q.dtype)
        if need and workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        _need(workspace, "workspace", torch.uint8, dev=q.device)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        args = [_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(step)]
        if eps is not None:
            args.append(float(eps))
        st = fn(*args, _ptr(h0), _ptr(o), _ptr(hT), B, T, H, dk, dv, CHUNK, _DT[q.dtype],
                _ptr(workspace), ws_bytes, s)
    _check(st, name)
    return o, hT


def kda_chunk_fwd(q, k, v, g, eta, eps: float = 1e-6, h0=None, *, o=None, hT=None,
                  return_state: bool = True, workspace=None, stream=None):
    """Per-channel-gate prefill as chunks (kla_kda_chunk_fwd): g [B,T,H,dk]
    fp32.  bf16 runs the tensor-core chunk path.  Returns (o, hT)."""
    return _kda_chunk(_native.lib().kla_kda_chunk_fwd, "kla_kda_chunk_fwd", q, k, v, g, eta,
                      eps, h0, o, hT, return_state, workspace, stream)


def kda_chunk_fwd_beta(q, k, v, g, beta, h0=None, *, o=None, hT=None, return_state: bool = True,
                       workspace=None, stream=None):
    """kda_chunk_fwd with beta given per token (kla_kda_chunk_fwd_beta)."""
    return _kda_chunk(_native.lib().kla_kda_chunk_fwd_beta, "kla_kda_chunk_fwd_beta", q, k, v,
                      g, beta, None, h0, o, hT, return_state, workspace, stream)


def _kda_decode(fn, name, q, k, v, g, step, eps, S, o, stream):
    _need(q, "q")
    if q.dtype not in _DT:
        raise ValueError("q, k, v must be bfloat16 or float32")
    B, H, dk = q.shape
    dv = v.shape[-1]
    d = q.device
    _need(k, "k", q.dtype, (B, H, dk), d)
    _need(v, "v", q.dtype, (B, H, dv), d)
    _need(g, "g", torch.float32, (B, H, dk), d)
    _need(step, "eta" if eps is not None else "beta", torch.float32, (B, H), d)
    _need(S, "S", torch.float32, (B, H, dk, dv), d)
    with _on(q, stream) as s:
        if o is None:
            o = torch.empty((B, H, dv), dtype=q.dtype, device=d)
        _need(o, "o", q.dtype, (B, H, dv), d)
        args = [_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(step)]
        if eps is not None:
            args.append(float(eps))
        st = fn(*args, _ptr(S), _ptr(o), B, H, dk, dv, _DT[q.dtype], s)
    _check(st, name)
    return o


def kda_decode_step(q, k, v, g, eta, S, eps: float = 1e-6, *, o=None, stream=None):
    """One per-channel-gated decode token (kla_kda_decode_step): g [B,H,dk];
    S is updated in place.  Returns o [B,H,dv]."""
    return _kda_decode(_native.lib().kla_kda_decode_step, "kla_kda_decode_step", q, k, v, g,
                       eta, eps, S, o, stream)


def kda_decode_step_beta(q, k, v, g, beta, S, *, o=None, stream=None):
    """Per-channel-gated decode token with beta given (kla_kda_decode_step_beta)."""
    return _kda_decode(_native.lib().kla_kda_decode_step_beta, "kla_kda_decode_step_beta",
                       q, k, v, g, beta, None, S, o, stream)


def check_device_error(stream=None):
    """Synchronise and raise KLAError if a kernel reported a timed-out wait
    (on the device of ``stream``; default: the current device's current
    stream)."""
    s = torch.cuda.current_stream() if stream is None else stream
    with torch.cuda.device(s.device):
        _check(_native.lib().kla_check_device_error(s.cuda_stream), "kla_check_device_error")
