"""Oracle for Kaczmarz Linear Attention -- TEST INFRASTRUCTURE ONLY.

A plain fp64 CPU evaluation of the KLA recurrence, token by token, compiled
from ``kla_oracle.c`` and called through ctypes.  Only the test-suite,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  It shares no code with the CUDA library; the only thing both
sides use is the seeded input generator, which holds none of the method's
arithmetic.

Sources of each formula (page title, section):
  * beta_t = eta_t / (||k_t||^2 + eps): "Kaczmarz Linear Attention", Abstract.
  * S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t:
    "Deep Dive into KDA", section 2.2 (Gated DeltaNet), which the KLA Abstract
    says KLA keeps unchanged apart from beta.
  * per-channel gate: S_t = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1}
    + beta_t v_t k_t^T, a_t = exp(g_t) per key channel (decay first, then the
    erase reads the decayed state): "Deep Dive into KDA", section 2.3 (KDA);
    the KLA Abstract names a preconditioned KDA (beta from the key norm).

Arrays follow the library's layouts: q, k ``[B, T, H, dk]``; v, o
``[B, T, H, dv]``; g, eta ``[B, T, H]``; states ``[B, H, dk, dv]`` holding
h = S^T.  Inputs may be numpy arrays or torch tensors of any float dtype; they
are widened exactly to float64 before use.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (fp64, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    dp = ctypes.POINTER(ctypes.c_double)
    i = ctypes.c_int
    lib.kla_oracle_beta.argtypes = [dp, dp, ctypes.c_double, dp, i, i, i, i]
    lib.kla_oracle_beta.restype = None
    lib.kla_oracle_gated_delta.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp,
                                           i, i, i, i, i]
    lib.kla_oracle_gated_delta.restype = None
    lib.kla_oracle_forward.argtypes = [dp, dp, dp, dp, dp, ctypes.c_double,
                                       dp, dp, dp, i, i, i, i, i]
    lib.kla_oracle_forward.restype = None
    lib.kla_oracle_kda.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, i, i, i, i, i]
    lib.kla_oracle_kda.restype = None
    lib.kla_oracle_backward.argtypes = [dp, dp, dp, dp, dp, ctypes.c_double, dp, dp, dp,
                                        dp, dp, dp, dp, dp, dp, i, i, i, i, i]
    lib.kla_oracle_backward.restype = None
    lib.kla_oracle_gated_delta_backward.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp,
                                                    dp, dp, dp, dp, dp, dp, i, i, i, i, i]
    lib.kla_oracle_gated_delta_backward.restype = None
    lib.kla_oracle_kda_backward.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp,
                                            dp, dp, dp, dp, dp, dp, i, i, i, i, i]
    lib.kla_oracle_kda_backward.restype = None
    lib.kla_oracle_num_threads.argtypes = []
    lib.kla_oracle_num_threads.restype = i
    _lib = lib
    return lib


def f64(x) -> np.ndarray:
    """Widen a numpy array or torch tensor exactly to contiguous float64."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: widen on the host, exactly
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def num_threads() -> int:
    return int(_load().kla_oracle_num_threads())


def beta(k, eta, eps: float) -> np.ndarray:
    """beta_t = eta_t / (||k_t||^2 + eps) per (b, t, h)."""
    k, eta = f64(k), f64(eta)
    B, T, H, dk = k.shape
    out = np.empty((B, T, H), dtype=np.float64)
    _load().kla_oracle_beta(_ptr(k), _ptr(eta), float(eps), _ptr(out), B, T, H, dk)
    return out


def gated_delta(q, k, v, g, beta_, h0=None):
    """Gated delta rule with beta given per token.  Returns (o, hT) in fp64."""
    q, k, v, g, beta_, h0 = map(f64, (q, k, v, g, beta_, h0))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == k.shape and v.shape[:3] == (B, T, H)
    assert g.shape == (B, T, H) and beta_.shape == (B, T, H)
    if h0 is not None:
        assert h0.shape == (B, H, dk, dv)
    o = np.empty((B, T, H, dv), dtype=np.float64)
    hT = np.empty((B, H, dk, dv), dtype=np.float64)
    _load().kla_oracle_gated_delta(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta_),
                                   _ptr(h0), _ptr(o), _ptr(hT), B, T, H, dk, dv)
    return o, hT


def forward(q, k, v, g, eta, eps: float, h0=None):
    """KLA prefill: returns (o [B,T,H,dv], hT [B,H,dk,dv]) in fp64."""
    q, k, v, g, eta, h0 = map(f64, (q, k, v, g, eta, h0))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == k.shape and v.shape[:3] == (B, T, H)
    assert g.shape == (B, T, H) and eta.shape == (B, T, H)
    if h0 is not None:
        assert h0.shape == (B, H, dk, dv)
    o = np.empty((B, T, H, dv), dtype=np.float64)
    hT = np.empty((B, H, dk, dv), dtype=np.float64)
    _load().kla_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(eta),
                               float(eps), _ptr(h0), _ptr(o), _ptr(hT),
                               B, T, H, dk, dv)
    return o, hT


def backward(q, k, v, g, eta, eps: float, h0, dout, dhT=None):
    """Gradients of KLA for dL/do = dout [B,T,H,dv] and dL/dh_T = dhT
    [B,H,dk,dv] (None = 0).  Returns dq, dk, dv, dg, deta, dh0 (fp64)."""
    q, k, v, g, eta, h0, dout, dhT = map(f64, (q, k, v, g, eta, h0, dout, dhT))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == k.shape and v.shape[:3] == (B, T, H) and dout.shape == v.shape
    out = dict(dq=np.empty_like(q), dk=np.empty_like(k), dv=np.empty_like(v),
               dg=np.empty((B, T, H)), deta=np.empty((B, T, H)),
               dh0=np.empty((B, H, dk, dv)))
    _load().kla_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(eta), float(eps),
                                _ptr(h0), _ptr(dout), _ptr(dhT), _ptr(out["dq"]),
                                _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]),
                                _ptr(out["deta"]), _ptr(out["dh0"]), B, T, H, dk, dv)
    return out


def gated_delta_backward(q, k, v, g, beta_, h0, dout, dhT=None):
    """Gradients of the gated delta rule (beta given per token) for
    dL/do = dout and dL/dh_T = dhT (None = 0).  Returns dq, dk, dv, dg,
    dbeta, dh0 (fp64)."""
    q, k, v, g, beta_, h0, dout, dhT = map(f64, (q, k, v, g, beta_, h0, dout, dhT))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == k.shape and v.shape[:3] == (B, T, H) and dout.shape == v.shape
    out = dict(dq=np.empty_like(q), dk=np.empty_like(k), dv=np.empty_like(v),
               dg=np.empty((B, T, H)), dbeta=np.empty((B, T, H)),
               dh0=np.empty((B, H, dk, dv)))
    _load().kla_oracle_gated_delta_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta_), _ptr(h0), _ptr(dout), _ptr(dhT),
        _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]),
        _ptr(out["dh0"]), B, T, H, dk, dv)
    return out


def kda_backward_beta(q, k, v, g, beta_, h0, dout, dhT=None):
    """Gradients of the per-channel-gate form with beta given (g [B,T,H,dk])
    for dL/do = dout and dL/dh_T = dhT (None = 0).  Returns dq, dk, dv, dg
    ([B,T,H,dk]), dbeta, dh0 (fp64)."""
    q, k, v, g, beta_, h0, dout, dhT = map(f64, (q, k, v, g, beta_, h0, dout, dhT))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == k.shape and g.shape == k.shape and dout.shape == v.shape
    out = dict(dq=np.empty_like(q), dk=np.empty_like(k), dv=np.empty_like(v),
               dg=np.empty_like(g), dbeta=np.empty((B, T, H)), dh0=np.empty((B, H, dk, dv)))
    _load().kla_oracle_kda_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta_), _ptr(h0), _ptr(dout), _ptr(dhT),
        _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]),
        _ptr(out["dh0"]), B, T, H, dk, dv)
    return out


def kda_backward(q, k, v, g, eta, eps: float, h0, dout, dhT=None):
    """Gradients of KLA with the per-channel gate (beta = eta / (||k||^2 +
    eps)): the beta-given gradients, then the step size's chain rule into
    deta and dk.  Returns dq, dk, dv, dg, deta, dh0 (fp64)."""
    kf = f64(k)
    n2 = (kf * kf).sum(-1)
    den = n2 + eps
    b = f64(eta) / den
    out = kda_backward_beta(q, k, v, g, b, h0, dout, dhT)
    db = out.pop("dbeta")
    out["deta"] = db / den
    out["dk"] = out["dk"] - (2.0 * db * f64(eta) / den ** 2)[..., None] * kf
    return out


def kda(q, k, v, g, beta_, h0=None):
    """Delta rule with a per-channel gate (KDA form), beta given per token:
    g [B,T,H,dk] (log-gate per key channel), beta [B,T,H].  Returns (o, hT)
    in fp64."""
    q, k, v, g, beta_, h0 = map(f64, (q, k, v, g, beta_, h0))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == k.shape and v.shape[:3] == (B, T, H)
    assert g.shape == (B, T, H, dk) and beta_.shape == (B, T, H)
    if h0 is not None:
        assert h0.shape == (B, H, dk, dv)
    o = np.empty((B, T, H, dv), dtype=np.float64)
    hT = np.empty((B, H, dk, dv), dtype=np.float64)
    _load().kla_oracle_kda(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta_), _ptr(h0),
                           _ptr(o), _ptr(hT), B, T, H, dk, dv)
    return o, hT


def kda_forward(q, k, v, g, eta, eps: float, h0=None):
    """KLA with the per-channel gate (preconditioned KDA): beta from the key
    norm, then :func:`kda`.  g is [B,T,H,dk].  Returns (o, hT) in fp64."""
    return kda(q, k, v, g, beta(k, eta, eps), h0)


def kda_decode_step(q, k, v, g, eta, eps: float, S):
    """One per-channel-gated decode token: g [B,H,dk].  Returns (o, S_new)."""
    q, k, v, g, eta, S = map(f64, (q, k, v, g, eta, S))
    o, S_new = kda_forward(q[:, None], k[:, None], v[:, None], g[:, None],
                           eta[:, None], eps, S)
    return o[:, 0], S_new


def decode_step(q, k, v, g, eta, eps: float, S):
    """One decode token: q, k [B,H,dk]; v [B,H,dv]; g, eta [B,H];
    S [B,H,dk,dv] (h-form).  Returns (o [B,H,dv], S_new) without touching S."""
    q, k, v, g, eta, S = map(f64, (q, k, v, g, eta, S))
    o, S_new = forward(q[:, None], k[:, None], v[:, None], g[:, None],
                       eta[:, None], eps, S)
    return o[:, 0], S_new


def rel_l2(x, ref) -> float:
    """||x - ref||_2 / ||ref||_2 over the whole tensor, in fp64."""
    x, ref = f64(x), f64(ref)
    den = float(np.linalg.norm(ref.ravel()))
    num = float(np.linalg.norm((x - ref).ravel()))
    return num / den if den > 0 else num
