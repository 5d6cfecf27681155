"""ctypes loader of libkla.so.  Raises loudly if the library is missing: the
product path has no fallback of any kind."""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkla.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "kla.h")

_lib = None

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t

SIGNATURES = {
    "kla_chunk_fwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "kla_chunk_fwd_segments": (_i, [_i, _i, _i, _i, _i, _i, _sz]),
    "kla_chunk_fwd_single_launch": (_i, [_i, _i, _i, _i, _i, _i, _sz]),
    "kla_chunk_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp,
                           _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "kla_chunk_fwd_states": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp, _vp,
                                  _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "kla_chunk_ut_transform": (_i, [_vp, _vp, _vp, _f, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "kla_chunk_ut_bound_check": (_i, [_vp, _vp, _vp, _f, _i, _i, _i, _i, _i, _vp, _sz, _vp,
                                      _vp]),
    "kla_chunk_state_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                 _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "kla_recurrent_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp,
                               _i, _i, _i, _i, _i, _i, _vp]),
    "kla_gdn_chunk_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                               _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "kla_gdn_decode_step": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                 _i, _i, _i, _i, _i, _vp]),
    "kla_decode_step": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp,
                             _i, _i, _i, _i, _i, _vp]),
    "kla_chunk_fwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp,
                                   _i, _i, _i, _i, _i, _i, _vp]),
    "kla_chunk_fwd_host_staging_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "kla_chunk_fwd_host": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp,
                                _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "kla_kda_chunk_fwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "kla_kda_chunk_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp,
                               _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "kla_kda_chunk_fwd_beta": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                    _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "kla_kda_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp,
                         _i, _i, _i, _i, _i, _i, _vp]),
    "kla_kda_fwd_beta": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                              _i, _i, _i, _i, _i, _i, _vp]),
    "kla_kda_decode_step": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp,
                                 _i, _i, _i, _i, _i, _vp]),
    "kla_kda_decode_step_beta": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                      _i, _i, _i, _i, _i, _vp]),
    "kla_recurrent_bwd_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "kla_recurrent_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp,
                               _vp, _vp, _vp, _vp, _vp, _vp,
                               _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "kla_gdn_recurrent_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                   _vp, _vp, _vp, _vp, _vp, _vp,
                                   _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "kla_kda_recurrent_bwd_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "kla_kda_recurrent_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp,
                                   _vp, _vp, _vp, _vp, _vp, _vp,
                                   _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "kla_kda_recurrent_bwd_beta": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                        _vp, _vp, _vp, _vp, _vp, _vp,
                                        _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "kla_chunk_bwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "kla_chunk_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp,
                           _vp, _vp, _vp, _vp, _vp, _vp,
                           _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "kla_gdn_chunk_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                               _vp, _vp, _vp, _vp, _vp, _vp,
                               _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "kla_check_device_error": (_i, [_vp]),
    "kla_selftest_wait_timeout": (_i, [ctypes.c_uint, _vp]),
    "kla_status_string": (ctypes.c_char_p, [_i]),
    "kla_version": (_i, []),
}


def header_symbols(path: str = HEADER):
    """Names of the entry points kla.h declares (KLA_API-prefixed)."""
    text = open(path).read()
    return re.findall(r"KLA_API\s+[\w\s\*]+?\b(kla_\w+)\s*\(", text)


def lib():
    """The loaded library (ctypes.CDLL).  Raises RuntimeError if unavailable."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            "libkla.so is not built (%s); run delta_rule_linear_kla_b200/build.py "
            "or __graft_entry__.build()" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L
