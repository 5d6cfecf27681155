"""Failure detection without a GPU fault: a bounded device-side wait that
runs out (a barrier phase nothing completes) reports KLA_ERR_TIMEOUT through
the device error word, the word is cleared by reading it, and the context
keeps working afterwards."""
import time

import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_kla_b200 import _native, api, inputs

from helpers import TOL, cuda, rel

pytestmark = pytest.mark.gpu
TIMEOUT = 4


def test_bounded_wait_times_out_and_context_survives():
    lib = _native.lib()
    st = torch.cuda.current_stream().cuda_stream
    api.check_device_error()  # start from a clear error word
    t0 = time.perf_counter()
    assert lib.kla_selftest_wait_timeout(50, st) == 0
    with pytest.raises(api.KLAError) as e:
        api.check_device_error()
    waited = time.perf_counter() - t0
    assert e.value.status == TIMEOUT
    assert 0.04 < waited < 10.0
    assert lib.kla_check_device_error(st) == 0  # reading cleared it
    # the context is intact: a decode step still matches the oracle
    w = inputs.DECODE.scaled(B=2, H=2, prefix_tokens=24)
    d = inputs.make_decode(w, steps=1)
    s = d["steps"]
    rng = np.random.Generator(np.random.PCG64(81))
    S0 = torch.from_numpy(rng.normal(0, 0.1, (w.B, w.H, w.dk, w.dv)).astype(np.float32))
    S = cuda(S0.clone())
    o = api.decode_step(*(cuda(s[n][0]) for n in ("q", "k", "v", "g", "eta")), S, d["eps"])
    api.check_device_error()
    o_ref, S_ref = oracle.decode_step(*(s[n][0] for n in ("q", "k", "v", "g", "eta")), d["eps"],
                                      S0)
    assert rel(o.cpu(), o_ref) < TOL["bf16"] and rel(S.cpu(), S_ref) < TOL["fp32"]
