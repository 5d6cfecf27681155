"""The seeded generators: determinism, shapes, dtypes and distribution facts."""
import numpy as np
import torch

from delta_rule_linear_kla_b200 import inputs


def test_prefill_deterministic_and_shaped():
    w = inputs.WORKLOADS["prefill_4k"].scaled(B=1, T=130, H=2)
    a = inputs.make_prefill(w)
    b = inputs.make_prefill(w)
    for key in ("q", "k", "v", "g", "eta"):
        assert torch.equal(a[key], b[key])
    assert a["q"].shape == (1, 130, 2, 128) and a["q"].dtype == torch.bfloat16
    assert a["g"].shape == (1, 130, 2) and a["g"].dtype == torch.float32
    assert a["h0"] is None and a["eps"] == 1e-6 and a["chunk"] == 64
    assert (a["g"] < 0).all() and ((a["eta"] > 0) & (a["eta"] < 1)).all()


def test_key_scale_ranges():
    w = inputs.WORKLOADS["prefill_4k"].scaled(B=1, T=512, H=4)
    x = inputs.make_prefill(w)
    n = x["k"].float().norm(dim=-1) / np.sqrt(128)
    assert 0.15 < float(n.min()) and float(n.max()) < 6.0
    s = inputs.make_prefill(inputs.WORKLOADS["stress"].scaled(B=1, T=512, H=4))
    ns = s["k"].float().norm(dim=-1)
    assert float(ns.min()) >= 0.0099 and float(ns.max()) <= 100.5
    assert s["h0"] is not None and s["h0"].shape == (1, 4, 64, 64)
    assert float((s["g"] == 0).float().mean()) > 0.4
    assert float(s["eta"].max()) > 1.5


def test_long_context_strong_forgets_shared_by_heads():
    w = inputs.WORKLOADS["prefill_65k"].scaled(T=4096, H=4)
    x = inputs.make_prefill(w)
    g = x["g"][0]  # [T, H]
    strong = (g <= -2.0) & (g >= -5.0) & (g == g[:, :1])
    rows = strong.all(dim=1)
    assert 10 < int(rows.sum()) < 100  # ~1% of 4096 tokens


def test_tiny_is_fp32():
    x = inputs.make_prefill(inputs.WORKLOADS["tiny"])
    assert x["q"].dtype == torch.float32 and x["q"].shape == (1, 256, 2, 64)


def test_decode_inputs():
    w = inputs.DECODE.scaled(B=2, H=3, prefix_tokens=16, steps=5)
    d = inputs.make_decode(w)
    assert d["prefix"]["k"].shape == (2, 16, 3, 128)
    assert d["steps"]["q"].shape == (5, 2, 3, 128)
    assert d["steps"]["g"].shape == (5, 2, 3)
    d2 = inputs.make_decode(w)
    assert torch.equal(d["steps"]["v"], d2["steps"]["v"])
