"""Test helpers: move seeded inputs to the GPU and compare with the oracle."""
import numpy as np
import torch

import oracle

TOL = {"bf16": 1e-2, "fp32": 1e-4}  # relative L2 bars for bf16 / fp32 I/O


def cuda(x):
    if x is None:
        return None
    if isinstance(x, dict):
        return {k: cuda(v) for k, v in x.items()}
    if isinstance(x, torch.Tensor):
        return x.cuda().contiguous()
    return x


def rel(x, ref):
    return oracle.rel_l2(x, ref)


def worst_head_rel(o, o_ref):
    """Largest relative L2 error over (b, h) slices of a [B,T,H,d] output."""
    o, o_ref = oracle.f64(o), oracle.f64(o_ref)
    B, _, H, _ = o.shape
    return max(rel(o[b, :, h], o_ref[b, :, h]) for b in range(B) for h in range(H))


def oracle_decode_state(dec_inputs):
    """State the prefix leaves (oracle, fp64 -> fp32 tensor)."""
    p = dec_inputs["prefix"]
    _, hT = oracle.forward(p["q"], p["k"], p["v"], p["g"], p["eta"], dec_inputs["eps"])
    return torch.from_numpy(hT.astype(np.float32))


class Padded:
    """A contiguous tensor view in the middle of a larger allocation whose
    borders hold a byte pattern (the canaries of an out-of-bounds write):
    ``t`` is the view, ``intact()`` says whether both borders are unchanged.
    The view starts ``pad_bytes`` into the allocation (a multiple of 256, so
    its alignment is that of a fresh allocation)."""

    PATTERN = 0x5B

    def __init__(self, shape, dtype, device, pad_bytes=4096):
        es = torch.empty((), dtype=dtype).element_size()
        n = int(np.prod(shape)) if len(shape) else 1
        assert pad_bytes % 256 == 0 and pad_bytes % es == 0
        self.lo, self.hi = pad_bytes, pad_bytes + n * es
        self.raw = torch.full((self.hi + pad_bytes,), self.PATTERN, dtype=torch.uint8,
                              device=device)
        self.t = self.raw[self.lo:self.hi].view(dtype).view(shape)

    def intact(self):
        b = self.raw.cpu()
        return bool((b[:self.lo] == self.PATTERN).all() and (b[self.hi:] == self.PATTERN).all())
