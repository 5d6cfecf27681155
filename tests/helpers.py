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


# Per-slice bars, looser than the whole-tensor bar (a slice has fewer
# elements to average its rounding over): every (b, h) slice, and every
# 64-token chunk of every (b, h) slice.  One wholly wrong token of a 4096-token
# head moves that head's rel-L2 by ~1/sqrt(64) per chunk, far above both.
HEAD_FACTOR, CHUNK_FACTOR = 2.0, 5.0


def _slice_rel(x, ref, floor):
    den = max(float(np.linalg.norm(ref.ravel())), floor)
    num = float(np.linalg.norm((x - ref).ravel()))
    return num / den if den > 0 else num


def parity_report(x, ref, chunks=True):
    """Whole-tensor rel-L2 of an output [B,T,H,d] against the oracle, the
    worst (b, h) slice and the worst 64-token chunk of any slice.  A chunk's
    denominator is floored at 1e-3 of its slice's RMS chunk norm, so chunks
    whose reference output is (nearly) zero are judged against the slice's
    scale instead of dividing by ~0."""
    x, ref = oracle.f64(x), oracle.f64(ref)
    B, T, H, _ = ref.shape
    worst_h, worst_c = (0.0, None), (0.0, None)
    for b in range(B):
        for h in range(H):
            xs, rs = x[b, :, h], ref[b, :, h]
            e = _slice_rel(xs, rs, 0.0)
            if e > worst_h[0]:
                worst_h = (e, (b, h))
            if not chunks:
                continue
            nck = (T + 63) // 64
            rms = float(np.linalg.norm(rs.ravel())) / np.sqrt(nck)
            for n in range(nck):
                sl = slice(64 * n, min(T, 64 * n + 64))
                e = _slice_rel(xs[sl], rs[sl], 1e-3 * rms)
                if e > worst_c[0]:
                    worst_c = (e, (b, h, n))
    return {"whole": rel(x, ref), "worst_head": worst_h, "worst_chunk": worst_c}


def assert_parity(x, ref, dtype, chunks=True, tol=None):
    """Output [B,T,H,d] against the oracle: rel-L2 <= tol over the whole
    tensor (the stated bar), <= HEAD_FACTOR * tol on every (b, h) slice and
    <= CHUNK_FACTOR * tol on every 64-token chunk of every slice."""
    t = TOL[dtype] if tol is None else tol
    r = parity_report(x, ref, chunks)
    assert r["whole"] <= t, r
    assert r["worst_head"][0] <= HEAD_FACTOR * t, r
    if chunks:
        assert r["worst_chunk"][0] <= CHUNK_FACTOR * t, r
    return r


def assert_state_parity(h, ref, dtype, tol=None):
    """States [B,H,dk,dv] against the oracle: whole tensor and every (b, h)
    state on its own."""
    t = TOL[dtype] if tol is None else tol
    h, ref = oracle.f64(h), oracle.f64(ref)
    whole = rel(h, ref)
    heads = [(_slice_rel(h[b, i], ref[b, i], 0.0), (b, i))
             for b in range(ref.shape[0]) for i in range(ref.shape[1])]
    worst = max(heads) if heads else (0.0, None)
    assert whole <= t and worst[0] <= HEAD_FACTOR * t, (whole, worst)
    return whole, worst


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
