"""Identities the per-channel-gate chunk kernels' blocking rests on, in fp64
on the CPU.  Within a chunk, a product decayed channel by channel,
sum_i x_ri y_si e^{G_ri - G_si} over s < r, factors for s before row r's
16-token sub-block through that sub-block's first row (the reference):
e^{G_ri - G_si} = e^{G_ri - G_ref,i} e^{G_ref,i - G_si}, both factors <= 1
since G does not increase along a chunk.  The forward prep kernel forms A
and P that way; the same factorization turns the reverse-mode sums of a
chunkwise per-channel-gate backward into plain products."""
import numpy as np

C, SB = 64, 16


def _setup(seed, dk=8):
    r = np.random.Generator(np.random.PCG64(seed))
    K = r.standard_normal((C, dk))
    Q = r.standard_normal((C, dk))
    G = np.cumsum(-np.log1p(np.exp(r.normal(1.0, 1.5, (C, dk)))), axis=0)
    w = r.standard_normal((C, C))
    low = np.tril(np.ones((C, C), dtype=bool), -1)
    E = np.exp(np.where(low[:, :, None], G[:, None, :] - G[None, :, :], 0.0)) * low[:, :, None]
    return K, Q, G, w * low, E


def _refs(G, R):
    r0 = R * SB
    return r0, np.exp(G[r0:r0 + SB] - G[r0]), np.exp(G[r0] - G[:r0])


def test_forward_products_factor_through_the_subblock_reference():
    K, Q, G, _, E = _setup(71)
    direct = np.einsum("ri,si,rsi->rs", Q, K, E)
    for R in range(1, C // SB):
        r0, a, b = _refs(G, R)
        assert a.max() <= 1.0 and b.max() <= 1.0
        blocked = (Q[r0:r0 + SB] * a) @ (K[:r0] * b).T
        assert np.abs(blocked - direct[r0:r0 + SB, :r0]).max() <= 1e-13 * np.abs(direct).max()


def test_reverse_sums_factor_through_the_subblock_reference():
    K, _, G, w, E = _setup(72)
    rows = np.einsum("rs,si,rsi->ri", w, K, E)
    cols = np.einsum("rs,ri,rsi->si", w, K, E)
    F = np.einsum("rs,ri,si,rsi->rsi", w, K, K, E)
    dG = F.sum(1) - F.sum(0)
    b_rows, b_cols, b_dG = np.zeros_like(K), np.zeros_like(K), np.zeros_like(K)
    for R in range(C // SB):
        r0 = R * SB
        sl = slice(r0, r0 + SB)
        if R:
            _, a, b = _refs(G, R)
            X = w[sl, :r0] @ (K[:r0] * b)
            Y = w[sl, :r0].T @ (K[sl] * a)
            b_rows[sl] += a * X
            b_cols[:r0] += b * Y
            b_dG[sl] += K[sl] * a * X
            b_dG[:r0] -= K[:r0] * b * Y
        Ed, wd = E[sl, sl], w[sl, sl]  # the diagonal sub-block: direct sums
        b_rows[sl] += np.einsum("rs,si,rsi->ri", wd, K[sl], Ed)
        b_cols[sl] += np.einsum("rs,ri,rsi->si", wd, K[sl], Ed)
        Fd = np.einsum("rs,ri,si,rsi->rsi", wd, K[sl], K[sl], Ed)
        b_dG[sl] += Fd.sum(1) - Fd.sum(0)
    for got, ref in ((b_rows, rows), (b_cols, cols), (b_dG, dG)):
        assert np.abs(got - ref).max() <= 1e-13 * np.abs(ref).max()
