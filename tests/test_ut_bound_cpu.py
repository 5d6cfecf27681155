"""The bound behind the UT kernel's debug check, pinned in fp64 on the CPU.

For one chunk, T = (I + A)^{-1} with A_rs = beta_r (k_r . k_s) e^{G_r - G_s}
(s < r) ("Deep Dive into KDA", section 3, with the step size beta =
eta / (||k||^2 + eps) of the "Kaczmarz Linear Attention" Abstract).  Solving
(I + A) x = b row by row shows that the strictly lower entries are

    T_rs = -beta_r e^{G_r - G_s} k_r^T P_rs k_s,
    P_rs = (I - beta_{r-1} k_{r-1} k_{r-1}^T) ... (I - beta_{s+1} k_{s+1} k_{s+1}^T),

a product of the erase factors of the tokens between s and r.  Each factor
has norm max(1, |1 - eta'_j|) with eta'_j = beta_j ||k_j||^2 <= eta_j, so for
eta in [0, 2], |T_rs| ||k_r|| / ||k_s|| <= eta'_r e^{G_r - G_s}.  These
tests check the closed form entry by entry against a plain inverse, the
bound on chunks drawn like the stress workload, and that it fails outside
its domain (eta = 4 with nearly collinear keys)."""
import numpy as np


def _chunk(seed, C=24, d=8, eta_hi=2.0, collinear=False):
    r = np.random.Generator(np.random.PCG64(seed))
    if collinear:
        k = r.standard_normal(d) + 0.01 * r.standard_normal((C, d))
    else:
        z = r.standard_normal((C, d))
        k = z / np.linalg.norm(z, axis=1, keepdims=True)
    k = k * np.exp(r.uniform(np.log(1e-2), np.log(1e2), (C, 1)))
    eta = np.full(C, eta_hi) if collinear else r.uniform(0.0, eta_hi, C)
    g = np.where(r.random(C) < 0.5, 0.0, -np.log1p(np.exp(r.normal(1.0, 2.0, C))))
    G = np.cumsum(g)
    n2 = (k * k).sum(1)
    beta = eta / (n2 + 1e-6)
    A = np.zeros((C, C))
    for i in range(C):
        for s in range(i):
            A[i, s] = beta[i] * (k[i] @ k[s]) * np.exp(G[i] - G[s])
    return k, beta, G, n2, np.linalg.inv(np.eye(C) + A)


def test_entries_are_products_of_erase_factors():
    for seed in range(5):
        k, beta, G, _, T = _chunk(seed, C=12)
        C, d = k.shape
        for i in range(C):
            for s in range(i):
                P = np.eye(d)
                for j in range(s + 1, i):  # later tokens multiply on the left
                    P = (np.eye(d) - beta[j] * np.outer(k[j], k[j])) @ P
                closed = -beta[i] * np.exp(G[i] - G[s]) * (k[i] @ P @ k[s])
                assert abs(T[i, s] - closed) <= 1e-9 * max(1.0, abs(T[i, s])), (seed, i, s)


def _worst_ratio(k, beta, G, n2, T):
    C = len(G)
    worst = 0.0
    for i in range(C):
        for s in range(i):
            bound = beta[i] * n2[i] * np.exp(G[i] - G[s]) * np.sqrt(n2[s] / n2[i])
            if bound > 0:
                worst = max(worst, abs(T[i, s]) / bound)
    return worst


def test_bound_holds_for_eta_in_zero_two():
    worst = max(_worst_ratio(*_chunk(seed, C=64, d=16)) for seed in range(40))
    assert 0.0 < worst <= 1.0 + 1e-9, worst
    collinear = max(_worst_ratio(*_chunk(seed, C=32, d=16, eta_hi=2.0, collinear=True))
                    for seed in range(10))
    assert collinear <= 1.0 + 1e-9, collinear


def test_bound_fails_beyond_eta_two():
    worst = max(_worst_ratio(*_chunk(seed, C=32, d=16, eta_hi=4.0, collinear=True))
                for seed in range(3))
    assert worst > 10.0, worst
