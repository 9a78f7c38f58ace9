"""The seeded synthetic inputs follow the stated recipe (CPU only).

Keys: key p = mu_j + 0.3 N(0, I) with j drawn from the drifting active set
{(floor(p M / L) + i) mod M : i < M / 4}.  Queries: a convex mix of three
centres plus 0.3 N(0, I).  Head weights: N(0, 1) * w_scale.  Every stream
is keyed by (seed, tag, 8192-position block), so any slice of positions is
the same whatever the chunking.
"""
import numpy as np

from synth import workloads as S

WL = S.scaled(S.WORKLOADS["tiny_fp32_L4k"], L=20000, T=500)


def test_slices_do_not_depend_on_chunking():
    full = S.keys_f64(WL)
    q_full, w_full = S.queries_f64(WL, 0, WL.L)
    g = np.random.default_rng(3)
    for _ in range(6):
        p0 = int(g.integers(0, WL.L - 1))
        p1 = int(g.integers(p0 + 1, min(WL.L, p0 + 20000) + 1))
        assert np.array_equal(S.keys_f64(WL, p0, p1), full[p0:p1])
        q, w = S.queries_f64(WL, p0, p1)
        assert np.array_equal(q, q_full[p0:p1]) and np.array_equal(w, w_full[p0:p1])
    # a block boundary (8192 positions) inside the slice
    assert np.array_equal(S.keys_f64(WL, 8000, 8400), full[8000:8400])


def test_keys_sit_on_an_active_centre():
    mu = S.centres(WL)
    keys = S.keys_f64(WL)
    # nearest centre of every key (centres are ~sqrt(2d) apart, noise ~0.3 sqrt(d))
    d2 = (keys * keys).sum(1)[:, None] - 2.0 * keys @ mu.T + (mu * mu).sum(1)[None, :]
    j = d2.argmin(1)
    p = np.arange(WL.L)
    base = (p * WL.M) // WL.L
    off = (j - base) % WL.M
    assert np.all(off < WL.M // 4), "a key's component lies outside its active set"
    # the active set drifts: the first eighth of the positions draws from
    # components [0, 3M/8), the middle eighth from [3M/8, 3M/4)
    early = set(j[: WL.L // 8].tolist())
    mid = set(j[3 * WL.L // 8: WL.L // 2].tolist())
    assert early.isdisjoint(mid)
    # noise scale 0.3 per coordinate
    resid = keys - mu[j]
    assert abs(resid.std() - 0.3) < 0.01


def test_queries_and_weights():
    mu = S.centres(WL)
    q, w = S.queries_f64(WL, 0, 4000)
    assert q.shape == (4000, WL.H, WL.d) and w.shape == (4000, WL.H)
    # head weights ~ N(0, 1) * w_scale
    assert abs(w.std() / WL.w_scale - 1.0) < 0.05
    assert abs(w.mean() / WL.w_scale) < 0.05
    # a Dirichlet(1, 1, 1) mix of three centres (unit-variance coordinates)
    # plus 0.3 N(0, 1) noise: per-coordinate variance 3 E[a^2] + 0.09 =
    # 3 * (1/6) + 0.09 = 0.59, mean 0 (weights summing to anything but 1,
    # or another Dirichlet parameter, moves the variance)
    cvar = mu.var()
    assert abs(q.var() - (0.5 * cvar + 0.09)) < 0.03
    assert abs(q.mean()) < 0.05
