"""The inequalities the GPU sweep's pruning and FP32 error bound rest on, checked in
FP64 on random and adversarial Hessians (CPU only).

With H_s = (H + H^T) / 2, D = diag(H), C = D^-1/2 H_s D^-1/2, mu <= lambda_min(C),
nu = the largest absolute row sum of C, z_a = sqrt(H_aa) dw_a:
  * E = dw^T H dw >= mu * sum_a H_aa dw_a^2 (the per-candidate lower bound);
  * T = sum_ab |H_s,ab| |dw_a| |dw_b| <= nu * |z|^2 <= (nu / mu) * E (so the FP32 form's
    error, at most 48 u T, is at most rho E with rho = 48 u nu / mu);
  * lambda_max(|C|) <= nu <= 16 and lambda_min(C) >= 2 - nu (Gershgorin);
and the class-wide bounds that end the sweep's walk over a mantissa class (below).
"""
import numpy as np
import pytest


def _hessians(rng):
    out = {}
    X = rng.standard_normal((2048, 16)) * rng.lognormal(0.0, 1.0, 16)
    out["independent"] = X.T @ X
    X = rng.standard_normal((4096, 16))
    X[:, 3] *= 5000.0
    out["dominant_channel"] = X.T @ X
    X = 0.3 * rng.standard_normal((1024, 16)) + rng.standard_normal((1024, 1))
    out["common_factor"] = X.T @ X
    X = rng.standard_normal((1024, 16))
    X[:, 1::2] = X[:, 0::2] + 1e-3 * rng.standard_normal((1024, 8))
    out["near_collinear"] = X.T @ X
    X = np.abs(rng.standard_normal((16384, 16))) * (rng.random((16384, 16)) < 0.4)
    out["sparse_nonnegative"] = X.T @ X
    X = rng.standard_normal((85, 16))
    out["few_tokens"] = X.T @ X
    return out


@pytest.mark.parametrize("name", ["independent", "dominant_channel", "common_factor", "near_collinear",
                                  "sparse_nonnegative", "few_tokens"])
def test_bounds_hold(name):
    rng = np.random.default_rng(7)
    H = _hessians(rng)[name]
    Hs = 0.5 * (H + H.T)
    d = np.sqrt(np.diag(H))
    C = Hs / d[:, None] / d[None, :]
    mu = float(np.linalg.eigvalsh(C).min())
    nu = float(np.abs(C).sum(axis=1).max())
    assert mu > 0
    assert float(np.linalg.eigvalsh(np.abs(C)).max()) <= nu * (1 + 1e-12)
    assert nu <= 16 * (1 + 1e-12)
    assert mu >= 2 - nu - 1e-12
    dws = rng.standard_normal((20000, 16)) * rng.lognormal(0.0, 2.0, (20000, 16))
    dws[:5000, rng.integers(0, 16)] = 0.0  # some zero components
    E = np.einsum("na,ab,nb->n", dws, H, dws)
    z2 = np.einsum("na,a->n", dws * dws, np.diag(H))
    T = np.einsum("na,ab,nb->n", np.abs(dws), np.abs(Hs), np.abs(dws))
    assert np.all(E >= mu * z2 * (1 - 1e-9))
    assert np.all(T <= nu * z2 * (1 + 1e-9))
    assert np.all(T <= (nu / mu) * E * (1 + 1e-9))


def test_nu_is_tight_for_weakly_correlated_channels():
    # the reason for nu over the worst case 16: for channels with independent tokens
    # the row sums of |C| stay near 1, so rho shrinks by an order of magnitude
    rng = np.random.default_rng(8)
    X = rng.standard_normal((2048, 16)) * rng.lognormal(0.0, 1.0, 16)
    H = X.T @ X
    d = np.sqrt(np.diag(H))
    nu = float((np.abs(H) / d[:, None] / d[None, :]).sum(axis=1).max())
    assert nu < 1.6


# ------------------------------------------------------------ class-wide walk bounds
# Within a mantissa class the candidate scales are 2^k s0. The upward walk stops on the
# distance of each quotient u = w / s0 to U_k = {0, 2^(k-1)} U {1, 1.5} 2^m (m >= k), which
# holds every larger candidate's grid; the downward walk on max(|w| - 3 2^k1 s0, 0).
def _u_grid(k, top):
    pts = {0.0, 2.0 ** (k - 1)}
    m = k
    while 2.0 ** m <= top:
        pts.add(2.0 ** m)
        pts.add(1.5 * 2.0 ** m)
        m += 1
    return np.array(sorted(pts))


def test_larger_scales_quantise_onto_u():
    # every grid point of a larger candidate (E2M1 values times 2^k', k' > k) lies in U_k
    import oracle
    e2m1 = sorted({abs(oracle.e2m1_rne(x)) for x in np.linspace(0, 7, 141)})
    for k in range(-3, 4):
        U = set(_u_grid(k, 2.0 ** 12).tolist())
        for kk in range(k + 1, k + 8):
            for v in e2m1:
                assert v * 2.0 ** kk in U, (k, kk, v)


def test_upward_distance_is_a_lower_bound_for_every_larger_scale():
    # |u - q_k'(u) 2^k'| >= dist(u, U_k) for all k' > k, and below 6 2^k the candidate's own
    # RNE point is the nearest point of U_k (so its |dw| is that distance)
    import oracle
    rng = np.random.default_rng(9)
    for k in (-2, 0, 3):
        U = _u_grid(k, 2.0 ** (k + 12))
        us = np.concatenate([rng.uniform(0, 64 * 2.0 ** k, 4000), rng.uniform(0, 2.0 ** k, 1000)])
        for u in us:
            d = float(np.min(np.abs(U - u)))
            for kk in range(k + 1, k + 8):
                q = oracle.e2m1_rne(u / 2.0 ** kk) * 2.0 ** kk
                assert abs(u - q) >= d * (1 - 1e-12), (k, kk, u)
            if u < 6 * 2.0 ** k:
                q = oracle.e2m1_rne(u / 2.0 ** k) * 2.0 ** k
                assert abs(abs(u - q) - d) <= 1e-12 * max(1.0, u), (k, u)


def test_downward_bound_for_every_smaller_scale():
    # every scale 2^k' s0 with k' < k1 quantises to at most 6 2^k' <= 3 2^k1 (in units of s0)
    import oracle
    rng = np.random.default_rng(10)
    for k1 in (-1, 2, 5):
        for u in rng.uniform(0, 40 * 2.0 ** k1, 3000):
            bound = max(u - 3 * 2.0 ** k1, 0.0)
            for kk in range(k1 - 6, k1):
                q = oracle.e2m1_rne(u / 2.0 ** kk) * 2.0 ** kk
                assert abs(u - q) >= bound * (1 - 1e-12), (k1, kk, u)
