"""The inequalities the GPU sweep's pruning and FP32 error bound rest on, checked in
FP64 on random and adversarial Hessians (CPU only).

With H_s = (H + H^T) / 2, D = diag(H), C = D^-1/2 H_s D^-1/2, mu <= lambda_min(C),
nu = the largest absolute row sum of C, z_a = sqrt(H_aa) dw_a:
  * E = dw^T H dw >= mu * sum_a H_aa dw_a^2 (the per-candidate lower bound);
  * T = sum_ab |H_s,ab| |dw_a| |dw_b| <= nu * |z|^2 <= (nu / mu) * E (so the FP32 form's
    error, at most 48 u T, is at most rho E with rho = 48 u nu / mu);
  * lambda_max(|C|) <= nu <= 16 and lambda_min(C) >= 2 - nu (Gershgorin).
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
