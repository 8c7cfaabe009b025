"""Pins for oracle.sh: real harmonics, frames and Wigner-D against closed forms,
a library routine and exact group identities."""
import math

import numpy as np
import pytest
from scipy.special import sph_harm_y, roots_legendre

from oracle import sh


def _dirs(n, seed=0):
    v = np.random.default_rng(seed).standard_normal((n, 3))
    return v / np.linalg.norm(v, axis=1, keepdims=True)


def test_real_sh_matches_scipy_complex_harmonics():
    # scipy's Y_l^m carries the Condon-Shortley phase; the real basis without it is
    # sqrt(2) (-1)^m Re/Im Y_l^|m|.
    v = _dirs(200)
    th, ph = np.arccos(v[:, 2]), np.arctan2(v[:, 1], v[:, 0])
    Y = sh.real_sh(8, v)
    for l in range(9):
        for m in range(-l, l + 1):
            c = sph_harm_y(l, abs(m), th, ph)
            if m == 0:
                ref = c.real
            elif m > 0:
                ref = math.sqrt(2) * (-1) ** m * c.real
            else:
                ref = math.sqrt(2) * (-1) ** m * c.imag
            np.testing.assert_allclose(Y[:, l * l + l + m], ref, atol=1e-13)


def test_real_sh_orthonormal_by_exact_quadrature():
    lmax = 6
    xg, wg = roots_legendre(lmax + 2)
    nphi = 2 * lmax + 3
    ph = 2 * np.pi * np.arange(nphi) / nphi
    z = np.repeat(xg, nphi)
    w = np.repeat(wg, nphi) * (2 * np.pi / nphi)
    p = np.tile(ph, len(xg))
    r = np.sqrt(1 - z * z)
    v = np.stack([r * np.cos(p), r * np.sin(p), z], 1)
    Y = sh.real_sh(lmax, v)
    G = (Y * w[:, None]).T @ Y
    np.testing.assert_allclose(G, np.eye(G.shape[0]), atol=1e-12)


def test_l1_is_y_z_x():
    v = _dirs(20)
    Y = sh.real_sh(1, v)
    np.testing.assert_allclose(Y[:, 1:4], math.sqrt(3 / (4 * math.pi)) * v[:, [1, 2, 0]], atol=1e-14)


def test_frame_rotates_edge_onto_z():
    v = np.concatenate([_dirs(100), [[0, 0, 1.0], [0, 0, -1.0], [1.0, 0, 0], [0, -1.0, 0]]])
    R = sh.frame(v)
    np.testing.assert_allclose(np.einsum("eij,ej->ei", R, v), np.tile([0, 0, 1.0], (len(v), 1)),
                               atol=1e-14)
    np.testing.assert_allclose(R @ np.swapaxes(R, 1, 2), np.tile(np.eye(3), (len(v), 1, 1)),
                               atol=1e-14)
    np.testing.assert_allclose(np.linalg.det(R), 1.0, atol=1e-14)


def test_wigner_defining_identity_and_orthogonality():
    rng = np.random.default_rng(1)
    R = np.stack([sh.random_rotation(rng) for _ in range(10)])
    D = sh.wigner_D(6, R)
    v = _dirs(30, 2)
    Y = sh.real_sh(6, v)
    Yr = sh.real_sh(6, np.einsum("rij,kj->rki", R, v))
    for l in range(7):
        sl = slice(l * l, (l + 1) ** 2)
        np.testing.assert_allclose(np.einsum("rmn,kn->rkm", D[l], Y[:, sl]), Yr[:, :, sl], atol=1e-12)
        DtD = np.swapaxes(D[l], 1, 2) @ D[l]
        np.testing.assert_allclose(DtD, np.tile(np.eye(2 * l + 1), (10, 1, 1)), atol=1e-13)


def test_wigner_edge_frame_leaves_only_m0():
    v = np.concatenate([_dirs(50, 3), [[0, 0, 1.0], [0, 0, -1.0]]])
    D = sh.wigner_D(6, sh.frame(v))
    Y = sh.real_sh(6, v)
    Yz = sh.real_sh(6, np.array([0, 0, 1.0]))
    for l in range(7):
        sl = slice(l * l, (l + 1) ** 2)
        got = np.einsum("emn,en->em", D[l], Y[:, sl])
        np.testing.assert_allclose(got, np.tile(Yz[sl], (len(v), 1)), atol=1e-12)
        off = np.delete(got, l, axis=1)
        assert off.size == 0 or np.abs(off).max() < 1e-12


def test_wigner_composition():
    rng = np.random.default_rng(4)
    for _ in range(5):
        R1, R2 = sh.random_rotation(rng), sh.random_rotation(rng)
        D1, D2, D12 = sh.wigner_D(5, R1), sh.wigner_D(5, R2), sh.wigner_D(5, R1 @ R2)
        for l in range(6):
            np.testing.assert_allclose(D12[l], D1[l] @ D2[l], atol=1e-12)


def test_wigner_l1_is_permuted_rotation_matrix():
    rng = np.random.default_rng(5)
    P = np.array([[0, 1.0, 0], [0, 0, 1.0], [1.0, 0, 0]])   # (x,y,z) -> (y,z,x)
    for _ in range(5):
        R = sh.random_rotation(rng)
        np.testing.assert_allclose(sh.wigner_D(1, R)[1], P @ R @ P.T, atol=1e-13)


@pytest.mark.parametrize("g", [0.3, 1.7, -2.5])
def test_wigner_about_z_closed_form(g):
    D = sh.wigner_D(6, sh.rot_z(g))
    for l in range(7):
        ref = np.zeros((2 * l + 1, 2 * l + 1))
        ref[l, l] = 1.0
        for m in range(1, l + 1):
            c, s = math.cos(m * g), math.sin(m * g)
            ref[l + m, l + m] = c
            ref[l + m, l - m] = -s
            ref[l - m, l + m] = s
            ref[l - m, l - m] = c
        np.testing.assert_allclose(D[l], ref, atol=1e-13)
