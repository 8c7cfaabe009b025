"""Real spherical harmonics, edge frames and Wigner-D matrices (fp64).

Test infrastructure only (see oracle/__init__.py).

Basis (a reading: the pages name the spherical-harmonic basis of the node
embeddings -- MALOQ Section III-C1, embeddings of size (L_max+1)^2 x E -- but
not its phase): orthonormal real harmonics ordered m = -l..l, coefficient
index l^2 + l + m,

    Y_{l,0}  = N_l0 P_l(cos t)
    Y_{l,m}  = sqrt(2) N_lm P_l^m(cos t) cos(m p)      m > 0
    Y_{l,-m} = sqrt(2) N_lm P_l^m(cos t) sin(m p)      m > 0

with P_l^m the associated Legendre function WITHOUT the Condon-Shortley
phase and N_lm = sqrt((2l+1)/(4 pi) (l-m)!/(l+m)!).  So Y_1 is proportional
to (y, z, x).

Wigner-D (MALOQ Section III-C1: a rotation R acts on the embeddings as the
direct sum of D^l(R)): the matrix with Y_l(R r) = D^l(R) Y_l(r) for every unit
vector r.  The oracle obtains it from that definition by least squares on a
fixed set of sample directions.

Frame (MALOQ Fig. 3(b,c) rotates each edge onto a common axis; this build
uses +z): R_e = R_y(-beta) R_z(-alpha) with alpha = atan2(y, x),
beta = acos(z), so that R_e r_e = z-hat.  At the poles alpha = 0.
"""
from __future__ import annotations

import math

import numpy as np


def _norm(l: int, m: int) -> float:
    return math.sqrt((2 * l + 1) / (4 * math.pi) * math.factorial(l - m) / math.factorial(l + m))


def assoc_legendre_reduced(lmax: int, z: np.ndarray):
    """Q[l][m] = P_l^m(z) / (1 - z^2)^(m/2) (no Condon-Shortley phase), m <= l <= lmax.

    Textbook recurrences: Q_m^m = (2m-1)!!, Q_{m+1}^m = (2m+1) z Q_m^m,
    (l-m) Q_l^m = (2l-1) z Q_{l-1}^m - (l+m-1) Q_{l-2}^m.
    """
    Q = {}
    for m in range(lmax + 1):
        dfact = 1.0
        for k in range(1, 2 * m, 2):
            dfact *= k
        Q[(m, m)] = np.full_like(z, dfact)
        if m + 1 <= lmax:
            Q[(m + 1, m)] = (2 * m + 1) * z * Q[(m, m)]
        for l in range(m + 2, lmax + 1):
            Q[(l, m)] = ((2 * l - 1) * z * Q[(l - 1, m)] - (l + m - 1) * Q[(l - 2, m)]) / (l - m)
    return Q


def real_sh(lmax: int, v: np.ndarray) -> np.ndarray:
    """Real spherical harmonics of unit vectors v[..., 3] -> [..., (lmax+1)^2]."""
    v = np.asarray(v, dtype=np.float64)
    x, y, z = v[..., 0], v[..., 1], v[..., 2]
    Q = assoc_legendre_reduced(lmax, z)
    out = np.zeros(v.shape[:-1] + ((lmax + 1) ** 2,))
    # (x + i y)^m = sin(t)^m e^{i m p}
    re = np.ones_like(x)
    im = np.zeros_like(x)
    powers = [(re, im)]
    for m in range(1, lmax + 1):
        re, im = re * x - im * y, re * y + im * x
        powers.append((re, im))
    for l in range(lmax + 1):
        out[..., l * l + l] = _norm(l, 0) * Q[(l, 0)]
        for m in range(1, l + 1):
            c = math.sqrt(2.0) * _norm(l, m) * Q[(l, m)]
            out[..., l * l + l + m] = c * powers[m][0]
            out[..., l * l + l - m] = c * powers[m][1]
    return out


def frame(rhat: np.ndarray) -> np.ndarray:
    """Rotation matrices R[..., 3, 3] with R @ rhat = z-hat (R_y(-beta) R_z(-alpha))."""
    rhat = np.asarray(rhat, dtype=np.float64)
    x, y, z = rhat[..., 0], rhat[..., 1], rhat[..., 2]
    rho = np.sqrt(x * x + y * y)
    pole = rho == 0.0
    ca = np.where(pole, 1.0, x / np.where(pole, 1.0, rho))
    sa = np.where(pole, 0.0, y / np.where(pole, 1.0, rho))
    cb, sb = z, rho
    Rz = np.zeros(rhat.shape[:-1] + (3, 3))
    Rz[..., 0, 0] = ca
    Rz[..., 0, 1] = sa
    Rz[..., 1, 0] = -sa
    Rz[..., 1, 1] = ca
    Rz[..., 2, 2] = 1.0
    Ry = np.zeros_like(Rz)
    Ry[..., 0, 0] = cb
    Ry[..., 0, 2] = -sb
    Ry[..., 1, 1] = 1.0
    Ry[..., 2, 0] = sb
    Ry[..., 2, 2] = cb
    return Ry @ Rz


def _sample_dirs(n: int = 64) -> np.ndarray:
    """Fixed, well-spread unit vectors (Fibonacci sphere) for the projection."""
    k = np.arange(n) + 0.5
    z = 1.0 - 2.0 * k / n
    r = np.sqrt(1.0 - z * z)
    p = k * math.pi * (3.0 - math.sqrt(5.0))
    return np.stack([r * np.cos(p), r * np.sin(p), z], axis=-1)


def wigner_D(lmax: int, R: np.ndarray):
    """List over l = 0..lmax of D^l(R)[..., 2l+1, 2l+1] with Y_l(R r) = D^l(R) Y_l(r).

    Solves Y_l(R p_k) = D Y_l(p_k) for D in the least-squares sense over fixed
    sample directions p_k (the system is consistent, so the solution is exact
    up to rounding).
    """
    R = np.asarray(R, dtype=np.float64)
    P = _sample_dirs(max(64, 4 * (2 * lmax + 1)))
    Y = real_sh(lmax, P)                                   # [K, (lmax+1)^2]
    Prot = np.einsum("...ij,kj->...ki", R, P)              # R p_k  -> [..., K, 3]
    Yrot = real_sh(lmax, Prot)                             # [..., K, (lmax+1)^2]
    out = []
    for l in range(lmax + 1):
        sl = slice(l * l, (l + 1) * (l + 1))
        pinv = np.linalg.pinv(Y[:, sl])                    # [(2l+1), K]
        DT = np.einsum("ik,...kj->...ij", pinv, Yrot[..., sl])
        out.append(np.swapaxes(DT, -1, -2))
    return out


def rot_z(g: float) -> np.ndarray:
    c, s = math.cos(g), math.sin(g)
    return np.array([[c, -s, 0.0], [s, c, 0.0], [0.0, 0.0, 1.0]])


def random_rotation(rng: np.random.Generator) -> np.ndarray:
    """Uniform random rotation (QR of a Gaussian matrix, det fixed to +1)."""
    q, r = np.linalg.qr(rng.standard_normal((3, 3)))
    q = q * np.sign(np.diag(r))
    if np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    return q
