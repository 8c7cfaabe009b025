"""Real Clebsch-Gordan coefficients for the real spherical-harmonic basis (fp64).

Test infrastructure only (see oracle/__init__.py).

MALOQ Section III-B1, Eq. (1): a block H^{ab} of size (2l_a+1) x (2l_b+1) is
the tensor product l_a (x) l_b, and a transformation T made of Clebsch-Gordan
coefficients writes it as the direct sum of |L, M> for L = |l_a-l_b|..l_a+l_b.

Here C^L (for fixed l_a, l_b, L) is the real matrix [(2l_a+1)(2l_b+1), 2L+1],
rows indexed a*(2l_b+1) + b (a, b the positions m+l), with

    (D^{l_a}(R) (x) D^{l_b}(R)) C^L = C^L D^L(R)   for all rotations R,
    C^L^T C^L = I.

For real irreducible representations this intertwiner is unique up to sign
(Schur); the oracle finds it as the null space of the stacked equations over a
few fixed rotations and fixes the sign so that the first non-zero entry of
column M = -L, in row order, is positive (a convention; the pages give none).
"""
from __future__ import annotations

import functools

import numpy as np

from . import sh as _sh


@functools.lru_cache(maxsize=None)
def real_cg(la: int, lb: int, L: int) -> np.ndarray:
    if not (abs(la - lb) <= L <= la + lb):
        raise ValueError("triangle rule violated")
    rng = np.random.Generator(np.random.PCG64(12345))
    na, nb, nl = 2 * la + 1, 2 * lb + 1, 2 * L + 1
    lm = max(la, lb, L)
    rows = []
    for _ in range(3):
        R = _sh.random_rotation(rng)
        D = _sh.wigner_D(lm, R)
        A = np.kron(D[la], D[lb])
        B = D[L]
        # row-major vec: vec(A C) = (A (x) I) vec C ; vec(C B) = (I (x) B^T) vec C
        rows.append(np.kron(A, np.eye(nl)) - np.kron(np.eye(na * nb), B.T))
    M = np.concatenate(rows, axis=0)
    _, s, vt = np.linalg.svd(M)
    if not (s[-1] < 1e-9 and (len(s) == 1 or s[-2] > 1e-6)):
        raise RuntimeError("intertwiner space is not one-dimensional")
    Cm = vt[-1].reshape(na * nb, nl)
    lam = np.trace(Cm.T @ Cm) / nl
    Cm = Cm / np.sqrt(lam)
    col = Cm[:, 0]
    first = np.nonzero(np.abs(col) > 1e-9)[0][0]
    if col[first] < 0:
        Cm = -Cm
    return Cm


def transform_T(la: int, lb: int) -> np.ndarray:
    """T = [C^{|la-lb|} ... C^{la+lb}], square orthogonal (2la+1)(2lb+1) matrix."""
    return np.concatenate([real_cg(la, lb, L) for L in range(abs(la - lb), la + lb + 1)], axis=1)
