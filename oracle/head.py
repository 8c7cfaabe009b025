"""Hamiltonian off-diagonal block head (fp64).

Test infrastructure only (see oracle/__init__.py).

MALOQ Section III-B1 and Eq. (1): each orbital block H^{ab}_{ij} of size
(2l_a+1) x (2l_b+1) is the Clebsch-Gordan image of labels |L, M>,
L = |l_a-l_b|..l_a+l_b; the labels of one block are concatenated into h_ij.
MALOQ Section III: edge messages are "used directly to update the embeddings
of edges (in the Edge blocks)", and Label->Matrix turns predicted labels into
H.  Readings (the pages give no formula for the head):
  * per directed edge e = (s -> d) an independent gated SO(2) convolution with
    the head's own weights (oracle.layer.so2_messages, no attention) gives
    t_e[L, M, c];
  * labels h_e[L, M, k] = sum_c U^L[k, c] t_e[L, M, c], one k per shell pair
    (a, b) that contains L, pairs in lexicographic order;
  * block H_e[(a, i), (b, j)] = sum_{L, M} C^L_{(l_a i)(l_b j), M} h_e[L, M, k(a,b,L)]
    with rows the destination atom's orbitals and columns the source atom's,
    every species sharing one orbital template (shell list).
"""
from __future__ import annotations

import numpy as np

from .cg import real_cg
from .layer import edge_geometry, so2_messages


def label_pairs(shells, lmax):
    """For L = 0..lmax the shell pairs (a, b) containing L, lexicographic (a outer)."""
    out = [[] for _ in range(lmax + 1)]
    for a, la in enumerate(shells):
        for b, lb in enumerate(shells):
            for L in range(abs(la - lb), la + lb + 1):
                if L > lmax:
                    raise ValueError("orbital template needs a larger lmax")
                out[L].append((a, b))
    return out


def labels_to_block(h, shells):
    """h: list over L of [E, 2L+1, mult_L] -> blocks [E, n_orb, n_orb]."""
    lmax = len(h) - 1
    pairs = label_pairs(shells, lmax)
    offs = np.concatenate([[0], np.cumsum([2 * l + 1 for l in shells])])
    E = h[0].shape[0] if h[0].size else next(x.shape[0] for x in h if x.size)
    n = int(offs[-1])
    H = np.zeros((E, n, n))
    for L in range(lmax + 1):
        for k, (a, b) in enumerate(pairs[L]):
            la, lb = shells[a], shells[b]
            Cm = real_cg(la, lb, L)                                  # [(2la+1)(2lb+1), 2L+1]
            blk = np.einsum("pm,em->ep", Cm, h[L][:, :, k]).reshape(E, 2 * la + 1, 2 * lb + 1)
            H[:, offs[a]:offs[a + 1], offs[b]:offs[b + 1]] += blk
    return H


def block_to_labels(H, shells, lmax):
    """Inverse of labels_to_block (C^L has orthonormal columns)."""
    pairs = label_pairs(shells, lmax)
    offs = np.concatenate([[0], np.cumsum([2 * l + 1 for l in shells])])
    E = H.shape[0]
    h = []
    for L in range(lmax + 1):
        hL = np.zeros((E, 2 * L + 1, len(pairs[L])))
        for k, (a, b) in enumerate(pairs[L]):
            Cm = real_cg(shells[a], shells[b], L)
            blk = H[:, offs[a]:offs[a + 1], offs[b]:offs[b + 1]].reshape(E, -1)
            hL[:, :, k] = blk @ Cm
        h.append(hL)
    return h


def hamiltonian_blocks(pos, box, row_ptr, src, shift, n_emb, W, shells, *, lmax, mmax, rcut,
                       n_rbf, atoms=None, frame_fn=None):
    """Blocks for every incoming edge of the listed destination atoms (all by default),
    concatenated in CSR order -> [E_sel, n_orb, n_orb]."""
    n_emb = np.asarray(n_emb, dtype=np.float64)
    pairs = label_pairs(shells, lmax)
    dests = range(len(n_emb)) if atoms is None else atoms
    n_orb = sum(2 * l + 1 for l in shells)
    blocks = []
    for d in dests:
        d = int(d)
        e0, e1 = int(row_ptr[d]), int(row_ptr[d + 1])
        if e1 == e0:
            continue
        s = src[e0:e1].astype(np.int64)
        dist, D = edge_geometry(pos, box, d, s, shift[e0:e1], lmax, frame_fn)
        z = np.concatenate([n_emb[s], np.broadcast_to(n_emb[d], (len(s),) + n_emb.shape[1:])],
                           axis=2)
        t, _ = so2_messages(z, dist, D, W, lmax, mmax, rcut, n_rbf)   # [E, L^2, C]
        h = []
        for L in range(lmax + 1):
            tL = t[:, L * L:(L + 1) * (L + 1), :]
            if pairs[L]:
                h.append(np.einsum("kc,emc->emk", W[f"U{L}"], tL))
            else:
                h.append(np.zeros((len(s), 2 * L + 1, 0)))
        blocks.append(labels_to_block(h, shells))
    if not blocks:
        return np.zeros((0, n_orb, n_orb))
    return np.concatenate(blocks, axis=0)


def assemble_hamiltonian(n_atoms, row_ptr, src, onsite, edge_blocks):
    """Gamma-point Hamiltonian of the whole structure as a dense matrix (fp64).

    MALOQ Section III-B (Label->Matrix: the predicted blocks placed at their atom
    pair's rows and columns of H, the orbital template fixing the slices); the
    review page of arXiv 2507.03840 (one matrix of 104,833 orbitals for the
    8,064-atom GeSbTe cell).  Readings (the pages give no formula): every atom d
    owns the rows of its n_orb orbitals; the on-site block of d and the blocks of
    all its incoming edges s -> d (rows d's orbitals, columns s's) are added at
    (d, d) and (d, s); periodic images of the same pair sum into one block (the
    k = 0 matrix).

    onsite[N, n_orb, n_orb]; edge_blocks[E, n_orb, n_orb] in CSR order.
    Returns H[N n_orb, N n_orb].
    """
    onsite = np.asarray(onsite, dtype=np.float64)
    edge_blocks = np.asarray(edge_blocks, dtype=np.float64)
    n_orb = onsite.shape[1]
    H = np.zeros((n_atoms * n_orb, n_atoms * n_orb))
    for d in range(n_atoms):
        r = slice(d * n_orb, (d + 1) * n_orb)
        H[r, r] += onsite[d]
        for e in range(int(row_ptr[d]), int(row_ptr[d + 1])):
            s = int(src[e])
            H[r, s * n_orb:(s + 1) * n_orb] += edge_blocks[e]
    return H
