"""Pins for oracle.cg and oracle.head: closed-form couplings, orthogonality,
intertwining with fresh rotations, round trips and block equivariance."""
import dataclasses
import math

import numpy as np
import pytest

import synth
from oracle import cg, graph, head, sh


def test_couplings_with_l0_are_identity():
    for l in range(5):
        np.testing.assert_allclose(cg.real_cg(0, l, l), np.eye(2 * l + 1), atol=1e-12)
        np.testing.assert_allclose(cg.real_cg(l, 0, l), np.eye(2 * l + 1), atol=1e-12)


def test_1x1_to_0_is_dot_product_and_1x1_to_1_is_cross_product():
    np.testing.assert_allclose(cg.real_cg(1, 1, 0)[:, 0], np.eye(3).ravel() / math.sqrt(3), atol=1e-12)
    eps = np.zeros((3, 3, 3))
    for i, j, k in [(0, 1, 2), (1, 2, 0), (2, 0, 1)]:
        eps[i, j, k], eps[i, k, j] = 1.0, -1.0
    # basis (y, z, x) is a cyclic relabelling of (x, y, z): same Levi-Civita symbol
    ref = np.einsum("Mab->abM", eps).reshape(9, 3) / math.sqrt(2)
    np.testing.assert_allclose(cg.real_cg(1, 1, 1), ref, atol=1e-12)


@pytest.mark.parametrize("la,lb", [(1, 1), (2, 2), (3, 3), (1, 2), (2, 3), (0, 3), (3, 1)])
def test_T_orthogonal_and_intertwining(la, lb):
    T = cg.transform_T(la, lb)
    np.testing.assert_allclose(T.T @ T, np.eye(T.shape[0]), atol=1e-12)
    rng = np.random.default_rng(77)
    for _ in range(3):
        Q = sh.random_rotation(rng)
        D = sh.wigner_D(la + lb, Q)
        for L in range(abs(la - lb), la + lb + 1):
            C = cg.real_cg(la, lb, L)
            np.testing.assert_allclose(np.kron(D[la], D[lb]) @ C, C @ D[L], atol=1e-11)


@pytest.mark.parametrize("l", [1, 2, 3])
def test_equal_degree_coupling_symmetry(l):
    # C^L_(a,b) is symmetric in (a, b) for even 2l - L and antisymmetric for odd
    for L in range(0, 2 * l + 1):
        C = cg.real_cg(l, l, L).reshape(2 * l + 1, 2 * l + 1, 2 * L + 1)
        sign = (-1) ** (2 * l - L)
        np.testing.assert_allclose(np.swapaxes(C, 0, 1), sign * C, atol=1e-12)


def test_label_multiplicities():
    p13 = head.label_pairs((0, 0, 1, 1, 2), 4)
    assert [len(x) for x in p13] == [9, 17, 13, 5, 1]
    assert sum(len(x) * (2 * L + 1) for L, x in enumerate(p13)) == 13 * 13
    p27 = head.label_pairs((0, 0, 0, 0, 1, 1, 2, 2, 3), 6)
    assert sum(len(x) * (2 * L + 1) for L, x in enumerate(p27)) == 27 * 27
    assert [len(x) for x in p27] == [len(x) for x in synth.shell_pairs_per_L((0, 0, 0, 0, 1, 1, 2, 2, 3), 6)]


def test_label_block_round_trip():
    shells = (0, 0, 1, 1, 2)
    rng = np.random.default_rng(3)
    H = rng.standard_normal((5, 13, 13))
    h = head.block_to_labels(H, shells, 4)
    np.testing.assert_allclose(head.labels_to_block(h, shells), H, atol=1e-12)


def test_block_equivariance_under_global_rotation():
    w = dataclasses.replace(synth.WORKLOADS["tiny"], lmax=4, mmax=2, channels=8, heads=1, n_rbf=8,
                            shells=(0, 1, 2), dtype="fp32")
    rng = np.random.default_rng(2)
    box = np.array([60.0, 60.0, 60.0])
    c = box / 2
    pos = c + np.array([[0, 0, 0], [1.9, 0.3, -0.4], [-0.7, 2.1, 0.9], [0.4, -1.2, 2.2]])
    n = rng.standard_normal((4, 25, 8))
    W = synth.make_head_weights(w, 1, bias_std=0.2)
    kw = dict(lmax=4, mmax=2, rcut=w.rcut, n_rbf=w.n_rbf)
    rp, src, shf = graph.neighbour_list_bruteforce(pos, box, w.rcut)
    Hb = head.hamiltonian_blocks(pos, box, rp, src, shf, n, W, w.shells, **kw)
    Q = sh.random_rotation(rng)
    D = sh.wigner_D(4, Q)
    n2 = np.empty_like(n)
    for l in range(5):
        n2[:, l * l:(l + 1) ** 2] = np.einsum("mn,anc->amc", D[l], n[:, l * l:(l + 1) ** 2])
    pos2 = c + (pos - c) @ Q.T
    rp2, src2, shf2 = graph.neighbour_list_bruteforce(pos2, box, w.rcut)
    np.testing.assert_array_equal(src2, src)
    Hb2 = head.hamiltonian_blocks(pos2, box, rp2, src2, shf2, n2, W, w.shells, **kw)
    Dorb = np.zeros((9, 9))
    o = 0
    for l in w.shells:
        Dorb[o:o + 2 * l + 1, o:o + 2 * l + 1] = D[l]
        o += 2 * l + 1
    np.testing.assert_allclose(Hb2, Dorb @ Hb @ Dorb.T, atol=1e-10)
    assert np.abs(Hb).max() > 1e-2


def test_assembly_two_atoms_by_hand():
    # two atoms, one s orbital each, edges 1 -> 0 (twice, two images) and 0 -> 1:
    # H = [[on0, e10a + e10b], [e01, on1]]
    from oracle.head import assemble_hamiltonian
    row_ptr = np.array([0, 2, 3])
    src = np.array([1, 1, 0])
    onsite = np.array([[[1.5]], [[-2.0]]])
    edges = np.array([[[0.25]], [[0.5]], [[-0.75]]])
    H = assemble_hamiltonian(2, row_ptr, src, onsite, edges)
    np.testing.assert_array_equal(H, [[1.5, 0.75], [-0.75, -2.0]])


def test_assembly_symmetric_for_transposed_reverse_edges():
    # random graph with every edge's reverse carrying the transposed block: H symmetric;
    # on-site blocks only on the block diagonal; trace from the on-site blocks alone
    from oracle.head import assemble_hamiltonian
    rng = np.random.default_rng(4)
    n, n_orb = 6, 4
    pairs = [(d, s) for d in range(n) for s in range(n) if d != s and rng.random() < 0.5]
    pairs = sorted(set(pairs) | {(s, d) for d, s in pairs})
    blk = {}
    for d, s in pairs:
        if (s, d) in blk:
            blk[(d, s)] = blk[(s, d)].T
        else:
            blk[(d, s)] = rng.standard_normal((n_orb, n_orb))
    row_ptr = np.zeros(n + 1, dtype=np.int64)
    src, edges = [], []
    for d in range(n):
        for dd, s in pairs:
            if dd == d:
                src.append(s)
                edges.append(blk[(d, s)])
        row_ptr[d + 1] = len(src)
    on = rng.standard_normal((n, n_orb, n_orb))
    on = on + on.transpose(0, 2, 1)
    H = assemble_hamiltonian(n, row_ptr, np.array(src), on, np.array(edges))
    np.testing.assert_allclose(H, H.T, atol=0)
    assert np.isclose(np.trace(H), sum(np.trace(o) for o in on))
    Hz = assemble_hamiltonian(n, row_ptr, np.array(src), np.zeros_like(on), np.array(edges))
    for d in range(n):
        assert np.all(Hz[d * n_orb:(d + 1) * n_orb, d * n_orb:(d + 1) * n_orb] == 0)
