"""Pins for oracle.layer: exact invariances, equivariances and special cases that a
dropped term, a wrong sign or index, or a transposed operand would break."""
import dataclasses
import math

import numpy as np
import pytest

import synth
from oracle import graph, layer, sh

SMALL = dataclasses.replace(synth.WORKLOADS["tiny"], name="small_l4", lmax=4, mmax=2, channels=8,
                            heads=2, n_rbf=8, rcut=6.0)


def _kw(w):
    return dict(lmax=w.lmax, mmax=w.mmax, rcut=w.rcut, n_rbf=w.n_rbf, heads=w.heads)


def _cluster(n=14, seed=0, box=60.0):
    rng = np.random.default_rng(seed)
    pts = []
    while len(pts) < n:
        p = rng.uniform(-4.5, 4.5, 3)
        if np.linalg.norm(p) < 4.5 and all(np.linalg.norm(p - q) > 1.4 for q in pts):
            pts.append(p)
    c = np.full(3, box / 2)
    return np.array(pts) + c, np.array([box, box, box]), c


def _rotate_embeddings(n, Q, lmax):
    D = sh.wigner_D(lmax, Q)
    out = np.empty_like(n)
    for l in range(lmax + 1):
        sl = slice(l * l, (l + 1) ** 2)
        out[:, sl, :] = np.einsum("mn,anc->amc", D[l], n[:, sl, :])
    return out


def _run(w, pos, box, n, W, **extra):
    rp, src, shf = graph.neighbour_list_bruteforce(pos, box, w.rcut)
    return layer.layer_forward(pos, box, rp, src, shf, n, W, **_kw(w), **extra)


@pytest.mark.parametrize("seed", [0, 1])
def test_global_rotation_equivariance(seed):
    w = SMALL
    pos, box, c = _cluster(seed=seed)
    n = np.random.default_rng(seed).standard_normal((len(pos), (w.lmax + 1) ** 2, w.channels))
    W = synth.make_layer_weights(w, seed, bias_std=0.3)
    out = _run(w, pos, box, n, W)
    Q = sh.random_rotation(np.random.default_rng(100 + seed))
    pos2 = c + (pos - c) @ Q.T
    out2 = _run(w, pos2, box, _rotate_embeddings(n, Q, w.lmax), W)
    np.testing.assert_allclose(out2, _rotate_embeddings(out, Q, w.lmax), atol=1e-10)
    assert np.abs(out - n).max() > 1e-2          # the layer did something


def test_roll_about_edge_axis_is_invisible():
    w = SMALL
    pos, _, box = synth.make_cell(w, 3, n_atoms=40)
    n = np.random.default_rng(3).standard_normal((len(pos), (w.lmax + 1) ** 2, w.channels))
    W = synth.make_layer_weights(w, 3, bias_std=0.3)
    out = _run(w, pos, box, n, W)
    rng = np.random.default_rng(7)

    def rolled(rhat):
        g = rng.uniform(-np.pi, np.pi, len(rhat))
        Rz = np.stack([sh.rot_z(x) for x in g])
        return Rz @ sh.frame(rhat)

    out2 = _run(w, pos, box, n, W, frame_fn=rolled)
    np.testing.assert_allclose(out2, out, atol=1e-12)


def test_atom_permutation_equivariance():
    w = SMALL
    pos, _, box = synth.make_cell(w, 4, n_atoms=40)
    n = np.random.default_rng(4).standard_normal((len(pos), (w.lmax + 1) ** 2, w.channels))
    W = synth.make_layer_weights(w, 4, bias_std=0.3)
    out = _run(w, pos, box, n, W)
    perm = np.random.default_rng(5).permutation(len(pos))
    out2 = _run(w, pos[perm], box, n[perm], W)
    np.testing.assert_allclose(out2, out[perm], atol=1e-12)


def test_softmax_weights_sum_to_one_per_atom_and_head():
    w = dataclasses.replace(SMALL, heads=4)
    pos, _, box = synth.make_cell(w, 5, n_atoms=40)
    n = np.random.default_rng(5).standard_normal((len(pos), (w.lmax + 1) ** 2, w.channels))
    W = synth.make_layer_weights(w, 5, bias_std=0.3)
    _, alphas = _run(w, pos, box, n, W, return_alpha=True)
    for d, a in alphas.items():
        if len(a):
            np.testing.assert_allclose(a.sum(0), np.ones(w.heads), atol=1e-13)
            assert np.all(a > 0)


def test_identity_weights_give_mean_of_sources():
    # lmax = mmax: every row kept, so D^T D = I.  W0, W_m1 copy the source half,
    # W_m2 = 0, gate = 1, logits = 0  =>  out_d = n_d + mean over incoming edges of n_s.
    w = synth.WORKLOADS["tiny"]
    pos, _, box = synth.make_cell(w, 0)
    L, C = w.lmax + 1, w.channels
    n = synth.make_embeddings(w, len(pos), 0)
    W = synth.make_layer_weights(w, 0)
    W["W2"][:] = 0.0
    W["b2"][:] = 1.0
    W["A"][:] = 0.0
    W["bA"][:] = 0.0
    W["W0"][:] = 0.0
    for l in range(L):
        W["W0"][l * C:(l + 1) * C, l * 2 * C:l * 2 * C + C] = np.eye(C)
    for m in range(1, w.mmax + 1):
        W[f"W{m}_1"][:] = 0.0
        W[f"W{m}_2"][:] = 0.0
        for i in range(L - m):
            W[f"W{m}_1"][i * C:(i + 1) * C, i * 2 * C:i * 2 * C + C] = np.eye(C)
    rp, src, shf = graph.neighbour_list_bruteforce(pos, box, w.rcut)
    out = layer.layer_forward(pos, box, rp, src, shf, n, W, **_kw(w))
    for d in range(len(pos)):
        s = src[rp[d]:rp[d + 1]]
        np.testing.assert_allclose(out[d], n[d] + n[s].mean(0), atol=1e-12)


def test_lmax0_is_scalar_graph_attention():
    w = dataclasses.replace(SMALL, lmax=0, mmax=0, heads=2, channels=6)
    pos, _, box = synth.make_cell(w, 6, n_atoms=30)
    n = np.random.default_rng(6).standard_normal((len(pos), 1, w.channels))
    W = synth.make_layer_weights(w, 6, bias_std=0.3)
    rp, src, shf = graph.neighbour_list_bruteforce(pos, box, w.rcut)
    out = layer.layer_forward(pos, box, rp, src, shf, n, W, **_kw(w))
    K, C, H = w.n_rbf, w.channels, w.heads
    for d in range(len(pos)):
        ref = n[d, 0].copy()
        logits, vals = [], []
        for e in range(rp[d], rp[d + 1]):
            s = src[e]
            r = pos[s] + shf[e] * box - pos[d]
            dist = math.sqrt((r * r).sum())
            rho = np.array([math.exp(-(dist - k * w.rcut / (K - 1)) ** 2 /
                                     (2 * (w.rcut / (K - 1)) ** 2)) for k in range(K)])
            h = W["W1"] @ rho + W["b1"]
            h = h / (1 + np.exp(-h))
            g = W["W2"] @ h + W["b2"]
            x = g * np.concatenate([n[s, 0], n[d, 0]])
            y = W["W0"] @ x
            sy = y / (1 + np.exp(-y))
            logits.append(W["A"] @ sy + W["bA"])
            vals.append(y)
        if logits:
            lg = np.array(logits)
            p = np.exp(lg - lg.max(0))
            p /= p.sum(0)
            for e in range(len(vals)):
                ref += np.repeat(p[e], C // H) * vals[e]
        np.testing.assert_allclose(out[d, 0], ref, atol=1e-12)


def test_two_atoms_radial_basis_closed_form():
    # two atoms 3.7 A apart; gate picks Gaussian k through SiLU; output
    # out_0 = n_0 + SiLU(rho_k(d)) * n_1 for the l = 0, channel-0 copy.
    w = dataclasses.replace(SMALL, lmax=0, mmax=0, heads=1, channels=1, n_rbf=7, rcut=6.0)
    box = np.array([40.0, 40.0, 40.0])
    pos = np.array([[10.0, 10.0, 10.0], [10.0 + 3.7, 10.0, 10.0]])
    n = np.array([[[0.4]], [[-1.3]]])
    for k in range(7):
        W = synth.make_layer_weights(w, 0)
        W["W1"][:] = 0.0
        W["W1"][0, k] = 1.0
        W["W2"][:] = np.array([[1.0], [0.0]])
        W["b2"][:] = 0.0
        W["W0"][:] = np.array([[1.0, 0.0]])
        out = _run(w, pos, box, n, W)
        mu, sig = k * 6.0 / 6, 6.0 / 6
        rho = math.exp(-(3.7 - mu) ** 2 / (2 * sig * sig))
        silu = rho / (1 + math.exp(-rho))
        assert abs(out[0, 0, 0] - (0.4 + silu * -1.3)) < 1e-14
        assert abs(out[1, 0, 0] - (-1.3 + silu * 0.4)) < 1e-14


def test_isolated_atom_keeps_its_embedding():
    w = SMALL
    box = np.array([40.0, 40.0, 40.0])
    pos = np.array([[5.0, 5.0, 5.0], [7.0, 5.0, 5.0], [30.0, 30.0, 30.0]])
    n = np.random.default_rng(8).standard_normal((3, (w.lmax + 1) ** 2, w.channels))
    W = synth.make_layer_weights(w, 8, bias_std=0.3)
    out = _run(w, pos, box, n, W)
    np.testing.assert_array_equal(out[2], n[2])
    assert np.abs(out[0] - n[0]).max() > 1e-3
