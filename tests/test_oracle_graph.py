"""Pins for oracle.graph: brute force against the cell list, symmetry of the
directed list, and the pages' average degree for amorphous HfO2."""
import json
import os

import numpy as np
import pytest

import synth
from oracle import graph


def _as_set(row_ptr, src, shift):
    out = set()
    for d in range(len(row_ptr) - 1):
        for e in range(row_ptr[d], row_ptr[d + 1]):
            out.add((d, int(src[e]), tuple(int(x) for x in shift[e])))
    return out


def test_tiny_has_multiple_images_and_symmetry():
    w = synth.WORKLOADS["tiny"]
    pos, _, box = synth.make_cell(w, 0)
    assert box[0] < 2 * w.rcut
    rp, src, sh = graph.neighbour_list_bruteforce(pos, box, w.rcut)
    edges = _as_set(rp, src, sh)
    assert len(edges) == rp[-1]
    for (d, s, t) in edges:                     # s->d with shift t  <=>  d->s with -t
        assert (s, d, tuple(-x for x in t)) in edges
    # some source appears twice in one segment (two images inside the cutoff)
    dup = any(len(set(src[rp[d]:rp[d + 1]])) < rp[d + 1] - rp[d] for d in range(len(pos)))
    assert dup
    # segments sorted by (s, shift)
    for d in range(len(pos)):
        keys = [(int(src[e]),) + tuple(int(x) for x in sh[e]) for e in range(rp[d], rp[d + 1])]
        assert keys == sorted(keys)


@pytest.mark.parametrize("seed", [0, 1])
def test_cell_list_equals_brute_force(seed):
    w = synth.WORKLOADS["hfo2_3000"]
    # 700-atom cell at the HfO2 density: box 20.2 A, 2 cells of 8 A is < 3 -> use rcut 6
    pos, _, box = synth.make_cell(w, seed, n_atoms=700)
    rcut = 6.0
    a = graph.neighbour_list_bruteforce(pos, box, rcut)
    b = graph.neighbour_list(pos, box, rcut)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_boundary_tie_is_excluded():
    # an exact-distance pair: |r| = rcut must not be an edge (strict <)
    box = np.array([20.0, 20.0, 20.0])
    pos = np.array([[1.0, 1.0, 1.0], [4.0, 5.0, 1.0], [1.0, 1.0, 5.999]])
    rp, src, sh = graph.neighbour_list_bruteforce(pos, box, 5.0)
    e = _as_set(rp, src, sh)
    assert (0, 1, (0, 0, 0)) not in e       # distance exactly 5
    assert (0, 2, (0, 0, 0)) in e           # 4.999 < 5


def test_empty_graph():
    box = np.array([50.0, 50.0, 50.0])
    pos = np.array([[1.0, 1.0, 1.0], [25.0, 25.0, 25.0]])
    rp, src, sh = graph.neighbour_list_bruteforce(pos, box, 5.0)
    assert rp.tolist() == [0, 0, 0] and len(src) == 0


def test_hfo2_average_degree_matches_pages(root):
    gold = json.load(open(os.path.join(root, "tests/golden/pages_structure.json")))["hfo2_degree"]
    w = synth.WORKLOADS["hfo2_3000"]
    pos, _, box = synth.make_cell(w, 0)
    sample = np.random.default_rng(0).choice(len(pos), 150, replace=False)
    counts, _, _ = graph.neighbour_list_bruteforce(pos, box, gold["rcut_A"], atoms=sample)
    deg = counts.mean()
    assert abs(deg - gold["average_degree"]) / gold["average_degree"] < 0.05, deg
    assert abs(deg * gold["atoms"] - gold["edges_approx"]) / gold["edges_approx"] < 0.05


def test_gst_template_matches_pages_orbital_count(root):
    gold = json.load(open(os.path.join(root, "tests/golden/pages_structure.json")))["gst_orbitals"]
    w = synth.WORKLOADS["gst_8064"]
    assert w.n_orb == 13
    assert abs(w.n_orb * gold["atoms"] - gold["orbitals"]) / gold["orbitals"] < 1e-3
