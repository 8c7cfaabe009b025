"""GPU neighbour list and Wigner rows against the oracle (bit-exact CSR)."""
import numpy as np
import pytest
import torch

import synth
from gpu_helpers import cell, gpu_graph, oracle_graph, sample_atoms
from oracle import graph as ograph
from oracle import sh as osh

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def egnn():
    from equivariant_gnn_electronic_b200 import egnn
    return egnn


@pytest.mark.parametrize("name", ["tiny", "hfo2_3000", "gst_8064", "mixed_12000"])
def test_csr_bit_exact(egnn, name):
    g = gpu_graph(egnn, name)
    rp, src, sh = oracle_graph(name)
    assert g.read_status() == 0
    assert g.n_edges == rp[-1]
    np.testing.assert_array_equal(g.row_ptr.cpu().numpy(), rp)
    np.testing.assert_array_equal(g.src[:g.n_edges].cpu().numpy(), src)
    np.testing.assert_array_equal(g.shift[:g.n_edges].cpu().numpy(), sh)


def test_csr_stress_sampled(egnn):
    name = "stress_40000"
    w = synth.WORKLOADS[name]
    pos, _, box = cell(name)
    g = gpu_graph(egnn, name)
    assert g.read_status() == 0
    rp = g.row_ptr.cpu().numpy()
    atoms = sample_atoms(len(pos), 60, 1)
    counts, src, sh = ograph.neighbour_list_bruteforce(pos, box, w.rcut, atoms=atoms)
    o = 0
    gsrc = g.src.cpu().numpy()
    gsh = g.shift.cpu().numpy()
    for a, c in zip(atoms, counts):
        assert rp[a + 1] - rp[a] == c
        np.testing.assert_array_equal(gsrc[rp[a]:rp[a + 1]], src[o:o + c])
        np.testing.assert_array_equal(gsh[rp[a]:rp[a + 1]], sh[o:o + c])
        o += c
    assert abs(g.n_edges - 7.2e6) / 7.2e6 < 0.1


def test_capacity_protocol(egnn):
    g = gpu_graph(egnn, "tiny", capacity=10)      # binding grows the arrays on EGNN_ERR_CAPACITY
    rp, _, _ = oracle_graph("tiny")
    assert g.n_edges == rp[-1] and g.capacity >= rp[-1]


def test_bad_position_is_reported(egnn):
    pos, species, box = cell("tiny")
    bad = pos.copy()
    bad[5, 1] = box[1] + 1.0
    with pytest.raises(egnn.EgnnError) as ei:
        egnn.build_graph(torch.from_numpy(bad).cuda(), torch.from_numpy(species).cuda(), box, 6.0, 2, 2)
    assert ei.value.code == egnn.EGNN_ERR_DEVICE_CHECK


def test_isolated_atoms_graph(egnn):
    box = np.array([100.0, 100.0, 100.0])
    pos = np.array([[1.0, 1.0, 1.0], [50.0, 50.0, 50.0], [52.0, 50.0, 50.0]])
    g = gpu_graph(egnn, "tiny", pos=pos, box=box)
    assert g.row_ptr.cpu().numpy().tolist() == [0, 0, 1, 2]


@pytest.mark.parametrize("name", ["gst_8064", "mixed_12000", "tiny"])
def test_wigner_rows_match_oracle(egnn, name):
    w = synth.WORKLOADS[name]
    pos, _, box = cell(name)
    g = gpu_graph(egnn, name)
    rp, src, sh = oracle_graph(name)
    E = g.n_edges
    eidx = np.unique(np.concatenate([np.random.default_rng(2).choice(E, 300, replace=False), [0, E - 1]]))
    dst = np.searchsorted(rp, eidx, side="right") - 1
    r = ograph.edge_vectors(pos, box, dst, src[eidx], sh[eidx])
    dist = np.sqrt((r * r).sum(1))
    D = osh.wigner_D(w.lmax, osh.frame(r / dist[:, None]))
    gw = g.wigner.cpu().numpy()[eidx]
    np.testing.assert_allclose(g.dist.cpu().numpy()[eidx], dist, rtol=1e-6)
    o = 0
    for l in range(w.lmax + 1):
        ml = min(l, w.mmax)
        rows = D[l][:, l - ml:l + ml + 1, :].reshape(len(eidx), -1)
        np.testing.assert_allclose(gw[:, o:o + rows.shape[1]], rows, atol=2e-5)
        o += rows.shape[1]
    assert o == gw.shape[1]
