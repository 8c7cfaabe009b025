"""Failure paths on the GPU, exercised without faulting it.

* A bounded wait that runs out: the pipelined kernels wait on mbarriers with a time
  limit and record EGNN_DEV_WAIT_TIMEOUT instead of hanging.  egnn_check_bounded_wait
  runs that same wait routine on an mbarrier nothing arrives on, with a 1 ms limit;
  the status word must report the timeout and the next layer call must run clean.
* An out-of-range source index, injected on the host into a built graph: the rotate
  kernel of the layer and the Wigner kernel of egnn_edge_geometry must report
  EGNN_DEV_INDEX_RANGE and skip the access (every read stays in bounds).
"""
import numpy as np
import pytest
import torch

import synth
from gpu_helpers import TOL, cell, check_layer, gpu_graph, oracle_graph, to_dev
from oracle import layer as olayer
from oracle import sh as osh
from oracle.graph import edge_vectors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def egnn():
    from equivariant_gnn_electronic_b200 import egnn
    return egnn


def _layer(egnn, g, w, n, W):
    desc = egnn.desc_for(w)
    return egnn.layer_forward(g, desc, egnn.pack_weights(W, desc), to_dev(n, torch.bfloat16))


def test_bounded_wait_runs_out_and_the_next_call_runs_clean(egnn):
    w = synth.WORKLOADS["hfo2_3000"]
    pos, _, box = cell("hfo2_3000", 0, 60)
    g = gpu_graph(egnn, "hfo2_3000", 0, 60)
    egnn.check_bounded_wait(g, 1000)
    code = g.read_status()
    assert code == egnn.EGNN_DEV_WAIT_TIMEOUT
    g.status.zero_()
    n = synth.make_embeddings(w, len(pos), 0)
    W = synth.make_layer_weights(w, 0, bias_std=0.1)
    out = _layer(egnn, g, w, n, W)
    torch.cuda.synchronize()
    assert g.read_status() == 0
    rp, src, sh = oracle_graph("hfo2_3000", 0, 60)
    ref = olayer.layer_forward(pos, box, rp, src, sh, n, W, lmax=w.lmax, mmax=w.mmax, rcut=w.rcut,
                               n_rbf=w.n_rbf, heads=w.heads)
    check_layer(out.float().cpu().numpy().astype(np.float64), ref, n, TOL["bf16"], heads=w.heads)


def test_bounded_wait_rejects_bad_limits(egnn):
    g = gpu_graph(egnn, "hfo2_3000", 0, 60)
    for bad in (0, 2_000_001):
        with pytest.raises(egnn.EgnnError):
            egnn.check_bounded_wait(g, bad)


def test_bad_source_index_is_reported_by_the_rotate_kernel(egnn):
    w = synth.WORKLOADS["hfo2_3000"]
    pos, _, _ = cell("hfo2_3000", 0, 60)
    g = gpu_graph(egnn, "hfo2_3000", 0, 60)
    assert g.read_status() == 0
    g.src[g.n_edges // 2] = len(pos) + 7
    n = synth.make_embeddings(w, len(pos), 0)
    out = _layer(egnn, g, w, n, synth.make_layer_weights(w, 0))
    torch.cuda.synchronize()
    assert g.read_status() == egnn.EGNN_DEV_INDEX_RANGE
    assert torch.isfinite(out.float()).all()


def test_bad_source_index_is_reported_by_the_wigner_kernel(egnn):
    pos, _, box = cell("hfo2_3000", 0, 60)
    g = gpu_graph(egnn, "hfo2_3000", 0, 60)
    g.src[3] = -2
    egnn.edge_geometry(torch.from_numpy(pos).cuda(), box, g)
    assert g.read_status() == egnn.EGNN_DEV_INDEX_RANGE


def test_edge_geometry_follows_moved_atoms(egnn):
    # same neighbour list, atoms displaced by up to 0.05 A: distances and Wigner rows
    # recomputed by egnn_edge_geometry against the oracle's frame of the new positions
    w = synth.WORKLOADS["hfo2_3000"]
    pos, _, box = cell("hfo2_3000", 0, 80)
    g = gpu_graph(egnn, "hfo2_3000", 0, 80)
    ref_w = g.wigner[:g.n_edges].clone()
    egnn.edge_geometry(torch.from_numpy(pos).cuda(), box, g)
    torch.cuda.synchronize()
    assert torch.equal(g.wigner[:g.n_edges], ref_w)      # same positions: same rows
    moved = np.mod(pos + np.random.default_rng(3).uniform(-0.05, 0.05, pos.shape), box)
    egnn.edge_geometry(torch.from_numpy(np.ascontiguousarray(moved)).cuda(), box, g)
    torch.cuda.synchronize()
    assert g.read_status() == 0
    rp, src, sh = oracle_graph("hfo2_3000", 0, 80)
    wig = g.wigner[:g.n_edges].cpu().numpy().astype(np.float64)
    dist = g.dist[:g.n_edges].cpu().numpy().astype(np.float64)
    for d in (0, 17, 79):
        e0, e1 = int(rp[d]), int(rp[d + 1])
        r = edge_vectors(moved, box, d, src[e0:e1].astype(np.int64), sh[e0:e1])
        rr = np.sqrt((r * r).sum(-1))
        np.testing.assert_allclose(dist[e0:e1], rr, rtol=1e-6)
        D = osh.wigner_D(w.lmax, osh.frame(r / rr[:, None]))
        o = 0
        for l in range(w.lmax + 1):
            ml = min(l, w.mmax)
            rows = D[l][:, l - ml:l + ml + 1, :].reshape(e1 - e0, -1)
            np.testing.assert_allclose(wig[e0:e1, o:o + rows.shape[1]], rows, atol=2e-5)
            o += rows.shape[1]
