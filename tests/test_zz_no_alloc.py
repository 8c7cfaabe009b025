"""egnn_build_graph_noalloc: the graph build for callers that cannot give the library
a device workspace (they may not call cudaMalloc themselves, for instance because
they only receive device pointers from their host application, or because they
forbid allocation after start-up).  Its scratch is a fixed array inside the library.

Checked through the C ABI against egnn_build_graph (which takes a workspace) on two
calls in a row: a large cell first, then a small one, so the second call runs on
scratch that still holds the first call's contents.  This file is collected last."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _inputs(name, seed=0):
    w = synth.WORKLOADS[name]
    pos, spc, box = synth.make_cell(w, seed)
    return w, torch.from_numpy(pos).cuda(), torch.from_numpy(spc).cuda(), box


def test_noalloc_matches_workspace_build_on_two_calls_in_a_row():
    from equivariant_gnn_electronic_b200 import egnn
    for name in ("hfo2_3000", "tiny"):
        w, pos, spc, box = _inputs(name)
        ref = egnn.build_graph(pos, spc, box, w.rcut, w.lmax, w.mmax)
        g = egnn.Graph(pos.shape[0], ref.capacity, w.lmax, w.mmax, pos.device)
        g.wigner.fill_(7.0)
        code = egnn.build_graph_noalloc(pos, spc, box, w.rcut, w.lmax, w.mmax, g)
        torch.cuda.synchronize()
        assert code == egnn.EGNN_OK, egnn.status_string(code)
        assert g.read_status() == 0
        E = ref.n_edges
        assert g.n_edges == E
        assert torch.equal(g.row_ptr, ref.row_ptr)
        assert torch.equal(g.src[:E], ref.src[:E])
        assert torch.equal(g.shift[:E], ref.shift[:E])
        # same kernels on the same inputs: the tolerance of the Wigner tests, met exactly here
        np.testing.assert_allclose(g.dist[:E].cpu().numpy(), ref.dist[:E].cpu().numpy(), rtol=1e-6)
        np.testing.assert_allclose(g.wigner[:E].cpu().numpy(), ref.wigner[:E].cpu().numpy(), atol=2e-5)


def test_noalloc_rejects_cells_above_its_limit():
    from equivariant_gnn_electronic_b200 import egnn
    w, pos, spc, box = _inputs("tiny")
    g = egnn.Graph(pos.shape[0], 16, w.lmax, w.mmax, pos.device)
    import ctypes
    boxarr = (ctypes.c_double * 3)(*[float(b) for b in box])
    code = egnn.lib.egnn_build_graph_noalloc(ctypes.c_void_p(pos.data_ptr()), ctypes.c_void_p(spc.data_ptr()),
                                             131073, boxarr, w.rcut, w.lmax, w.mmax, ctypes.byref(g.s), None)
    assert code == egnn.EGNN_ERR_UNSUPPORTED


def test_noalloc_capacity_protocol_and_retry():
    # arrays too small: EGNN_ERR_CAPACITY with n_edges set, then grow and call again;
    # the retried build matches egnn_build_graph bit for bit
    from equivariant_gnn_electronic_b200 import egnn
    w, pos, spc, box = _inputs("tiny")
    ref = egnn.build_graph(pos, spc, box, w.rcut, w.lmax, w.mmax)
    g = egnn.Graph(pos.shape[0], 8, w.lmax, w.mmax, pos.device)
    code = egnn.build_graph_noalloc(pos, spc, box, w.rcut, w.lmax, w.mmax, g)
    assert code == egnn.EGNN_ERR_CAPACITY
    assert g.n_edges == ref.n_edges
    g._alloc(g.n_edges)
    g._sync_struct()
    code = egnn.build_graph_noalloc(pos, spc, box, w.rcut, w.lmax, w.mmax, g)
    torch.cuda.synchronize()
    assert code == egnn.EGNN_OK and g.read_status() == 0
    E = ref.n_edges
    assert torch.equal(g.row_ptr, ref.row_ptr)
    assert torch.equal(g.src[:E], ref.src[:E])
    assert torch.equal(g.shift[:E], ref.shift[:E])
    assert torch.equal(g.wigner[:E], ref.wigner[:E])


def test_noalloc_cell_without_edges():
    # isolated atoms: E = 0, row_ptr all zero, as egnn_build_graph gives
    from equivariant_gnn_electronic_b200 import egnn
    w = synth.WORKLOADS["tiny"]
    box = np.array([100.0, 100.0, 100.0])
    pos = torch.tensor([[1.0, 1.0, 1.0], [50.0, 50.0, 50.0], [20.0, 80.0, 40.0]], dtype=torch.float64).cuda()
    spc = torch.zeros(3, dtype=torch.int32).cuda()
    ref = egnn.build_graph(pos, spc, box, w.rcut, w.lmax, w.mmax)
    g = egnn.Graph(3, 4, w.lmax, w.mmax, pos.device)
    g.row_ptr.fill_(-1)
    code = egnn.build_graph_noalloc(pos, spc, box, w.rcut, w.lmax, w.mmax, g)
    torch.cuda.synchronize()
    assert code == egnn.EGNN_OK and g.read_status() == 0
    assert ref.n_edges == 0 and g.n_edges == 0
    assert torch.equal(g.row_ptr, ref.row_ptr)
