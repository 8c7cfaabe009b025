"""Label <-> block conversion and Hamiltonian assembly on the GPU, against the oracle.

Matrix -> Label and Label -> Matrix follow the Clebsch-Gordan transform of the
head (oracle.head.block_to_labels / labels_to_block); the assembly follows
oracle.head.assemble_hamiltonian (dense k = 0 matrix).  fp32 on the GPU against
fp64: relative tolerance 1e-5 (sums of at most 49 products, or of a few dozen
blocks per atom pair)."""
import numpy as np
import pytest
import torch

import synth
from gpu_helpers import cell, gpu_graph, oracle_graph, rel_err
from oracle import head as ohead

pytestmark = pytest.mark.gpu
TOL = 1e-5
TEMPLATES = [(0, 1), (0, 0, 1, 1, 2), (0, 0, 0, 0, 1, 1, 2, 2, 3), (0,) * 8 + (1,) * 8]


@pytest.fixture(scope="module")
def egnn():
    from equivariant_gnn_electronic_b200 import egnn
    return egnn


def _flat_labels(h):
    # oracle labels: list over L of [n, 2L+1, mult_L] -> [n, n_lab] in the C ABI order
    return np.concatenate([x.reshape(x.shape[0], -1) for x in h if x.shape[2] > 0], axis=1)


def _unflat(flat, shells):
    lmax = 2 * max(shells)
    pairs = ohead.label_pairs(shells, lmax)
    out, o = [], 0
    for L in range(lmax + 1):
        m = len(pairs[L])
        out.append(flat[:, o:o + (2 * L + 1) * m].reshape(-1, 2 * L + 1, m))
        o += (2 * L + 1) * m
    return out


@pytest.mark.parametrize("shells", TEMPLATES)
def test_blocks_to_labels_matches_oracle(egnn, shells):
    n_orb = sum(2 * l + 1 for l in shells)
    H = np.random.default_rng(len(shells)).standard_normal((300, n_orb, n_orb))
    got = egnn.blocks_to_labels(torch.from_numpy(H.astype(np.float32)).cuda(), shells).cpu().numpy()
    ref = _flat_labels(ohead.block_to_labels(H.astype(np.float32).astype(np.float64), shells, 2 * max(shells)))
    assert got.shape == ref.shape == (300, egnn.label_count(shells))
    assert rel_err(got, ref) < TOL


@pytest.mark.parametrize("shells", TEMPLATES)
def test_labels_to_blocks_matches_oracle_and_round_trips(egnn, shells):
    n_lab = egnn.label_count(shells)
    h = np.random.default_rng(7 + len(shells)).standard_normal((257, n_lab)).astype(np.float32)
    got = egnn.labels_to_blocks(torch.from_numpy(h).cuda(), shells)
    ref = ohead.labels_to_block(_unflat(h.astype(np.float64), shells), shells)
    assert rel_err(got.cpu().numpy(), ref) < TOL
    back = egnn.blocks_to_labels(got, shells).cpu().numpy()
    assert rel_err(back, h) < TOL


def test_conversion_of_no_blocks(egnn):
    shells = (0, 1)
    out = egnn.blocks_to_labels(torch.zeros(0, 4, 4, device="cuda"), shells)
    assert out.shape == (0, egnn.label_count(shells))


@pytest.mark.parametrize("name,n_atoms", [("tiny", None), ("hfo2_3000", 60)])
def test_assembly_matches_dense_oracle(egnn, name, n_atoms):
    # tiny: box 11.1 A < 2 r_cut, so atom pairs appear through several periodic images
    # and atoms see their own images (summed into the on-site block)
    w = synth.WORKLOADS[name]
    pos, _, box = cell(name, 0, n_atoms)
    g = gpu_graph(egnn, name, 0, n_atoms)
    rp, src, sh = oracle_graph(name, 0, n_atoms)
    N, E, n_orb = len(pos), g.n_edges, 5
    rng = np.random.default_rng(11)
    on = rng.standard_normal((N, n_orb, n_orb)).astype(np.float32)
    eb = rng.standard_normal((E, n_orb, n_orb)).astype(np.float32)
    row_ptr, col, val = egnn.assemble_hamiltonian(g, torch.from_numpy(on).cuda(), torch.from_numpy(eb).cuda())
    torch.cuda.synchronize()
    row_ptr = row_ptr.cpu().numpy()
    nnzb = int(row_ptr[-1])
    col, val = col[:nnzb].cpu().numpy(), val[:nnzb].cpu().numpy()
    dense = np.zeros((N * n_orb, N * n_orb))
    for d in range(N):
        cols = col[row_ptr[d]:row_ptr[d + 1]]
        assert np.all(np.diff(cols) > 0) and d in cols          # ascending, on-site present
        for j in range(row_ptr[d], row_ptr[d + 1]):
            dense[d * n_orb:(d + 1) * n_orb, col[j] * n_orb:(col[j] + 1) * n_orb] = val[j]
    ref = ohead.assemble_hamiltonian(N, rp, src, on, eb)
    assert rel_err(dense, ref) < TOL
    # block count: one on-site block per atom plus one per distinct source s != d
    expect = sum(1 + len(set(src[rp[d]:rp[d + 1]]) - {d}) for d in range(N))
    assert nnzb == expect
    if name == "tiny":
        assert nnzb < N + E                                       # images were merged


def test_assembly_of_head_blocks_gst_cell_size(egnn):
    # the 8,064-atom GeSbTe-like cell with its 13-orbital template: H has 104,832 rows
    w = synth.WORKLOADS["gst_8064"]
    pos, _, box = cell("gst_8064")
    g = gpu_graph(egnn, "gst_8064")
    desc = egnn.desc_for(w)
    n = synth.make_embeddings(w, len(pos), 0)
    HW = synth.make_head_weights(w, 0)
    from gpu_helpers import to_dev
    blocks = egnn.hamiltonian_blocks(g, desc, egnn.pack_weights(HW, desc, attention=False), w.shells,
                                     to_dev(n, torch.bfloat16))
    on = torch.zeros(len(pos), w.n_orb, w.n_orb, device="cuda")
    row_ptr, col, val = egnn.assemble_hamiltonian(g, on, blocks)
    torch.cuda.synchronize()
    assert g.read_status() == 0
    assert len(pos) * w.n_orb == 104_832
    nnzb = int(row_ptr[-1])
    rp, src, _ = oracle_graph("gst_8064")
    for d in (0, 4000, len(pos) - 1):
        b, e = int(row_ptr[d]), int(row_ptr[d + 1])
        cols = col[b:e].cpu().numpy()
        ref_cols = sorted(set(src[rp[d]:rp[d + 1]].tolist()) | {d})
        assert cols.tolist() == ref_cols
        # each off-diagonal block is the sum of that source's edge blocks
        for j, s in enumerate(cols):
            if s == d:
                continue
            es = [k for k in range(rp[d], rp[d + 1]) if src[k] == s]
            ref = blocks[es].sum(0)
            assert torch.allclose(val[b + j], ref, rtol=1e-5, atol=1e-6)
    assert nnzb <= len(pos) + g.n_edges
