"""GPU eSCN layer and Hamiltonian head against the oracle.

Small cells are compared element by element over every atom; the full-size
workloads on a seeded sample of destination atoms (the layer is local to each
destination atom, so a sampled atom's output is exact, not statistical).
Tolerances: fp32 1e-4, bf16 storage / fp32 accumulation 2e-2, as max relative
error max|gpu - ref| / max|ref|, applied to the output and to the update
out - n_d, and to each (degree, attention head) block of both (check_layer)."""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from gpu_helpers import TOL, cell, check_layer, gpu_graph, oracle_graph, rel_err, sample_atoms, to_dev
from oracle import head as ohead
from oracle import layer as olayer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def egnn():
    from equivariant_gnn_electronic_b200 import egnn
    return egnn


def _kw(w):
    return dict(lmax=w.lmax, mmax=w.mmax, rcut=w.rcut, n_rbf=w.n_rbf)


def run_layer(egnn, name, w, seed=0, n_atoms=None, atoms=None, bias_std=0.0):
    pos, _, box = cell(name, seed, n_atoms)
    g = gpu_graph(egnn, name, seed, n_atoms, lmax=w.lmax, mmax=w.mmax)
    desc = egnn.desc_for(w)
    dt = egnn.torch_dtype(desc)
    n = synth.make_embeddings(w, len(pos), seed)
    W = synth.make_layer_weights(w, seed, bias_std=bias_std)
    out = egnn.layer_forward(g, desc, egnn.pack_weights(W, desc), to_dev(n, dt))
    torch.cuda.synchronize()
    assert g.read_status() == 0
    got = out.float().cpu().numpy().astype(np.float64)
    rp, src, sh = oracle_graph(name, seed, n_atoms)
    sel = np.arange(len(pos)) if atoms is None else atoms
    ref = olayer.layer_forward(pos, box, rp, src, sh, n, W, **_kw(w), heads=w.heads, atoms=sel)
    return got[sel], ref, n[sel]


def check(got, ref, nd, tol, heads=1):
    check_layer(got, ref, nd, tol, heads=heads)


def test_layer_tiny_fp32_every_atom(egnn):
    w = synth.WORKLOADS["tiny"]
    got, ref, nd = run_layer(egnn, "tiny", w, bias_std=0.2)
    check(got, ref, nd, TOL["fp32"])


@pytest.mark.parametrize("seed", [1, 2])
def test_layer_tiny_more_seeds(egnn, seed):
    w = synth.WORKLOADS["tiny"]
    got, ref, nd = run_layer(egnn, "tiny", w, seed=seed)
    check(got, ref, nd, TOL["fp32"])


def test_layer_small_bf16_every_atom(egnn):
    # 300-atom HfO2-density cell, full C=128, lmax 4: many chunks per atom
    w = synth.WORKLOADS["hfo2_3000"]
    got, ref, nd = run_layer(egnn, "hfo2_3000", w, n_atoms=300, bias_std=0.1)
    check(got, ref, nd, TOL["bf16"], heads=w.heads)


@pytest.mark.parametrize("name", ["hfo2_3000", "gst_8064", "mixed_12000", "stress_40000"])
def test_layer_full_size_sampled(egnn, name):
    w = synth.WORKLOADS[name]
    pos, _, _ = cell(name)
    atoms = np.concatenate([[0, len(pos) - 1], sample_atoms(len(pos), 30, 3)])
    got, ref, nd = run_layer(egnn, name, w, atoms=np.unique(atoms))
    check(got, ref, nd, TOL["bf16"], heads=w.heads)


def test_layer_isolated_atom_keeps_embedding(egnn):
    w = synth.WORKLOADS["tiny"]
    box = np.array([100.0, 100.0, 100.0])
    pos = np.array([[1.0, 1.0, 1.0], [50.0, 50.0, 50.0], [52.0, 50.0, 50.0], [50.0, 53.0, 50.0]])
    g = gpu_graph(egnn, "tiny", pos=pos, box=box)
    desc = egnn.desc_for(w)
    n = np.random.default_rng(0).standard_normal((4, 9, 16))
    W = synth.make_layer_weights(w, 0)
    out = egnn.layer_forward(g, desc, egnn.pack_weights(W, desc), to_dev(n, torch.float32)).cpu().numpy()
    np.testing.assert_array_equal(out[0], n[0].astype(np.float32))
    from oracle import graph as og
    rp, src, sh = og.neighbour_list_bruteforce(pos, box, w.rcut)
    ref = olayer.layer_forward(pos, box, rp, src, sh, n, W, **_kw(w), heads=w.heads)
    assert rel_err(out, ref) < TOL["fp32"]


@pytest.mark.parametrize("lmax,mmax", [(1, 1), (2, 2), (3, 1), (5, 2), (6, 0)])
def test_layer_bf16_degrees(egnn, lmax, mmax):
    # tensor-core layer at the other degree / order limits it accepts, every atom of a
    # 100-atom HfO2-density cell
    w = dataclasses.replace(synth.WORKLOADS["hfo2_3000"], lmax=lmax, mmax=mmax)
    pos, _, box = cell("hfo2_3000", 0, 100)
    g = gpu_graph(egnn, "hfo2_3000", 0, 100, lmax=lmax, mmax=mmax)
    desc = egnn.desc_for(w)
    n = synth.make_embeddings(w, len(pos), 0)
    W = synth.make_layer_weights(w, 0, bias_std=0.1)
    out = egnn.layer_forward(g, desc, egnn.pack_weights(W, desc), to_dev(n, torch.bfloat16))
    torch.cuda.synchronize()
    assert g.read_status() == 0
    rp, src, sh = oracle_graph("hfo2_3000", 0, 100)
    ref = olayer.layer_forward(pos, box, rp, src, sh, n, W, **_kw(w), heads=w.heads)
    check(out.float().cpu().numpy().astype(np.float64), ref, n, TOL["bf16"], heads=w.heads)


@pytest.mark.parametrize("heads", [1, 16])
def test_layer_bf16_head_counts(egnn, heads):
    # tensor-core layer at the fewest and the most attention heads it accepts
    w = dataclasses.replace(synth.WORKLOADS["hfo2_3000"], heads=heads)
    pos, _, box = cell("hfo2_3000", 0, 100)
    g = gpu_graph(egnn, "hfo2_3000", 0, 100)
    desc = egnn.desc_for(w)
    n = synth.make_embeddings(w, len(pos), 0)
    W = synth.make_layer_weights(w, 0, bias_std=0.1)
    out = egnn.layer_forward(g, desc, egnn.pack_weights(W, desc), to_dev(n, torch.bfloat16))
    torch.cuda.synchronize()
    assert g.read_status() == 0
    rp, src, sh = oracle_graph("hfo2_3000", 0, 100)
    ref = olayer.layer_forward(pos, box, rp, src, sh, n, W, **_kw(w), heads=w.heads)
    check(out.float().cpu().numpy().astype(np.float64), ref, n, TOL["bf16"], heads=w.heads)


def test_layer_is_deterministic(egnn):
    w = synth.WORKLOADS["hfo2_3000"]
    pos, species, box = cell("hfo2_3000", 0, 300)
    g = gpu_graph(egnn, "hfo2_3000", 0, 300)
    desc = egnn.desc_for(w)
    n = to_dev(synth.make_embeddings(w, len(pos), 0), torch.bfloat16)
    Wp = egnn.pack_weights(synth.make_layer_weights(w, 0), desc)
    a = egnn.layer_forward(g, desc, Wp, n).clone()
    b = egnn.layer_forward(g, desc, Wp, n)
    assert torch.equal(a, b)


def run_head(egnn, name, w, seed=0, n_atoms=None, atoms=None, bias_std=0.0, shells=None):
    shells = w.shells if shells is None else shells
    pos, _, box = cell(name, seed, n_atoms)
    g = gpu_graph(egnn, name, seed, n_atoms, lmax=w.lmax, mmax=w.mmax)
    desc = egnn.desc_for(w)
    dt = egnn.torch_dtype(desc)
    n = synth.make_embeddings(w, len(pos), seed)
    HW = synth.make_head_weights(w, seed, bias_std=bias_std, shells=shells)
    blocks = egnn.hamiltonian_blocks(g, desc, egnn.pack_weights(HW, desc, attention=False), shells,
                                     to_dev(n, dt))
    torch.cuda.synchronize()
    assert g.read_status() == 0
    got = blocks.cpu().numpy().astype(np.float64)
    rp, src, sh = oracle_graph(name, seed, n_atoms)
    sel = np.arange(len(pos)) if atoms is None else atoms
    ref = ohead.hamiltonian_blocks(pos, box, rp, src, sh, n, HW, shells, **_kw(w), atoms=sel)
    idx = np.concatenate([np.arange(rp[a], rp[a + 1]) for a in sel])
    return got[idx], ref


def test_head_tiny_fp32_every_edge(egnn):
    w = synth.WORKLOADS["tiny"]
    got, ref = run_head(egnn, "tiny", w, bias_std=0.2)
    assert rel_err(got, ref) < TOL["fp32"]


@pytest.mark.parametrize("name", ["gst_8064", "mixed_12000"])
def test_head_full_size_sampled(egnn, name):
    w = synth.WORKLOADS[name]
    pos, _, _ = cell(name)
    got, ref = run_head(egnn, name, w, atoms=sample_atoms(len(pos), 4, 5))
    assert rel_err(got, ref) < TOL["bf16"]


def test_head_bf16_every_edge(egnn):
    # tensor-core head, labels folded into the SO(2) weights, every edge of a 150-atom cell
    w = synth.WORKLOADS["hfo2_3000"]
    got, ref = run_head(egnn, "hfo2_3000", w, n_atoms=150, bias_std=0.1)
    assert rel_err(got, ref) < TOL["bf16"]


def test_head_bf16_wide_template(egnn):
    # 8 s + 8 p shells (32 orbitals): 384 label rows for |m| = 0 and 256 per half for
    # |m| = 1, i.e. a full 512-column accumulator
    w = synth.WORKLOADS["hfo2_3000"]
    shells = (0,) * 8 + (1,) * 8
    got, ref = run_head(egnn, "hfo2_3000", w, n_atoms=120, bias_std=0.1, shells=shells)
    assert rel_err(got, ref) < TOL["bf16"]


def test_head_bf16_channel_space(egnn):
    # lmax 2 with ten p shells: the label record (960 floats) is larger than the
    # channel-space record (768), so the head rotates y back per channel instead
    w = dataclasses.replace(synth.WORKLOADS["hfo2_3000"], lmax=2, shells=(1,) * 10)
    got, ref = run_head(egnn, "hfo2_3000", w, n_atoms=120, bias_std=0.1)
    assert rel_err(got, ref) < TOL["bf16"]


def _cluster_cell(n, box=60.0, seed=0, spread=4.0):
    rng = np.random.default_rng(seed)
    pts = []
    while len(pts) < n:
        p = rng.uniform(-spread, spread, 3)
        if all(np.linalg.norm(p - q) > 1.5 for q in pts):
            pts.append(p)
    return np.array(pts) + box / 2, np.array([box, box, box])


@pytest.mark.parametrize("n_atoms", [3, 9])
def test_layer_bf16_fewer_edges_than_one_tile(egnn, n_atoms):
    # tensor-core path with a single ragged tile (E < 128) and an isolated atom
    w = synth.WORKLOADS["hfo2_3000"]
    pos, box = _cluster_cell(n_atoms)
    pos = np.concatenate([pos, [[2.0, 2.0, 2.0]]])
    g = gpu_graph(egnn, "hfo2_3000", pos=pos, box=box)
    assert 0 < g.n_edges < 128
    desc = egnn.desc_for(w)
    n = synth.round_bf16(np.random.default_rng(n_atoms).standard_normal((len(pos), 25, 128)))
    W = synth.make_layer_weights(w, 1, bias_std=0.1)
    out = egnn.layer_forward(g, desc, egnn.pack_weights(W, desc), to_dev(n, torch.bfloat16))
    torch.cuda.synchronize()
    assert g.read_status() == 0
    from oracle import graph as og
    rp, src, sh = og.neighbour_list_bruteforce(pos, box, w.rcut)
    ref = olayer.layer_forward(pos, box, rp, src, sh, n, W, **_kw(w), heads=w.heads)
    got = out.float().cpu().numpy().astype(np.float64)
    check(got, ref, n, TOL["bf16"], heads=w.heads)
    np.testing.assert_array_equal(got[-1], n[-1])


def test_layer_bf16_no_edges(egnn):
    w = synth.WORKLOADS["hfo2_3000"]
    box = np.array([100.0, 100.0, 100.0])
    pos = np.array([[1.0, 1.0, 1.0], [50.0, 50.0, 50.0]])
    g = gpu_graph(egnn, "hfo2_3000", pos=pos, box=box)
    assert g.n_edges == 0
    desc = egnn.desc_for(w)
    n = synth.round_bf16(np.random.default_rng(0).standard_normal((2, 25, 128)))
    W = synth.make_layer_weights(w, 0)
    out = egnn.layer_forward(g, desc, egnn.pack_weights(W, desc), to_dev(n, torch.bfloat16))
    np.testing.assert_array_equal(out.float().cpu().numpy(), n.astype(np.float32))
