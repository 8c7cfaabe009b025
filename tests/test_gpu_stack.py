"""Layer stacks and the head as the benchmark runs them, against the oracle.

The benchmark chains a workload's layers through two ping-pong buffers and one
reused workspace, then runs the Hamiltonian head on the last layer's output.
These tests run exactly that chain through the C ABI and compare it with the
oracle run over the same chain.

Small cells: every atom, every layer, checked two ways.  Per layer: the oracle
recomputes layer k from the GPU's stored layer k-1 output, so both sides start
from the same bf16 tensor and the check (check_layer) isolates that layer's
error.  End to end: the oracle runs the whole chain from the initial embeddings,
keeping each layer's output in bf16 (the workloads' storage precision); the GPU's
last output and blocks must be within the tolerance of that chain, normwise, with
the errors of all layers accumulated.

Full-size cells: the chain runs on the GPU; then, for sampled destination atoms,
the oracle recomputes layer k from the GPU's stored layer k-1 output (so both
sides start from the same bf16 tensor) and the head from the GPU's last layer
output.  The layer is local to each destination atom, so a sampled atom's value
is exact, not statistical.

Tolerances as in the single-layer tests (check_layer): bf16 storage with fp32
accumulation 2e-2, on the output, the update and every (degree, head) block."""
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


def gpu_chain(egnn, w, g, n0, seed, bias_std):
    """The benchmark's chain: layer i with its own weights, ping-pong buffers, one
    workspace for every layer; then the head on the last output.  Returns the
    outputs of every layer (host copies) and the blocks."""
    desc = egnn.desc_for(w)
    dt = egnn.torch_dtype(desc)
    x = to_dev(n0, dt)
    bufs = [torch.empty_like(x), torch.empty_like(x)]
    ws = torch.empty(egnn.workspace_bytes(egnn.EGNN_WS_LAYER, desc, g.n_atoms, g.n_edges), dtype=torch.uint8,
                     device=x.device)
    Ws = [synth.make_layer_weights(w, seed, layer=i, bias_std=bias_std) for i in range(w.n_layers)]
    outs = []
    for i in range(w.n_layers):
        y = bufs[i % 2]
        egnn.layer_forward(g, desc, egnn.pack_weights(Ws[i], desc), x, y, workspace=ws)
        outs.append(y.float().cpu().numpy().astype(np.float64))
        x = y
    HW = synth.make_head_weights(w, seed, bias_std=bias_std)
    blocks = egnn.hamiltonian_blocks(g, desc, egnn.pack_weights(HW, desc, attention=False), w.shells, x)
    torch.cuda.synchronize()
    assert g.read_status() == 0
    return outs, Ws, HW, blocks.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("name,n_atoms", [("hfo2_3000", 120), ("gst_8064", 100), ("mixed_12000", 90)])
def test_chain_small_cell_every_atom(egnn, name, n_atoms):
    # hfo2 / gst: 4 layers at lmax 4 + the 13-orbital head; mixed: 6 layers at lmax 6
    # + the 27-orbital head
    w = synth.WORKLOADS[name]
    pos, _, box = cell(name, 0, n_atoms)
    g = gpu_graph(egnn, name, 0, n_atoms)
    n0 = synth.make_embeddings(w, len(pos), 0)
    outs, Ws, HW, blocks = gpu_chain(egnn, w, g, n0, seed=0, bias_std=0.1)
    rp, src, sh = oracle_graph(name, 0, n_atoms)
    x, xo = n0, n0
    for i in range(w.n_layers):
        ref = olayer.layer_forward(pos, box, rp, src, sh, x, Ws[i], **_kw(w), heads=w.heads)
        check_layer(outs[i], ref, x, TOL["bf16"], heads=w.heads)
        x = outs[i]
        xo = synth.round_bf16(olayer.layer_forward(pos, box, rp, src, sh, xo, Ws[i], **_kw(w), heads=w.heads))
    assert rel_err(outs[-1], xo) < TOL["bf16"]
    refb = ohead.hamiltonian_blocks(pos, box, rp, src, sh, x, HW, w.shells, **_kw(w))
    assert rel_err(blocks, refb) < TOL["bf16"]
    refb_chain = ohead.hamiltonian_blocks(pos, box, rp, src, sh, xo, HW, w.shells, **_kw(w))
    assert rel_err(blocks, refb_chain) < TOL["bf16"]


@pytest.mark.parametrize("name", ["gst_8064", "mixed_12000"])
def test_chain_full_size_sampled(egnn, name):
    # every layer k of the benchmarked chain from the GPU's own layer k-1 output, and the
    # head from its last layer, on sampled destination atoms of the full cell
    w = synth.WORKLOADS[name]
    pos, _, box = cell(name)
    g = gpu_graph(egnn, name)
    n0 = synth.make_embeddings(w, len(pos), 0)
    outs, Ws, HW, blocks = gpu_chain(egnn, w, g, n0, seed=0, bias_std=0.0)
    rp, src, sh = oracle_graph(name)
    x = n0
    for i in range(w.n_layers):
        atoms = np.unique(np.concatenate([[0, len(pos) - 1], sample_atoms(len(pos), 10, 100 + i)]))
        ref = olayer.layer_forward(pos, box, rp, src, sh, x, Ws[i], **_kw(w), heads=w.heads, atoms=atoms)
        check_layer(outs[i][atoms], ref, x[atoms], TOL["bf16"], heads=w.heads)
        x = outs[i]
    atoms = sample_atoms(len(pos), 3, 7)
    refb = ohead.hamiltonian_blocks(pos, box, rp, src, sh, x, HW, w.shells, **_kw(w), atoms=atoms)
    idx = np.concatenate([np.arange(rp[a], rp[a + 1]) for a in atoms])
    assert rel_err(blocks[idx], refb) < TOL["bf16"]


@pytest.mark.parametrize("scale,attn", [(1e2, 1e-2), (1e4, 1e-4), (3e5, 1.0 / 3e5), (1e4, 0.0)])
def test_layer_large_magnitude_inputs(egnn, scale, attn):
    # Embeddings far outside N(0, 1), up to values beyond the fp16 range (65,504).
    # The attention matrix is scaled by `attn` so that the logits stay of order one:
    # softmax of logits of order `scale` is ill-conditioned (a relative error e of the
    # logits moves the weights by e * scale), which would test the conditioning of
    # softmax, not the range of the path.  attn = 0 gives uniform weights.
    w = synth.WORKLOADS["hfo2_3000"]
    pos, _, box = cell("hfo2_3000", 0, 100)
    g = gpu_graph(egnn, "hfo2_3000", 0, 100)
    desc = egnn.desc_for(w)
    n = synth.round_bf16(synth.make_embeddings(w, len(pos), 0) * scale)
    W = dict(synth.make_layer_weights(w, 0, bias_std=0.1))
    W["A"] = synth.round_bf16(W["A"] * attn)
    W["bA"] = synth.round_bf16(W["bA"] * attn)
    out = egnn.layer_forward(g, desc, egnn.pack_weights(W, desc), to_dev(n, torch.bfloat16))
    torch.cuda.synchronize()
    assert g.read_status() == 0
    got = out.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    rp, src, sh = oracle_graph("hfo2_3000", 0, 100)
    ref = olayer.layer_forward(pos, box, rp, src, sh, n, W, **_kw(w), heads=w.heads)
    check_layer(got, ref, n, TOL["bf16"], heads=w.heads)


@pytest.mark.parametrize("scale", [1e4, 3e5])
def test_head_large_magnitude_inputs(egnn, scale):
    # the head is linear in the embeddings (no attention): its blocks scale with them
    w = synth.WORKLOADS["hfo2_3000"]
    pos, _, box = cell("hfo2_3000", 0, 100)
    g = gpu_graph(egnn, "hfo2_3000", 0, 100)
    desc = egnn.desc_for(w)
    n = synth.round_bf16(synth.make_embeddings(w, len(pos), 0) * scale)
    HW = synth.make_head_weights(w, 0, bias_std=0.1)
    blocks = egnn.hamiltonian_blocks(g, desc, egnn.pack_weights(HW, desc, attention=False), w.shells,
                                     to_dev(n, torch.bfloat16))
    torch.cuda.synchronize()
    assert g.read_status() == 0
    got = blocks.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    rp, src, sh = oracle_graph("hfo2_3000", 0, 100)
    ref = ohead.hamiltonian_blocks(pos, box, rp, src, sh, n, HW, w.shells, **_kw(w))
    assert rel_err(got, ref) < TOL["bf16"]
