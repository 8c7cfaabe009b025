"""Shared set-up for the GPU parity tests: seeded inputs -> CUDA path and oracle."""
from __future__ import annotations

import functools

import numpy as np
import torch

import synth
from oracle import graph as ograph

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def rel_err(got, ref):
    """Normwise-infinity relative error max|got - ref| / max|ref|."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max()
    return float(np.abs(got - ref).max() / (den if den > 0 else 1.0))


def check_layer(got, ref, nd, tol, heads=1, bf16_out=None):
    """Layer output parity, as asserted by every layer test.

    got, ref, nd: [atoms, (lmax+1)^2, C] (GPU output, oracle output, layer input n_d).
    Normwise-infinity relative error (max|got - ref| / max|ref|) below ``tol``:
      * on the whole output;
      * on the update out - n_d, after allowing each element the rounding of a bf16
        output (2^-8 |ref|, half an ulp), which is relative to |out|, not to the
        smaller update;
      * on every block of one degree l and one attention head's channels, for the
        output and for the update, so that small blocks (high l, one head) are pinned
        by their own magnitude rather than by the largest block's.
    Returns the largest of these errors."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    nd = np.asarray(nd, dtype=np.float64)
    bf16_out = tol > 1e-3 if bf16_out is None else bf16_out
    diff = np.abs(got - ref)
    allow = (2.0 ** -8) * np.abs(ref) if bf16_out else np.zeros_like(ref)
    upd = ref - nd

    def upd_err(sl):
        den = np.abs(upd[sl]).max()
        num = max(0.0, float((diff[sl] - allow[sl]).max()))
        return num / den if den > 0 else num

    errs = {"out": rel_err(got, ref), "update": upd_err(np.s_[:])}
    L = int(round(np.sqrt(got.shape[1])))
    C = got.shape[2]
    hc = C // heads
    for l in range(L):
        for h in range(heads):
            sl = np.s_[:, l * l:(l + 1) * (l + 1), h * hc:(h + 1) * hc]
            errs[f"out l={l} h={h}"] = rel_err(got[sl], ref[sl])
            errs[f"update l={l} h={h}"] = upd_err(sl)
    worst = max(errs, key=errs.get)
    assert errs[worst] < tol, (worst, errs[worst])
    return errs[worst]


@functools.lru_cache(maxsize=8)
def cell(name: str, seed: int = 0, n_atoms: int | None = None):
    w = synth.WORKLOADS[name]
    return synth.make_cell(w, seed, n_atoms=n_atoms)


@functools.lru_cache(maxsize=4)
def oracle_graph(name: str, seed: int = 0, n_atoms: int | None = None):
    pos, _, box = cell(name, seed, n_atoms)
    w = synth.WORKLOADS[name]
    return ograph.neighbour_list(pos, box, w.rcut)


def gpu_graph(egnn, name, seed=0, n_atoms=None, lmax=None, mmax=None, capacity=None, pos=None, box=None,
              rcut=None):
    w = synth.WORKLOADS[name]
    if pos is None:
        pos, species, box = cell(name, seed, n_atoms)
    else:
        species = np.zeros(len(pos), dtype=np.int32)
    g = egnn.build_graph(torch.from_numpy(pos).cuda(), torch.from_numpy(species).cuda(), box,
                         w.rcut if rcut is None else rcut, w.lmax if lmax is None else lmax,
                         w.mmax if mmax is None else mmax, capacity=capacity)
    torch.cuda.synchronize()
    return g


def to_dev(x: np.ndarray, dtype):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dtype).cuda().contiguous()


def sample_atoms(n: int, k: int, seed: int = 0):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(n, size=min(k, n), replace=False))
