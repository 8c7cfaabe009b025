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
