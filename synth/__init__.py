"""Seeded synthetic inputs shared by the CUDA path, its tests and the oracle.

This module only draws random numbers and arranges them into arrays of the
documented shapes.  It holds none of the layer's arithmetic: no spherical
harmonics, rotations, neighbour searches, contractions or softmax.  Both the
CUDA path (through ``bench.py`` and the GPU tests) and the oracle consume what
it returns as plain inputs.

Workloads (the pages' datasets -- amorphous HfO2, GeSbTe, OMol molecules --
are not available, so seeded random cells with their density, minimum
distance, species mix and cutoff stand in for them):

* ``tiny``         96 atoms, species 1:2, 0.07 atoms/A^3, d_min 1.8 A, r_cut 6 A,
                   lmax 2, mmax 2, C 16, 1 head, 16 Gaussians, fp32.
* ``hfo2_3000``    3,000 atoms, 1:2, 0.085 atoms/A^3, d_min 1.9, r_cut 8,
                   lmax 4, mmax 2, C 128, 8 heads, 32 Gaussians, 4 layers, bf16.
* ``gst_8064``     8,064 atoms, 2:2:5, 0.033 atoms/A^3, d_min 2.4, r_cut 10,
                   lmax 4, mmax 2, C 128, 8 heads, 32 Gaussians, 4 layers,
                   13-orbital head {s,s,p,p,d}, bf16.
* ``mixed_12000``  12,000 atoms, 5 species 0.3/0.25/0.2/0.15/0.1,
                   0.06 atoms/A^3, d_min 2.0, r_cut 8, lmax 6, mmax 2, C 128,
                   8 heads, 32 Gaussians, 6 layers, 27-orbital head
                   {s,s,s,s,p,p,d,d,f}, bf16.
* ``stress_40000`` 40,000 atoms, 1:2, 0.085 atoms/A^3, d_min 1.9, r_cut 8,
                   lmax 4, mmax 2, C 128, 8 heads, 32 Gaussians, 1 layer, bf16.

Recipe: random sequential addition of uniform points in a periodic cubic box
of side (N/rho)^(1/3), rejecting a candidate closer than d_min (minimum image)
to any accepted point; atoms then sorted by a 4 A cell grid (x-major) so that
neighbouring atoms sit near each other in memory.  Species are exact counts
from the ratios, shuffled.  Node embeddings ~ N(0,1); weights ~ N(0, 1/fan_in),
biases zero unless asked.  bf16 workloads round embeddings and weights to
bf16 here, so every consumer sees the same representable values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Sequence, Tuple

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "make_cell", "make_embeddings", "make_layer_weights",
    "make_head_weights", "round_bf16", "shell_pairs_per_L", "LAYER_WEIGHT_ORDER",
    "HEAD_WEIGHT_ORDER",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n_atoms: int
    species_ratio: Tuple[float, ...]
    density: float          # atoms / A^3
    d_min: float            # A
    rcut: float             # A
    lmax: int
    mmax: int
    channels: int
    heads: int
    n_rbf: int
    n_layers: int
    shells: Tuple[int, ...]  # orbital template (angular momentum of each shell); () = no head
    dtype: str               # "fp32" or "bf16"

    @property
    def box(self) -> float:
        return (self.n_atoms / self.density) ** (1.0 / 3.0)

    @property
    def n_orb(self) -> int:
        return sum(2 * l + 1 for l in self.shells)


WORKLOADS: Dict[str, Workload] = {
    w.name: w for w in [
        Workload("tiny", 96, (1, 2), 0.07, 1.8, 6.0, 2, 2, 16, 1, 16, 1, (0, 1), "fp32"),
        Workload("hfo2_3000", 3000, (1, 2), 0.085, 1.9, 8.0, 4, 2, 128, 8, 32, 4,
                 (0, 0, 1, 1, 2), "bf16"),
        Workload("gst_8064", 8064, (2, 2, 5), 0.033, 2.4, 10.0, 4, 2, 128, 8, 32, 4,
                 (0, 0, 1, 1, 2), "bf16"),
        Workload("mixed_12000", 12000, (0.3, 0.25, 0.2, 0.15, 0.1), 0.06, 2.0, 8.0, 6, 2,
                 128, 8, 32, 6, (0, 0, 0, 0, 1, 1, 2, 2, 3), "bf16"),
        Workload("stress_40000", 40000, (1, 2), 0.085, 1.9, 8.0, 4, 2, 128, 8, 32, 1,
                 (), "bf16"),
    ]
}


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even); returned as float64."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float64).numpy()


def _species_counts(n: int, ratio: Sequence[float]) -> List[int]:
    r = np.asarray(ratio, dtype=np.float64)
    r = r / r.sum()
    counts = [int(math.floor(n * x + 1e-9)) for x in r]
    i = 0
    while sum(counts) < n:       # hand out the remainder in order
        counts[i % len(counts)] += 1
        i += 1
    return counts


def make_cell(w: Workload, seed: int = 0, n_atoms: int | None = None,
              box: float | None = None):
    """Random sequential addition cell.  Returns (pos[N,3] f64, species[N] i32, box[3] f64).

    ``n_atoms``/``box`` override the workload's (for small test cells); the
    density then follows from them.
    """
    n = w.n_atoms if n_atoms is None else n_atoms
    L = w.box if box is None else box
    if n_atoms is not None and box is None:
        L = (n / w.density) ** (1.0 / 3.0)
    rng = np.random.Generator(np.random.PCG64(seed))
    dmin2 = w.d_min * w.d_min
    ng = max(1, int(L // max(w.d_min, 1e-9)))
    cw = L / ng
    grid: Dict[Tuple[int, int, int], List[int]] = {}
    pts = np.zeros((n, 3))
    cnt = 0
    attempts = 0
    while cnt < n:
        cand = rng.random((4096, 3)) * L
        for p in cand:
            attempts += 1
            if attempts > 400 * n + 100000:
                raise RuntimeError("random sequential addition did not converge")
            c = (int(p[0] // cw) % ng, int(p[1] // cw) % ng, int(p[2] // cw) % ng)
            ok = True
            for dx in (-1, 0, 1):
                for dy in (-1, 0, 1):
                    for dz in (-1, 0, 1):
                        lst = grid.get(((c[0] + dx) % ng, (c[1] + dy) % ng, (c[2] + dz) % ng))
                        if not lst:
                            continue
                        q = pts[lst]
                        d = p - q
                        d -= L * np.round(d / L)
                        if np.any((d * d).sum(1) < dmin2):
                            ok = False
                            break
                    if not ok:
                        break
                if not ok:
                    break
            if ok:
                pts[cnt] = p
                grid.setdefault(c, []).append(cnt)
                cnt += 1
                if cnt == n:
                    break
    # spatial order: 4 A cells, x-major
    nc = max(1, int(L // 4.0))
    cidx = np.minimum((pts / (L / nc)).astype(np.int64), nc - 1)
    key = (cidx[:, 0] * nc + cidx[:, 1]) * nc + cidx[:, 2]
    order = np.argsort(key, kind="stable")
    pts = pts[order]
    counts = _species_counts(n, w.species_ratio)
    species = np.concatenate([np.full(c, i, dtype=np.int32) for i, c in enumerate(counts)])
    rng.shuffle(species)
    return np.ascontiguousarray(pts), species.astype(np.int32), np.array([L, L, L], dtype=np.float64)


def make_embeddings(w: Workload, n_atoms: int, seed: int = 0) -> np.ndarray:
    """Node embeddings [N][(lmax+1)^2][C] ~ N(0,1) (bf16-rounded for bf16 workloads)."""
    rng = np.random.Generator(np.random.PCG64(10_000 + seed))
    x = rng.standard_normal((n_atoms, (w.lmax + 1) ** 2, w.channels))
    return round_bf16(x) if w.dtype == "bf16" else x


# Order in which the layer's weights are drawn and packed (row-major [out][in]).
LAYER_WEIGHT_ORDER = ("W1", "b1", "W2", "b2", "W0", "Wm", "A", "bA")
HEAD_WEIGHT_ORDER = ("W1", "b1", "W2", "b2", "W0", "Wm", "U")


def _shapes(w: Workload) -> Dict[str, tuple]:
    L, C, K = w.lmax + 1, w.channels, w.n_rbf
    s = {
        "W1": (C, K), "b1": (C,), "W2": (L * 2 * C, C), "b2": (L * 2 * C,),
        "W0": (L * C, L * 2 * C),
    }
    for m in range(1, w.mmax + 1):
        nm = L - m
        s[f"W{m}_1"] = (nm * C, nm * 2 * C)
        s[f"W{m}_2"] = (nm * C, nm * 2 * C)
    return s


def _fan_in(shape: tuple) -> int:
    return shape[1] if len(shape) == 2 else 1


def _draw(rng, shape, bias_std, is_bias):
    if is_bias:
        return rng.standard_normal(shape) * bias_std if bias_std > 0 else np.zeros(shape)
    return rng.standard_normal(shape) / math.sqrt(_fan_in(shape))


def make_layer_weights(w: Workload, seed: int = 0, layer: int = 0,
                       bias_std: float = 0.0) -> Dict[str, np.ndarray]:
    """One layer's weights, drawn in LAYER_WEIGHT_ORDER from PCG64(seed, layer).

    Keys: W1[C,K] b1[C] W2[L*2C,C] b2[L*2C] W0[L*C,L*2C] W{m}_1, W{m}_2 [n_m*C, n_m*2C]
    (m = 1..mmax, n_m = lmax+1-m) A[H,L*C] bA[H].
    """
    rng = np.random.Generator(np.random.PCG64([seed, 1000 + layer]))
    shapes = _shapes(w)
    shapes["A"] = (w.heads, (w.lmax + 1) * w.channels)
    shapes["bA"] = (w.heads,)
    out = {}
    for k, shp in shapes.items():
        out[k] = _draw(rng, shp, bias_std, k.startswith("b"))
    if w.dtype == "bf16":
        out = {k: round_bf16(v) for k, v in out.items()}
    return out


def shell_pairs_per_L(shells: Sequence[int], lmax: int) -> List[List[Tuple[int, int]]]:
    """For each L = 0..lmax, the (alpha, beta) shell pairs with |l_a - l_b| <= L <= l_a + l_b,
    in lexicographic order (alpha outer).  Its lengths are the label multiplicities mult_L."""
    out: List[List[Tuple[int, int]]] = [[] for _ in range(lmax + 1)]
    for a, la in enumerate(shells):
        for b, lb in enumerate(shells):
            for L in range(abs(la - lb), la + lb + 1):
                if L <= lmax:
                    out[L].append((a, b))
    return out


def make_head_weights(w: Workload, seed: int = 0, bias_std: float = 0.0,
                      shells: Sequence[int] | None = None) -> Dict[str, np.ndarray]:
    """Hamiltonian-head weights: the SO(2) block (same keys/shapes as a layer, no attention)
    plus U{L}[mult_L, C] for L = 0..lmax, drawn from PCG64(seed, 9999)."""
    shells = w.shells if shells is None else tuple(shells)
    rng = np.random.Generator(np.random.PCG64([seed, 9999]))
    shapes = _shapes(w)
    for L, pairs in enumerate(shell_pairs_per_L(shells, w.lmax)):
        if pairs:
            shapes[f"U{L}"] = (len(pairs), w.channels)
    out = {}
    for k, shp in shapes.items():
        out[k] = _draw(rng, shp, bias_std, k.startswith("b"))
    if w.dtype == "bf16":
        out = {k: round_bf16(v) for k, v in out.items()}
    return out
