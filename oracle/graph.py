"""Periodic radius graph in the destination-sorted ("incoming edge") layout (fp64).

Test infrastructure only (see oracle/__init__.py).

Graph (MALOQ Section I and Table II: atoms joined within a cutoff radius,
periodic cells; review page of arXiv 2507.03840, "What carries the argument":
each node owns every edge directed INTO it).  A directed edge e = (s -> d,
shift) exists when

    r_e = (x_s + shift * box) - x_d,   ((r_x*r_x + r_y*r_y) + r_z*r_z) < rcut*rcut

evaluated in fp64 in exactly that order with separately rounded products and
sums, for every periodic image shift in Z^3, excluding (s, shift) = (d, 0).
Edges are grouped by destination d (CSR row_ptr) and, inside a segment,
sorted by (s, shift_x, shift_y, shift_z) ascending.  This tie-break and the
operation order are a reading (the pages fix neither) chosen so that the
CUDA builder can reproduce the list bit for bit.
"""
from __future__ import annotations

import itertools
import math

import numpy as np


def _shift_range(box: np.ndarray, rcut: float):
    S = [int(math.ceil(rcut / b)) for b in box]
    return np.array(list(itertools.product(*[range(-s, s + 1) for s in S])), dtype=np.int64)


def _segment(d: int, pos: np.ndarray, box: np.ndarray, rcut2: float, cand_s: np.ndarray,
             cand_shift: np.ndarray):
    """Exact inclusion test for candidate (s, shift) pairs of destination d; sorted output."""
    img = pos[cand_s] + cand_shift.astype(np.float64) * box[None, :]
    r = img - pos[d][None, :]
    d2 = (r[:, 0] * r[:, 0] + r[:, 1] * r[:, 1]) + r[:, 2] * r[:, 2]
    keep = d2 < rcut2
    keep &= ~((cand_s == d) & np.all(cand_shift == 0, axis=1))
    s = cand_s[keep]
    sh = cand_shift[keep]
    order = np.lexsort((sh[:, 2], sh[:, 1], sh[:, 0], s))
    return s[order], sh[order]


def neighbour_list_bruteforce(pos, box, rcut, atoms=None):
    """O(N^2 * images) list.  Returns (row_ptr[N+1] or counts, src[E], shift[E,3]).

    With ``atoms`` given, only those destination segments are built and
    (counts[len(atoms)], src, shift) is returned, concatenated in that order.
    """
    pos = np.asarray(pos, dtype=np.float64)
    box = np.asarray(box, dtype=np.float64)
    n = len(pos)
    shifts = _shift_range(box, rcut)
    rcut2 = float(rcut) * float(rcut)
    all_s = np.repeat(np.arange(n, dtype=np.int64), len(shifts))
    all_sh = np.tile(shifts, (n, 1))
    dests = range(n) if atoms is None else atoms
    srcs, shs, counts = [], [], []
    for d in dests:
        s, sh = _segment(int(d), pos, box, rcut2, all_s, all_sh)
        srcs.append(s)
        shs.append(sh)
        counts.append(len(s))
    src = np.concatenate(srcs).astype(np.int32) if srcs else np.zeros(0, np.int32)
    shift = (np.concatenate(shs) if shs else np.zeros((0, 3))).astype(np.int8)
    counts = np.array(counts, dtype=np.int64)
    if atoms is not None:
        return counts, src, shift
    row_ptr = np.zeros(n + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    return row_ptr, src, shift


def neighbour_list(pos, box, rcut):
    """Cell-list version of the same list (identical output; faster for large cells).

    Cells of side >= rcut, at least 3 per dimension (else brute force); each
    atom's candidates come from the 27 surrounding cells, each with the one
    periodic shift that places that cell next to the destination cell.
    """
    pos = np.asarray(pos, dtype=np.float64)
    box = np.asarray(box, dtype=np.float64)
    n = len(pos)
    nc = np.array([int(b // (rcut * 1.000001)) for b in box])
    if np.any(nc < 3):
        return neighbour_list_bruteforce(pos, box, rcut)
    cell = np.minimum((pos / (box / nc)).astype(np.int64), nc - 1)
    cell = np.maximum(cell, 0)
    lin = (cell[:, 0] * nc[1] + cell[:, 1]) * nc[2] + cell[:, 2]
    order = np.argsort(lin, kind="stable")
    starts = np.searchsorted(lin[order], np.arange(nc.prod() + 1))
    rcut2 = float(rcut) * float(rcut)
    offs = np.array(list(itertools.product((-1, 0, 1), repeat=3)), dtype=np.int64)
    srcs, shs, counts = [], [], []
    for d in range(n):
        c = cell[d]
        cand_s, cand_sh = [], []
        for o in offs:
            t = c + o
            sh = np.floor_divide(t, nc)
            w = t - sh * nc
            li = (w[0] * nc[1] + w[1]) * nc[2] + w[2]
            members = order[starts[li]:starts[li + 1]]
            cand_s.append(members)
            cand_sh.append(np.tile(sh, (len(members), 1)))
        cs = np.concatenate(cand_s)
        csh = np.concatenate(cand_sh)
        s, sh = _segment(d, pos, box, rcut2, cs, csh)
        srcs.append(s)
        shs.append(sh)
        counts.append(len(s))
    row_ptr = np.zeros(n + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    src = np.concatenate(srcs).astype(np.int32)
    shift = np.concatenate(shs).astype(np.int8)
    return row_ptr, src, shift


def edge_vectors(pos, box, d, src, shift):
    """r_e = (x_s + shift*box) - x_d for the given destination(s) d (scalar or per-edge)."""
    pos = np.asarray(pos, dtype=np.float64)
    box = np.asarray(box, dtype=np.float64)
    return (pos[src] + shift.astype(np.float64) * box[None, :]) - pos[d]
