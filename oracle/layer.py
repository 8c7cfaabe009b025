"""One eSCN (SO(2)-equivariant) message-passing layer, incoming-edge layout (fp64).

Test infrastructure only (see oracle/__init__.py).

What the pages fix: node embeddings are spherical-harmonic coefficients of
size (L_max+1)^2 x E (MALOQ Section III-C1); messages are built from the
concatenated pair n_i (+) n_j (MALOQ Section III-D, Fig. 4(b)); each edge is
rotated onto a common axis by Wigner-D matrices so that the SO(3) interaction
reduces to SO(2) "constrained linear layers" (MALOQ Sections II-B1 and III,
Fig. 3); messages are aggregated onto their target nodes (MALOQ Section III);
the target node owns its incoming edges so attention and aggregation are local
(review page of arXiv 2507.03840, "What carries the argument").

Readings taken where the pages are silent:
  * edge vector r_e = x_s + shift*box - x_d points from the receiver d to the
    sender s; frame R_e with R_e r_e/|r_e| = z-hat (oracle.sh.frame);
  * concatenation order [n_s || n_d] along channels (2C input channels);
  * radial basis: K Gaussians, mu_k = k rcut/(K-1), sigma = rcut/(K-1), no
    envelope; gate g = W2 SiLU(W1 rho + b1) + b2, g in R^{(lmax+1) x 2C},
    scaling the rotated input x[l, m, c2] by g[l, c2];
  * SO(2) linear: m = 0 mixes all l and channels, y0 = W0 x0; for 0 < m <= mmax
    the (+m, -m) pair mixes as y+ = W_m1 x+ - W_m2 x-, y- = W_m2 x+ + W_m1 x-
    (x+- stacked over l = m..lmax); rows with |m| > mmax are dropped;
  * attention logit a_{e,h} = sum_j A[h, j] SiLU(y0)_j + bA[h]; softmax over the
    incoming edges of each atom and head; head h covers channels
    [h C/H, (h+1) C/H);
  * rotate back with the transpose of the kept rows of D^l(R_e); residual
    out_d = n_d + sum_e alpha_{e, h(c)} msg_e; an atom with no incoming edge
    keeps out_d = n_d.
"""
from __future__ import annotations

import numpy as np

from . import sh as _sh
from .graph import edge_vectors


def silu(x):
    return x / (1.0 + np.exp(-x))


def rbf(dist, rcut, K):
    """Gaussian radial basis rho_k(d) = exp(-(d - mu_k)^2 / (2 sigma^2))."""
    mu = np.arange(K) * (rcut / (K - 1))
    sigma = rcut / (K - 1)
    return np.exp(-((dist[:, None] - mu[None, :]) ** 2) / (2.0 * sigma * sigma))


def edge_geometry(pos, box, d, src, shift, lmax, frame_fn=None):
    """Per-edge distance and Wigner-D list for destination atom d."""
    r = edge_vectors(pos, box, d, src, shift)
    dist = np.sqrt((r * r).sum(-1))
    rhat = r / dist[:, None]
    R = _sh.frame(rhat) if frame_fn is None else frame_fn(rhat)
    return dist, _sh.wigner_D(lmax, R)


def so2_messages(z, dist, D, W, lmax, mmax, rcut, K):
    """Gated SO(2) convolution of the edge inputs, rotated back.

    z[E, (lmax+1)^2, 2C] = [n_s || n_d]; D = list of D^l [E, 2l+1, 2l+1].
    Returns (msg[E, (lmax+1)^2, C], y0[E, (lmax+1) C]).
    """
    E = z.shape[0]
    C2 = z.shape[2]
    C = C2 // 2
    L = lmax + 1
    hid = silu(rbf(dist, rcut, K) @ W["W1"].T + W["b1"])
    g = (hid @ W["W2"].T + W["b2"]).reshape(E, L, C2)
    # rotate into the edge frame, keep |m| <= mmax, gate
    x = {}
    for l in range(L):
        zl = z[:, l * l:(l + 1) * (l + 1), :]
        rot = np.einsum("emn,enc->emc", D[l], zl)
        for m in range(-min(l, mmax), min(l, mmax) + 1):
            x[(l, m)] = rot[:, l + m, :] * g[:, l, :]
    # SO(2) linear
    y = {}
    x0 = np.concatenate([x[(l, 0)] for l in range(L)], axis=1)
    y0 = x0 @ W["W0"].T
    for l in range(L):
        y[(l, 0)] = y0[:, l * C:(l + 1) * C]
    for m in range(1, mmax + 1):
        xp = np.concatenate([x[(l, m)] for l in range(m, L)], axis=1)
        xm = np.concatenate([x[(l, -m)] for l in range(m, L)], axis=1)
        W1, W2 = W[f"W{m}_1"], W[f"W{m}_2"]
        yp = xp @ W1.T - xm @ W2.T
        ym = xp @ W2.T + xm @ W1.T
        for i, l in enumerate(range(m, L)):
            y[(l, m)] = yp[:, i * C:(i + 1) * C]
            y[(l, -m)] = ym[:, i * C:(i + 1) * C]
    # rotate back: msg^l[m'] = sum_{|m| <= mmax} D^l[m, m'] y[l, m]
    msg = np.zeros((E, L * L, C))
    for l in range(L):
        for m in range(-min(l, mmax), min(l, mmax) + 1):
            msg[:, l * l:(l + 1) * (l + 1), :] += D[l][:, l + m, :, None] * y[(l, m)][:, None, :]
    return msg, y0


def layer_forward(pos, box, row_ptr, src, shift, n_in, W, *, lmax, mmax, rcut, n_rbf, heads,
                  atoms=None, frame_fn=None, return_alpha=False):
    """out[d] for each destination atom d (all atoms, or the listed ``atoms``).

    n_in[N, (lmax+1)^2, C]; W as drawn by synth.make_layer_weights.
    With return_alpha, also returns {d: alpha[E_d, H]}.
    """
    n_in = np.asarray(n_in, dtype=np.float64)
    C = n_in.shape[2]
    dests = range(len(n_in)) if atoms is None else atoms
    out = np.zeros((len(dests),) + n_in.shape[1:])
    alphas = {}
    hc = C // heads
    for i, d in enumerate(dests):
        d = int(d)
        e0, e1 = int(row_ptr[d]), int(row_ptr[d + 1])
        out[i] = n_in[d]
        if e1 == e0:
            alphas[d] = np.zeros((0, heads))
            continue
        s = src[e0:e1].astype(np.int64)
        dist, D = edge_geometry(pos, box, d, s, shift[e0:e1], lmax, frame_fn)
        z = np.concatenate([n_in[s], np.broadcast_to(n_in[d], (len(s),) + n_in.shape[1:])], axis=2)
        msg, y0 = so2_messages(z, dist, D, W, lmax, mmax, rcut, n_rbf)
        a = silu(y0) @ W["A"].T + W["bA"]                      # [E, H]
        a = a - a.max(axis=0, keepdims=True)
        p = np.exp(a)
        alpha = p / p.sum(axis=0, keepdims=True)
        alphas[d] = alpha
        wch = np.repeat(alpha, hc, axis=1)                     # [E, C]
        out[i] += (wch[:, None, :] * msg).sum(axis=0)
    return (out, alphas) if return_alpha else out
