"""Float64 oracle of the interatomic potential's message-passing step.

Test infrastructure only (see ``oracle/__init__``).

The model (per-edge equivariant SO(2) convolution of a machine-learned
interatomic potential with lmax = 3, as in the DPA4-Neo "first-order SO(2)
input-gradient path" page; the pages give no formulas, so each step is the
plainest reading of the model description of the seeded workloads):

  radial basis   e_n(d) = u(d/rc) sin(n pi d / rc) / d,  n = 1..8
                 u(x) = 1 - 28 x^6 + 48 x^7 - 21 x^8 (x < 1), 0 otherwise
  radial MLP     R = W3 SiLU(W2 SiLU(W1 e))  in R^{4C}, one scale per (l, c);
                 bias-free; one network per layer (per species pair when the
                 model has pair radial networks)
  rotate in      u = D(R_e) x_send  (per degree block), x~ = R (.) u
  SO(2) mixing   m = 0:  y0 = W0 x~0                      (4C x 4C)
                 m > 0:  y+ = Wr x+ - Wi x-,  y- = Wi x+ + Wr x-
                         ((4-m)C x (4-m)C each)
  rotate back    msg = D(R_e)^T y
  aggregate      agg_i = (1/158) sum_{e: recv(e)=i} msg_e
  update         no gate: h = agg;  gated: x <- x + G(agg),
                 G(a)[l=0] = SiLU(a0), G(a)[l>0] = a * SiLU(a0) (per channel)
  readout        e_i = w_o . SiLU(W_ro h_i[l=0]);  E = sum_i e_i
  input          x_0[l=0] = emb[species], higher degrees zero

r_e = x_send + S L - x_recv; R_e is any rotation with R_e r_hat = z (the result
does not depend on the choice).  Forces F = -dE/dx by a hand-written reverse
mode; the edge-direction gradient uses the frame-free identity
a_k = -<g_D, D J_k>, g_r = (dE/dd) r_hat + (a x r)/|r|^2.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

from . import sh

NC = sh.NCOMP


def silu(z):
    return z / (1.0 + np.exp(-z))


def dsilu(z):
    s = 1.0 / (1.0 + np.exp(-z))
    return s * (1.0 + z * (1.0 - s))


# ------------------------------------------------------------------ radial part
def envelope(x, p: int = 6):
    """Polynomial envelope of degree p (p = 6: 1 - 28x^6 + 48x^7 - 21x^8), 0 for x >= 1."""
    a = (p + 1) * (p + 2) / 2.0
    b = p * (p + 2)
    c = p * (p + 1) / 2.0
    u = 1.0 - a * x ** p + b * x ** (p + 1) - c * x ** (p + 2)
    return np.where(x < 1.0, u, 0.0)


def denvelope(x, p: int = 6):
    a = (p + 1) * (p + 2) / 2.0
    b = p * (p + 2)
    c = p * (p + 1) / 2.0
    du = -a * p * x ** (p - 1) + b * (p + 1) * x ** p - c * (p + 2) * x ** (p + 1)
    return np.where(x < 1.0, du, 0.0)


def bessel_basis(d, rc: float, n_basis: int = 8, p: int = 6):
    """[E] -> [E, n_basis]."""
    n = np.arange(1, n_basis + 1)
    x = d / rc
    return envelope(x, p)[:, None] * np.sin(np.pi * n[None, :] * d[:, None] / rc) / d[:, None]


def dbessel_basis(d, rc: float, n_basis: int = 8, p: int = 6):
    n = np.arange(1, n_basis + 1)
    x = d / rc
    arg = np.pi * n[None, :] * d[:, None] / rc
    s, c = np.sin(arg), np.cos(arg)
    u = envelope(x, p)[:, None]
    du = denvelope(x, p)[:, None] / rc
    dd = d[:, None]
    return du * s / dd + u * ((np.pi * n[None, :] / rc) * c / dd - s / (dd * dd))


def radial_forward(e, W1, W2, W3):
    z1 = e @ W1.T
    h1 = silu(z1)
    z2 = h1 @ W2.T
    h2 = silu(z2)
    R = h2 @ W3.T
    return R, (z1, h1, z2, h2)


def radial_backward(gR, cache, W1, W2, W3):
    z1, h1, z2, h2 = cache
    g_h2 = gR @ W3
    g_z2 = g_h2 * dsilu(z2)
    g_h1 = g_z2 @ W2
    g_z1 = g_h1 * dsilu(z1)
    return g_z1 @ W1


# ------------------------------------------------------------------ SO(2) mixing
def m_block_index(m: int) -> List[int]:
    """Component indices (lm) of the +m (or, for m<0, -|m|) entries, l = |m|..3."""
    return [sh.lm_index(l, m) for l in range(abs(m), sh.LMAX + 1)]


def so2_apply(xt: np.ndarray, W: Dict[str, np.ndarray], t: int, transpose: bool = False) -> np.ndarray:
    """x~ [E,16,C] -> y [E,16,C] (or the transpose map for gradients)."""
    E, _, C = xt.shape
    y = np.zeros_like(xt)
    idx0 = m_block_index(0)
    X0 = xt[:, idx0, :].reshape(E, -1)                    # (l, c) order
    W0 = W[f"so2_{t}_W0"].astype(np.float64)
    Y0 = X0 @ (W0 if transpose else W0.T)
    y[:, idx0, :] = Y0.reshape(E, len(idx0), C)
    for m in (1, 2, 3):
        ip, im = m_block_index(m), m_block_index(-m)
        Xp = xt[:, ip, :].reshape(E, -1)
        Xm = xt[:, im, :].reshape(E, -1)
        Wr = W[f"so2_{t}_Wr{m}"].astype(np.float64)
        Wi = W[f"so2_{t}_Wi{m}"].astype(np.float64)
        if not transpose:
            Yp = Xp @ Wr.T - Xm @ Wi.T
            Ym = Xp @ Wi.T + Xm @ Wr.T
        else:
            Yp = Xp @ Wr + Xm @ Wi
            Ym = -Xp @ Wi + Xm @ Wr
        y[:, ip, :] = Yp.reshape(E, len(ip), C)
        y[:, im, :] = Ym.reshape(E, len(im), C)
    return y


def rotate(Dl_list, v: np.ndarray, transpose: bool = False) -> np.ndarray:
    """Apply block-diagonal D (list of [E,2l+1,2l+1]) to v [E,16,C]."""
    out = np.empty_like(v)
    for l, Dl in enumerate(Dl_list):
        b = sh.block(l)
        out[:, b, :] = np.matmul(np.swapaxes(Dl, 1, 2) if transpose else Dl, v[:, b, :])
    return out


# ------------------------------------------------------------------ conv layer
@dataclasses.dataclass
class EdgeGeom:
    r: np.ndarray        # [E,3]
    d: np.ndarray        # [E]
    rhat: np.ndarray     # [E,3]
    Dl: list             # per l: [E,2l+1,2l+1]


def edge_geometry(r: np.ndarray, frame=None) -> EdgeGeom:
    r = np.asarray(r, dtype=np.float64)
    d = np.sqrt(np.einsum("ij,ij->i", r, r))
    rhat = r / d[:, None]
    Re = sh.edge_frame(rhat) if frame is None else frame
    Dl = [sh.wigner_D_l(l, Re) for l in range(sh.LMAX + 1)]
    return EdgeGeom(r=r, d=d, rhat=rhat, Dl=Dl)


def pair_index(a, b, n_species):
    lo, hi = np.minimum(a, b), np.maximum(a, b)
    return lo * n_species - lo * (lo - 1) // 2 + (hi - lo)


def radial_of_edges(spec, W, t, d, pair):
    """R [E,4,C] for layer t, plus what the backward needs."""
    e = bessel_basis(d, spec.cutoff, spec.n_basis, spec.env_p)
    R = np.empty((d.shape[0], 4 * spec.C))
    caches = {}
    for p in np.unique(pair):
        sel = pair == p
        W1 = W[f"rad{t}_{p}_W1"].astype(np.float64)
        W2 = W[f"rad{t}_{p}_W2"].astype(np.float64)
        W3 = W[f"rad{t}_{p}_W3"].astype(np.float64)
        R[sel], caches[p] = radial_forward(e[sel], W1, W2, W3)
    return R.reshape(-1, 4, spec.C), caches


def _expand_R(R):
    """[E,4,C] per-degree scales -> [E,16,C] (repeated over m)."""
    return np.repeat(R, [2 * l + 1 for l in range(4)], axis=1)


def conv_forward(spec, W, t, x, recv, send, geom: EdgeGeom, pair, n_atoms):
    """One interaction layer: returns agg [N,16,C] (already divided by avg_degree)."""
    R, _ = radial_of_edges(spec, W, t, geom.d, pair)
    u = rotate(geom.Dl, x[send])
    xt = _expand_R(R) * u
    y = so2_apply(xt, W, t)
    msg = rotate(geom.Dl, y, transpose=True)
    agg = np.zeros((n_atoms,) + x.shape[1:])
    np.add.at(agg, recv, msg)
    return agg / spec.avg_degree


def conv_backward(spec, W, t, x, g_agg, recv, send, geom: EdgeGeom, pair, n_atoms,
                  need_gx: bool = True):
    """Reverse of :func:`conv_forward` given dE/d(agg).

    Returns (g_x [N,16,C] or None, g_r [E,3])."""
    C = spec.C
    e = bessel_basis(geom.d, spec.cutoff, spec.n_basis, spec.env_p)
    de = dbessel_basis(geom.d, spec.cutoff, spec.n_basis, spec.env_p)
    R, caches = radial_of_edges(spec, W, t, geom.d, pair)
    xs = x[send]
    u = rotate(geom.Dl, xs)
    Rx = _expand_R(R)
    xt = Rx * u
    y = so2_apply(xt, W, t)
    g_m = g_agg[recv] / spec.avg_degree
    g_y = rotate(geom.Dl, g_m)
    g_xt = so2_apply(g_y, W, t, transpose=True)
    # radial scale gradient and the rotated-input gradient
    g_R = np.zeros((xs.shape[0], 4, C))
    for l in range(4):
        b = sh.block(l)
        g_R[:, l, :] = np.sum(g_xt[:, b, :] * u[:, b, :], axis=1)
    g_u = Rx * g_xt
    g_x = None
    if need_gx:
        g_xs = rotate(geom.Dl, g_u, transpose=True)
        g_x = np.zeros((n_atoms,) + x.shape[1:])
        np.add.at(g_x, send, g_xs)
    # gradient with respect to the block-diagonal D, then the frame-free edge torque
    a = np.zeros((xs.shape[0], 3))
    for l in range(1, 4):
        b = sh.block(l)
        gD = np.einsum("eac,ebc->eab", y[:, b, :], g_m[:, b, :]) \
            + np.einsum("eac,ebc->eab", g_u[:, b, :], xs[:, b, :])
        for k in range(3):
            DJ = np.matmul(geom.Dl[l], sh.J_GEN[k][b, b])
            a[:, k] -= np.einsum("eab,eab->e", gD, DJ)
    # radial: dE/dd
    g_e = np.empty((xs.shape[0], spec.n_basis))
    gRf = g_R.reshape(-1, 4 * C)
    for p, cache in caches.items():
        sel = pair == p
        g_e[sel] = radial_backward(gRf[sel], cache, W[f"rad{t}_{p}_W1"].astype(np.float64),
                                   W[f"rad{t}_{p}_W2"].astype(np.float64),
                                   W[f"rad{t}_{p}_W3"].astype(np.float64))
    dEdd = np.sum(g_e * de, axis=1)
    g_r = dEdd[:, None] * geom.rhat + np.cross(a, geom.r) / (geom.d ** 2)[:, None]
    return g_x, g_r


# ------------------------------------------------------------------ full model
def gate(a):
    s = silu(a[:, 0, :])
    out = a * s[:, None, :]
    out[:, 0, :] = s
    return out


def gate_backward(a, g):
    a0 = a[:, 0, :]
    s, ds = silu(a0), dsilu(a0)
    ga = g * s[:, None, :]
    ga[:, 0, :] = g[:, 0, :] * ds + np.sum(g[:, 1:, :] * a[:, 1:, :], axis=1) * ds
    return ga


def readout(W, h):
    z = h[:, 0, :] @ W["ro_W"].astype(np.float64).T
    return silu(z) @ W["ro_w"].astype(np.float64), z


def initial_features(spec, W, species):
    x = np.zeros((species.shape[0], NC, spec.C))
    x[:, 0, :] = W["emb"].astype(np.float64)[species]
    return x


@dataclasses.dataclass
class Result:
    energy: float
    atom_energy: np.ndarray
    forces: np.ndarray
    virial: np.ndarray
    g_r: np.ndarray


def energy_forces(spec, W, species, recv, send, r, n_atoms, chunk: int = 8192,
                  want_forces: bool = True, frame=None) -> Result:
    """Energy, per-atom energies, forces F = -dE/dx and virial W = -sum r (x) g."""
    species = np.asarray(species)
    recv = np.asarray(recv)
    send = np.asarray(send)
    E_n = r.shape[0]
    pair = pair_index(species[recv], species[send], spec.n_species) if spec.pair_radial \
        else np.zeros(E_n, dtype=np.int64)
    chunks = [slice(s, min(s + chunk, E_n)) for s in range(0, E_n, chunk)]
    geoms = [edge_geometry(r[c], None if frame is None else frame[c]) for c in chunks]
    xs = [initial_features(spec, W, species)]
    aggs = []
    for t in range(spec.n_layers):
        agg = np.zeros_like(xs[-1])
        for c, g in zip(chunks, geoms):
            agg += conv_forward(spec, W, t, xs[-1], recv[c], send[c], g, pair[c], n_atoms)
        aggs.append(agg)
        xs.append(xs[-1] + gate(agg) if spec.gated else agg)
    h = xs[-1]
    e_atom, z = readout(W, h)
    energy = float(np.sum(e_atom))
    if not want_forces:
        return Result(energy, e_atom, None, None, None)
    g = np.zeros_like(h)
    g[:, 0, :] = (W["ro_w"].astype(np.float64) * dsilu(z)) @ W["ro_W"].astype(np.float64)
    g_r = np.zeros((E_n, 3))
    for t in reversed(range(spec.n_layers)):
        g_agg = gate_backward(aggs[t], g) if spec.gated else g
        g_next = g.copy() if spec.gated else np.zeros_like(g)
        for c, gm in zip(chunks, geoms):
            gx, gr = conv_backward(spec, W, t, xs[t], g_agg, recv[c], send[c], gm, pair[c],
                                   n_atoms, need_gx=t > 0)
            g_r[c] += gr
            if gx is not None:
                g_next += gx
        g = g_next
    F = np.zeros((n_atoms, 3))
    np.add.at(F, recv, g_r)
    np.subtract.at(F, send, g_r)
    virial = -np.einsum("ea,eb->ab", r, g_r)
    return Result(energy, e_atom, F, virial, g_r)


def energy_only(spec, W, species, recv, send, r, n_atoms, chunk: int = 8192) -> float:
    return energy_forces(spec, W, species, recv, send, r, n_atoms, chunk, want_forces=False).energy


def single_layer(spec, W, t, x, recv, send, r, species, n_atoms, frame=None, chunk: int = 8192):
    """The one-layer convolution (mp_forward): agg [N,16,C] for given features x."""
    species = np.asarray(species)
    E_n = r.shape[0]
    pair = pair_index(species[recv], species[send], spec.n_species) if spec.pair_radial \
        else np.zeros(E_n, dtype=np.int64)
    agg = np.zeros((n_atoms, NC, spec.C))
    for s in range(0, E_n, chunk):
        c = slice(s, min(s + chunk, E_n))
        g = edge_geometry(r[c], None if frame is None else frame[c])
        agg += conv_forward(spec, W, t, np.asarray(x, dtype=np.float64), recv[c], send[c], g,
                            pair[c], n_atoms)
    return agg
