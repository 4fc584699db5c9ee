"""Certified radial tables (float64).

Test infrastructure only (see ``oracle/__init__``).

Follows the FastMACE page, "Rewrite screens: adopted and rejected", rows OPT6-T04 and
OPT6-T05 (radial tables): per species pair and interaction, the radial chain from the
edge length up to the output of the hidden layers is replaced by float64-fitted
piecewise Chebyshev tables of degree 10 on dyadic pieces, whose values and
r-derivatives are within 1e-7 of their local scale; the tables are opt-in, float32 on
the device, and are judged by a certificate: the float32 table's error divided by the
float32 network's error, both against the float64 network.

For the model here the tabulated function is h2(d) in R^64, the output of the radial
MLP's hidden layers (basis e_n(d) with the polynomial envelope, W1, SiLU, W2, SiLU);
the head W3 (64 -> 4C) stays a matrix product.  Readings (the page gives the rule, not
its constants):
  * the range is [0, rc]; the pieces are the dyadic intervals [i rc / 2^L, (i+1) rc / 2^L]
    met by bisecting [0, rc] until a piece passes;
  * a piece passes when, at N_CHECK points of it (Chebyshev extrema, the ends included),
    every output's interpolant and
    its d-derivative are within TOL of that output's local scale: the largest magnitude
    the output (or its derivative) reaches on the piece, never taken below FLOOR times
    its largest magnitude on the whole range (so that outputs passing through zero keep
    a finite scale);
  * the interpolant of degree 10 is the one through the 11 Chebyshev points of the first
    kind mapped onto the piece.
"""
from __future__ import annotations

import numpy as np
from scipy import special

from . import model

DEGREE = 10
TOL = 1e-7
FLOOR = 1e-3
N_CHECK = 48
MAX_LEVEL = 14


# ------------------------------------------------------------------ Chebyshev series on [-1, 1]
def cheb_nodes(n: int) -> np.ndarray:
    """The n Chebyshev points of the first kind, cos(pi (2k+1) / (2n)), k = 0..n-1."""
    k = np.arange(n)
    return np.cos(np.pi * (2 * k + 1) / (2 * n))


def cheb_fit(f_nodes: np.ndarray) -> np.ndarray:
    """Coefficients c_0..c_{n-1} of the interpolant sum_k c_k T_k(t) through the values
    f_nodes [n, ...] at cheb_nodes(n) (discrete orthogonality of the cosines)."""
    n = f_nodes.shape[0]
    theta = np.pi * (2 * np.arange(n) + 1) / (2 * n)
    Tm = np.cos(np.outer(np.arange(n), theta))                # [k, j] = T_k(t_j)
    c = (2.0 / n) * np.tensordot(Tm, f_nodes, axes=(1, 0))
    c[0] *= 0.5
    return c


def cheb_eval(c: np.ndarray, t: np.ndarray) -> np.ndarray:
    """sum_k c_k T_k(t) by Clenshaw's recurrence; c [n, m], t [p] -> [p, m]."""
    b1 = np.zeros((t.shape[0], c.shape[1]))
    b2 = np.zeros_like(b1)
    for k in range(c.shape[0] - 1, 0, -1):
        b1, b2 = 2.0 * t[:, None] * b1 - b2 + c[k][None, :], b1
    return t[:, None] * b1 - b2 + c[0][None, :]


def cheb_deriv(c: np.ndarray) -> np.ndarray:
    """Coefficients of d/dt of sum_k c_k T_k(t) (one degree lower):
    d_{k-1} = d_{k+1} + 2 k c_k from the top, then d_0 halved."""
    n = c.shape[0]
    d = np.zeros((n + 1,) + c.shape[1:])
    for k in range(n - 1, 0, -1):
        d[k - 1] = d[k + 1] + 2.0 * k * c[k]
    d[0] *= 0.5
    return d[: n - 1]


# ------------------------------------------------------------------ the tabulated function
def basis(spec, d: np.ndarray):
    """The radial basis e_n(d) = u(d/rc) sin(k_n d) / d (k_n = n pi / rc) and its d-derivative,
    written with spherical Bessel functions so that both stay accurate as d -> 0:
    sin(k d) / d = k j0(k d) and d/dd [sin(k d) / d] = -k^2 j1(k d)."""
    rc = float(spec.cutoff)
    k = np.pi * np.arange(1, spec.n_basis + 1) / rc
    x = (k[None, :] * d[:, None])
    u = model.envelope(d / rc, spec.env_p)[:, None]
    du = model.denvelope(d / rc, spec.env_p)[:, None] / rc
    j0 = special.spherical_jn(0, x)
    j1 = special.spherical_jn(1, x)
    return u * k * j0, du * k * j0 - u * k * k * j1


def radial_hidden(spec, W, t: int, p: int, d: np.ndarray):
    """h2(d) [E,64] of layer t's radial network p and its derivative dh2/dd (forward mode)."""
    d = np.asarray(d, dtype=np.float64)
    e, de = basis(spec, d)
    W1 = W[f"rad{t}_{p}_W1"].astype(np.float64)
    W2 = W[f"rad{t}_{p}_W2"].astype(np.float64)
    z1 = e @ W1.T
    h1 = model.silu(z1)
    dh1 = (de @ W1.T) * model.dsilu(z1)
    z2 = h1 @ W2.T
    return model.silu(z2), (dh1 @ W2.T) * model.dsilu(z2)


# ------------------------------------------------------------------ building a table
def _fit_piece(f, a: float, b: float, deg: int):
    t = cheb_nodes(deg + 1)
    vals, _ = f(0.5 * (a + b) + 0.5 * (b - a) * t)
    c = cheb_fit(vals)
    dc = cheb_deriv(c) * (2.0 / (b - a))                    # d/dd = (2 / (b - a)) d/dt
    return c, dc


def _check_points(a: float, b: float, n: int = N_CHECK) -> np.ndarray:
    """n Chebyshev extrema on [a, b], the ends included (where the derivative's error peaks)."""
    return a + 0.5 * (b - a) * (1.0 - np.cos(np.pi * np.arange(n) / (n - 1)))


def build_table(f, lo: float, hi: float, deg: int = DEGREE, tol: float = TOL, floor: float = FLOOR,
                max_level: int = MAX_LEVEL):
    """Dyadic piecewise Chebyshev table of f: d -> (values [p, m], d-derivatives [p, m]) on [lo, hi].

    Returns a list of pieces (a, b, level, c [deg+1, m], dc [deg, m]) ordered by a."""
    grid = lo + (hi - lo) * (np.arange(4096) + 0.5) / 4096
    v, dv = f(grid)
    gscale = np.abs(v).max(axis=0)
    gdscale = np.abs(dv).max(axis=0)
    pieces = []
    stack = [(lo, hi, 0)]
    while stack:
        a, b, level = stack.pop()
        c, dc = _fit_piece(f, a, b, deg)
        x = _check_points(a, b)
        fv, fd = f(x)
        tt = (2.0 * x - a - b) / (b - a)
        pv, pd = cheb_eval(c, tt), cheb_eval(dc, tt)
        s = np.maximum(np.abs(fv).max(axis=0), floor * gscale)
        sd = np.maximum(np.abs(fd).max(axis=0), floor * gdscale)
        ok = np.all(np.abs(pv - fv) <= tol * s) and np.all(np.abs(pd - fd) <= tol * sd)
        if ok or level >= max_level:
            pieces.append((a, b, level, c, dc))
        else:
            m = 0.5 * (a + b)
            stack.append((m, b, level + 1))
            stack.append((a, m, level + 1))
    pieces.sort(key=lambda q: q[0])
    return pieces


def table_eval(pieces, d: np.ndarray):
    """Values and d-derivatives of a table at d (each point in its piece)."""
    d = np.asarray(d, dtype=np.float64)
    m = pieces[0][3].shape[1]
    v = np.empty((d.shape[0], m))
    dv = np.empty_like(v)
    starts = np.array([q[0] for q in pieces])
    idx = np.clip(np.searchsorted(starts, d, side="right") - 1, 0, len(pieces) - 1)
    for k in np.unique(idx):
        a, b, _, c, dc = pieces[k]
        sel = idx == k
        t = (2.0 * d[sel] - a - b) / (b - a)
        v[sel] = cheb_eval(c, t)
        dv[sel] = cheb_eval(dc, t)
    return v, dv


def radial_table(spec, W, t: int, p: int, **kw):
    """The certified table of layer t's radial network p: h2 and dh2/dd on [0, rc]."""
    return build_table(lambda d: radial_hidden(spec, W, t, p, d), 0.0, float(spec.cutoff), **kw)


def certificate(approx, network, exact, scale) -> float:
    """max |approx - exact| / max |network - exact|, each output measured in its own scale
    (the float32 table's error over the float32 network's error, against float64)."""
    ea = (np.abs(approx - exact) / scale).max()
    en = (np.abs(network - exact) / scale).max()
    return float(ea / en)
