"""Real spherical harmonics, Wigner-D matrices and rotation generators (float64).

Test infrastructure only (see ``oracle/__init__``).

Convention (the model rotates neighbour irreps with lmax = 3 into the edge
frame; the pages fix neither basis nor phase, so this plain reading is used):
real, orthonormal on the unit sphere, z the polar axis, components ordered
m = -l..l, no Condon-Shortley phase: m > 0 ~ P_l^m(cos t) cos(m p), m < 0 ~
P_l^|m|(cos t) sin(|m| p), each with a positive constant.  Degree 1 is thus
sqrt(3/4pi) * (y, z, x).  The 16 components of lmax = 3 are indexed
lm = l*l + l + m.

Wigner-D: for a rotation Q, D(Q) is defined by Y(Q r) = D(Q) Y(r) for all unit r.
It is obtained here by least-squares fitting over a fixed set of generic
points P: D_l(Q) = Y_l(Q P) Y_l(P)^+ (exact up to rounding because Y_l(P) has
full row rank).

Generators: J_k = d/de D(exp(e [e_k]x)) at e = 0, taken by a complex step of the
fitted D (exact up to rounding for these polynomial maps).
"""
from __future__ import annotations

import math

import numpy as np

LMAX = 3
NCOMP = 16


def lm_index(l: int, m: int) -> int:
    return l * l + l + m


def block(l: int) -> slice:
    return slice(l * l, (l + 1) * (l + 1))


def sh_l(l: int, v: np.ndarray) -> np.ndarray:
    """Y_l at points v [...,3] on the unit sphere -> [..., 2l+1] (also valid for
    complex v: the expressions are polynomials)."""
    x, y, z = v[..., 0], v[..., 1], v[..., 2]
    pi = math.pi
    if l == 0:
        return (0.5 * math.sqrt(1.0 / pi)) * np.ones_like(x)[..., None]
    if l == 1:
        c = math.sqrt(3.0 / (4.0 * pi))
        return np.stack([c * y, c * z, c * x], axis=-1)
    if l == 2:
        c1 = 0.5 * math.sqrt(15.0 / pi)
        c0 = 0.25 * math.sqrt(5.0 / pi)
        c2 = 0.25 * math.sqrt(15.0 / pi)
        return np.stack([
            c1 * x * y,
            c1 * y * z,
            c0 * (2 * z * z - x * x - y * y),
            c1 * x * z,
            c2 * (x * x - y * y),
        ], axis=-1)
    if l == 3:
        c3 = 0.25 * math.sqrt(35.0 / (2.0 * pi))
        c2 = 0.5 * math.sqrt(105.0 / pi)
        c1 = 0.25 * math.sqrt(21.0 / (2.0 * pi))
        c0 = 0.25 * math.sqrt(7.0 / pi)
        c2b = 0.25 * math.sqrt(105.0 / pi)
        r2 = x * x + y * y
        return np.stack([
            c3 * y * (3 * x * x - y * y),
            c2 * x * y * z,
            c1 * y * (4 * z * z - r2),
            c0 * z * (2 * z * z - 3 * r2),
            c1 * x * (4 * z * z - r2),
            c2b * z * (x * x - y * y),
            c3 * x * (x * x - 3 * y * y),
        ], axis=-1)
    raise ValueError(l)


def sh_all(v: np.ndarray) -> np.ndarray:
    return np.concatenate([sh_l(l, v) for l in range(LMAX + 1)], axis=-1)


def _fit_points(n: int = 24) -> np.ndarray:
    """Deterministic generic unit vectors (Fibonacci sphere, rotated off-axis)."""
    k = np.arange(n) + 0.5
    z = 1.0 - 2.0 * k / n
    phi = k * math.pi * (3.0 - math.sqrt(5.0)) + 0.3
    rho = np.sqrt(1.0 - z * z)
    return np.stack([rho * np.cos(phi), rho * np.sin(phi), z], axis=-1)


FIT_P = _fit_points()
_PINV = [np.linalg.pinv(sh_l(l, FIT_P).T) for l in range(LMAX + 1)]   # [npts, 2l+1]


def wigner_D_l(l: int, Q: np.ndarray) -> np.ndarray:
    """D_l(Q) for rotation(s) Q [...,3,3] -> [..., 2l+1, 2l+1]."""
    QP = np.einsum("...ij,pj->...pi", Q, FIT_P)            # [..., npts, 3]
    Y = sh_l(l, QP)                                        # [..., npts, 2l+1]
    return np.einsum("...pa,pb->...ab", Y, _PINV[l])       # Y(QP)^T (2l+1 x npts) @ pinv


def wigner_D(Q: np.ndarray) -> np.ndarray:
    """Block-diagonal 16x16 D(Q)."""
    Q = np.asarray(Q)
    out = np.zeros(Q.shape[:-2] + (NCOMP, NCOMP), dtype=np.result_type(Q, np.float64))
    for l in range(LMAX + 1):
        out[..., block(l), block(l)] = wigner_D_l(l, Q)
    return out


def skew(v) -> np.ndarray:
    x, y, z = v
    return np.array([[0.0, -z, y], [z, 0.0, -x], [-y, x, 0.0]])


def generators() -> np.ndarray:
    """J[k] (k = x, y, z), each block-diagonal 16x16, by complex step."""
    h = 1e-30
    J = np.zeros((3, NCOMP, NCOMP))
    for k in range(3):
        e = np.zeros(3)
        e[k] = 1.0
        Q = np.eye(3) + 1j * h * skew(e)
        J[k] = np.imag(wigner_D(Q)) / h
    return J


J_GEN = generators()


def rot_x(a):
    c, s = math.cos(a), math.sin(a)
    return np.array([[1, 0, 0], [0, c, -s], [0, s, c]], dtype=np.float64)


def rot_y(a):
    c, s = math.cos(a), math.sin(a)
    return np.array([[c, 0, s], [0, 1, 0], [-s, 0, c]], dtype=np.float64)


def rot_z(a):
    c, s = math.cos(a), math.sin(a)
    return np.array([[c, -s, 0], [s, c, 0], [0, 0, 1]], dtype=np.float64)


def random_rotation(rng: np.random.Generator) -> np.ndarray:
    q = rng.standard_normal(4)
    q /= np.linalg.norm(q)
    a, b, c, d = q
    return np.array([
        [a * a + b * b - c * c - d * d, 2 * (b * c - a * d), 2 * (b * d + a * c)],
        [2 * (b * c + a * d), a * a - b * b + c * c - d * d, 2 * (c * d - a * b)],
        [2 * (b * d - a * c), 2 * (c * d + a * b), a * a - b * b - c * c + d * d],
    ])


def edge_frame(rhat: np.ndarray) -> np.ndarray:
    """A rotation R_e with R_e rhat = z, Euler form R_y(-beta) R_z(-alpha), with
    cos(beta) = z, sin(beta) = rho, cos(alpha) = x/rho, sin(alpha) = y/rho
    (alpha = 0 on the pole).  Batched over [...,3]."""
    x, y, z = rhat[..., 0], rhat[..., 1], rhat[..., 2]
    rho = np.sqrt(x * x + y * y)
    safe = rho > 0
    ca = np.where(safe, x / np.where(safe, rho, 1.0), 1.0)
    sa = np.where(safe, y / np.where(safe, rho, 1.0), 0.0)
    cb, sb = z, rho
    Rz = np.zeros(rhat.shape[:-1] + (3, 3))
    Rz[..., 0, 0] = ca
    Rz[..., 0, 1] = sa
    Rz[..., 1, 0] = -sa
    Rz[..., 1, 1] = ca
    Rz[..., 2, 2] = 1.0
    Ry = np.zeros_like(Rz)
    Ry[..., 0, 0] = cb
    Ry[..., 0, 2] = -sb
    Ry[..., 1, 1] = 1.0
    Ry[..., 2, 0] = sb
    Ry[..., 2, 2] = cb
    return Ry @ Rz
