"""Pins for real spherical harmonics, Wigner-D and generators: quadrature
orthonormality, the textbook associated-Legendre form (scipy), the degree-1
rotation matrix, group properties, the Lie algebra and its Casimir."""
import math

import numpy as np
import pytest
from scipy.special import lpmv, roots_legendre

from oracle import sh

RNG = np.random.default_rng(5)


def _unit(v):
    return v / np.linalg.norm(v, axis=-1, keepdims=True)


def _sphere_quadrature():
    # exact for polynomials of degree <= 15 in cos(theta) and trigonometric degree < 16 in phi
    ct, wt = roots_legendre(8)
    phi = np.arange(16) * 2 * math.pi / 16
    CT, PH = np.meshgrid(ct, phi, indexing="ij")
    st = np.sqrt(1 - CT ** 2)
    pts = np.stack([st * np.cos(PH), st * np.sin(PH), CT], -1).reshape(-1, 3)
    w = (wt[:, None] * np.full(16, 2 * math.pi / 16)[None, :]).ravel()
    return pts, w


def test_orthonormal_on_sphere():
    pts, w = _sphere_quadrature()
    Y = sh.sh_all(pts)
    G = (Y * w[:, None]).T @ Y
    assert np.abs(G - np.eye(16)).max() < 1e-13


def test_matches_associated_legendre():
    v = _unit(RNG.standard_normal((50, 3)))
    theta = np.arccos(v[:, 2])
    phi = np.arctan2(v[:, 1], v[:, 0])
    Y = sh.sh_all(v)
    for l in range(4):
        for m in range(-l, l + 1):
            am = abs(m)
            N = math.sqrt((2 * l + 1) / (4 * math.pi) * math.factorial(l - am) / math.factorial(l + am))
            P = lpmv(am, l, np.cos(theta)) * (-1) ** am         # remove the Condon-Shortley phase
            if m == 0:
                ref = N * P
            elif m > 0:
                ref = math.sqrt(2) * N * P * np.cos(m * phi)
            else:
                ref = math.sqrt(2) * N * P * np.sin(am * phi)
            assert np.abs(Y[:, sh.lm_index(l, m)] - ref).max() < 1e-13, (l, m)


def test_degree_one_order_is_y_z_x():
    v = _unit(RNG.standard_normal((10, 3)))
    c = math.sqrt(3 / (4 * math.pi))
    assert np.allclose(sh.sh_l(1, v), c * v[:, [1, 2, 0]], atol=1e-15)


def test_wigner_group_properties():
    Q1, Q2 = sh.random_rotation(RNG), sh.random_rotation(RNG)
    D1, D2, D12 = sh.wigner_D(Q1), sh.wigner_D(Q2), sh.wigner_D(Q1 @ Q2)
    assert np.abs(D1 @ D1.T - np.eye(16)).max() < 1e-12
    assert np.abs(D12 - D1 @ D2).max() < 1e-12
    assert np.abs(sh.wigner_D(np.eye(3)) - np.eye(16)).max() < 1e-12
    assert np.abs(sh.wigner_D(Q1.T) - D1.T).max() < 1e-12


def test_wigner_degree_one_is_permuted_rotation():
    Q = sh.random_rotation(RNG)
    P = np.array([[0, 1, 0], [0, 0, 1], [1, 0, 0]], float)
    assert np.abs(sh.wigner_D_l(1, Q) - P @ Q @ P.T).max() < 1e-13


def test_wigner_transforms_harmonics():
    Q = sh.random_rotation(RNG)
    v = _unit(RNG.standard_normal((40, 3)))
    lhs = sh.sh_all(v @ Q.T)
    rhs = sh.sh_all(v) @ sh.wigner_D(Q).T
    assert np.abs(lhs - rhs).max() < 1e-12


def test_z_rotation_acts_on_m_pairs():
    g = 0.7
    D = sh.wigner_D(sh.rot_z(g))
    for l in range(1, 4):
        for m in range(1, l + 1):
            p, q = sh.lm_index(l, m), sh.lm_index(l, -m)
            blk = D[np.ix_([p, q], [p, q])]
            ref = np.array([[math.cos(m * g), -math.sin(m * g)], [math.sin(m * g), math.cos(m * g)]])
            assert np.abs(blk - ref).max() < 1e-12


def test_generators_lie_algebra():
    J = sh.J_GEN
    for k in range(3):
        assert np.abs(J[k] + J[k].T).max() < 1e-12
    assert np.abs(J[0] @ J[1] - J[1] @ J[0] - J[2]).max() < 1e-12
    assert np.abs(J[1] @ J[2] - J[2] @ J[1] - J[0]).max() < 1e-12
    assert np.abs(J[2] @ J[0] - J[0] @ J[2] - J[1]).max() < 1e-12
    cas = sum(J[k] @ J[k] for k in range(3))
    ref = -np.diag(np.concatenate([np.full(2 * l + 1, l * (l + 1.0)) for l in range(4)]))
    assert np.abs(cas - ref).max() < 1e-11
    P = np.array([[0, 1, 0], [0, 0, 1], [1, 0, 0]], float)
    for k in range(3):
        e = np.zeros(3)
        e[k] = 1
        assert np.abs(J[k][1:4, 1:4] - P @ sh.skew(e) @ P.T).max() < 1e-13


def test_generator_is_derivative_of_rotation():
    h = 1e-6
    for k, R in enumerate([sh.rot_x, sh.rot_y, sh.rot_z]):
        fd = (sh.wigner_D(R(h)) - sh.wigner_D(R(-h))) / (2 * h)
        assert np.abs(fd - sh.J_GEN[k]).max() < 1e-8


@pytest.mark.parametrize("v", [[0, 0, 1], [0, 0, -1], [1e-9, 0, 1], [0.3, -0.4, 0.866], [1, 0, 0],
                               [-0.2, 0.1, -0.97]])
def test_edge_frame_maps_direction_to_z(v):
    rhat = _unit(np.array(v, float))
    R = sh.edge_frame(rhat)
    assert np.abs(R @ rhat - np.array([0, 0, 1.0])).max() < 1e-13
    assert np.abs(R @ R.T - np.eye(3)).max() < 1e-13
    assert abs(np.linalg.det(R) - 1) < 1e-13
