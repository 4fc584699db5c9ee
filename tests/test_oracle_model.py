"""Pins for the model oracle: envelope and basis closed forms, frame (gauge)
independence, rotation equivariance and invariance, the SH addition theorem for
a single edge, the scalar-only pair-potential special case, finite-difference
forces and strain-derivative virial."""
import math

import numpy as np
import pytest

import synth
from oracle import model, nl, sh

RNG = np.random.default_rng(9)


def test_envelope_closed_form():
    x = np.array([0.0, 1.0])
    assert np.allclose(model.envelope(x), [1.0, 0.0], atol=1e-15)
    assert abs(model.denvelope(np.array([1.0 - 1e-12]))[0]) < 1e-9
    # triple root at x = 1 (value, slope and curvature vanish at the cutoff): u(1-h) ~ h^3
    h = 1e-3
    ratio = model.envelope(np.array([1 - h]))[0] / model.envelope(np.array([1 - h / 2]))[0]
    assert abs(ratio - 8.0) < 0.05
    assert model.envelope(np.array([1.3]))[0] == 0.0
    xs = np.linspace(0.05, 0.95, 7)
    fd = (model.envelope(xs + 1e-6) - model.envelope(xs - 1e-6)) / 2e-6
    assert np.abs(fd - model.denvelope(xs)).max() < 1e-8


def test_bessel_basis_limits_and_derivative():
    rc = 6.0
    e = model.bessel_basis(np.array([1e-7]), rc)[0]
    assert np.allclose(e, np.pi * np.arange(1, 9) / rc, rtol=1e-6)   # sin(x)/x -> 1
    assert np.abs(model.bessel_basis(np.array([rc]), rc)).max() == 0.0
    d = np.linspace(0.8, 5.9, 11)
    fd = (model.bessel_basis(d + 1e-6, rc) - model.bessel_basis(d - 1e-6, rc)) / 2e-6
    assert np.abs(fd - model.dbessel_basis(d, rc)).max() < 1e-7
    # the sine factors are orthogonal on [0, rc]: int sin(n pi d/rc) sin(k pi d/rc) = rc/2 delta
    t, w = np.polynomial.legendre.leggauss(64)
    dd = (t + 1) * rc / 2
    s = model.bessel_basis(dd, rc) * dd[:, None] / model.envelope(dd / rc)[:, None]
    G = (s * (w * rc / 2)[:, None]).T @ s
    assert np.abs(G - rc / 2 * np.eye(8)).max() < 1e-10


def test_radial_network_vanishes_at_cutoff():
    w = synth.small_workload(C=8)
    R, _ = model.radial_of_edges(w.spec, w.weights, 0, np.array([w.spec.cutoff, 2.0]), np.zeros(2, int))
    assert np.abs(R[0]).max() == 0.0 and np.abs(R[1]).max() > 0


def test_pair_index_is_upper_triangle():
    a = np.array([0, 0, 0, 1, 1, 2, 2, 1])
    b = np.array([0, 1, 2, 1, 2, 2, 0, 0])
    assert list(model.pair_index(a, b, 3)) == [0, 1, 2, 3, 4, 5, 2, 1]


def _random_edges(n_atoms=5, n_edges=30, C=4):
    recv = np.sort(RNG.integers(0, n_atoms, n_edges))
    send = RNG.integers(0, n_atoms, n_edges)
    r = RNG.standard_normal((n_edges, 3)) * 1.5
    r *= (RNG.uniform(1.0, 5.5, n_edges) / np.linalg.norm(r, axis=1))[:, None]
    return recv, send, r


def test_so2_mixing_commutes_with_z_rotation():
    spec = synth.ModelSpec(C=4, n_layers=1)
    W = synth.draw_weights(spec, np.random.default_rng(1))
    x = RNG.standard_normal((6, 16, 4))
    Dz = sh.wigner_D(sh.rot_z(0.83))
    lhs = model.so2_apply(np.einsum("ab,ebc->eac", Dz, x), W, 0)
    rhs = np.einsum("ab,ebc->eac", Dz, model.so2_apply(x, W, 0))
    assert np.abs(lhs - rhs).max() < 1e-12
    # the transpose map is the adjoint
    g = RNG.standard_normal(x.shape)
    assert abs(np.sum(model.so2_apply(x, W, 0) * g) - np.sum(x * model.so2_apply(g, W, 0, True))) < 1e-10


def test_messages_do_not_depend_on_the_edge_frame():
    spec = synth.ModelSpec(C=4, n_layers=1)
    W = synth.draw_weights(spec, np.random.default_rng(2))
    recv, send, r = _random_edges()
    x = RNG.standard_normal((5, 16, 4))
    sp = np.zeros(5, int)
    a = model.single_layer(spec, W, 0, x, recv, send, r, sp, 5)
    rhat = r / np.linalg.norm(r, axis=1, keepdims=True)
    frames = np.stack([sh.rot_z(g) @ F for g, F in zip(RNG.uniform(0, 6.3, r.shape[0]),
                                                        sh.edge_frame(rhat))])
    b = model.single_layer(spec, W, 0, x, recv, send, r, sp, 5, frame=frames)
    assert np.abs(a - b).max() < 1e-12 * max(1.0, np.abs(a).max())


def test_layer_is_rotation_equivariant():
    spec = synth.ModelSpec(C=4, n_layers=1)
    W = synth.draw_weights(spec, np.random.default_rng(3))
    recv, send, r = _random_edges()
    x = RNG.standard_normal((5, 16, 4))
    sp = np.zeros(5, int)
    Q = sh.random_rotation(RNG)
    D = sh.wigner_D(Q)
    a = model.single_layer(spec, W, 0, x, recv, send, r, sp, 5)
    b = model.single_layer(spec, W, 0, np.einsum("ab,ebc->eac", D, x), recv, send, r @ Q.T, sp, 5)
    assert np.abs(np.einsum("ab,ebc->eac", D, a) - b).max() < 1e-12


def test_single_edge_message_follows_addition_theorem():
    # scalar input on the sender: y has only m = 0 entries, and the rotated-back
    # message of degree l is sqrt(4 pi/(2l+1)) Y_l(r_hat) times y[l, m=0]
    spec = synth.ModelSpec(C=3, n_layers=1)
    W = synth.draw_weights(spec, np.random.default_rng(4))
    r = np.array([[1.1, -2.0, 0.7]])
    x = np.zeros((2, 16, 3))
    x[1, 0, :] = [0.5, -1.0, 2.0]
    agg = model.single_layer(spec, W, 0, x, np.array([0]), np.array([1]), r, np.zeros(2, int), 2)
    d = np.linalg.norm(r)
    R, _ = model.radial_of_edges(spec, W, 0, np.array([d]), np.zeros(1, int))
    xt0 = R[0, 0] * x[1, 0]                                   # l = 0 rotated input, scaled
    W0 = W["so2_0_W0"].astype(np.float64)
    y_m0 = (W0[:, :3] @ xt0).reshape(4, 3)                    # rows (l, c), input column block l' = 0
    Y = sh.sh_all(r[0] / d)
    for l in range(4):
        ref = math.sqrt(4 * math.pi / (2 * l + 1)) * np.outer(Y[sh.block(l)], y_m0[l]) / spec.avg_degree
        assert np.abs(agg[0, sh.block(l)] - ref).max() < 1e-13


def test_scalar_only_single_layer_is_a_pair_potential():
    # one layer, no gate, scalar node inputs: e_i depends only on l=0 messages, i.e. on
    # W0's (l=0 -> l=0) block and the l=0 radial scale -- no rotation is involved.
    w = synth.small_workload(ncell=1, C=8, n_layers=1, gated=False, sigma=0.1)
    st, spec, W = w.structure, w.spec, w.weights
    g = nl.brute_force(st.pos, st.box, spec.cutoff)
    res = model.energy_forces(spec, W, st.species, g.recv, g.send, g.r, st.pos.shape[0])
    d = np.linalg.norm(g.r, axis=1)
    R, _ = model.radial_of_edges(spec, W, 0, d, np.zeros_like(d, dtype=int))
    emb = W["emb"].astype(np.float64)[st.species]
    W00 = W["so2_0_W0"].astype(np.float64)[:spec.C, :spec.C]
    msg = (R[:, 0, :] * emb[g.send]) @ W00.T
    h0 = np.zeros((st.pos.shape[0], spec.C))
    np.add.at(h0, g.recv, msg)
    h0 /= spec.avg_degree
    e = model.silu(h0 @ W["ro_W"].astype(np.float64).T) @ W["ro_w"].astype(np.float64)
    assert abs(e.sum() - res.energy) < 1e-12 * abs(res.energy)


def _setup(ncell=1, C=6, n_layers=2, gated=True, sigma=0.1, n_species=1, pair=False):
    w = synth.small_workload(ncell=ncell, C=C, n_layers=n_layers, gated=gated, sigma=sigma,
                             n_species=n_species, pair_radial=pair)
    st = w.structure
    g = nl.brute_force(st.pos, st.box, w.spec.cutoff)
    return w, st, g


def _energy_at(w, st, g, pos):
    r = (pos[g.send] - pos[g.recv]) + g.shift * st.box[None, :]
    return model.energy_only(w.spec, w.weights, st.species, g.recv, g.send, r, pos.shape[0])


@pytest.mark.parametrize("n_species,pair", [(1, False), (2, True)])
def test_forces_match_finite_differences(n_species, pair):
    w, st, g = _setup(n_species=n_species, pair=pair)
    res = model.energy_forces(w.spec, w.weights, st.species, g.recv, g.send, g.r, st.pos.shape[0])
    h = 1e-5
    fd = np.zeros_like(res.forces)
    for a in range(st.pos.shape[0]):
        for k in range(3):
            p = st.pos.copy()
            p[a, k] += h
            ep = _energy_at(w, st, g, p)
            p[a, k] -= 2 * h
            em = _energy_at(w, st, g, p)
            fd[a, k] = -(ep - em) / (2 * h)
    scale = np.abs(res.forces).max()
    assert scale > 0
    assert np.abs(fd - res.forces).max() < 1e-6 * scale
    assert np.abs(res.forces.sum(axis=0)).max() < 1e-12 * scale * st.pos.shape[0]


def test_energy_invariant_and_forces_covariant_under_rotation():
    w, st, g = _setup()
    n = st.pos.shape[0]
    a = model.energy_forces(w.spec, w.weights, st.species, g.recv, g.send, g.r, n)
    Q = sh.random_rotation(RNG)
    b = model.energy_forces(w.spec, w.weights, st.species, g.recv, g.send, g.r @ Q.T, n)
    assert abs(a.energy - b.energy) < 1e-12 * abs(a.energy)
    assert np.abs(a.forces @ Q.T - b.forces).max() < 1e-10 * np.abs(a.forces).max()


def test_virial_is_minus_strain_derivative():
    w, st, g = _setup()
    n = st.pos.shape[0]
    res = model.energy_forces(w.spec, w.weights, st.species, g.recv, g.send, g.r, n)
    h = 1e-6
    for a in range(3):
        for b in range(3):
            eps = np.zeros((3, 3))
            eps[a, b] = h
            ep = model.energy_only(w.spec, w.weights, st.species, g.recv, g.send, g.r @ (np.eye(3) + eps).T, n)
            em = model.energy_only(w.spec, w.weights, st.species, g.recv, g.send, g.r @ (np.eye(3) - eps).T, n)
            assert abs(-(ep - em) / (2 * h) - res.virial[b, a]) < 1e-6 * np.abs(res.virial).max()
    assert np.abs(res.virial - res.virial.T).max() < 1e-10 * np.abs(res.virial).max()


def test_n64_forces_sampled_finite_differences():
    w = synth.workload("n64_diamond")
    st = w.structure
    g = nl.brute_force(st.pos, st.box, w.spec.cutoff)
    res = model.energy_forces(w.spec, w.weights, st.species, g.recv, g.send, g.r, 64)
    h = 1e-5
    for a, k in [(0, 0), (17, 1), (40, 2), (63, 0)]:
        p = st.pos.copy()
        p[a, k] += h
        ep = _energy_at(w, st, g, p)
        p[a, k] -= 2 * h
        em = _energy_at(w, st, g, p)
        assert abs(-(ep - em) / (2 * h) - res.forces[a, k]) < 1e-6 * np.abs(res.forces).max()
