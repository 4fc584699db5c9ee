"""Pins for the certified-radial-table oracle (oracle/tables.py): Chebyshev interpolation
against closed forms (exact polynomials, the Chebyshev coefficients of exp, the derivative
of T_n, the interpolation error bound), the tabulated function against finite differences
and against the model's own radial network, and the table against its own rule (dyadic
pieces covering the range, every piece within tolerance at fresh points)."""
import math

import numpy as np
import pytest
from scipy import special

import synth
from oracle import model as omodel
from oracle import tables as tb


def test_degree_10_polynomials_are_reproduced_exactly():
    rng = np.random.default_rng(0)
    coef = rng.standard_normal((11, 3))                       # monomial coefficients
    poly = lambda t: np.stack([np.polynomial.polynomial.polyval(t, coef[:, j]) for j in range(3)], axis=1)
    c = tb.cheb_fit(poly(tb.cheb_nodes(11)))
    t = rng.uniform(-1, 1, 200)
    assert np.abs(tb.cheb_eval(c, t) - poly(t)).max() <= 1e-12 * np.abs(poly(t)).max()
    # T_3 is the third basis function
    c3 = tb.cheb_fit((4 * tb.cheb_nodes(11) ** 3 - 3 * tb.cheb_nodes(11))[:, None])
    assert np.abs(c3[:, 0] - np.eye(11)[3]).max() <= 1e-14


def test_chebyshev_coefficients_of_exp_are_modified_bessel_values():
    """exp(t) = I_0(1) + 2 sum_k I_k(1) T_k(t); the degree-10 interpolant's coefficients differ
    from these only by the aliased higher terms."""
    c = tb.cheb_fit(np.exp(tb.cheb_nodes(11))[:, None])[:, 0]
    want = np.array([special.iv(0, 1.0)] + [2 * special.iv(k, 1.0) for k in range(1, 11)])
    # at the 11 points T_{22-k} takes the values of -T_k: the interpolant's c_k differs from the
    # series' by about 2 I_{22-k}(1) (1e-12 for k = 10, far smaller below)
    alias = np.array([2 * special.iv(22 - k, 1.0) for k in range(11)])
    assert np.all(np.abs(c - want) <= 1.5 * alias + 1e-15)


def test_derivative_of_t5_is_five_u4():
    c = np.zeros((6, 1))
    c[5, 0] = 1.0
    dc = tb.cheb_deriv(c)
    t = np.linspace(-0.99, 0.99, 101)
    u4 = 16 * t ** 4 - 12 * t ** 2 + 1                        # Chebyshev polynomial of the second kind
    assert np.abs(tb.cheb_eval(dc, t)[:, 0] - 5 * u4).max() <= 1e-12


def test_interpolation_error_within_the_textbook_bound():
    """|f - p| <= max|f^(11)| ((b - a) / 2)^11 / (2^10 11!) at the Chebyshev points; sin has
    max|f^(11)| <= 1, and the bound is nearly attained."""
    a, b = 0.3, 2.1
    f = lambda d: (np.sin(d)[:, None], np.cos(d)[:, None])
    c, _ = tb._fit_piece(f, a, b, 10)
    x = np.linspace(a, b, 2001)
    err = np.abs(tb.cheb_eval(c, (2 * x - a - b) / (b - a))[:, 0] - np.sin(x)).max()
    bound = ((b - a) / 2) ** 11 / (2 ** 10 * math.factorial(11))
    assert err <= bound and err >= 1e-3 * bound


def test_basis_is_the_models_basis_and_has_the_small_distance_limits():
    w = synth.small_workload(ncell=1, C=32, n_layers=2, sigma=0.1)
    spec = w.spec
    d = np.linspace(0.5, 6.5, 61)
    e, de = tb.basis(spec, d)
    assert np.abs(e - omodel.bessel_basis(d, spec.cutoff, spec.n_basis, spec.env_p)).max() <= 1e-13
    assert np.abs(de - omodel.dbessel_basis(d, spec.cutoff, spec.n_basis, spec.env_p)).max() <= 1e-12
    # d -> 0: sin(k d) / d -> k, its derivative -> -k^3 d / 3 -> 0 (the envelope is flat there)
    k = np.pi * np.arange(1, 9) / spec.cutoff
    e0, de0 = tb.basis(spec, np.array([0.0, 1e-9]))
    assert np.allclose(e0[0], k, rtol=0, atol=1e-15) and np.allclose(e0[1], k, rtol=1e-15)
    assert np.abs(de0[1] + k ** 3 * 1e-9 / 3).max() <= 1e-15


def test_radial_hidden_is_the_models_hidden_output_and_its_derivative():
    w = synth.small_workload(ncell=1, C=32, n_layers=2, sigma=0.1)
    spec, W = w.spec, w.weights
    d = np.linspace(0.7, 5.9, 57)
    h2, dh2 = tb.radial_hidden(spec, W, 1, 0, d)
    e = omodel.bessel_basis(d, spec.cutoff, spec.n_basis, spec.env_p)
    _, (_, _, _, h2_model) = omodel.radial_forward(e, W["rad1_0_W1"].astype(float), W["rad1_0_W2"].astype(float),
                                                   W["rad1_0_W3"].astype(float))
    assert np.abs(h2 - h2_model).max() <= 1e-14
    h = 1e-6
    fd = (tb.radial_hidden(spec, W, 1, 0, d + h)[0] - tb.radial_hidden(spec, W, 1, 0, d - h)[0]) / (2 * h)
    assert np.abs(dh2 - fd).max() <= 1e-7 * np.abs(dh2).max()


@pytest.mark.parametrize("name,t", [("n4096_diamond", 0), ("n4096_diamond", 2), ("ternary_n2000", 1)])
def test_table_pieces_are_dyadic_and_within_tolerance(name, t):
    w = synth.workload(name)
    spec, W = w.spec, w.weights
    p = w.spec.n_pairs - 1
    pieces = tb.radial_table(spec, W, t, p)
    rc = float(spec.cutoff)
    # dyadic pieces that tile [0, rc]
    assert pieces[0][0] == 0.0 and pieces[-1][1] == rc
    for (a, b, level, c, dc), nxt in zip(pieces, pieces[1:] + [None]):
        width = rc / 2 ** level
        assert abs((b - a) - width) <= 1e-12 * rc and abs(a / width - round(a / width)) <= 1e-9
        assert level < tb.MAX_LEVEL
        if nxt is not None:
            assert nxt[0] == b
        assert c.shape == (tb.DEGREE + 1, 64) and dc.shape == (tb.DEGREE, 64)
    # fresh points (not the check points): values and derivatives within tolerance of the local scale
    f = lambda d: tb.radial_hidden(spec, W, t, p, d)
    gv, gd = f(np.linspace(1e-3, rc - 1e-3, 4096))
    gs, gds = np.abs(gv).max(axis=0), np.abs(gd).max(axis=0)
    rng = np.random.default_rng(7)
    for a, b, level, c, dc in pieces:
        x = rng.uniform(a, b, 40)
        fv, fd = f(x)
        pv, pd = tb.table_eval(pieces, x)
        s = np.maximum(np.abs(f(np.linspace(a, b, 200)[1:-1])[0]).max(axis=0), tb.FLOOR * gs)
        sd = np.maximum(np.abs(f(np.linspace(a, b, 200)[1:-1])[1]).max(axis=0), tb.FLOOR * gds)
        assert np.all(np.abs(pv - fv) <= 2 * tb.TOL * s)
        assert np.all(np.abs(pd - fd) <= 2 * tb.TOL * sd)
