"""Pins for the radial-chain oracle: the fold identity in float64 (the page prints
a max difference of 1e-15), the adjoint identity of the input gradient, and the
page's intermediate size and flop count."""
import json
import os

import numpy as np

import synth
from oracle import chain

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_numbers.json")))


def test_fold_identity_forward_and_backward():
    ci = synth.chain_inputs(E=3000, seed=3)
    kc_u, y0_u = chain.unfolded_forward(ci.x, ci.U, ci.M)
    W_eff = chain.fold(ci.U, ci.M)
    assert W_eff.shape == (128, 25)
    kc_f, y0_f = chain.folded_forward(ci.x, W_eff, ci.U[0])
    scale = np.abs(kc_u).max()
    assert np.abs(kc_u - kc_f).max() <= 1e-12 * scale
    assert np.abs(y0_u - y0_f).max() <= 1e-14 * np.abs(y0_u).max()
    gx_u = chain.unfolded_backward(ci.g_kc, ci.g_y0, ci.U, ci.M)
    gx_f = chain.folded_backward(ci.g_kc, ci.g_y0, W_eff, ci.U[0])
    assert np.abs(gx_u - gx_f).max() <= 1e-12 * np.abs(gx_u).max()
    # the page's float64 identity figure is of the same order
    assert np.abs(kc_u - kc_f).max() < 1000 * GOLD["fold_identity_float64"]["max_abs_diff"] * scale


def test_input_gradient_is_the_adjoint():
    ci = synth.chain_inputs(E=500, seed=8)
    kc, y0 = chain.unfolded_forward(ci.x, ci.U, ci.M)
    gx = chain.unfolded_backward(ci.g_kc, ci.g_y0, ci.U, ci.M)
    lhs = np.sum(gx * ci.x.astype(np.float64))
    rhs = np.sum(ci.g_kc * kc) + np.sum(ci.g_y0 * y0)
    assert abs(lhs - rhs) < 1e-10 * abs(rhs)


def test_unfolded_chain_matches_plain_loops():
    ci = synth.chain_inputs(E=4, seed=1)
    kc, y0 = chain.unfolded_forward(ci.x, ci.U, ci.M)
    for e in range(4):
        up = [[sum(float(ci.x[e, l, k]) * float(ci.U[l, k, h]) for k in range(32)) for h in range(64)]
              for l in range(4)]
        flat = [up[l][h] for l in range(4) for h in range(64)]
        for j in range(25):
            assert abs(sum(flat[i] * float(ci.M[i, j]) for i in range(256)) - kc[e, j]) < 1e-12
        assert np.allclose(up[0], y0[e], atol=1e-13)


def test_page_sizes():
    g = GOLD["radial_chain"]
    E = g["E"]
    assert round(chain.unfolded_intermediate_bytes(E) / 1e6) == 663  # "662 MB" (662.7e6 B)
    assert int(chain.unfolded_intermediate_bytes(E) / 1e6) == g["intermediate_MB"]
    assert round(chain.unfolded_flops(E) / 1e9) == g["chain_GFLOP_approx"]
