"""Pins for the weight-gradient oracle (oracle/grads.py): central finite differences of the
oracle's energy with respect to sampled entries of every weight tensor (two small models:
one radial network per layer, and per-pair radial networks), the energy it returns, and the
gradients the model's structure forces to zero (the first layer's input and the last
layer's read-out use degree 0 only, so neither sees the m > 0 mixing blocks)."""
import numpy as np
import pytest

import synth
from oracle import grads as og
from oracle import model as om
from oracle import nl as onl


def _setup(**kw):
    w = synth.small_workload(ncell=1, C=16, sigma=0.1, **kw)
    st = w.structure
    g = onl.brute_force(st.pos, st.box, w.spec.cutoff)
    return w, st, g


@pytest.mark.parametrize("kw", [dict(n_layers=3, gated=True), dict(n_layers=2, gated=True, n_species=3, pair_radial=True),
                                dict(n_layers=2, gated=False)])
def test_weight_gradients_match_central_differences(kw):
    w, st, g = _setup(**kw)
    n = st.pos.shape[0]
    E, gr = og.energy_weight_grad(w.spec, w.weights, st.species, g.recv, g.send, g.r, n)
    E_ref = om.energy_only(w.spec, w.weights, st.species, g.recv, g.send, g.r, n)
    assert abs(E - E_ref) <= 1e-12 * abs(E_ref)
    assert set(gr) == set(w.weights)
    rng = np.random.default_rng(11)
    h = 1e-5
    for name, Wt in w.weights.items():
        flat = np.asarray(Wt, dtype=np.float64).ravel()
        scale = np.abs(gr[name]).max()
        for idx in rng.choice(flat.size, size=min(3, flat.size), replace=False):
            Wp = dict(w.weights)
            Wm = dict(w.weights)
            a, b = flat.copy(), flat.copy()
            a[idx] += h
            b[idx] -= h
            Wp[name] = a.reshape(np.shape(Wt))
            Wm[name] = b.reshape(np.shape(Wt))
            fd = (om.energy_only(w.spec, Wp, st.species, g.recv, g.send, g.r, n)
                  - om.energy_only(w.spec, Wm, st.species, g.recv, g.send, g.r, n)) / (2 * h)
            got = gr[name].ravel()[idx]
            assert abs(got - fd) <= 1e-6 * max(scale, 1e-12) + 1e-9, (name, idx, got, fd)


def test_structural_zeros():
    w, st, g = _setup(n_layers=3, gated=True)
    _, gr = og.energy_weight_grad(w.spec, w.weights, st.species, g.recv, g.send, g.r, st.pos.shape[0])
    C = w.spec.C
    for m in (1, 2, 3):
        for t in (0, 2):                            # first layer: degree-0 input; last: degree-0 read-out
            assert np.all(gr[f"so2_{t}_Wr{m}"] == 0.0) and np.all(gr[f"so2_{t}_Wi{m}"] == 0.0)
        assert np.abs(gr[f"so2_1_Wr{m}"]).max() > 0 and np.abs(gr[f"so2_1_Wi{m}"]).max() > 0
    # first layer: only the degree-0 input columns of W0; last layer: only its degree-0 output rows
    assert np.all(gr["so2_0_W0"][:, C:] == 0.0) and np.abs(gr["so2_0_W0"][:, :C]).max() > 0
    assert np.all(gr["so2_2_W0"][C:, :] == 0.0) and np.abs(gr["so2_2_W0"][:C, :]).max() > 0
    # the first layer's radial scales enter through degree 0 only
    assert np.all(gr["rad0_0_W3"][C:, :] == 0.0)
