"""Certified radial tables on the GPU (opt-in; FastMACE page, "Rewrite screens: adopted and
rejected", OPT6-T04 / OPT6-T05): the certificate of the float32 tables against the float32
radial network, both measured against the float64 oracle, and the energy and forces with the
tables on against the float64 oracle of the exact model (same tolerances as without tables).

Certificate = max |table - float64| / max |network - float64| over a dense grid of edge lengths,
each of the 64 hidden outputs measured in its own scale (its largest magnitude on the grid); for
the length derivative, the projection onto a random dE/dh2 (what the backward consumes).  The
page's gate is that the tables are no less accurate than the float32 network: certificate <= 1.
"""
import numpy as np
import pytest

import synth
from oracle import model as omodel
from oracle import nl as onl
from oracle import tables as otab

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import edge_message_passing_b200 as emp  # noqa: E402


def _h2(model, t, p, d, g):
    hi, lo, dEdd = emp.mp_radial_hidden(model, t, p, torch.from_numpy(d.astype(np.float32)).cuda(),
                                        torch.from_numpy(g).cuda())
    return hi.double().cpu().numpy() + lo.double().cpu().numpy(), dEdd.double().cpu().numpy()


@pytest.mark.parametrize("name,t,p", [("n4096_diamond", 0, 0), ("n4096_diamond", 1, 0), ("n4096_diamond", 2, 0),
                                      ("ternary_n2000", 1, 5), ("ternary_n2000", 2, 2)])
def test_table_certificate(name, t, p):
    w = synth.workload(name)
    model = emp.Model(w.spec, w.weights)
    d = np.linspace(0.7, w.spec.cutoff - 1e-3, 4096).astype(np.float32).astype(np.float64)
    g = np.random.default_rng(t + 3 * p).standard_normal((d.shape[0], 64)).astype(np.float32)
    h64, dh64 = otab.radial_hidden(w.spec, w.weights, t, p, d)
    gd64 = np.einsum("ej,ej->e", g.astype(np.float64), dh64)
    net, net_d = _h2(model, t, p, d, g)
    n_pieces = model.radial_tables(otab.TOL)
    tab, tab_d = _h2(model, t, p, d, g)
    ref_pieces = sum(len(otab.radial_table(w.spec, w.weights, tt, pp))
                     for tt in range(w.spec.n_layers) for pp in range(w.spec.n_pairs))
    assert abs(n_pieces - ref_pieces) <= max(2, ref_pieces // 20)        # the same rule, host double
    scale = np.abs(h64).max(axis=0)
    cert = otab.certificate(tab, net, h64, scale)
    cert_d = otab.certificate(tab_d[:, None], net_d[:, None], gd64[:, None], np.abs(gd64).max())
    print(f"{name} layer {t} pair {p}: certificate {cert:.3f} (values), {cert_d:.3f} (length derivative)")
    assert cert <= 1.0 and cert_d <= 1.0


def _check(w, tables: bool):
    st = w.structure
    g = emp.nl_build(torch.from_numpy(st.pos).cuda(), st.box, w.spec.cutoff)
    ref_g = onl.brute_force(st.pos, st.box, w.spec.cutoff) if st.pos.shape[0] <= 600 else \
        onl.cell_list(st.pos, st.box, w.spec.cutoff)
    model = emp.Model(w.spec, w.weights)
    if tables:
        assert model.radial_tables(otab.TOL) > 0
    e, f, v, _ = emp.mp_energy_forces(model, g, torch.from_numpy(st.species).cuda(), virial=True)
    ref = omodel.energy_forces(w.spec, w.weights, st.species, ref_g.recv, ref_g.send, ref_g.r, st.pos.shape[0])
    E, F = float(e.cpu()[0]), f.cpu().numpy()
    assert abs(E - ref.energy) <= 1e-5 * abs(ref.energy)
    assert np.abs(F - ref.forces).max() <= 1e-4 * np.abs(ref.forces).max()
    assert np.abs(v.cpu().numpy() - ref.virial).max() <= 1e-4 * np.abs(ref.virial).max()
    assert emp.last_device_error() == 0
    return model, g, (e.clone(), f.clone())


def test_energy_forces_with_tables_n512():
    _check(synth.workload("n512_diamond"), tables=True)


def test_energy_forces_with_tables_per_pair_networks():
    _check(synth.small_workload(ncell=1, C=32, n_layers=3, gated=True, n_species=3, pair_radial=True, sigma=0.1),
           tables=True)


def test_tables_off_gives_the_network_back_bit_for_bit():
    w = synth.small_workload(ncell=1, C=32, n_layers=3, gated=True, sigma=0.1)
    model, g, (e0, f0) = _check(w, tables=False)
    sp = torch.from_numpy(w.structure.species).cuda()
    model.radial_tables(otab.TOL)
    e1, f1, _, _ = emp.mp_energy_forces(model, g, sp)
    assert not torch.equal(f1, f0)                    # the tables are in use
    assert model.radial_tables(0.0) == 0
    e2, f2, _, _ = emp.mp_energy_forces(model, g, sp)
    assert torch.equal(e2, e0) and torch.equal(f2, f0)
