"""Weight gradients of the energy on the GPU (mp_energy_weight_grad) against the float64
oracle's reverse mode (oracle/grads.py, pinned by finite differences): every weight tensor,
max |d| <= 1e-4 max |ref| (FP32 sums over up to E edges; the forces' tolerance), the energy
and forces of the same call as mp_energy_forces's, and two calls agreeing bit for bit."""
import numpy as np
import pytest

import synth
from oracle import grads as og
from oracle import nl as onl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import edge_message_passing_b200 as emp  # noqa: E402


def _run(w, cohort=None):
    spec = w.spec if cohort is None else synth.ModelSpec(**{**w.spec.__dict__, "cohort_edges": cohort})
    st = w.structure
    g = emp.nl_build(torch.from_numpy(st.pos).cuda(), st.box, spec.cutoff)
    model = emp.Model(spec, w.weights)
    sp = torch.from_numpy(st.species).cuda()
    e, f, gr = emp.mp_energy_weight_grad(model, g, sp)
    ref_g = onl.brute_force(st.pos, st.box, spec.cutoff)
    E_ref, ref = og.energy_weight_grad(spec, w.weights, st.species, ref_g.recv, ref_g.send, ref_g.r, st.pos.shape[0])
    assert abs(float(e.cpu()[0]) - E_ref) <= 1e-5 * abs(E_ref)
    for name, r in ref.items():
        got = gr[name].double().cpu().numpy()
        scale = np.abs(r).max()
        if scale == 0.0:
            assert np.all(got == 0.0), name
        else:
            assert np.abs(got - r).max() <= 1e-4 * scale, (name, np.abs(got - r).max() / scale)
    e2, f2, _, _ = emp.mp_energy_forces(model, g, sp)
    assert torch.equal(e, e2) and torch.equal(f, f2)
    e3, f3, gr3 = emp.mp_energy_weight_grad(model, g, sp)
    for name in gr:
        assert torch.equal(gr[name], gr3[name])
    assert emp.last_device_error() == 0


@pytest.mark.parametrize("n_layers", [1, 2, 3])
def test_weight_grad_small_gated(n_layers):
    _run(synth.small_workload(ncell=1, C=32, n_layers=n_layers, gated=n_layers > 1, sigma=0.1), cohort=256)


def test_weight_grad_per_pair_radial():
    _run(synth.small_workload(ncell=1, C=32, n_layers=3, gated=True, n_species=3, pair_radial=True, sigma=0.1),
         cohort=128)


def test_weight_grad_n512():
    _run(synth.workload("n512_diamond"))
