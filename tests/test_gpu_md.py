"""Neighbour-list reuse with a skin (the MD loop): a graph built with cutoff rc + skin and
refreshed at new positions gives the energy and forces of the float64 oracle at those
positions with cutoff rc (the longer edges contribute exactly zero), the refreshed edge
vectors equal a fresh build's bit for bit, and a displacement beyond skin / 2 asks for a
rebuild."""
import numpy as np
import pytest

import synth
from oracle import model as omodel
from oracle import nl as onl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import edge_message_passing_b200 as emp  # noqa: E402


def test_skin_refresh_matches_the_oracle_and_a_fresh_build():
    w = synth.small_workload(ncell=1, C=32, n_layers=3, gated=True, sigma=0.1)
    st, spec = w.structure, w.spec
    skin = 0.6
    model = emp.Model(spec, w.weights)
    sp = torch.from_numpy(st.species).cuda()
    cache = emp.NeighbourCache(st.box, spec.cutoff, skin)
    g = cache.update(torch.from_numpy(st.pos).cuda())
    rng = np.random.default_rng(5)
    pos1 = st.pos + rng.uniform(-0.12, 0.12, st.pos.shape)         # every atom moves < skin / 2
    g1 = cache.update(torch.from_numpy(pos1).cuda())
    assert cache.builds == 1 and g1 is g
    # the refreshed vectors are those a fresh build (same cutoff) computes for the same edges
    fresh = emp.nl_build(torch.from_numpy(pos1).cuda(), st.box, spec.cutoff + skin)
    if fresh.n_edges == g1.n_edges and torch.equal(fresh.send, g1.send) and torch.equal(fresh.shift, g1.shift):
        assert torch.equal(fresh.vec.view(torch.int32), g1.vec.view(torch.int32))
    e, f, _, _ = emp.mp_energy_forces(model, g1, sp)
    ref_g = onl.brute_force(pos1, st.box, spec.cutoff)
    ref = omodel.energy_forces(spec, w.weights, st.species, ref_g.recv, ref_g.send, ref_g.r, pos1.shape[0])
    assert abs(float(e.cpu()[0]) - ref.energy) <= 1e-5 * abs(ref.energy)
    assert np.abs(f.cpu().numpy() - ref.forces).max() <= 1e-4 * np.abs(ref.forces).max()
    # one atom beyond skin / 2: rebuilt
    pos2 = pos1.copy()
    pos2[3] += np.array([0.35, 0.0, 0.0])
    cache.update(torch.from_numpy(pos2).cuda())
    assert cache.builds == 2
    assert emp.last_device_error() == 0
