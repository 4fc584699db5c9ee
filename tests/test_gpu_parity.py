"""GPU parity of the CUDA path (through the C-ABI) against the float64 oracle.

Tolerances (FP32 path vs float64 oracle):
  neighbour list, edge order, shifts, mirror, float32 r_e: bit-exact;
  energy: |dE| <= 1e-5 |E|;  forces: max|dF| <= 1e-4 max|F|  (the target stated
  for this path);
  single-layer aggregates and SO(2) mixing: max|d| <= 2e-5 max|ref| (FP32 /
  3xTF32 dot products of length <= 16C with N(0,1/fan_in) weights; rounding
  error ~ sqrt(K) 2^-23 relative, well below this bound);
  radial chain: max|d| <= 1e-5 max|ref| (length-128 FP32 dot products).
"""
import json
import os

import numpy as np
import pytest

import synth
from oracle import chain as ochain
from oracle import model as omodel
from oracle import nl as onl
from oracle import sh

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import edge_message_passing_b200 as emp  # noqa: E402

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _cuda(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def _graph(st, rc=6.0):
    return emp.nl_build(_cuda(st.pos, torch.float64), st.box, rc)


def _assert_graph_equal(g, ref):
    assert g.n_edges == ref.n_edges
    assert np.array_equal(g.recv.cpu().numpy(), ref.recv)
    assert np.array_equal(g.send.cpu().numpy(), ref.send)
    assert np.array_equal(g.shift.cpu().numpy(), ref.shift)
    assert np.array_equal(g.mirror.cpu().numpy(), ref.mirror)
    assert np.array_equal(g.recv_off.cpu().numpy(), ref.recv_off)
    v = g.vec.cpu().numpy()
    assert np.array_equal(v.view(np.uint32), ref.vec.view(np.uint32))


# ------------------------------------------------------------------ neighbour list
@pytest.mark.parametrize("case", ["single_atom", "simple_cubic", "strict"])
def test_nl_tiny_cases(case):
    if case == "single_atom":
        pos, box, rc = np.array([[0.3, 0.4, 0.5]]), np.ones(3), 1.8
    elif case == "simple_cubic":
        pos = np.array([[i, j, k] for i in range(3) for j in range(3) for k in range(3)], float)
        box, rc = np.full(3, 3.0), 1.5
    else:
        pos, box, rc = np.array([[1.0, 1.0, 1.0], [3.0, 1.0, 1.0], [1.0, 2.999999, 1.0]]), np.full(3, 50.0), 2.0
    g = emp.nl_build(_cuda(pos, torch.float64), box, rc)
    _assert_graph_equal(g, onl.brute_force(pos, box, rc))


@pytest.mark.parametrize("name", ["n64_diamond", "n512_diamond", "ternary_n2000", "n4096_diamond"])
def test_nl_bit_exact(name):
    st = synth.workload(name).structure
    ref = onl.cell_list(st.pos, st.box, 6.0) if name == "ternary_n2000" else onl.brute_force(st.pos, st.box, 6.0)
    _assert_graph_equal(_graph(st), ref)


def test_nl_capacity_two_phase_and_errors():
    st = synth.workload("n64_diamond").structure
    g = emp.nl_build(_cuda(st.pos, torch.float64), st.box, 6.0, capacity=100)   # grows to 10112
    assert g.n_edges == 10112
    bad = st.pos.copy()
    bad[3, 1] = np.nan
    with pytest.raises(emp.EmpError, match="non-finite"):
        emp.nl_build(_cuda(bad, torch.float64), st.box, 6.0)


# ------------------------------------------------------------------ SO(2) mixing
def _to_cols(x, C):
    """[M,16,C] component layout -> [M,16C] m-major column layout."""
    M = x.shape[0]
    out = np.zeros((M, 16 * C), dtype=x.dtype)
    for l in range(4):
        for m in range(-l, l + 1):
            a = abs(m)
            off = {0: 0, 1: 4, 2: 10, 3: 14}[a] + ((4 - a) if m < 0 else 0) + (l - a)
            out[:, off * C:(off + 1) * C] = x[:, sh.lm_index(l, m), :]
    return out


@pytest.mark.parametrize("C,M", [(32, 300), (64, 128), (96, 257), (128, 1000), (256, 300)])
@pytest.mark.parametrize("transpose", [False, True])
def test_so2_mix_matches_oracle(C, M, transpose):
    spec = synth.ModelSpec(C=C, n_layers=1)
    W = synth.draw_weights(spec, np.random.default_rng(C + M))
    model = emp.Model(spec, W)
    x = np.random.default_rng(1).standard_normal((M, 16, C)).astype(np.float32)
    ref = omodel.so2_apply(x.astype(np.float64), W, 0, transpose=transpose)
    y = emp.mp_so2_mix(model, 0, _cuda(_to_cols(x, C)), transpose=transpose).cpu().numpy()
    refc = _to_cols(ref, C)
    assert np.abs(y - refc).max() <= 2e-5 * np.abs(refc).max()


# ------------------------------------------------------------------ one layer
@pytest.mark.parametrize("C,cohort,layer", [(32, 8192, 0), (32, 128, 1), (64, 256, 0)])
def test_single_layer_matches_oracle(C, cohort, layer):
    w = synth.small_workload(ncell=1, C=C, n_layers=2, cohort_edges=cohort, sigma=0.1)
    st = w.structure
    g = _graph(st)
    ref_g = onl.brute_force(st.pos, st.box, 6.0)
    x = synth.random_features(st.pos.shape[0], C, seed=5)
    model = emp.Model(w.spec, w.weights)
    agg = emp.mp_forward(model, g, layer, _cuda(st.species), _cuda(x)).cpu().numpy()
    ref = omodel.single_layer(w.spec, w.weights, layer, x, ref_g.recv, ref_g.send, ref_g.r, st.species,
                              st.pos.shape[0])
    assert np.abs(agg - ref).max() <= 2e-5 * np.abs(ref).max()


def test_single_layer_n64_full_features():
    w = synth.workload("n64_diamond")
    st = w.structure
    g = _graph(st)
    ref_g = onl.brute_force(st.pos, st.box, 6.0)
    x = synth.random_features(64, w.spec.C, seed=6)
    model = emp.Model(w.spec, w.weights)
    agg = emp.mp_forward(model, g, 0, _cuda(st.species), _cuda(x)).cpu().numpy()
    ref = omodel.single_layer(w.spec, w.weights, 0, x, ref_g.recv, ref_g.send, ref_g.r, st.species, 64)
    assert np.abs(agg - ref).max() <= 2e-5 * np.abs(ref).max()


# ------------------------------------------------------------------ energy and forces
def _check_ef(w, cohort=None, virial=True):
    spec = w.spec if cohort is None else synth.ModelSpec(**{**w.spec.__dict__, "cohort_edges": cohort})
    st = w.structure
    n = st.pos.shape[0]
    g = _graph(st, spec.cutoff)
    ref_g = onl.brute_force(st.pos, st.box, spec.cutoff)
    model = emp.Model(spec, w.weights)
    e, f, v, ea = emp.mp_energy_forces(model, g, _cuda(st.species), virial=virial, atom_energy=True)
    ref = omodel.energy_forces(spec, w.weights, st.species, ref_g.recv, ref_g.send, ref_g.r, n)
    E = float(e.cpu().numpy()[0])
    F = f.cpu().numpy()
    assert abs(E - ref.energy) <= 1e-5 * abs(ref.energy), (E, ref.energy)
    assert np.abs(F - ref.forces).max() <= 1e-4 * np.abs(ref.forces).max()
    assert np.abs(ea.cpu().numpy() - ref.atom_energy).max() <= 1e-5 * np.abs(ref.atom_energy).max()
    if virial:
        assert np.abs(v.cpu().numpy() - ref.virial).max() <= 1e-4 * np.abs(ref.virial).max()
    return model, g, (E, F)


@pytest.mark.parametrize("n_layers", [2, 3])
@pytest.mark.parametrize("cohort", [8192, 128])
def test_energy_forces_small_gated(cohort, n_layers):
    """Two layers: the first (degree-0 input) and the last (degree-0 output) alone; three: also
    a layer between them, run over edge cohorts (128 edges: many cohorts and a ragged tail)."""
    _check_ef(synth.small_workload(ncell=1, C=32, n_layers=n_layers, gated=True, sigma=0.1), cohort=cohort)


def test_energy_forces_ungated_three_layers():
    _check_ef(synth.small_workload(ncell=1, C=32, n_layers=3, gated=False, sigma=0.1), cohort=256)


def _cluster_workload(n_layers=3, far=True, seed=9):
    """A small random cluster in a large periodic box, plus (far=True) one atom out of every
    other atom's reach: a receiver (and sender) with no edges at all."""
    rng = np.random.default_rng(seed)
    w = synth.small_workload(ncell=1, C=32, n_layers=n_layers, gated=True, sigma=0.1)
    pts = [rng.uniform(0.0, 4.0, 3)]
    while len(pts) < 10:
        p = rng.uniform(0.0, 4.0, 3)
        if min(np.linalg.norm(p - q) for q in pts) > 1.2:
            pts.append(p)
    if far:
        pts.append(np.array([15.0, 15.0, 15.0]))
    pos = np.array(pts) + 2.0
    st = synth.Structure(pos=pos, box=np.full(3, 30.0), species=np.zeros(len(pts), dtype=np.int32))
    return synth.Workload(name="cluster", structure=st, spec=w.spec, weights=w.weights)


def test_energy_forces_isolated_atom():
    w = _cluster_workload()
    _, g, (E, F) = _check_ef(w, cohort=128)
    ro = g.recv_off.cpu().numpy()
    assert ro[-1] - ro[-2] == 0                      # the far atom receives no edge
    assert np.all(F[-1] == 0.0)


def test_energy_forces_no_edges():
    """E = 0: the energy is the readout of the embeddings, forces and virial vanish."""
    st = synth.Structure(pos=np.array([[1.0, 1.0, 1.0], [15.0, 15.0, 15.0]]), box=np.full(3, 30.0),
                         species=np.zeros(2, dtype=np.int32))
    w0 = synth.small_workload(ncell=1, C=32, n_layers=3, gated=True, sigma=0.1)
    w = synth.Workload(name="pair", structure=st, spec=w0.spec, weights=w0.weights)
    g = _graph(st)
    assert g.n_edges == 0
    model = emp.Model(w.spec, w.weights)
    e, f, v, ea = emp.mp_energy_forces(model, g, _cuda(st.species), virial=True, atom_energy=True)
    ref = omodel.energy_forces(w.spec, w.weights, st.species, np.zeros(0, int), np.zeros(0, int),
                               np.zeros((0, 3)), 2)
    assert abs(float(e.cpu()[0]) - ref.energy) <= 1e-5 * abs(ref.energy)
    assert np.all(f.cpu().numpy() == 0.0) and np.all(v.cpu().numpy() == 0.0)


@pytest.mark.parametrize("C", [96, 256])
def test_energy_forces_other_widths(C):
    """Channel counts off the bench's: 96 (one channel per thread in the backward edge
    kernel, 192-wide product tiles) and 256 (the largest the library accepts)."""
    _check_ef(synth.small_workload(ncell=1, C=C, n_layers=2, gated=True, sigma=0.1), cohort=512)


def test_energy_forces_small_pair_radial():
    _check_ef(synth.small_workload(ncell=1, C=32, n_layers=2, gated=True, n_species=3, pair_radial=True,
                                   sigma=0.1), cohort=256)


def test_energy_forces_n64():
    _check_ef(synth.workload("n64_diamond"))


@pytest.mark.parametrize("n_layers", [3, 4])
def test_kept_and_recomputed_mixing_outputs_agree_bit_for_bit(n_layers):
    """In the workspace of mp_workspace_bytes the per-edge layers keep their mixing outputs y
    from the forward; in that of mp_workspace_bytes_min the backward recomputes them: the same
    products, so the same bits (128-edge cohorts: many cohort pairs and a ragged tail)."""
    w = synth.small_workload(ncell=1, C=32, n_layers=n_layers, gated=True, sigma=0.1)
    spec = synth.ModelSpec(**{**w.spec.__dict__, "cohort_edges": 128})
    g = _graph(w.structure, spec.cutoff)
    sp = _cuda(w.structure.species)
    model = emp.Model(spec, w.weights)
    assert model.workspace_bytes_min(g.n_edges, g.n_atoms) < model.workspace_bytes(g.n_edges, g.n_atoms)
    a = [t.clone() for t in emp.mp_energy_forces(model, g, sp, virial=True, atom_energy=True)]
    b = emp.mp_energy_forces(model, g, sp, virial=True, atom_energy=True, compact=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert emp.last_device_error() == 0


def test_results_are_deterministic_and_inputs_untouched():
    w = synth.small_workload(ncell=1, C=32, n_layers=2, gated=True, sigma=0.1)
    st = w.structure
    pos = _cuda(st.pos, torch.float64)
    pos0 = pos.clone()
    g = emp.nl_build(pos, st.box, 6.0)
    snap = [t.clone() for t in (g.recv, g.send, g.mirror, g.recv_off, g.shift, g.vec)]
    sp = _cuda(st.species)
    model = emp.Model(w.spec, w.weights)
    a = emp.mp_energy_forces(model, g, sp, virial=True)
    b = emp.mp_energy_forces(model, g, sp, virial=True)
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)
    assert torch.equal(pos, pos0)
    for t0, t1 in zip(snap, (g.recv, g.send, g.mirror, g.recv_off, g.shift, g.vec)):
        assert torch.equal(t0, t1)
    assert emp.last_device_error() == 0


# ------------------------------------------------------------------ radial chain
def test_radial_chain_full_size():
    ci = synth.chain_inputs()
    ch = emp.Chain(ci.U, ci.M)
    kc, y0, gx = emp.mp_radial_chain(ch, _cuda(ci.x), _cuda(ci.g_kc), _cuda(ci.g_y0))
    W_eff = ochain.fold(ci.U, ci.M)
    rk, ry = ochain.folded_forward(ci.x, W_eff, ci.U[0])
    rg = ochain.folded_backward(ci.g_kc, ci.g_y0, W_eff, ci.U[0])
    assert np.abs(kc.cpu().numpy() - rk).max() <= 1e-5 * np.abs(rk).max()
    assert np.abs(y0.cpu().numpy() - ry).max() <= 1e-5 * np.abs(ry).max()
    assert np.abs(gx.cpu().numpy() - rg).max() <= 1e-5 * np.abs(rg).max()


def test_radial_chain_ragged_and_empty():
    ci = synth.chain_inputs(E=333, seed=12)
    ch = emp.Chain(ci.U, ci.M)
    kc, y0, gx = emp.mp_radial_chain(ch, _cuda(ci.x), _cuda(ci.g_kc), _cuda(ci.g_y0))
    ru, ry = ochain.unfolded_forward(ci.x, ci.U, ci.M)
    rg = ochain.unfolded_backward(ci.g_kc, ci.g_y0, ci.U, ci.M)
    assert np.abs(kc.cpu().numpy() - ru).max() <= 1e-5 * np.abs(ru).max()
    assert np.abs(gx.cpu().numpy() - rg).max() <= 1e-5 * np.abs(rg).max()
    e = torch.empty((0, 4, 32), device="cuda")
    kc, y0, _ = emp.mp_radial_chain(ch, e)
    assert kc.shape == (0, 25)


# edges per tile: 128 rows; sizes around one tile and with an uneven number of tiles per SM
@pytest.mark.parametrize("E", [1, 127, 128, 129, 148 * 128 * 3 + 77])
def test_radial_chain_tile_edges(E):
    ci = synth.chain_inputs(E=E, seed=20 + E % 7)
    ch = emp.Chain(ci.U, ci.M)
    kc, y0, gx = emp.mp_radial_chain(ch, _cuda(ci.x), _cuda(ci.g_kc), _cuda(ci.g_y0))
    W_eff = ochain.fold(ci.U, ci.M)
    rk, ry = ochain.folded_forward(ci.x, W_eff, ci.U[0])
    rg = ochain.folded_backward(ci.g_kc, ci.g_y0, W_eff, ci.U[0])
    for got, ref in ((kc, rk), (y0, ry), (gx, rg)):
        assert np.abs(got.cpu().numpy().reshape(ref.shape) - ref).max() <= 1e-5 * np.abs(ref).max()
    assert emp.last_device_error() == 0


# ------------------------------------------------------------------ full-size workloads
def _stored_oracle(name):
    path = os.path.join(GOLD, f"{name}_oracle.npz")
    if not os.path.exists(path):
        pytest.skip(f"{path} not generated (tests/golden/make_oracle_refs.py)")
    return np.load(path)


@pytest.mark.parametrize("name", ["n512_diamond", "n4096_diamond", "ternary_n2000"])
def test_energy_forces_full_size_against_stored_oracle(name):
    """The benchmark workloads at full size, in the launch configuration bench.py times."""
    ref = _stored_oracle(name)
    w = synth.workload(name)
    st = w.structure
    g = _graph(st, w.spec.cutoff)
    assert g.n_edges == int(ref["n_edges"])
    model = emp.Model(w.spec, w.weights)
    e, f, v, ea = emp.mp_energy_forces(model, g, _cuda(st.species), virial=True, atom_energy=True)
    E = float(e.cpu().numpy()[0])
    F = f.cpu().numpy()
    rE, rF = float(ref["energy"]), ref["forces"]
    assert abs(E - rE) <= 1e-5 * abs(rE), (E, rE)
    assert np.abs(F - rF).max() <= 1e-4 * np.abs(rF).max()
    assert np.abs(ea.cpu().numpy() - ref["atom_energy"]).max() <= 1e-5 * np.abs(ref["atom_energy"]).max()
    assert np.abs(v.cpu().numpy() - ref["virial"]).max() <= 1e-4 * np.abs(ref["virial"]).max()
    assert emp.last_device_error() == 0


def test_graph_replay_matches_eager_ternary_per_pair_networks():
    """Per-pair radial networks are captured too (their row ranges stay on the device)."""
    ref = _stored_oracle("ternary_n2000")
    w = synth.workload("ternary_n2000")
    st = w.structure
    g = _graph(st, w.spec.cutoff)
    sp = _cuda(st.species)
    model = emp.Model(w.spec, w.weights)
    e, f, _, _ = emp.mp_energy_forces(model, g, sp)
    e, f = e.clone(), f.clone()
    efg = emp.EnergyForcesGraph(model, g, sp)
    for _ in range(2):
        e2, f2, _, _ = efg.replay()
        torch.cuda.synchronize()
        assert torch.equal(e, e2) and torch.equal(f, f2)
    assert abs(float(e2.cpu()[0]) - float(ref["energy"])) <= 1e-5 * abs(float(ref["energy"]))
    assert np.abs(f2.cpu().numpy() - ref["forces"]).max() <= 1e-4 * np.abs(ref["forces"]).max()
    assert emp.last_device_error() == 0


def test_graph_replay_matches_eager_n4096():
    """The launch configuration bench.py times: the step captured once as a CUDA graph and
    replayed gives the eager call's results bit for bit (and so the stored oracle's)."""
    ref = _stored_oracle("n4096_diamond")
    w = synth.workload("n4096_diamond")
    st = w.structure
    g = _graph(st, w.spec.cutoff)
    sp = _cuda(st.species)
    model = emp.Model(w.spec, w.weights)
    e, f, _, _ = emp.mp_energy_forces(model, g, sp)
    e, f = e.clone(), f.clone()
    ec, fc, _, _ = emp.mp_energy_forces(model, g, sp, compact=True)    # y recomputed in the backward
    assert torch.equal(e, ec) and torch.equal(f, fc)
    efg = emp.EnergyForcesGraph(model, g, sp)
    assert efg.launches > 0
    for _ in range(2):
        e2, f2, _, _ = efg.replay()
        torch.cuda.synchronize()
        assert torch.equal(e, e2) and torch.equal(f, f2)
    E = float(e2.cpu().numpy()[0])
    assert abs(E - float(ref["energy"])) <= 1e-5 * abs(float(ref["energy"]))
    assert np.abs(f2.cpu().numpy() - ref["forces"]).max() <= 1e-4 * np.abs(ref["forces"]).max()
    assert emp.last_device_error() == 0


def test_single_layer_n4096_sampled_receivers():
    """Full-size single layer with random full features (all degrees): the oracle computes the
    aggregates of a sample of receivers from their own edges."""
    w = synth.workload("n4096_diamond")
    st = w.structure
    g = _graph(st)
    ref_g = onl.brute_force(st.pos, st.box, 6.0)
    x = synth.random_features(st.pos.shape[0], w.spec.C, seed=8)
    model = emp.Model(w.spec, w.weights)
    agg = emp.mp_forward(model, g, 1, _cuda(st.species), _cuda(x)).cpu().numpy()
    rng = np.random.default_rng(3)
    sample = np.sort(rng.choice(st.pos.shape[0], 24, replace=False))
    for i in sample:
        sl = slice(int(ref_g.recv_off[i]), int(ref_g.recv_off[i + 1]))
        ref = omodel.single_layer(w.spec, w.weights, 1, x, ref_g.recv[sl], ref_g.send[sl], ref_g.r[sl], st.species,
                                  st.pos.shape[0])[i]
        assert np.abs(agg[i] - ref).max() <= 2e-5 * np.abs(ref).max()


def test_tf32_rounding_matches_the_conversion_instruction():
    """The 3xTF32 split rounds on the bits (integer add and mask); over every non-NaN 32-bit
    pattern it must give what cvt.rna.tf32.f32 gives."""
    assert emp.tf32_split_selftest() == 0
