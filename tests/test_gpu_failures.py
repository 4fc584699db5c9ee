"""Failure detection through the C ABI, without a GPU fault.

Each case makes the failure on the host side (a buffer too small, a pointer off its
alignment, a neighbour list the key or the sort buffer cannot hold) or lets a bounded
device wait run out on an mbarrier that nothing arrives on; every case checks the
status returned and that the device stays usable afterwards.
"""
import ctypes

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import edge_message_passing_b200 as emp  # noqa: E402

EMP_ERR_ARG, EMP_ERR_TIMEOUT, EMP_ERR_WORKSPACE = -1, -4, -6


def _small_model(n_layers=3):
    w = synth.small_workload(ncell=1, C=32, n_layers=n_layers, gated=True, sigma=0.1, cohort_edges=128)
    st = w.structure
    g = emp.nl_build(torch.from_numpy(st.pos).cuda(), st.box, w.spec.cutoff)
    return w, g, emp.Model(w.spec, w.weights)


def _still_usable():
    w, g, model = _small_model()
    e, f, _, _ = emp.mp_energy_forces(model, g, torch.from_numpy(w.structure.species).cuda())
    torch.cuda.synchronize()
    assert np.isfinite(float(e.cpu()[0])) and torch.isfinite(f).all()
    assert emp.last_device_error() == 0


def test_bounded_wait_runs_out_and_reports_timeout():
    assert emp.last_device_error() == 0
    emp.set_wait_limit(2_000_000)              # about a millisecond
    try:
        assert emp.wait_selftest() == EMP_ERR_TIMEOUT
    finally:
        emp.set_wait_limit(0)                  # back to the default bound
    assert emp.last_device_error() == 0        # the word was cleared by the read
    _still_usable()


def test_workspace_too_small_is_rejected():
    w, g, model = _small_model()
    L = emp.lib()
    gc = g.c()
    need = model.workspace_bytes_min(g.n_edges, g.n_atoms)     # the least any call runs in
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    N, C = g.n_atoms, w.spec.C
    sp = torch.from_numpy(w.structure.species).cuda()
    x = torch.zeros((N, 16, C), device="cuda")
    agg = torch.empty_like(x)
    e = torch.empty(1, dtype=torch.float64, device="cuda")
    f = torch.empty((N, 3), device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert L.mp_forward(model.handle, ctypes.byref(gc), 1, sp.data_ptr(), x.data_ptr(), agg.data_ptr(),
                        ws.data_ptr(), ws.numel(), s) == EMP_ERR_WORKSPACE
    assert L.mp_energy_forces(model.handle, ctypes.byref(gc), sp.data_ptr(), e.data_ptr(), f.data_ptr(), None, None,
                              ws.data_ptr(), ws.numel(), s) == EMP_ERR_WORKSPACE
    X = torch.zeros((100, 16 * C), device="cuda")
    Y = torch.empty_like(X)
    small = torch.empty(2 * X.numel() * 4, dtype=torch.uint8, device="cuda")      # 256 bytes short
    assert L.mp_so2_mix(model.handle, 0, 0, 100, X.data_ptr(), Y.data_ptr(), small.data_ptr(), small.numel(),
                        s) == EMP_ERR_WORKSPACE
    assert emp.last_device_error() == 0


def test_misaligned_chain_buffers_are_rejected():
    ci = synth.chain_inputs(E=64, seed=5)
    ch = emp.Chain(ci.U, ci.M)
    L = emp.lib()
    raw = torch.zeros(64 * 128 + 1, device="cuda")
    x_off = raw[1:]                             # 4 bytes past a 16-byte boundary
    kc = torch.empty((64, 25), device="cuda")
    y0 = torch.empty((64, 64), device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert L.mp_radial_chain(ch.handle, 64, x_off.data_ptr(), kc.data_ptr(), y0.data_ptr(), None, None, None,
                             s) == EMP_ERR_ARG
    x = torch.zeros((64, 4, 32), device="cuda")
    assert L.mp_radial_chain(ch.handle, 64, x.data_ptr(), kc.data_ptr(), y0.data_ptr(), None, None, None, s) == 0
    torch.cuda.synchronize()
    assert emp.last_device_error() == 0


def test_nl_more_neighbours_than_the_sort_holds():
    """100 atoms in a 3 A cube with a 7 A cutoff: about 5300 neighbours per atom (> 4096)."""
    pos = np.random.default_rng(2).uniform(0.0, 3.0, (100, 3))
    with pytest.raises(emp.EmpError, match="device-side check failed"):
        emp.nl_build(torch.from_numpy(pos).cuda(), np.full(3, 3.0), 7.0)
    _still_usable()


def test_nl_image_shift_beyond_the_key_range():
    """One atom in a 0.04 A thin box: its own images up to 149 box lengths away are edges."""
    pos = np.array([[0.01, 5.0, 5.0]])
    with pytest.raises(emp.EmpError, match="unsupported"):
        emp.nl_build(torch.from_numpy(pos).cuda(), np.array([0.04, 100.0, 100.0]), 6.0)
    _still_usable()
