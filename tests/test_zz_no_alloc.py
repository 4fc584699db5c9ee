"""nl_build_noalloc: the neighbour list for callers that cannot allocate device
memory (their device memory comes from a host program's own pool, or they must
avoid the device-wide synchronisation of cudaMalloc / cudaFree).  Its cell-list
scratch is a fixed array inside the library.  Checked through the C ABI against
nl_build (which uses caller scratch) on two calls in a row; the neighbour list
is bit-exact, so the comparison is exact.  Kept in a file of its own, collected
last."""
import ctypes

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import edge_message_passing_b200 as emp  # noqa: E402


def _noalloc(pos_np, box, rc, cap):
    L = emp.lib()
    N = pos_np.shape[0]
    pos = torch.from_numpy(pos_np).cuda()
    bufs = [torch.full((cap,), -7, dtype=torch.int32, device="cuda") for _ in range(3)]
    off = torch.full((N + 1,), -7, dtype=torch.int32, device="cuda")
    shift = torch.full((cap, 3), -7, dtype=torch.int32, device="cuda")
    vec = torch.full((cap, 3), -7.0, dtype=torch.float32, device="cuda")
    g = emp.GraphC(bufs[0].data_ptr(), bufs[1].data_ptr(), bufs[2].data_ptr(), off.data_ptr(), shift.data_ptr(),
                   vec.data_ptr(), 0, N)
    p = emp.NlParams(N, (ctypes.c_double * 3)(*[float(b) for b in box]), float(rc), cap)
    ne = ctypes.c_int64(0)
    st = L.nl_build_noalloc(ctypes.byref(p), pos.data_ptr(), ctypes.byref(g), ctypes.byref(ne),
                            torch.cuda.current_stream().cuda_stream)
    assert st == 0, L.emp_status_string(st)
    E = ne.value
    torch.cuda.synchronize()
    return E, bufs[0][:E], bufs[1][:E], bufs[2][:E], off, shift[:E], vec[:E]


def _check_same(st, rc):
    ref = emp.nl_build(torch.from_numpy(st.pos).cuda(), st.box, rc)
    E, recv, send, mirror, off, shift, vec = _noalloc(st.pos, st.box, rc, ref.n_edges)
    assert E == ref.n_edges
    for a, b in ((recv, ref.recv), (send, ref.send), (mirror, ref.mirror), (off, ref.recv_off), (shift, ref.shift)):
        assert torch.equal(a, b)
    assert torch.equal(vec.view(torch.int32), ref.vec.view(torch.int32))


def test_noalloc_matches_nl_build_on_two_calls_in_a_row():
    _check_same(synth.workload("n512_diamond").structure, 6.0)     # 512 atoms, 80896 edges
    _check_same(synth.workload("n64_diamond").structure, 6.0)      # then a smaller cell: no stale scratch


def test_noalloc_rejects_too_many_atoms():
    L = emp.lib()
    N = 65536 + 1                                   # one above the documented maximum
    p = emp.NlParams(N, (ctypes.c_double * 3)(10.0, 10.0, 10.0), 6.0, 0)
    g = emp.GraphC()
    ne = ctypes.c_int64(0)
    dummy = torch.zeros(3, dtype=torch.float64, device="cuda")
    assert L.nl_build_noalloc(ctypes.byref(p), dummy.data_ptr(), ctypes.byref(g), ctypes.byref(ne), None) == -6
