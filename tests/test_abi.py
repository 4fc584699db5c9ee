"""Host-side checks of the C-ABI library: it loads, exports every function that
include/emp.h declares, and rejects bad arguments before touching a device."""
import ctypes
import os
import re

import numpy as np
import pytest

import synth
import edge_message_passing_b200 as emp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "emp.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"^\s*typedef[^;]*;", "", src, flags=re.M)          # function-pointer types are not exports
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_expected_entry_points():
    names = _declared()
    for n in ("nl_build", "mp_forward", "mp_energy_forces", "mp_radial_chain", "mp_so2_mix"):
        assert n in names
    assert sorted(emp.SYMBOLS) == names


def test_library_exports_every_declared_symbol():
    L = emp.lib()
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings():
    L = emp.lib()
    assert L.emp_status_string(0) == b"ok"
    assert L.emp_status_string(-2).startswith(b"graph capacity")
    assert L.emp_status_string(12345) == b"unknown status"


@pytest.mark.parametrize("name", ["n64_diamond", "n512_diamond", "ternary_n2000"])
def test_weight_count_matches_blob_layout(name):
    w = synth.workload(name)
    sc = emp.spec_c(w.spec)
    n = emp.lib().mp_weight_count(ctypes.byref(sc))
    assert n == sum(np.asarray(w.weights[k]).size for k in emp.weight_order(w.spec))
    assert set(emp.weight_order(w.spec)) == set(w.weights)


def test_null_arguments_are_rejected_on_the_host():
    L = emp.lib()
    ne = ctypes.c_int64(0)
    assert L.nl_build(None, None, None, ctypes.byref(ne), None, 0, None) == -1
    assert L.mp_model_create(None, None, 0, None) == -1
    assert L.mp_forward(None, None, 0, None, None, None, None, 0, None) == -1
    assert L.mp_energy_forces(None, None, None, None, None, None, None, None, 0, None) == -1
    assert L.mp_radial_chain(None, 0, None, None, None, None, None, None, None) == -1
    assert L.mp_so2_mix(None, 0, 0, 0, None, None, None, 0, None) == -1
    assert L.mp_workspace_bytes(None, 10, 10) == 0
    assert L.mp_workspace_bytes_min(None, 10, 10) == 0
    assert L.mp_sharded_workspace_bytes(None, 10, 10, 10) == 0
    assert L.mp_weight_grad_workspace_bytes(None, 10, 10) == 0
    assert L.nl_workspace_bytes(100) > 0
