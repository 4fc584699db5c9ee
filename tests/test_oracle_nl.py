"""Pins for the neighbour-list oracle: brute force vs an independent cell list,
hand-countable lattices, strictness of the cutoff, mirror symmetry, and the
page-printed edge and cohort counts."""
import json
import math
import os

import numpy as np
import pytest

import synth
from oracle import nl

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_numbers.json")))


def _same(a, b):
    return (np.array_equal(a.recv, b.recv) and np.array_equal(a.send, b.send)
            and np.array_equal(a.shift, b.shift) and np.array_equal(a.r, b.r)
            and np.array_equal(a.mirror, b.mirror) and np.array_equal(a.recv_off, b.recv_off))


@pytest.mark.parametrize("name,n", [("n64_diamond", 64), ("n512_diamond", 512)])
def test_diamond_every_atom_has_158_neighbours(name, n):
    st = synth.workload(name).structure
    g = nl.brute_force(st.pos, st.box, 6.0)
    assert st.pos.shape[0] == n
    # diamond shells up to 5.848 A hold 158 neighbours; the next shell is at 6.18 A
    assert np.all(np.diff(g.recv_off) == 158)
    assert g.n_edges == 158 * n


def test_edge_count_near_page_value():
    st = synth.workload("n64_diamond").structure
    g = nl.brute_force(st.pos, st.box, 6.0)
    assert abs(g.n_edges - GOLD["n64_edges_approx"]["value"]) <= 2


def test_cohort_counts_match_pages():
    for E, cohort, n in GOLD["cohorts_observed"]["rows"]:
        assert math.ceil(E / cohort) == n


@pytest.mark.parametrize("name", ["n64_diamond", "n512_diamond"])
def test_brute_force_equals_cell_list(name):
    st = synth.workload(name).structure
    assert _same(nl.brute_force(st.pos, st.box, 6.0), nl.cell_list(st.pos, st.box, 6.0))


def test_brute_force_equals_cell_list_random_cell():
    rng = np.random.default_rng(11)
    st = synth.random_cell(120, 0.08, 1.7, (40, 40, 40), rng)
    assert _same(nl.brute_force(st.pos, st.box, 6.0), nl.cell_list(st.pos, st.box, 6.0))


def test_single_atom_self_images():
    # one atom in a unit cube: images at distance 1 (6 faces), sqrt2 (12 edges), sqrt3 (8 corners)
    pos = np.array([[0.3, 0.4, 0.5]])
    box = np.ones(3)
    assert nl.brute_force(pos, box, 1.5).n_edges == 18
    assert nl.brute_force(pos, box, 1.8).n_edges == 26
    assert nl.brute_force(pos, box, 0.99).n_edges == 0
    g = nl.brute_force(pos, box, 1.5)
    assert _same(g, nl.cell_list(pos, box, 1.5))
    keys = [tuple(s) for s in g.shift]
    assert keys == sorted(keys)


def test_simple_cubic_shells():
    a = 1.0
    pos = np.array([[i, j, k] for i in range(3) for j in range(3) for k in range(3)], float) * a
    box = np.full(3, 3 * a)
    g = nl.brute_force(pos, box, 1.1)
    assert np.all(np.diff(g.recv_off) == 6)
    g = nl.brute_force(pos, box, 1.5)
    assert np.all(np.diff(g.recv_off) == 18)
    g = nl.brute_force(pos, box, 1.8)
    assert np.all(np.diff(g.recv_off) == 26)


def test_cutoff_is_strict():
    box = np.full(3, 50.0)
    pos = np.array([[1.0, 1.0, 1.0], [3.0, 1.0, 1.0]])       # distance exactly 2
    assert nl.brute_force(pos, box, 2.0).n_edges == 0
    assert nl.brute_force(pos, box, np.nextafter(2.0, 3.0)).n_edges == 2


def test_mirror_and_order():
    st = synth.workload("n64_diamond").structure
    g = nl.brute_force(st.pos, st.box, 6.0)
    e = np.arange(g.n_edges)
    assert np.array_equal(g.mirror[g.mirror], e)
    assert np.array_equal(g.recv[g.mirror], g.send)
    assert np.array_equal(g.shift[g.mirror], -g.shift)
    assert np.array_equal(g.r[g.mirror], -g.r)          # IEEE negation symmetry of the definition
    key = np.stack([g.recv, g.send, g.shift[:, 0], g.shift[:, 1], g.shift[:, 2]], 1)
    assert all(tuple(key[i]) < tuple(key[i + 1]) for i in range(g.n_edges - 1))
    assert np.array_equal(g.vec, g.r.astype(np.float32))
    assert np.all(np.sqrt(np.sum(g.r ** 2, axis=1)) < 6.0)


def test_ternary_cell_degree():
    w = synth.workload("ternary_n2000")
    st = w.structure
    g = nl.cell_list(st.pos, st.box, 6.0)
    deg = np.diff(g.recv_off)
    # mean degree of a homogeneous cell: density * (4/3) pi rc^3
    assert abs(deg.mean() - 0.08 * 4.0 / 3.0 * math.pi * 216.0) < 2.0
    assert deg.max() > deg.min()                         # ragged
    d = st.pos[:, None, :] - st.pos[None, :, :]
    d -= st.box[0] * np.round(d / st.box[0])
    dist = np.sqrt((d ** 2).sum(-1)) + np.eye(st.pos.shape[0]) * 99
    assert dist.min() >= 1.7
