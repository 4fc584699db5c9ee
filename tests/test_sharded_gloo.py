"""Receiver-range sharding, the exchange scheme of mp_energy_forces_sharded, with two gloo
ranks on CPU against the single-rank result (float64 oracle arithmetic; the library's kernels
need a GPU and are covered by tests/test_gpu_sharded.py).

Each rank takes the edges of a contiguous receiver range (edgewise balanced,
receiver_ranges of the binding), computes each layer's receiver sums from its edges and adds
them over the ranks (every receiver's row comes from one rank), updates all node features,
computes in the backward the layer's input gradient from its edges (the residual part on rank
0 only) and adds it over the ranks, and finally adds the per-edge gradients placed at their
edges of the whole graph; the energy, forces and virial then follow on every rank."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth
from oracle import model as om
from oracle import nl as onl
import edge_message_passing_b200 as emp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _allreduce(a):
    t = torch.from_numpy(np.ascontiguousarray(a))
    dist.all_reduce(t)
    return t.numpy()


def _sharded_oracle(w, g, rank, world):
    spec, W, st = w.spec, w.weights, w.structure
    n = st.pos.shape[0]
    a, b = emp.receiver_ranges(g.recv_off, world)[rank]
    e0, e1 = int(g.recv_off[a]), int(g.recv_off[b])
    recv, send, r = g.recv[e0:e1], g.send[e0:e1], g.r[e0:e1]
    pair = np.zeros(e1 - e0, dtype=np.int64)
    geom = om.edge_geometry(r) if e1 > e0 else None
    xs, aggs = [om.initial_features(spec, W, st.species)], []
    for t in range(spec.n_layers):
        agg = om.conv_forward(spec, W, t, xs[-1], recv, send, geom, pair, n) if e1 > e0 else np.zeros_like(xs[-1])
        agg = _allreduce(agg)
        aggs.append(agg)
        xs.append(xs[-1] + om.gate(agg) if spec.gated else agg)
    e_atom, z = om.readout(W, xs[-1])
    g_h = np.zeros_like(xs[-1])
    g_h[:, 0, :] = (W["ro_w"].astype(np.float64) * om.dsilu(z)) @ W["ro_W"].astype(np.float64)
    g_r = np.zeros((e1 - e0, 3))
    gcur = g_h
    for t in reversed(range(spec.n_layers)):
        g_agg = om.gate_backward(aggs[t], gcur) if spec.gated else gcur
        g_next = gcur.copy() if (spec.gated and rank == 0) else np.zeros_like(gcur)
        if e1 > e0:
            gx, gr = om.conv_backward(spec, W, t, xs[t], g_agg, recv, send, geom, pair, n, need_gx=t > 0)
            g_r += gr
            if gx is not None:
                g_next += gx
        gcur = _allreduce(g_next) if t > 0 else g_next
    g_all = np.zeros((g.recv.shape[0], 3))
    g_all[e0:e1] = g_r
    g_all = _allreduce(g_all)
    F = np.zeros((n, 3))
    np.add.at(F, g.recv, g_all)
    np.subtract.at(F, g.send, g_all)
    return float(np.sum(e_atom)), F, -np.einsum("ea,eb->ab", g.r, g_all)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    w = synth.small_workload(ncell=1, C=16, n_layers=3, gated=True, sigma=0.1)
    g = onl.brute_force(w.structure.pos, w.structure.box, w.spec.cutoff)
    out[rank] = _sharded_oracle(w, g, rank, world)
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_step_equals_the_single_rank_step(world):
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    w = synth.small_workload(ncell=1, C=16, n_layers=3, gated=True, sigma=0.1)
    st = w.structure
    g = onl.brute_force(st.pos, st.box, w.spec.cutoff)
    ref = om.energy_forces(w.spec, w.weights, st.species, g.recv, g.send, g.r, st.pos.shape[0])
    for r in range(world):
        E, F, V = out[r]
        assert abs(E - ref.energy) <= 1e-12 * abs(ref.energy)
        assert np.abs(F - ref.forces).max() <= 1e-10 * np.abs(ref.forces).max()
        assert np.abs(V - ref.virial).max() <= 1e-10 * np.abs(ref.virial).max()


def test_receiver_ranges_cover_every_atom_once_and_balance_edges():
    rng = np.random.default_rng(0)
    deg = rng.integers(0, 200, 1000)
    deg[100:140] = 0                                   # isolated atoms
    ro = np.concatenate([[0], np.cumsum(deg)])
    for world in (1, 2, 3, 8):
        rr = emp.receiver_ranges(ro, world)
        assert rr[0][0] == 0 and rr[-1][1] == 1000 and all(rr[k][1] == rr[k + 1][0] for k in range(world - 1))
        edges = [ro[b] - ro[a] for a, b in rr]
        assert sum(edges) == ro[-1] and max(edges) - min(edges) <= 2 * deg.max()
    assert emp.receiver_ranges(np.zeros(5, dtype=np.int64), 2) in ([(0, 0), (0, 4)], [(0, 4), (4, 4)])
