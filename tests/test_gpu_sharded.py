"""mp_energy_forces_sharded on the GPU.

* One rank over NCCL: the rank's view is the whole graph and the sums over ranks are
  identities, so the result equals mp_energy_forces bit for bit.
* Two ranks sharing this GPU, the sums over ranks through gloo on host copies (between kernel
  launches, so no kernel of one rank waits on another's): both ranks return the same energy,
  forces and virial, within the standard tolerances of the stored float64 oracle result of
  the N=512 diamond (the layer between the first and the last runs over cohorts, so every
  exchange of the scheme is exercised).
Each case runs in child processes (spawned), so no process group outlives it."""
import os
import socket

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, backend, port, name, out):
    import datetime
    import torch.distributed as dist
    import edge_message_passing_b200 as emp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group(backend, rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    w = synth.workload(name)
    st = w.structure
    g = emp.nl_build(torch.from_numpy(st.pos).cuda(), st.box, w.spec.cutoff)
    model = emp.Model(w.spec, w.weights)
    sp = torch.from_numpy(st.species).cuda()
    e, f, v = emp.mp_energy_forces_sharded(model, g, sp, rank, world, virial=True)
    res = [e.cpu().numpy(), f.cpu().numpy(), v.cpu().numpy()]
    if world == 1:
        e1, f1, v1, _ = emp.mp_energy_forces(model, g, sp, virial=True)
        res.append(bool(torch.equal(e, e1) and torch.equal(f, f1) and torch.equal(v, v1)))
    res.append(emp.last_device_error())
    out[rank] = res
    dist.barrier()
    dist.destroy_process_group()


def _spawn(world, backend, name):
    import torch.multiprocessing as mp
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, backend, _free_port(), name, out), nprocs=world, join=True)
    return dict(out)


def test_one_rank_over_nccl_equals_the_unsharded_call():
    out = _spawn(1, "nccl", "n512_diamond")
    assert out[0][3] is True and out[0][4] == 0


def test_two_ranks_on_one_gpu_over_gloo():
    out = _spawn(2, "gloo", "n512_diamond")
    ref = np.load(os.path.join(GOLD, "n512_diamond_oracle.npz"))
    for r in (0, 1):
        E, F, V, err = out[r]
        assert err == 0
        assert abs(float(E[0]) - float(ref["energy"])) <= 1e-5 * abs(float(ref["energy"]))
        assert np.abs(F - ref["forces"]).max() <= 1e-4 * np.abs(ref["forces"]).max()
        assert np.abs(V - ref["virial"]).max() <= 1e-4 * np.abs(ref["virial"]).max()
    assert np.array_equal(out[0][1], out[1][1]) and np.array_equal(out[0][0], out[1][0])
