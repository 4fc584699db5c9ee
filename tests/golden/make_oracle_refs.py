"""Write oracle reference results for the full-size workloads (float64, CPU).

    python tests/golden/make_oracle_refs.py [n4096_diamond ternary_n2000 ...]

Calls only oracle/ (and the shared seeded inputs in synth/).  The GPU parity tests
compare the CUDA path with these stored values, because the float64 oracle takes
minutes at these sizes.  Output: tests/golden/<workload>_oracle.npz with energy,
per-atom energies, forces and virial.
"""
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import synth  # noqa: E402
from oracle import model as omodel  # noqa: E402
from oracle import nl as onl  # noqa: E402


def make(name: str) -> str:
    w = synth.workload(name)
    st = w.structure
    t0 = time.time()
    g = onl.cell_list(st.pos, st.box, w.spec.cutoff)
    res = omodel.energy_forces(w.spec, w.weights, st.species, g.recv, g.send, g.r, st.pos.shape[0])
    out = os.path.join(HERE, f"{name}_oracle.npz")
    np.savez_compressed(out, energy=np.float64(res.energy), atom_energy=res.atom_energy, forces=res.forces,
                        virial=res.virial, n_edges=np.int64(g.n_edges))
    print(f"{name}: E={res.energy:.12g} edges={g.n_edges} in {time.time() - t0:.0f} s -> {out}")
    return out


if __name__ == "__main__":
    for n in (sys.argv[1:] or ["n4096_diamond"]):
        make(n)
