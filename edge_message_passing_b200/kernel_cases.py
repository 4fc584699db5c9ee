"""Small, self-contained invocations of single kernel families, for profilers.

    python -m edge_message_passing_b200.kernel_cases <case> [--iters K]

Cases (seeded synthetic inputs, sizes chosen so that buffers exceed the 126 MB L2
while the device footprint stays at a few GB):
  so2      one 8192-row cohort of the SO(2) mixing (C = 128), forward map
  so2t     the same, transpose (adjoint) map
  step512  one energy + force step of the N=512 diamond model (C = 128, 3 layers)
  step4096 one energy + force step of the N=4096 diamond model (the benchmark workload;
           for one-pass launch lists only: its workspace is several GB)
  chain    the folded radial chain at E = 647170, forward + input gradient
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def main() -> int:
    import torch

    import edge_message_passing_b200 as emp
    import synth

    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["so2", "so2t", "step512", "step4096", "chain"])
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args()
    torch.cuda.set_device(0)
    if a.case in ("so2", "so2t"):
        spec = synth.ModelSpec(C=128, n_layers=1)
        model = emp.Model(spec, synth.draw_weights(spec, np.random.default_rng(0)))
        X = torch.randn((8192, 16 * 128), device="cuda")
        for _ in range(a.iters):
            emp.mp_so2_mix(model, 0, X, transpose=a.case == "so2t")
    elif a.case in ("step512", "step4096"):
        w = synth.workload("n512_diamond" if a.case == "step512" else "n4096_diamond")
        model = emp.Model(w.spec, w.weights)
        g = emp.nl_build(torch.from_numpy(w.structure.pos).cuda(), w.structure.box, w.spec.cutoff)
        sp = torch.from_numpy(w.structure.species).cuda()
        for _ in range(a.iters):
            emp.mp_energy_forces(model, g, sp)
    else:
        ci = synth.chain_inputs()
        ch = emp.Chain(ci.U, ci.M)
        x, gk, gy = (torch.from_numpy(t).cuda() for t in (ci.x, ci.g_kc, ci.g_y0))
        for _ in range(a.iters):
            emp.mp_radial_chain(ch, x, gk, gy)
    torch.cuda.synchronize()
    err = emp.last_device_error()
    print(f"{a.case}: done, device error word {err}")
    return 0 if err == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
