"""Plain, slow, float64 CPU oracle for the equivariant edge message-passing path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never calls it, and the two share no code: no kernels, headers, helpers,
constant tables or pre/post-processing.  The only shared module is ``synth``,
which draws seeded inputs and holds none of the method's arithmetic.

What it computes follows the subject pages (deepmd-kit PR "first-order SO(2)
input-gradient path" for the DPA4-Neo SO(2) convolution with 8192-edge cohorts;
deepmd-kit PR #6108 "radial head fold") and the model definition of the seeded
workloads: cell-list neighbour list, Bessel radial basis with polynomial
envelope and radial MLP, Wigner-D rotation of neighbour irreps (lmax = 3) into
the edge frame, per-m SO(2) channel mixing, rotation back, normalised sum onto
receivers, gated residual updates, per-atom readout energy, and forces and
virial by a hand-written reverse mode.

Modules
  nl     neighbour list: brute force (the definition) and an independent cell list
  sh     real spherical harmonics, Wigner-D by fitting, rotation generators
  model  radial basis/MLP, SO(2) convolution, gate, readout, energy, forces
  chain  the radial projection chain, unfolded and folded

Every function is pinned by ``tests/test_oracle_*.py`` to something other than
itself (closed forms, invariants, library special cases, brute force, finite
differences).  Parity unpinned: absolute energies and forces of the seeded
workloads (the pages print none); they are pinned only through invariances,
finite differences and the special cases listed in the tests.
"""
