"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This module only draws random numbers and lays out lattices.  It holds none of
the message-passing arithmetic: no radial basis, no spherical harmonics, no
rotations, no mixing.  Both the float64 oracle and the CUDA library consume the
arrays it returns, so the two never generate inputs on their own.

Workloads (stand-ins for the structures measured on the pages, which are not
available here):

* ``n64_diamond``    2x2x2 conventional diamond cells, a = 3.567 A, seed 0,
                     C = 64, one interaction layer, no gate.
* ``n512_diamond``   4x4x4 cells, seed 1, C = 128, three gated residual layers,
                     virial reported.
* ``n4096_diamond``  8x8x8 cells, seed 2, C = 128, three gated residual layers,
                     8192-edge receiver-sorted cohorts.
* ``radial_chain``   the radial projection chain alone: x ~ N(0,1) of shape
                     [647170, 4, 32], seed 3.
* ``ternary_n2000``  2000 atoms of three species (400:400:1200) placed by
                     random sequential addition in a periodic cube of density
                     0.08 / A^3 with minimum image distance 1.7 A, seed 4,
                     per-species-pair radial networks.

Random stream convention: ``numpy.random.default_rng(seed)`` (PCG64).  Positions
(or the chain's x) are drawn first, then the weights in the declaration order of
:func:`weight_shapes`, each as float64 normals rounded to float32 so that the
oracle (float64 arithmetic) and the GPU (float32) see identical values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Tuple

import numpy as np

DIAMOND_A = 3.567  # conventional cubic cell edge of diamond carbon, angstrom
# fractional coordinates of the 8-atom conventional diamond cell
DIAMOND_BASIS = np.array(
    [
        [0.00, 0.00, 0.00],
        [0.00, 0.50, 0.50],
        [0.50, 0.00, 0.50],
        [0.50, 0.50, 0.00],
        [0.25, 0.25, 0.25],
        [0.25, 0.75, 0.75],
        [0.75, 0.25, 0.75],
        [0.75, 0.75, 0.25],
    ],
    dtype=np.float64,
)


@dataclasses.dataclass(frozen=True)
class ModelSpec:
    """Hyper-parameters of the interatomic potential (one interaction block type)."""

    C: int                      # channels per irrep component
    n_layers: int               # stacked interaction layers
    n_species: int = 1
    lmax: int = 3               # fixed: 16 = (lmax+1)^2 components
    n_basis: int = 8            # Bessel functions
    radial_hidden: int = 64     # radial MLP width
    readout_hidden: int = 0     # 0 -> C
    gated: bool = False         # residual + SiLU gate between layers
    pair_radial: bool = False   # one radial MLP per unordered species pair
    cutoff: float = 6.0
    env_p: int = 6              # polynomial envelope exponent
    avg_degree: float = 158.0   # aggregation normaliser
    cohort_edges: int = 8192    # receiver-sorted edge cohort size

    @property
    def H_ro(self) -> int:
        return self.readout_hidden if self.readout_hidden > 0 else self.C

    @property
    def n_pairs(self) -> int:
        s = self.n_species
        return s * (s + 1) // 2 if self.pair_radial else 1


@dataclasses.dataclass
class Structure:
    pos: np.ndarray        # [N,3] float64, not wrapped into the box
    box: np.ndarray        # [3] float64, orthorhombic periodic box edges
    species: np.ndarray    # [N] int32


def weight_shapes(spec: ModelSpec) -> List[Tuple[str, Tuple[int, ...], int]]:
    """Declaration order of the weights: (name, shape, fan_in).

    All linear maps are bias-free and stored (out, in).
    """
    C, H = spec.C, spec.radial_hidden
    out: List[Tuple[str, Tuple[int, ...], int]] = [("emb", (spec.n_species, C), spec.n_species)]
    for t in range(spec.n_layers):
        for p in range(spec.n_pairs):
            out.append((f"rad{t}_{p}_W1", (H, spec.n_basis), spec.n_basis))
            out.append((f"rad{t}_{p}_W2", (H, H), H))
            out.append((f"rad{t}_{p}_W3", (4 * C, H), H))
        out.append((f"so2_{t}_W0", (4 * C, 4 * C), 4 * C))
        for m in (1, 2, 3):
            k = (4 - m) * C
            out.append((f"so2_{t}_Wr{m}", (k, k), 2 * k))
            out.append((f"so2_{t}_Wi{m}", (k, k), 2 * k))
    out.append(("ro_W", (spec.H_ro, C), C))
    out.append(("ro_w", (spec.H_ro,), spec.H_ro))
    return out


def draw_weights(spec: ModelSpec, rng: np.random.Generator) -> Dict[str, np.ndarray]:
    """Weights ~ N(0, 1/fan_in), float32 values (returned as float32 arrays)."""
    w: Dict[str, np.ndarray] = {}
    for name, shape, fan_in in weight_shapes(spec):
        w[name] = (rng.standard_normal(shape) / math.sqrt(fan_in)).astype(np.float32)
    return w


def diamond(ncell: int, sigma: float, rng: np.random.Generator) -> Structure:
    """ncell^3 conventional diamond cells with iid N(0, sigma^2) noise per component."""
    cells = np.array([(i, j, k) for i in range(ncell) for j in range(ncell) for k in range(ncell)],
                     dtype=np.float64)
    frac = (cells[:, None, :] + DIAMOND_BASIS[None, :, :]).reshape(-1, 3)
    pos = frac * DIAMOND_A
    pos = pos + rng.normal(0.0, sigma, size=pos.shape)
    n = pos.shape[0]
    box = np.full(3, ncell * DIAMOND_A)
    return Structure(pos=pos, box=box, species=np.zeros(n, dtype=np.int32))


def random_cell(n: int, density: float, dmin: float, counts: Tuple[int, ...],
                rng: np.random.Generator) -> Structure:
    """Random sequential addition in a periodic cube; species in index blocks."""
    L = (n / density) ** (1.0 / 3.0)
    pos = np.empty((n, 3))
    k = 0
    while k < n:
        cand = rng.uniform(0.0, L, size=3)
        if k:
            d = pos[:k] - cand
            d -= L * np.round(d / L)
            if np.min(np.einsum("ij,ij->i", d, d)) < dmin * dmin:
                continue
        pos[k] = cand
        k += 1
    species = np.concatenate([np.full(c, s, dtype=np.int32) for s, c in enumerate(counts)])
    assert species.shape[0] == n
    return Structure(pos=pos, box=np.full(3, L), species=species)


@dataclasses.dataclass
class Workload:
    name: str
    spec: ModelSpec
    structure: Structure
    weights: Dict[str, np.ndarray]


def workload(name: str) -> Workload:
    """The named seeded workload (structure + model + weights)."""
    if name == "n64_diamond":
        rng = np.random.default_rng(0)
        st = diamond(2, 0.02, rng)
        spec = ModelSpec(C=64, n_layers=1, gated=False)
    elif name == "n512_diamond":
        rng = np.random.default_rng(1)
        st = diamond(4, 0.02, rng)
        spec = ModelSpec(C=128, n_layers=3, gated=True)
    elif name == "n4096_diamond":
        rng = np.random.default_rng(2)
        st = diamond(8, 0.02, rng)
        spec = ModelSpec(C=128, n_layers=3, gated=True)
    elif name == "ternary_n2000":
        rng = np.random.default_rng(4)
        st = random_cell(2000, 0.08, 1.7, (400, 400, 1200), rng)
        spec = ModelSpec(C=128, n_layers=3, n_species=3, gated=True, pair_radial=True)
    else:
        raise KeyError(name)
    return Workload(name, spec, st, draw_weights(spec, rng))


def small_workload(ncell: int = 1, C: int = 16, n_layers: int = 2, gated: bool = True,
                   n_species: int = 1, pair_radial: bool = False, cutoff: float = 6.0,
                   sigma: float = 0.05, seed: int = 7, cohort_edges: int = 8192) -> Workload:
    """A tiny diamond workload for fast tests (same recipe, smaller sizes)."""
    rng = np.random.default_rng(seed)
    st = diamond(ncell, sigma, rng)
    if n_species > 1:
        st.species = (np.arange(st.pos.shape[0]) % n_species).astype(np.int32)
    spec = ModelSpec(C=C, n_layers=n_layers, gated=gated, n_species=n_species,
                     pair_radial=pair_radial, cutoff=cutoff, cohort_edges=cohort_edges)
    return Workload(f"small_c{C}_l{n_layers}", spec, st, draw_weights(spec, rng))


# ----------------------------------------------------------------- radial chain
CHAIN_E = 647170


@dataclasses.dataclass
class ChainInputs:
    x: np.ndarray      # [E,4,32] float32
    U: np.ndarray      # [4,32,64] float32: per-degree up-projection (in, out)
    M: np.ndarray      # [256,25] float32: degree mixing (in, out)
    g_kc: np.ndarray   # [E,25] float32 upstream gradient
    g_y0: np.ndarray   # [E,64] float32 upstream gradient


def chain_inputs(E: int = CHAIN_E, seed: int = 3) -> ChainInputs:
    """x ~ N(0,1); U ~ N(0,1/32); M ~ N(0,1/256); upstream gradients ~ N(0,1)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((E, 4, 32), dtype=np.float32)
    U = (rng.standard_normal((4, 32, 64)) / math.sqrt(32)).astype(np.float32)
    M = (rng.standard_normal((256, 25)) / math.sqrt(256)).astype(np.float32)
    g_kc = rng.standard_normal((E, 25), dtype=np.float32)
    g_y0 = rng.standard_normal((E, 64), dtype=np.float32)
    return ChainInputs(x, U, M, g_kc, g_y0)


def random_features(n: int, C: int, seed: int) -> np.ndarray:
    """Full node features [n,16,C] (all degrees non-zero), float32 ~ N(0,1)."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal((n, 16, C), dtype=np.float32)
