"""Neighbour list oracle (test infrastructure only; see ``oracle/__init__``).

Definition (the bit-exact cell-list neighbour list of the SO(2) message-passing
step; deepmd-kit PR "first-order SO(2) input-gradient path", workload section:
N64 diamond, E ~ 10114):

  an edge is a triple (i, j, S), i the receiver, j the sender, S an integer
  image shift, such that with r = (x_j - x_i) + S * L evaluated per Cartesian
  component in float64 (one rounding for the difference, one for the product
  S*L, one for the sum) and d2 = (rx*rx + ry*ry) + rz*rz (separate roundings,
  no fused multiply-add), d2 < rc*rc strictly; (i, i, 0) is excluded.

Edges are ordered by receiver i, then sender j, then S lexicographically.
``recv_off`` is the CSR offset array over receivers; ``mirror[e]`` is the index
of (j, i, -S).  ``vec`` is r rounded to float32.
"""
from __future__ import annotations

import dataclasses
import itertools
import math

import numpy as np


@dataclasses.dataclass
class Graph:
    recv: np.ndarray      # [E] int32
    send: np.ndarray      # [E] int32
    shift: np.ndarray     # [E,3] int32
    r: np.ndarray         # [E,3] float64  (the definition's r)
    vec: np.ndarray       # [E,3] float32  (r rounded to nearest)
    recv_off: np.ndarray  # [N+1] int64
    mirror: np.ndarray    # [E] int64

    @property
    def n_edges(self) -> int:
        return int(self.recv.shape[0])


def _shift_range(pos: np.ndarray, box: np.ndarray, rc: float) -> np.ndarray:
    """Largest |S_d| that can give |r| < rc: |S_d L_d| < rc + span_d."""
    span = pos.max(axis=0) - pos.min(axis=0)
    return np.array([int(math.floor((rc + span[d]) / box[d])) for d in range(3)])


def _finish(pos, box, rc, recv, send, shift) -> Graph:
    n = pos.shape[0]
    order = np.lexsort((shift[:, 2], shift[:, 1], shift[:, 0], send, recv))
    recv, send, shift = recv[order], send[order], shift[order]
    r = (pos[send] - pos[recv]) + shift * box[None, :]
    counts = np.bincount(recv, minlength=n)
    recv_off = np.zeros(n + 1, dtype=np.int64)
    recv_off[1:] = np.cumsum(counts)
    key = {}
    for e in range(recv.shape[0]):
        key[(int(recv[e]), int(send[e]), int(shift[e, 0]), int(shift[e, 1]), int(shift[e, 2]))] = e
    mirror = np.array([key[(int(send[e]), int(recv[e]), -int(shift[e, 0]), -int(shift[e, 1]),
                            -int(shift[e, 2]))] for e in range(recv.shape[0])], dtype=np.int64)
    return Graph(recv=recv.astype(np.int32), send=send.astype(np.int32),
                 shift=shift.astype(np.int32), r=r, vec=r.astype(np.float32),
                 recv_off=recv_off, mirror=mirror)


def _within(pos, box, rc2, i_idx, j_idx, S):
    """The definition's test for arrays of candidate (i, j) with one shift S."""
    rx = (pos[j_idx, 0] - pos[i_idx, 0]) + S[0] * box[0]
    ry = (pos[j_idx, 1] - pos[i_idx, 1]) + S[1] * box[1]
    rz = (pos[j_idx, 2] - pos[i_idx, 2]) + S[2] * box[2]
    d2 = (rx * rx + ry * ry) + rz * rz
    return d2 < rc2


def brute_force(pos: np.ndarray, box: np.ndarray, rc: float) -> Graph:
    """All (i, j, S) over a shift range that provably contains every edge."""
    pos = np.asarray(pos, dtype=np.float64)
    box = np.asarray(box, dtype=np.float64)
    n = pos.shape[0]
    rc2 = rc * rc
    k = _shift_range(pos, box, rc)
    R, Sd, Jd = [], [], []
    ii, jj = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    ii = ii.ravel()
    jj = jj.ravel()
    for S in itertools.product(*(range(-k[d], k[d] + 1) for d in range(3))):
        S = np.array(S, dtype=np.float64)
        ok = _within(pos, box, rc2, ii, jj, S)
        if not S.any():
            ok &= ii != jj
        sel = np.nonzero(ok)[0]
        R.append(ii[sel])
        Jd.append(jj[sel])
        Sd.append(np.repeat(S[None, :].astype(np.int64), sel.shape[0], axis=0))
    recv = np.concatenate(R)
    send = np.concatenate(Jd)
    shift = np.concatenate(Sd)
    return _finish(pos, box, rc, recv, send, shift)


def cell_list(pos: np.ndarray, box: np.ndarray, rc: float) -> Graph:
    """Independent second path: bins atoms (wrapped) into cells of edge >= rc and
    enumerates the periodic 3^3 (or wider) stencil.  Candidate (j, S) pairs are
    then tested with the same definition; must equal :func:`brute_force`."""
    pos = np.asarray(pos, dtype=np.float64)
    box = np.asarray(box, dtype=np.float64)
    n = pos.shape[0]
    rc2 = rc * rc
    wrap = np.floor(pos / box).astype(np.int64)          # image of each raw position
    frac = pos / box - wrap                                # in [0, 1)
    nc = np.maximum(1, np.floor(box / (rc * (1 + 1e-9))).astype(np.int64))
    cell = np.minimum((frac * nc).astype(np.int64), nc - 1)
    s = np.ceil(rc * (1 + 1e-9) / (box / nc)).astype(np.int64)
    members = {}
    for a in range(n):
        members.setdefault(tuple(cell[a]), []).append(a)
    R, J, S_all = [], [], []
    for i in range(n):
        ci = cell[i]
        for d in itertools.product(*(range(-s[q], s[q] + 1) for q in range(3))):
            u = ci + np.array(d)
            T = np.floor_divide(u, nc)
            c = tuple(u - T * nc)
            js = members.get(c)
            if not js:
                continue
            js = np.array(js)
            S = T[None, :] - wrap[js] + wrap[i][None, :]      # raw-frame shift
            Sf = S.astype(np.float64)
            ii = np.full(js.shape[0], i)
            rx = (pos[js, 0] - pos[ii, 0]) + Sf[:, 0] * box[0]
            ry = (pos[js, 1] - pos[ii, 1]) + Sf[:, 1] * box[1]
            rz = (pos[js, 2] - pos[ii, 2]) + Sf[:, 2] * box[2]
            keep = ((rx * rx + ry * ry) + rz * rz) < rc2
            keep &= ~((js == i) & ~S.any(axis=1))
            R.extend([i] * int(keep.sum()))
            J.extend(js[keep].tolist())
            S_all.extend(S[keep].tolist())
    return _finish(pos, box, rc, np.array(R), np.array(J), np.array(S_all, dtype=np.int64).reshape(-1, 3))
