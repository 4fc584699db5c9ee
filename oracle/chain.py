"""Radial projection chain, unfolded and folded (float64).

Test infrastructure only (see ``oracle/__init__``).

Follows deepmd-kit PR #6108 ("radial head fold"), section "What": the raw basis
x (E,4,32) is up-projected per degree to (E,4,64) and the flattened (E,256)
result is multiplied by a (256,25) degree-mixing matrix; because both weights are
frozen, their product W_eff (128x25) can be formed once, giving
kc = x_flat @ W_eff, plus the l = 0 slice projection (E,32) @ (32,64), which is
the only up-projected row the rest of the model consumes.  No biases (the page
states none).  The input gradient is the transpose map.
"""
from __future__ import annotations

import numpy as np


def unfolded_forward(x, U, M):
    """x [E,4,32], U [4,32,64] (in,out), M [256,25] -> (kc [E,25], y0 [E,64])."""
    x = np.asarray(x, dtype=np.float64)
    up = np.einsum("elk,lkh->elh", x, U.astype(np.float64))     # [E,4,64]
    kc = up.reshape(x.shape[0], 256) @ M.astype(np.float64)
    return kc, up[:, 0, :]


def unfolded_backward(g_kc, g_y0, U, M):
    """Input gradient of :func:`unfolded_forward` -> g_x [E,4,32]."""
    g_up = (np.asarray(g_kc, dtype=np.float64) @ M.astype(np.float64).T).reshape(-1, 4, 64)
    g_up[:, 0, :] += g_y0
    return np.einsum("elh,lkh->elk", g_up, U.astype(np.float64))


def fold(U, M):
    """W_eff = vstack_l(U_l @ M_l), M_l the l-th 64-row slab of M -> [128,25]."""
    U = U.astype(np.float64)
    M = M.astype(np.float64)
    return np.concatenate([U[l] @ M[64 * l:64 * (l + 1)] for l in range(4)], axis=0)


def folded_forward(x, W_eff, U0):
    x = np.asarray(x, dtype=np.float64)
    E = x.shape[0]
    return x.reshape(E, 128) @ W_eff, x[:, 0, :] @ U0.astype(np.float64)


def folded_backward(g_kc, g_y0, W_eff, U0):
    g = np.asarray(g_kc, dtype=np.float64) @ W_eff.T                 # [E,128]
    g = g.reshape(-1, 4, 32)
    g[:, 0, :] += np.asarray(g_y0, dtype=np.float64) @ U0.astype(np.float64).T
    return g


def unfolded_flops(E: int) -> int:
    """Forward flops of the two-step chain: up-projection + degree mixing."""
    return 2 * E * (4 * 32 * 64 + 256 * 25)


def unfolded_intermediate_bytes(E: int) -> int:
    """FP32 bytes of the (E,4,64) up-projected intermediate."""
    return 4 * E * 4 * 64
