"""Weight gradients of the energy (float64): dE/dW for every weight of the model.

Test infrastructure only (see ``oracle/__init__``).

The pages keep the training path (weight gradients) on the old code path ("first-order
SO(2) input-gradient path", section "Implementation and scope": only the input gradient
is moved); this module is the plain reverse mode of the model of ``oracle.model`` with
respect to its weights, written out layer by layer:

  readout   e_i = w_o . SiLU(z_i), z_i = W_ro h_i[0]:
            dE/dw_o = sum_i SiLU(z_i);  dE/dW_ro = sum_i (w_o (.) SiLU'(z_i)) (x) h_i[0]
  SO(2)     y0 = W0 x~0; y+ = Wr x+ - Wi x-, y- = Wi x+ + Wr x- (per edge), g_y = D g_m:
            dE/dW0 = sum_e g_y0 (x) x~0;  dE/dWr = sum_e (g_y+ (x) x~+ + g_y- (x) x~-);
            dE/dWi = sum_e (g_y- (x) x~+ - g_y+ (x) x~-)
  radial    R = W3 h2, h2 = SiLU(W2 h1), h1 = SiLU(W1 e):  dE/dW3 = sum_e g_R (x) h2,
            dE/dW2 = sum_e g_z2 (x) h1, dE/dW1 = sum_e g_z1 (x) e
  embedding x_0[i][l=0] = emb[species_i]:  dE/demb[s] = sum_{i: species_i = s} dE/dx_0[i][0]

Energy only: gradients of force terms (mixed second derivatives) are not part of it.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from . import model as om
from . import sh


def energy_weight_grad(spec, W, species, recv, send, r, n_atoms) -> (float, Dict[str, np.ndarray]):
    """(E, {weight name: dE/dweight}) for the weights of synth.weight_shapes(spec)."""
    species = np.asarray(species)
    recv = np.asarray(recv)
    send = np.asarray(send)
    E_n = r.shape[0]
    C = spec.C
    pair = om.pair_index(species[recv], species[send], spec.n_species) if spec.pair_radial \
        else np.zeros(E_n, dtype=np.int64)
    geom = om.edge_geometry(r)
    e_basis = om.bessel_basis(geom.d, spec.cutoff, spec.n_basis, spec.env_p)
    grads = {k: np.zeros(np.shape(v)) for k, v in W.items()}
    # ---- forward, keeping what the weight gradients need
    xs = [om.initial_features(spec, W, species)]
    aggs, keep = [], []
    for t in range(spec.n_layers):
        R, caches = om.radial_of_edges(spec, W, t, geom.d, pair)
        u = om.rotate(geom.Dl, xs[-1][send])
        Rx = om._expand_R(R)
        xt = Rx * u
        y = om.so2_apply(xt, W, t)
        msg = om.rotate(geom.Dl, y, transpose=True)
        agg = np.zeros_like(xs[-1])
        np.add.at(agg, recv, msg)
        agg /= spec.avg_degree
        aggs.append(agg)
        keep.append((R, caches, u, Rx, xt))
        xs.append(xs[-1] + om.gate(agg) if spec.gated else agg)
    h = xs[-1]
    ro_W = W["ro_W"].astype(np.float64)
    ro_w = W["ro_w"].astype(np.float64)
    z = h[:, 0, :] @ ro_W.T
    energy = float(np.sum(om.silu(z) @ ro_w))
    # ---- readout
    grads["ro_w"] = om.silu(z).sum(axis=0)
    g_z = ro_w[None, :] * om.dsilu(z)
    grads["ro_W"] = g_z.T @ h[:, 0, :]
    g = np.zeros_like(h)
    g[:, 0, :] = g_z @ ro_W
    # ---- layers in reverse
    for t in reversed(range(spec.n_layers)):
        R, caches, u, Rx, xt = keep[t]
        g_agg = om.gate_backward(aggs[t], g) if spec.gated else g
        g_next = g.copy() if spec.gated else np.zeros_like(g)
        g_m = g_agg[recv] / spec.avg_degree
        g_y = om.rotate(geom.Dl, g_m)
        # SO(2) weights
        i0 = om.m_block_index(0)
        grads[f"so2_{t}_W0"] = g_y[:, i0, :].reshape(E_n, -1).T @ xt[:, i0, :].reshape(E_n, -1)
        for m in (1, 2, 3):
            ip, im = om.m_block_index(m), om.m_block_index(-m)
            Gp, Gm = g_y[:, ip, :].reshape(E_n, -1), g_y[:, im, :].reshape(E_n, -1)
            Xp, Xm = xt[:, ip, :].reshape(E_n, -1), xt[:, im, :].reshape(E_n, -1)
            grads[f"so2_{t}_Wr{m}"] = Gp.T @ Xp + Gm.T @ Xm
            grads[f"so2_{t}_Wi{m}"] = Gm.T @ Xp - Gp.T @ Xm
        # radial weights
        g_xt = om.so2_apply(g_y, W, t, transpose=True)
        g_R = np.zeros((E_n, 4, C))
        for l in range(4):
            b = sh.block(l)
            g_R[:, l, :] = np.sum(g_xt[:, b, :] * u[:, b, :], axis=1)
        gRf = g_R.reshape(E_n, 4 * C)
        for p, (z1, h1, z2, h2) in caches.items():
            sel = pair == p
            W2 = W[f"rad{t}_{p}_W2"].astype(np.float64)
            W3 = W[f"rad{t}_{p}_W3"].astype(np.float64)
            grads[f"rad{t}_{p}_W3"] = gRf[sel].T @ h2
            g_z2 = (gRf[sel] @ W3) * om.dsilu(z2)
            grads[f"rad{t}_{p}_W2"] = g_z2.T @ h1
            g_z1 = (g_z2 @ W2) * om.dsilu(z1)
            grads[f"rad{t}_{p}_W1"] = g_z1.T @ e_basis[sel]
        # input gradient of the layer
        g_xs = om.rotate(geom.Dl, Rx * g_xt, transpose=True)
        g_x = np.zeros_like(g)
        np.add.at(g_x, send, g_xs)
        g = g_next + g_x
    # ---- embedding
    demb = np.zeros((spec.n_species, C))
    np.add.at(demb, species, g[:, 0, :])
    grads["emb"] = demb
    return energy, grads
