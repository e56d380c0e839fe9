"""Neighbour list and CSR edge layout (oracle; test infrastructure only).

Brute force over every (receiver, sender, periodic image) triple. The
inclusion test is fixed so that two independent implementations can agree bit
for bit (the reading recorded in the design notes):

    s   = ((S0 * cell[0] + S1 * cell[1]) + S2 * cell[2])        (float64)
    r   = (pos[j] - pos[i]) + s                                 (float64, from float32 positions)
    d2  = (r_x * r_x + r_y * r_y) + r_z * r_z                   (float64, no fused multiply-add)
    include  iff  d2 < float64(r_cut)^2  and not (i == j and S == 0)

Stored edge vector: float32(r), pointing from the receiver i to the sender j.
Canonical order: by (receiver, sender, S0, S1, S2); the transposed order is the
stable re-sort by sender, i.e. by (sender, receiver, S).
"""
import itertools
import math

import numpy as np


def image_range(cell, pbc, r_cut):
    """Per-axis number of periodic images to scan: ceil(r_cut / plane spacing)."""
    n = [0, 0, 0]
    if cell is None:
        return n
    cell = np.asarray(cell, dtype=np.float64)
    vol = abs(np.linalg.det(cell))
    for a in range(3):
        if pbc[a]:
            b, c = cell[(a + 1) % 3], cell[(a + 2) % 3]
            spacing = vol / np.linalg.norm(np.cross(b, c))
            n[a] = int(math.ceil(float(r_cut) / spacing))
    return n


def shift_list(cell, pbc, r_cut):
    n = image_range(cell, pbc, r_cut)
    return [s for s in itertools.product(range(-n[0], n[0] + 1), range(-n[1], n[1] + 1),
                                         range(-n[2], n[2] + 1))]


def neighbors(pos, cell, pbc, r_cut, receivers=None):
    """Brute-force neighbour list.

    pos: [N, 3] float32; cell: [3, 3] float64 rows = lattice vectors, or None;
    pbc: 3 bools; r_cut: float32 scalar. ``receivers``: optional sorted subset
    of receiver indices (for sampled checks on large systems).
    Returns dict with int64 arrays receiver, sender, shift [E,3] and float32
    edge_vec [E,3], in canonical order.
    """
    pos = np.asarray(pos, dtype=np.float32).astype(np.float64)
    n_atoms = pos.shape[0]
    rc2 = np.float64(np.float32(r_cut)) * np.float64(np.float32(r_cut))
    cellv = np.zeros((3, 3)) if cell is None else np.asarray(cell, dtype=np.float64)
    shifts = shift_list(cell, pbc, r_cut)
    recv_list = range(n_atoms) if receivers is None else receivers
    out_r, out_s, out_sh, out_v = [], [], [], []
    j_all = np.arange(n_atoms)
    for i in recv_list:
        rows = []
        for s in shifts:
            sv = (s[0] * cellv[0] + s[1] * cellv[1]) + s[2] * cellv[2]
            dx = (pos[:, 0] - pos[i, 0]) + sv[0]
            dy = (pos[:, 1] - pos[i, 1]) + sv[1]
            dz = (pos[:, 2] - pos[i, 2]) + sv[2]
            d2 = (dx * dx + dy * dy) + dz * dz
            keep = d2 < rc2
            if s == (0, 0, 0):
                keep &= j_all != i
            jj = np.nonzero(keep)[0]
            for j in jj:
                rows.append((int(j), s, (dx[j], dy[j], dz[j])))
        rows.sort(key=lambda t: (t[0], t[1]))
        for j, s, v in rows:
            out_r.append(i)
            out_s.append(j)
            out_sh.append(s)
            out_v.append(v)
    e = len(out_r)
    return {
        "receiver": np.asarray(out_r, dtype=np.int64).reshape(e),
        "sender": np.asarray(out_s, dtype=np.int64).reshape(e),
        "shift": np.asarray(out_sh, dtype=np.int64).reshape(e, 3),
        "edge_vec": np.asarray(out_v, dtype=np.float64).reshape(e, 3).astype(np.float32),
    }


def csr(receiver, sender, n_nodes):
    """row_ptr, transposed row pointer and permutation for canonical-order edges."""
    receiver = np.asarray(receiver, dtype=np.int64)
    sender = np.asarray(sender, dtype=np.int64)
    row_ptr = np.zeros(n_nodes + 1, dtype=np.int64)
    np.add.at(row_ptr, receiver + 1, 1)
    row_ptr = np.cumsum(row_ptr)
    t_perm = np.argsort(sender, kind="stable")
    t_row_ptr = np.zeros(n_nodes + 1, dtype=np.int64)
    np.add.at(t_row_ptr, sender + 1, 1)
    t_row_ptr = np.cumsum(t_row_ptr)
    return row_ptr, t_row_ptr, t_perm


def forces_from_edge_grads(grad_edge_vec, receiver, sender, n_nodes):
    """F_k = sum_{e: recv=k} g_e - sum_{e: send=k} g_e  (F = -dL/dpos, r_e = pos_send - pos_recv + S)."""
    f = np.zeros((n_nodes, 3))
    g = np.asarray(grad_edge_vec, dtype=np.float64)
    np.add.at(f, np.asarray(receiver), g)
    np.add.at(f, np.asarray(sender), -g)
    return f
