"""Test helpers that build every expected value from the oracle and the seeded workloads only."""
import numpy as np

from oracle.conv import ConvSpec, conv_forward, conv_vjp
from oracle.graph import csr, neighbors

TOL = 1e-5   # per irrep block: max|gpu - ref| <= TOL * max|ref|


def spec_of(wl):
    return ConvSpec(wl.irreps, wl.lmax, wl.irreps, wl.n_basis, float(wl.r_cut))


def full_graph(wl):
    nb = neighbors(wl.pos, wl.cell, wl.pbc, wl.r_cut)
    row_ptr, t_row_ptr, t_perm = csr(nb["receiver"], nb["sender"], wl.n_nodes)
    return dict(nb, row_ptr=row_ptr, t_row_ptr=t_row_ptr, t_perm=t_perm)


def given_graph(wl):
    """Canonical order of a given edge list: stable by (receiver, sender)."""
    order = np.lexsort((wl.given_sender, wl.given_receiver))
    receiver = wl.given_receiver[order]
    sender = wl.given_sender[order]
    row_ptr, t_row_ptr, t_perm = csr(receiver, sender, wl.n_nodes)
    return dict(receiver=receiver, sender=sender, edge_vec=wl.given_edge_vec[order], perm=order,
                row_ptr=row_ptr, t_row_ptr=t_row_ptr, t_perm=t_perm)


def rows_subgraph(n_nodes, receiver, sender, edge_vec):
    """CSR over all n_nodes holding only the given (receiver-sorted) edges."""
    row_ptr = np.zeros(n_nodes + 1, dtype=np.int64)
    np.add.at(row_ptr, np.asarray(receiver) + 1, 1)
    return np.cumsum(row_ptr), np.asarray(sender), np.asarray(edge_vec)


def sampled_rows(wl, sample):
    """Oracle neighbour rows of the sampled receivers (brute force)."""
    return neighbors(wl.pos, wl.cell, wl.pbc, wl.r_cut, receivers=sorted(int(s) for s in sample))


def sender_edges(rows):
    """All edges whose sender is a sampled node, from the sampled nodes' own rows.

    The inclusion test is symmetric and exact under negation: (i <- j, S) is an edge iff
    (j <- i, -S) is, with edge vector exactly -r. So the edges sent by j are the mirror images of
    receiver j's row."""
    recv = rows["sender"].copy()           # mirrored: the old sender becomes the receiver
    send = rows["receiver"].copy()
    shift = -rows["shift"]
    vec = -rows["edge_vec"]
    key = np.lexsort((shift[:, 2], shift[:, 1], shift[:, 0], send, recv))
    return recv[key], send[key], shift[key], vec[key]


def forward_ref(wl, spec, x, W, graph=None, sample=None):
    if sample is None:
        return conv_forward(spec, graph["row_ptr"], graph["sender"], graph["edge_vec"], x, W)
    rows = sampled_rows(wl, sample)
    rp, snd, vec = rows_subgraph(wl.n_nodes, rows["receiver"], rows["sender"], rows["edge_vec"])
    return conv_forward(spec, rp, snd, vec, x, W, receivers=sorted(int(s) for s in sample)), rows


def block_errors(gpu, ref, channels, lmax):
    out = []
    for l in range(lmax + 1):
        sl = slice(channels * l * l, channels * (l + 1) ** 2)
        err = float(np.abs(np.asarray(gpu, np.float64)[:, sl] - ref[:, sl]).max()) if ref.size else 0.0
        scale = float(np.abs(ref[:, sl]).max()) if ref.size else 0.0
        out.append((l, err, scale))
    return out


def assert_blocks_close(gpu, ref, channels, lmax, what, tol=TOL):
    for l, err, scale in block_errors(gpu, ref, channels, lmax):
        assert err <= tol * scale, f"{what}: block l={l} max|err|={err:.3e} > {tol:g} * max|ref|={scale:.3e}"


def assert_close_rel(gpu, ref, what, tol=TOL):
    gpu = np.asarray(gpu, np.float64)
    err = float(np.abs(gpu - ref).max()) if ref.size else 0.0
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    assert err <= tol * scale, f"{what}: max|err|={err:.3e} > {tol:g} * max|ref|={scale:.3e}"


__all__ = ["TOL", "spec_of", "full_graph", "given_graph", "rows_subgraph", "sampled_rows", "sender_edges",
           "forward_ref", "block_errors", "assert_blocks_close", "assert_close_rel", "conv_vjp"]


def assert_irrep_blocks_close(gpu, ref, spec, side, what, tol=TOL):
    """Per irrep block of a general spec (side: 'in' or 'out'), the same bound as above."""
    blocks = spec.blocks_in if side == "in" else spec.blocks_out
    sl_of = spec.in_slice if side == "in" else spec.out_slice
    gpu = np.asarray(gpu, np.float64)
    for b, (mul, l, par) in enumerate(blocks):
        sl = sl_of(b)
        err = float(np.abs(gpu[:, sl] - ref[:, sl]).max()) if ref.size else 0.0
        scale = float(np.abs(ref[:, sl]).max()) if ref.size else 0.0
        assert err <= tol * scale, f"{what}: block {mul}x{l}{'e' if par > 0 else 'o'} max|err|={err:.3e} > " \
                                   f"{tol:g} * max|ref|={scale:.3e}"


__all__.append("assert_irrep_blocks_close")
