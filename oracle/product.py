"""Node-local tensor products (test infrastructure only; never imported by the product path).

The path-reduced "uvu" product of two node features, the building block of the product ladder in
"FlashCart" (Fig. 3b and Fig. E1): for every node and channel u,

    P[l3, m3, u] = sum_{p = (l1, l2, l3)} W[p, u] sum_{m1, m2} C^{l1 l2 l3}_{m1 m2 m3} B[l1, m1, u] A[l2, m2, u]

with the real Clebsch-Gordan coefficients and the path set of the edge convolution (l1, l2, l3 <= L,
triangle rule, l1 + l2 + l3 even). Features are laid out [N][(l, m)][C] like the convolution's
node rows. The ladder of correlation order nu reuses the same atomic basis A at every step:

    B_1 = A,   B_{q+1} = P(B_q, A; W_q),   out = sum_{q=1..nu} B_q

(each step's output enters the next product and also contributes to the final sum; the linear
maps between steps of the full architecture are left out, as in the path-reduced curves of
Fig. 3b). float64 throughout.

The full ladder (the dashed curves of Fig. 3b; Fig. E1 (b): the tensor-product outputs of the
retained coupling paths are compressed by W^(q) to d channels per retained rank) keeps the
per-path products without a weight,

    T_p[m3, u] = sum_{m1, m2} C^{l1 l2 l3}_{m1 m2 m3} B[l1, m1, u] A[l2, m2, u],

and maps them with one matrix per output rank l3 that mixes the paths of that rank and the
channels (d = C, the fixed width):

    B'[l3, m3, v] = sum_{p of rank l3} sum_u W_l3[v, p' C + u] T_p[m3, u]

(p' = the index of p among the paths of rank l3, in path order); the ladder recursion is unchanged.
"""
import numpy as np

from .cg import cg_real


def product_paths(lmax):
    """(l1, l2, l3) in lexicographic order: triangle rule, l1 + l2 + l3 even, all <= lmax."""
    out = []
    for l1 in range(lmax + 1):
        for l2 in range(lmax + 1):
            for l3 in range(lmax + 1):
                if abs(l1 - l2) <= l3 <= l1 + l2 and (l1 + l2 + l3) % 2 == 0:
                    out.append((l1, l2, l3))
    return out


def _block(x, l, c):
    """[N, 2l+1, C] view of rank-l components of a [N, (L+1)^2 C] feature array."""
    return x[:, l * l * c:(l + 1) * (l + 1) * c].reshape(x.shape[0], 2 * l + 1, c)


def node_product(lmax, channels, B, A, W):
    """P(B, A; W) for [N, (L+1)^2 C] inputs and W [n_paths, C]."""
    B = np.asarray(B, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    n, c = B.shape[0], channels
    out = np.zeros((n, (lmax + 1) ** 2 * c))
    for p, (l1, l2, l3) in enumerate(product_paths(lmax)):
        cg = cg_real(l1, l2, l3)
        t = np.einsum("abk,nau,nbu->nku", cg, _block(B, l1, c), _block(A, l2, c)) * W[p][None, None, :]
        out[:, l3 * l3 * c:(l3 + 1) * (l3 + 1) * c] += t.reshape(n, -1)
    return out


def node_ladder(lmax, channels, A, Ws):
    """out = sum_q B_q with B_1 = A and B_{q+1} = P(B_q, A; W_q); Ws: [nu - 1, n_paths, C]."""
    A = np.asarray(A, dtype=np.float64)
    b = A.copy()
    out = A.copy()
    for W in np.asarray(Ws, dtype=np.float64):
        b = node_product(lmax, channels, b, A, W)
        out += b
    return out


def paths_of_rank(lmax, l3):
    """Indices into product_paths(lmax) of the paths with output rank l3, in path order."""
    return [p for p, (_, _, c) in enumerate(product_paths(lmax)) if c == l3]


def full_step_sizes(lmax, channels):
    """Floats of each rank's compression matrix W_l3 [C][P_l3 C] (row-major), l3 = 0..L."""
    return [channels * len(paths_of_rank(lmax, l3)) * channels for l3 in range(lmax + 1)]


def split_full_step(lmax, channels, w):
    """A flat step of weights (the l3 matrices one after another, each [C][P_l3 C] row-major) as a
    list of [C, P_l3 C] matrices."""
    w = np.asarray(w, dtype=np.float64).ravel()
    out, off = [], 0
    for l3, size in enumerate(full_step_sizes(lmax, channels)):
        out.append(w[off:off + size].reshape(channels, -1))
        off += size
    assert off == w.size, "weights do not match the path set"
    return out


def node_product_full(lmax, channels, B, A, w):
    """One step of the full ladder: the unweighted per-path products T_p, then per output rank the
    path- and channel-mixing matrix. w: a flat step (see split_full_step)."""
    B = np.asarray(B, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    n, c = B.shape[0], channels
    paths = product_paths(lmax)
    mats = split_full_step(lmax, c, w)
    out = np.zeros((n, (lmax + 1) ** 2 * c))
    for l3 in range(lmax + 1):
        ps = paths_of_rank(lmax, l3)
        t = np.zeros((n, 2 * l3 + 1, len(ps), c))     # [node, m3, p', u]
        for j, p in enumerate(ps):
            l1, l2, _ = paths[p]
            t[:, :, j, :] = np.einsum("abk,nau,nbu->nku", cg_real(l1, l2, l3), _block(B, l1, c), _block(A, l2, c))
        res = t.reshape(n, 2 * l3 + 1, len(ps) * c) @ mats[l3].T   # [node, m3, v]
        out[:, l3 * l3 * c:(l3 + 1) * (l3 + 1) * c] = res.reshape(n, -1)
    return out


def node_ladder_full(lmax, channels, A, Ws):
    """out = sum_q B_q with B_1 = A and B_{q+1} = P_full(B_q, A; W_q); Ws: [nu - 1] flat steps."""
    A = np.asarray(A, dtype=np.float64)
    b = A.copy()
    out = A.copy()
    for w in Ws:
        b = node_product_full(lmax, channels, b, A, w)
        out += b
    return out
